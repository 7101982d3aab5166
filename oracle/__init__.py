"""fp64 CPU oracle for exact attention -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never imports it and shares no code with it.

The arithmetic lives in ``attn_oracle.c`` (plain C, IEEE double); this module
compiles it with gcc on first use and marshals numpy arrays.  Every input is
passed as float32 values (bf16 and fp32 inputs are exact in float32) and every
output comes back as float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    if True:
        P = ctypes.c_void_p
        I = ctypes.c_int
        Dd = ctypes.c_double
        I64 = ctypes.c_int64
        lib.oracle_rope_f64.argtypes = [P, P, P, I, I, I, Dd]
        lib.oracle_attn_fwd_f64.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Dd, I, Dd, I, P, I64]
        lib.oracle_attn_fwd_tiled_f64.argtypes = [P, P, P, P, P, I, I, I, I, I, I, Dd, I, I, I]
        lib.oracle_decode_f64.argtypes = [P, P, P, P, P, P, I, I, I, I, I, Dd]
        lib.oracle_decode_split_f64.argtypes = [P, P, P, P, P, P, I, I, I, I, I, Dd, I]
        lib.oracle_attn_bwd_f64.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, Dd, I, Dd, I]
        lib.oracle_attn_fwd_mask_f64.argtypes = [P, P, P, P, I64, I64, P, P, I, I, I, I, I, I, Dd, I, Dd, I]
        lib.oracle_attn_bwd_mask_f64.argtypes = [P, P, P, P, P, I64, I64, P, P, P, I, I, I, I, I, I, Dd, I, Dd, I]
        lib.oracle_attn_bwd_sampled_f64.argtypes = [P, P, P, P, I, I, I, I, I, I, Dd, I, Dd, I, I, I, P, I, P, I,
                                                    P, P, P]
        for f in (lib.oracle_rope_f64, lib.oracle_attn_fwd_f64, lib.oracle_attn_fwd_tiled_f64,
                  lib.oracle_decode_f64, lib.oracle_decode_split_f64, lib.oracle_attn_bwd_f64,
                  lib.oracle_attn_fwd_mask_f64, lib.oracle_attn_bwd_mask_f64, lib.oracle_attn_bwd_sampled_f64):
            f.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def swap_library(path):
    """Bind the functions of this module to another build of ``attn_oracle.c`` (``path``;
    None restores the default build).  Used only to check that the pins reject builds with
    planted mistakes."""
    global _lib
    _lib = None if path is None else _bind(path)


class OracleError(RuntimeError):
    pass


_STATUS = {1: "invalid argument", 2: "dimension mismatch", 3: "empty KV", 9: "out of memory"}


def _check(st: int):
    if st != 0:
        raise OracleError(_STATUS.get(st, f"status {st}"))


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    """Bound the OpenMP threads the oracle uses in later calls from this thread (the
    environment variable for a runtime not started yet, omp_set_num_threads for a running one)."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))
    try:
        ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))
    except OSError:
        pass


def threads() -> int:
    """OpenMP threads the next oracle call from this thread will use."""
    try:
        return int(ctypes.CDLL("libgomp.so.1").omp_get_max_threads())
    except OSError:
        return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def rope(x, pos, base: float) -> np.ndarray:
    """x [T,H,D] rotated at positions pos[T] (interleaved pairs); float64 result."""
    x = _f32(x)
    T, H, D = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    out = np.empty((T, H, D), dtype=np.float64)
    _check(_load().oracle_rope_f64(_ptr(x), _ptr(pos), _ptr(out), T, H, D, float(base)))
    return out


def attn_fwd(q, k, v, scale: float, causal: bool, rope_base: float = 0.0, q_pos0: int = 0,
             rows=None):
    """Exact attention, fp64.  q [B,Sq,Hq,D], k/v [B,Skv,Hkv,D].

    rows=None: returns (o [B,Sq,Hq,D], lse [B,Hq,Sq]).
    rows = int64 array of flat (b*Hq + hq)*Sq + i: returns (o [n,D], lse [n]).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, Skv, Hkv, D) or v.shape != k.shape:
        raise OracleError("dimension mismatch")
    if rows is None:
        o = np.empty((B, Sq, Hq, D), dtype=np.float64)
        lse = np.empty((B, Hq, Sq), dtype=np.float64)
        rp, n = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        o = np.empty((n, D), dtype=np.float64)
        lse = np.empty((n,), dtype=np.float64)
        rp = _ptr(rows)
    _check(_load().oracle_attn_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv,
                                       Sq, Skv, D, float(scale), int(bool(causal)), float(rope_base),
                                       int(q_pos0), rp, n))
    return o, lse


def attn_fwd_masked(q, k, v, mask, scale: float, causal: bool, rope_base: float = 0.0, q_pos0: int = 0):
    """attn_fwd with an additive mask on the scaled scores.  mask: [Sq, Skv], [B, Sq, Skv] (shared
    by the heads) or [B, Hq, Sq, Skv].  Returns (o [B,Sq,Hq,D], lse [B,Hq,Sq]) in float64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    m = _f32(mask)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    if m.shape[-2:] != (Sq, Skv):
        raise OracleError("mask shape")
    if m.ndim == 2:
        bs, hs = 0, 0
    elif m.ndim == 3:
        bs, hs = Sq * Skv, 0
    else:
        bs, hs = Hq * Sq * Skv, Sq * Skv
    o = np.empty((B, Sq, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq, Sq), dtype=np.float64)
    _check(_load().oracle_attn_fwd_mask_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(m), bs, hs, _ptr(o), _ptr(lse), B, Hq,
                                            Hkv, Sq, Skv, D, float(scale), int(bool(causal)), float(rope_base),
                                            int(q_pos0)))
    return o, lse


def _mask_strides(m, B, Hq, Sq, Skv):
    if m.shape[-2:] != (Sq, Skv):
        raise OracleError("mask shape")
    if m.ndim == 2:
        return 0, 0
    if m.ndim == 3:
        return Sq * Skv, 0
    return Hq * Sq * Skv, Sq * Skv


def attn_bwd_masked(q, k, v, dout, mask, scale: float, causal: bool, rope_base: float = 0.0, q_pos0: int = 0):
    """attn_bwd for the forward with an additive mask (see attn_fwd_masked)."""
    q, k, v, dout, m = _f32(q), _f32(k), _f32(v), _f32(dout), _f32(mask)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    bs, hs = _mask_strides(m, B, Hq, Sq, Skv)
    dq = np.empty((B, Sq, Hq, D), dtype=np.float64)
    dk = np.empty((B, Skv, Hkv, D), dtype=np.float64)
    dv = np.empty((B, Skv, Hkv, D), dtype=np.float64)
    _check(_load().oracle_attn_bwd_mask_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(m), bs, hs, _ptr(dq),
                                            _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Skv, D, float(scale),
                                            int(bool(causal)), float(rope_base), int(q_pos0)))
    return dq, dk, dv


def attn_fwd_tiled(q, k, v, scale: float, causal: bool, bq: int, bkv: int):
    """The online-softmax recurrence over (bq x bkv) blocks, fp64; same outputs as attn_fwd."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    o = np.empty((B, Sq, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq, Sq), dtype=np.float64)
    _check(_load().oracle_attn_fwd_tiled_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                             Hkv, Sq, Skv, D, float(scale), int(bool(causal)),
                                             int(bq), int(bkv)))
    return o, lse


def decode(q, kcache, vcache, seqlens, scale: float):
    """One query per (b, hq) against cache rows [0, seqlens[b]).  Returns (o [B,Hq,D], lse [B,Hq])."""
    q, kc, vc = _f32(q), _f32(kcache), _f32(vcache)
    B, Hq, D = q.shape
    Smax, Hkv = kc.shape[1], kc.shape[2]
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    o = np.empty((B, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    _check(_load().oracle_decode_f64(_ptr(q), _ptr(kc), _ptr(vc), _ptr(seqlens), _ptr(o), _ptr(lse),
                                     B, Hq, Hkv, Smax, D, float(scale)))
    return o, lse


def decode_split(q, kcache, vcache, seqlens, scale: float, num_tiles: int):
    """Split-KV decode (per-tile partials + LSE combine) with num_tiles tiles per sequence."""
    q, kc, vc = _f32(q), _f32(kcache), _f32(vcache)
    B, Hq, D = q.shape
    Smax, Hkv = kc.shape[1], kc.shape[2]
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    o = np.empty((B, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    _check(_load().oracle_decode_split_f64(_ptr(q), _ptr(kc), _ptr(vc), _ptr(seqlens), _ptr(o),
                                           _ptr(lse), B, Hq, Hkv, Smax, D, float(scale),
                                           int(num_tiles)))
    return o, lse


def attn_bwd(q, k, v, dout, scale: float, causal: bool, rope_base: float = 0.0, q_pos0: int = 0):
    """Gradients (dq [B,Sq,Hq,D], dk, dv [B,Skv,Hkv,D], float64) of the forward's o for the
    upstream gradient dout [B,Sq,Hq,D] -- the definition, see oracle_attn_bwd_f64."""
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, Skv, Hkv, D) or v.shape != k.shape or dout.shape != q.shape:
        raise OracleError("dimension mismatch")
    dq = np.empty((B, Sq, Hq, D), dtype=np.float64)
    dk = np.empty((B, Skv, Hkv, D), dtype=np.float64)
    dv = np.empty((B, Skv, Hkv, D), dtype=np.float64)
    _check(_load().oracle_attn_bwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                       B, Hq, Hkv, Sq, Skv, D, float(scale), int(bool(causal)),
                                       float(rope_base), int(q_pos0)))
    return dq, dk, dv


def attn_bwd_sampled(q, k, v, dout, scale: float, causal: bool, rope_base: float, q_pos0: int, b: int, kvh: int,
                     rows, keys):
    """The backward of one (batch b, kv head kvh) group at chosen places, fp64: dq of every q head
    of the group at query rows `rows` ([g, len(rows), D]), dk and dv of the kv head at keys `keys`
    ([len(keys), D] each).  Same definition as attn_bwd, for full-size problems."""
    q, k, v, g_ = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    keys = np.ascontiguousarray(keys, dtype=np.int64)
    g = Hq // Hkv
    dq = np.empty((g, rows.shape[0], D), dtype=np.float64)
    dk = np.empty((keys.shape[0], D), dtype=np.float64)
    dv = np.empty((keys.shape[0], D), dtype=np.float64)
    _check(_load().oracle_attn_bwd_sampled_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(g_), B, Hq, Hkv, Sq, Skv, D,
                                               float(scale), int(bool(causal)), float(rope_base), int(q_pos0),
                                               int(b), int(kvh), _ptr(rows), rows.shape[0], _ptr(keys),
                                               keys.shape[0], _ptr(dq), _ptr(dk), _ptr(dv)))
    return dq, dk, dv


def kv_append(kcache, vcache, seqlens, k_new, v_new, q=None, rope_base: float = 0.0):
    """The decode step's cache update (scirs2-neural 0.4.4 grouped_query_attention.rs,
    forward_with_cache / concat_cache: the new keys and values follow the cached ones and the new
    queries and keys are rotated at the cache offset; whisper-apr 0.3.1 lfm2 KvCache: an append
    past the capacity is an error).

    kcache/vcache [B,Smax,Hkv,D], seqlens [B], k_new/v_new [B,T,Hkv,D], q [B,T,Hq,D] or None.
    For each sequence b with L = seqlens[b]: if 0 <= L and L + T <= Smax, rows [L, L+T) take
    k_new[b] rotated at positions L..L+T-1 (rope_base > 0; unrotated otherwise) and v_new[b];
    q[b] is rotated at the same positions; the length becomes L + T.  Otherwise sequence b is
    left as it is and reported.  Returns float64 copies (kcache, vcache, seqlens, q, overflow[B]).
    """
    kc = np.array(kcache, dtype=np.float64)
    vc = np.array(vcache, dtype=np.float64)
    sl = np.array(seqlens, dtype=np.int64)
    kn, vn = np.asarray(k_new, dtype=np.float64), np.asarray(v_new, dtype=np.float64)
    qo = None if q is None else np.array(q, dtype=np.float64)
    B, Smax = kc.shape[0], kc.shape[1]
    T = kn.shape[1]
    overflow = np.zeros(B, dtype=bool)
    for b in range(B):
        L = int(sl[b])
        if L < 0 or L + T > Smax:
            overflow[b] = True
            continue
        pos = np.arange(L, L + T, dtype=np.int32)
        kc[b, L:L + T] = rope(kn[b], pos, rope_base) if rope_base > 0 else kn[b]
        vc[b, L:L + T] = vn[b]
        if qo is not None and rope_base > 0:
            qo[b] = rope(qo[b], pos, rope_base)
        sl[b] = L + T
    return kc, vc, sl, qo, overflow
