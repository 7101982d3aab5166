"""B200-native exact attention: Python binding of libattn_b200.so (the C ABI in include/attn_b200.h).

This module only marshals arguments: torch tensors supply device memory and the CUDA stream,
every computation runs in the library's sm_100a kernels.  There is no fallback: if the library
is missing or no CUDA device is present, calls raise.

Entry points (same names as the C ABI):
    attn_fwd(q, k, v, scale, causal, o=None, lse=None)                 -> (o, lse)
    attn_fwd_ex(q, k, v, scale, causal, rope_base, q_pos0, ...)        -> (o, lse)
    attn_decode(q, kcache, vcache, seqlens, scale, num_splits, ...)    -> (o, lse)
    rope_apply(x, pos, base)                                           -> x (in place)
Layouts: q/o [B, Sq, Hq, D]; k/v [B, Skv, Hkv, D]; lse [B, Hq, Sq] float32;
decode q/o [B, Hq, D], caches [B, Smax, Hkv, D], seqlens int32 [B], lse [B, Hq];
rope x [T, H, D], pos int32 [T].
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_b200.so")

ATTN_BF16, ATTN_FP32, ATTN_BF16_OUT_F32 = 0, 1, 2
STATUS = {0: "ok", 1: "invalid argument", 2: "dimension mismatch", 3: "empty KV",
          4: "unsupported configuration", 5: "workspace missing or too small", 6: "CUDA error",
          7: "device wait timed out"}

# symbols the library exports (kept in step with include/attn_b200.h)
EXPORTS = ("attn_fwd", "attn_fwd_ex", "attn_fwd_ex_workspace_size", "attn_decode",
           "attn_decode_workspace_size", "attn_decode_noalloc", "rope_apply", "attn_status_string",
           "attn_last_error", "attn_selftest_wait_timeout", "attn_read_device_status", "attn_kv_append",
           "attn_bwd", "attn_bwd_workspace_size", "attn_fwd_masked", "attn_bwd_masked",
           "attn_fwd_kv_splits")

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = ""
        if status == 6 and _lib is not None:
            detail = " -- " + _lib.attn_last_error().decode(errors="replace")
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status}){detail}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and type the C ABI.  Raises if the library was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} not found: build it with `python -m exact_attention_160_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, P]
    lib.attn_fwd_ex.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, F, I, P, Z, P]
    lib.attn_fwd_ex_workspace_size.argtypes = [I, I, I, I, I, I, I, F, I]
    lib.attn_fwd_ex_workspace_size.restype = Z
    lib.attn_fwd_kv_splits.argtypes = [I, I, I, I, I]
    lib.attn_fwd_kv_splits.restype = I
    lib.attn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, P, Z, I, P]
    lib.attn_decode_workspace_size.argtypes = [I, I, I, I]
    lib.attn_decode_workspace_size.restype = Z
    lib.attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P]
    lib.attn_decode_noalloc.restype = I
    lib.rope_apply.argtypes = [P, P, I, I, I, F, I, P]
    lib.attn_status_string.argtypes = [I]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_read_device_status.argtypes = [P]
    I64 = ctypes.c_int64
    lib.attn_fwd_masked.argtypes = [P, P, P, P, I64, I64, P, P, I, I, I, I, I, I, F, I, I, F, I, P, Z, P]
    lib.attn_fwd_masked.restype = I
    lib.attn_bwd_masked.argtypes = [P, P, P, P, I64, I64, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, F, I, P, Z, P]
    lib.attn_bwd_masked.restype = I
    lib.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, F, I, P, Z, P]
    lib.attn_bwd.restype = I
    lib.attn_bwd_workspace_size.argtypes = [I, I, I, I, I, I, I, F, I]
    lib.attn_bwd_workspace_size.restype = Z
    lib.attn_kv_append.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_kv_append.restype = I
    lib.attn_selftest_wait_timeout.argtypes = [I, P]
    lib.attn_selftest_wait_timeout.restype = I
    lib.attn_last_error.argtypes = []
    lib.attn_last_error.restype = ctypes.c_char_p
    for f in (lib.attn_fwd, lib.attn_fwd_ex, lib.attn_decode, lib.rope_apply, lib.attn_read_device_status):
        f.restype = I
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor, o: torch.Tensor = None) -> int:
    """dtype code of the C ABI: inputs' storage type, and for bf16 inputs the output's."""
    if t.dtype == torch.bfloat16:
        if o is not None and o.dtype == torch.float32:
            return ATTN_BF16_OUT_F32
        if o is not None and o.dtype != torch.bfloat16:
            raise TypeError(f"unsupported output dtype {o.dtype}")
        return ATTN_BF16
    if t.dtype == torch.float32:
        if o is not None and o.dtype != torch.float32:
            raise TypeError("fp32 inputs take an fp32 output")
        return ATTN_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(st: int, what: str):
    if st != 0:
        raise AttnError(st, what)


def _shape(t):
    return tuple(t.shape)


def _check_qkv(q, k, v, o=None, lse=None, same_dtype_o=False):
    """Shapes and dtypes the C ABI cannot see (it takes pointers and sizes): q [B, Sq, Hq, D],
    k and v [B, Skv, Hkv, D] of q's dtype, o like q, lse [B, Hq, Sq] fp32."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dim() != 4:
            raise ValueError(f"{name} must be [B, S, H, D], got {_shape(t)}")
    if _shape(k) != _shape(v):
        raise ValueError(f"k {_shape(k)} and v {_shape(v)} differ")
    if q.shape[0] != k.shape[0] or q.shape[3] != k.shape[3]:
        raise ValueError(f"q {_shape(q)} and k {_shape(k)} disagree on the batch or the head dim")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError(f"q, k and v must share one dtype ({q.dtype}, {k.dtype}, {v.dtype})")
    B, Sq, Hq, _ = q.shape
    if o is not None:
        if _shape(o) != _shape(q):
            raise ValueError(f"o {_shape(o)} must have q's shape {_shape(q)}")
        if same_dtype_o and o.dtype != q.dtype:
            raise TypeError(f"o must have q's dtype {q.dtype}")
    if lse is not None and (lse.dtype != torch.float32 or _shape(lse) != (B, Hq, Sq)):
        raise ValueError(f"lse must be float32 [B, Hq, Sq] = {(B, Hq, Sq)}, got {lse.dtype} {_shape(lse)}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def attn_fwd(q, k, v, scale: float, causal: bool, o=None, lse=None, want_lse: bool = True, out_dtype=None,
             stream=None, kv_split: bool = True):
    """Exact attention forward.  Returns (o, lse); lse is None when want_lse is False.
    out_dtype: torch.float32 to take a bf16 problem's output in fp32 (default: q's dtype).
    kv_split=False runs a small problem unsplit (the C attn_fwd, no workspace)."""
    return attn_fwd_ex(q, k, v, scale, causal, 0.0, 0, o=o, lse=lse, want_lse=want_lse, out_dtype=out_dtype,
                       stream=stream, kv_split=kv_split)


def fwd_kv_splits(q, k, out_dtype=None) -> int:
    """Key splits attn_fwd_ex uses for these shapes when it has its workspace (1: unsplit)."""
    lib = load_library()
    B, Sq, Hq, _ = q.shape
    return int(lib.attn_fwd_kv_splits(B, Hq, Sq, k.shape[1], _out_code(q, out_dtype)))


def _out_code(q, out_dtype):
    return _dtype_code(q) if out_dtype is None or q.dtype != torch.bfloat16 else (
        ATTN_BF16_OUT_F32 if out_dtype == torch.float32 else ATTN_BF16)


def fwd_workspace_bytes(q, k, rope_base: float, q_pos0: int, out_dtype=None) -> int:
    lib = load_library()
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    return int(lib.attn_fwd_ex_workspace_size(B, Hq, Hkv, Sq, Skv, D, _out_code(q, out_dtype), float(rope_base),
                                              int(q_pos0)))


def attn_fwd_ex(q, k, v, scale: float, causal: bool, rope_base: float, q_pos0: int = 0, o=None, lse=None,
                want_lse: bool = True, workspace=None, out_dtype=None, stream=None, kv_split: bool = True):
    """Exact attention forward with RoPE on Q (positions q_pos0 + i) and K (positions j).
    kv_split=False (without RoPE, D 64 or 128) calls the C attn_fwd: no workspace, no key splits."""
    lib = load_library()
    _check_qkv(q, k, v, o, lse)
    _need_cuda(q, k, v, o, lse, workspace)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    ws_bytes = 0
    if not kv_split and rope_base <= 0 and D in (64, 128):
        need, workspace = 0, None
    else:
        need = fwd_workspace_bytes(q, k, rope_base, q_pos0, o.dtype)
    if need > 0 or workspace is not None:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    if rope_base > 0 or need > 0:
        st = lib.attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Skv, D,
                             float(scale), int(bool(causal)), _dtype_code(q, o), float(rope_base), int(q_pos0),
                             _ptr(workspace), ws_bytes, _stream(stream))
        _check(st, "attn_fwd_ex")
    else:
        st = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Skv, D,
                          float(scale), int(bool(causal)), _dtype_code(q, o), _stream(stream))
        _check(st, "attn_fwd")
    return o, lse


def _mask_strides(mask, Sq: int, Skv: int):
    """(batch, head) element strides of a float32 mask [Sq, Skv], [B, Sq, Skv] or [B, Hq, Sq, Skv]
    (size-1 or expanded dims broadcast); rows must be contiguous."""
    if mask.dtype != torch.float32 or not mask.is_cuda or mask.shape[-2:] != (Sq, Skv) or mask.stride(-1) != 1 \
            or mask.stride(-2) != Skv:
        raise ValueError("mask must be a float32 CUDA tensor [..., Sq, Skv] with contiguous rows")
    if mask.dim() == 2:
        return 0, 0
    if mask.dim() == 3:
        return (mask.stride(0) if mask.shape[0] > 1 else 0), 0
    if mask.dim() == 4:
        return (mask.stride(0) if mask.shape[0] > 1 else 0), (mask.stride(1) if mask.shape[1] > 1 else 0)
    raise ValueError("mask must have 2, 3 or 4 dims")


def attn_fwd_masked(q, k, v, mask, scale: float, causal: bool, rope_base: float = 0.0, q_pos0: int = 0, o=None,
                    lse=None, workspace=None, out_dtype=None, stream=None):
    """Exact attention with an additive fp32 mask on the scaled scores.  mask: [Sq, Skv] (shared),
    [B, Sq, Skv] (per batch, shared by the heads) or [B, Hq, Sq, Skv]; rows must be contiguous."""
    lib = load_library()
    _check_qkv(q, k, v, o, lse)
    _need_cuda(q, k, v, o, lse, workspace)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    bs, hs = _mask_strides(mask, Sq, Skv)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    need = fwd_workspace_bytes(q, k, rope_base, q_pos0, o.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(mask), bs, hs, _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Skv,
                             D, float(scale), int(bool(causal)), _dtype_code(q, o), float(rope_base), int(q_pos0),
                             _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "attn_fwd_masked")
    return o, lse


def decode_workspace_bytes(B: int, Hq: int, D: int, num_splits: int) -> int:
    return int(load_library().attn_decode_workspace_size(B, Hq, D, num_splits))


def attn_decode(q, kcache, vcache, seqlens, scale: float, num_splits: int, o=None, lse=None,
                want_lse: bool = True, workspace=None, out_dtype=None, stream=None):
    """Split-KV decode of one token per (sequence, q head).  Returns (o, lse)."""
    lib = load_library()
    if q.dim() != 3 or kcache.dim() != 4 or _shape(kcache) != _shape(vcache):
        raise ValueError(f"q must be [B, Hq, D] and the caches one [B, Smax, Hkv, D] shape, got {_shape(q)}, "
                         f"{_shape(kcache)}, {_shape(vcache)}")
    if kcache.shape[0] != q.shape[0] or kcache.shape[3] != q.shape[2]:
        raise ValueError(f"q {_shape(q)} and the caches {_shape(kcache)} disagree on the batch or the head dim")
    if q.dtype != torch.bfloat16 or kcache.dtype != torch.bfloat16 or vcache.dtype != torch.bfloat16:
        raise TypeError("attn_decode takes bf16 q and caches")
    if seqlens.dtype != torch.int32 or _shape(seqlens) != (q.shape[0],):
        raise ValueError(f"seqlens must be int32 [B], got {seqlens.dtype} {_shape(seqlens)}")
    if o is not None and _shape(o) != _shape(q):
        raise ValueError(f"o {_shape(o)} must have q's shape {_shape(q)}")
    if lse is not None and (lse.dtype != torch.float32 or _shape(lse) != _shape(q)[:2]):
        raise ValueError(f"lse must be float32 [B, Hq], got {lse.dtype} {_shape(lse)}")
    _need_cuda(q, kcache, vcache, seqlens, o, lse, workspace)
    B, Hq, D = q.shape
    Smax, Hkv = kcache.shape[1], kcache.shape[2]
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib.attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(o), _ptr(lse), B, Hq, Hkv,
                         Smax, D, float(scale), int(num_splits), _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _dtype_code(q, o), _stream(stream))
    _check(st, "attn_decode")
    return o, lse


def rope_apply(x, pos, base: float, stream=None):
    """Rotate x [T, H, D] in place at positions pos [T] (int32)."""
    lib = load_library()
    if x.dim() != 3 or pos.dtype != torch.int32 or _shape(pos) != (x.shape[0],):
        raise ValueError(f"x must be [T, H, D] and pos int32 [T], got {_shape(x)}, {pos.dtype} {_shape(pos)}")
    _need_cuda(x, pos)
    T, H, D = x.shape
    st = lib.rope_apply(_ptr(x), _ptr(pos), T, H, D, float(base), _dtype_code(x), _stream(stream))
    _check(st, "rope_apply")
    return x


def bwd_workspace_bytes(q, k, rope_base: float = 0.0, q_pos0: int = 0, grad_dtype=None) -> int:
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    code = ATTN_FP32 if q.dtype == torch.float32 else (
        ATTN_BF16_OUT_F32 if grad_dtype == torch.float32 else ATTN_BF16)
    return int(load_library().attn_bwd_workspace_size(B, Hq, Hkv, Sq, Skv, D, code, float(rope_base), int(q_pos0)))


def attn_bwd(q, k, v, o, lse, dout, scale: float, causal: bool, rope_base: float = 0.0, q_pos0: int = 0,
             grad_dtype=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of the forward for the upstream gradient dout.  o and lse are the
    forward's outputs.  grad_dtype: torch.float32 to take a bf16 problem's gradients in fp32
    (default: q's dtype)."""
    lib = load_library()
    _check_qkv(q, k, v, o, lse, same_dtype_o=True)
    _check_qkv(q, k, v, dout, None, same_dtype_o=True)
    gd = q.dtype if grad_dtype is None else grad_dtype
    if q.dtype == torch.float32 and gd != torch.float32:
        raise TypeError("fp32 inputs take fp32 gradients")
    _need_cuda(q, k, v, o, lse, dout, workspace)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    code = ATTN_FP32 if q.dtype == torch.float32 else (ATTN_BF16_OUT_F32 if gd == torch.float32 else ATTN_BF16)
    dq = torch.empty(q.shape, dtype=gd, device=q.device)
    dk = torch.empty(k.shape, dtype=gd, device=q.device)
    dv = torch.empty(v.shape, dtype=gd, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(bwd_workspace_bytes(q, k, rope_base, q_pos0, gd), 1), dtype=torch.uint8,
                                device=q.device)
    st = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, Hq,
                      Hkv, Sq, Skv, D, float(scale), int(bool(causal)), code, float(rope_base), int(q_pos0),
                      _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "attn_bwd")
    return dq, dk, dv


def attn_bwd_masked(q, k, v, mask, o, lse, dout, scale: float, causal: bool, rope_base: float = 0.0,
                    q_pos0: int = 0, grad_dtype=None, workspace=None, stream=None):
    """attn_bwd for attn_fwd_masked (same mask)."""
    lib = load_library()
    _check_qkv(q, k, v, o, lse, same_dtype_o=True)
    _check_qkv(q, k, v, dout, None, same_dtype_o=True)
    gd0 = q.dtype if grad_dtype is None else grad_dtype
    if q.dtype == torch.float32 and gd0 != torch.float32:
        raise TypeError("fp32 inputs take fp32 gradients")
    _need_cuda(q, k, v, o, lse, dout, workspace)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    bs, hs = _mask_strides(mask, Sq, Skv)
    gd = q.dtype if grad_dtype is None else grad_dtype
    code = ATTN_FP32 if q.dtype == torch.float32 else (ATTN_BF16_OUT_F32 if gd == torch.float32 else ATTN_BF16)
    dq = torch.empty(q.shape, dtype=gd, device=q.device)
    dk = torch.empty(k.shape, dtype=gd, device=q.device)
    dv = torch.empty(v.shape, dtype=gd, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(bwd_workspace_bytes(q, k, rope_base, q_pos0, gd), 1), dtype=torch.uint8,
                                device=q.device)
    st = lib.attn_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(mask), bs, hs, _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                             _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Skv, D, float(scale), int(bool(causal)), code,
                             float(rope_base), int(q_pos0), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "attn_bwd_masked")
    return dq, dk, dv


def kv_append(kcache, vcache, seqlens, k_new, v_new, q=None, rope_base: float = 0.0, stream=None):
    """Append k_new/v_new [B, T, Hkv, D] (bf16) to the caches [B, Smax, Hkv, D] after each
    sequence's length, rotating keys (and q [B, T, Hq, D], in place) at positions L_b + t when
    rope_base > 0; advances seqlens [B] (int32, device).  Overflowing sequences are skipped and
    flagged in the device status word."""
    lib = load_library()
    if kcache.dim() != 4 or _shape(kcache) != _shape(vcache) or k_new.dim() != 4 or _shape(k_new) != _shape(v_new):
        raise ValueError(f"caches [B, Smax, Hkv, D] and new rows [B, T, Hkv, D] of one shape each, got "
                         f"{_shape(kcache)}, {_shape(vcache)}, {_shape(k_new)}, {_shape(v_new)}")
    if (k_new.shape[0], k_new.shape[2], k_new.shape[3]) != (kcache.shape[0], kcache.shape[2], kcache.shape[3]):
        raise ValueError(f"new rows {_shape(k_new)} do not fit the caches {_shape(kcache)}")
    if q is not None and (q.dim() != 4 or q.shape[0] != k_new.shape[0] or q.shape[1] != k_new.shape[1]
                          or q.shape[3] != k_new.shape[3]):
        raise ValueError(f"q must be [B, T, Hq, D] for new rows {_shape(k_new)}, got {_shape(q)}")
    if _shape(seqlens) != (kcache.shape[0],):
        raise ValueError(f"seqlens must be [B], got {_shape(seqlens)}")
    _need_cuda(kcache, vcache, seqlens, k_new, v_new, q)
    for t in (kcache, vcache, k_new, v_new, q):
        if t is not None and t.dtype != torch.bfloat16:
            raise TypeError("kv_append takes bf16 tensors")
    if seqlens.dtype != torch.int32:
        raise TypeError("seqlens must be int32")
    B, Smax, Hkv, D = kcache.shape
    T = k_new.shape[1]
    Hq = q.shape[2] if q is not None else Hkv
    st = lib.attn_kv_append(_ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(k_new), _ptr(v_new), _ptr(q), B, T,
                            Hq, Hkv, Smax, D, float(rope_base), _stream(stream))
    _check(st, "attn_kv_append")
    return kcache, vcache, seqlens


def read_device_status(stream=None) -> int:
    """Read and clear the library's device status word (synchronises the stream)."""
    return int(load_library().attn_read_device_status(_stream(stream)))
