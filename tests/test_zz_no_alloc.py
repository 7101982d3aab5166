"""attn_decode_noalloc: the decode entry point for callers that cannot allocate device memory
(code inside a host framework that owns all device allocations and hands a plugin only its inputs
and outputs, or a serving path that must not call cudaMalloc because it can synchronise the device
and take unbounded time).  It keeps the split partials in a scratch array the library owns.

Called here through the C ABI and compared with attn_decode (the caller's workspace) bit for bit:
both run the same split and combine kernels in the same order, so any difference is a bug in
where the scratch partials are put or read.  attn_decode gets a workspace filled with NaN, so a
slot its combine read without the split kernel having written it in the same call would show.
Two calls in a row per head dim: first every split slot of every (sequence, head) is written
(long sequences, the most splits), then short sequences use only the first split or two, so the
stale partials of the first call sit in the very slots a wrong combine would read.  The second call
must also leave the device's free memory and torch's allocator exactly as they were, and one
result is checked against the fp64 oracle.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, bits_to_dev, compare

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 16 << 20   # ATTN_NOALLOC_SCRATCH_BYTES


def _noalloc(lib, w, q, kc, vc, sl, o, lse):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.attn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
                                   ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(sl.data_ptr()),
                                   ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                                   w.B, w.Hq, w.Hkv, w.Smax, w.D, w.scale, w.num_splits,
                                   ea.ATTN_BF16_OUT_F32, stream)


def _reference(w, q, kc, vc, sl):
    """attn_decode with a caller workspace that starts out all NaN."""
    ws = torch.full((ea.decode_workspace_bytes(w.B, w.Hq, w.D, w.num_splits) // 4,), float("nan"),
                    dtype=torch.float32, device="cuda")
    return ea.attn_decode(q, kc, vc, sl, w.scale, w.num_splits, out_dtype=torch.float32, workspace=ws)


def _oracle_check(w, d, sl_host, o, lse):
    o_ref = np.empty((w.B, w.Hq, w.D))
    l_ref = np.empty((w.B, w.Hq))
    for b in range(w.B):
        L = int(sl_host[b])
        ob, lb = oracle.decode(d["q"][b:b + 1], si.bf16_bits_to_f32(d["k_bits"][b:b + 1, :L]),
                               si.bf16_bits_to_f32(d["v_bits"][b:b + 1, :L]), np.array([L], np.int32), w.scale)
        o_ref[b], l_ref[b] = ob[0], lb[0]
    compare(o.cpu().double().numpy(), o_ref, lse.cpu().double().numpy(), l_ref, TOL_BF16_O, TOL_BF16_LSE,
            f"noalloc D={w.D}")


@pytest.mark.parametrize("D", [64, 128])
def test_noalloc_decode_bit_exact_twice_and_allocates_nothing(D):
    lib = ea.load_library()
    B, Hq, Hkv, Smax, ns = 4, 32, 8, 8192, 16
    w = si.Decode(f"noalloc_d{D}", B, Hq, Hkv, D, Smax, 1, Smax, 1.0 / np.sqrt(D), ns, seed=30 + D)
    assert lib.attn_decode_workspace_size(B, Hq, D, ns) <= NOALLOC_BYTES
    long_len = np.full(B, Smax, np.int32)                     # 16 splits per (sequence, head)
    short_len = np.array([1, 700, 1100, 1535], np.int32)      # 1, 1, 2, 2 splits
    d = si.decode_inputs(w, seqlens=long_len)                 # cache rows past Smax: none; NaN-free
    q, kc, vc = bits_to_dev(d["q_bits"]), bits_to_dev(d["k_bits"]), bits_to_dev(d["v_bits"])
    o = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")

    # call 1: every split slot written
    sl = torch.from_numpy(long_len).cuda()
    assert _noalloc(lib, w, q, kc, vc, sl, o, lse) == 0, lib.attn_last_error().decode()
    o_ref, lse_ref = _reference(w, q, kc, vc, sl)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    if D == 64:
        _oracle_check(w, d, long_len, o, lse)

    # call 2: short sequences read only their first split slots; stale partials lie beyond them
    sl2 = torch.from_numpy(short_len).cuda()
    o2 = torch.empty_like(o)
    lse2 = torch.empty_like(lse)
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    assert _noalloc(lib, w, q, kc, vc, sl2, o2, lse2) == 0, lib.attn_last_error().decode()
    torch.cuda.synchronize()
    free1, alloc1 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    assert free1 == free0 and alloc1 == alloc0, (free0, free1, alloc0, alloc1)
    o2_ref, lse2_ref = _reference(w, q, kc, vc, sl2)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    assert torch.isfinite(o2).all()
    assert torch.equal(o2, o2_ref) and torch.equal(lse2, lse2_ref)
    if D == 128:
        _oracle_check(w, d, short_len, o2, lse2)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    lib = ea.load_library()
    w = si.Decode("small", 2, 8, 2, 64, 600, 1, 600, 0.125, 4, seed=33)
    d = si.decode_inputs(w)
    q, kc, vc = bits_to_dev(d["q_bits"]), bits_to_dev(d["k_bits"]), bits_to_dev(d["v_bits"])
    sl = torch.from_numpy(d["seqlens"]).cuda()
    o = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    # B * Hq * num_splits * (D + 1) * 4 bytes > 16 MiB
    big = si.Decode("too_big", 64, 64, 8, 64, 600, 1, 600, 0.125, 1024)
    assert lib.attn_decode_workspace_size(big.B, big.Hq, big.D, big.num_splits) > NOALLOC_BYTES
    assert _noalloc(lib, big, q, kc, vc, sl, o, lse) == 5
    assert b"built-in scratch" in lib.attn_last_error()
    # the same argument rules as attn_decode: a zero split count is an invalid argument for both
    bad = si.Decode("bad", 2, 8, 2, 64, 600, 1, 600, 0.125, 0)
    assert _noalloc(lib, bad, q, kc, vc, sl, o, lse) == 1
