"""attn_decode_noalloc: the decode entry point for callers that cannot allocate device memory
(code inside a host framework that owns all device allocations, or a latency-bound serving path
that must not call cudaMalloc).  It keeps the split partials in scratch memory the library owns.

Called here through the C ABI and compared with attn_decode (caller workspace) on two calls in a
row with different inputs, so the second call also shows that what the first left in the shared
scratch does not leak into its result.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, bits_to_dev

pytestmark = pytest.mark.gpu


def _inputs(seed, B=4, Hq=32, Hkv=8, D=64, Smax=6000, ns=16):
    w = si.Decode("noalloc", B, Hq, Hkv, D, Smax, 1, Smax, 1.0 / np.sqrt(D), ns, seed=seed)
    d = si.decode_inputs(w)
    return w, (bits_to_dev(d["q_bits"]), bits_to_dev(d["k_bits"]), bits_to_dev(d["v_bits"]),
               torch.from_numpy(d["seqlens"]).cuda())


def _noalloc(lib, w, q, kc, vc, sl, o, lse):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.attn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
                                   ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(sl.data_ptr()),
                                   ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                                   w.B, w.Hq, w.Hkv, w.Smax, w.D, w.scale, w.num_splits,
                                   ea.ATTN_BF16_OUT_F32, stream)


def test_noalloc_decode_matches_workspace_decode_twice():
    lib = ea.load_library()
    for seed, D in ((31, 64), (32, 128)):
        w, (q, kc, vc, sl) = _inputs(seed, D=D)
        o = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        st = _noalloc(lib, w, q, kc, vc, sl, o, lse)
        assert st == 0, lib.attn_last_error().decode()
        o_ref, lse_ref = ea.attn_decode(q, kc, vc, sl, w.scale, w.num_splits, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert ea.read_device_status() == 0
        assert torch.isfinite(o).all()
        assert (o - o_ref).abs().max().item() <= TOL_BF16_O
        assert (lse - lse_ref).abs().max().item() <= TOL_BF16_LSE


def test_noalloc_rejects_problems_larger_than_its_scratch():
    lib = ea.load_library()
    w, (q, kc, vc, sl) = _inputs(33, B=2, Hq=8, Hkv=2, Smax=600, ns=4)
    o = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    # B * Hq * num_splits * (D + 1) * 4 bytes > 16 MiB
    big = si.Decode("too_big", 64, 64, 8, 64, 600, 1, 600, 0.125, 1024)
    assert lib.attn_decode_workspace_size(big.B, big.Hq, big.D, big.num_splits) > (16 << 20)
    st = _noalloc(lib, big, q, kc, vc, sl, o, lse)
    assert st == 5
    assert b"built-in scratch" in lib.attn_last_error()
