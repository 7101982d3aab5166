"""Head dims other than 64 and 128 (zero-padded to the kernels' tile width inside the library):
forward and backward against the fp64 oracle at the true head dim, including D=36 (Moonshine's
head dim, whisper-apr lfm2 gqa.rs pad_head_dim_to) and RoPE, whose frequencies stay those of D."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, TOL_F32, bits_to_dev, compare, make_prefill, to_host_f64

pytestmark = pytest.mark.gpu

P = si.Prefill
FWD = [
    P("d36_moonshine_causal", "bf16", 2, 8, 8, 150, 150, 36, True, 1 / 6.0, seed=301),
    P("d36_rope_gqa", "bf16", 1, 8, 2, 130, 130, 36, True, 1 / 6.0, rope_base=10000.0, seed=302),
    P("d40_noncausal", "bf16", 1, 4, 4, 100, 90, 40, False, 0.158, seed=303),
    P("d96_rope_offset", "bf16", 1, 4, 2, 120, 200, 96, True, 0.102, rope_base=10000.0, q_pos0=80, seed=304),
    P("d112_mqa", "bf16", 2, 4, 1, 70, 140, 112, True, 0.0945, seed=305),
    P("d8_tiny", "bf16", 1, 2, 2, 40, 40, 8, True, 0.35, seed=306),
    P("d36_fp32", "fp32", 1, 2, 2, 90, 90, 36, True, 1 / 6.0, seed=307),
    P("d80_fp32_rope", "fp32", 1, 2, 1, 70, 100, 80, True, 0.11, rope_base=10000.0, q_pos0=30, seed=308),
]


@pytest.mark.parametrize("w", FWD, ids=lambda w: w.name)
def test_padded_forward_matches_oracle(w):
    x, dev = make_prefill(w)
    out_dtype = torch.float32
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                            out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    assert o.shape[-1] == w.D
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0)
    tol_o, tol_l = (TOL_F32, TOL_F32) if w.dtype == "fp32" else (TOL_BF16_O, TOL_BF16_LSE)
    compare(to_host_f64(o), ro, to_host_f64(lse), rl, tol_o, tol_l, w.name)


def test_padded_forward_bf16_output():
    w = FWD[0]
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, 0.0, 0)
    torch.cuda.synchronize()
    assert o.dtype == torch.bfloat16 and o.shape[-1] == 36
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
    compare(to_host_f64(o), ro, to_host_f64(lse), rl, TOL_BF16_O, TOL_BF16_LSE, "bf16 out")


@pytest.mark.parametrize("w", [FWD[1], FWD[3], FWD[6]], ids=lambda w: w.name)
def test_padded_backward_matches_oracle(w):
    x, dev = make_prefill(w)
    if w.dtype == "fp32":
        g = si.normal_f32(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))
        dout = torch.from_numpy(g).cuda()
        tol = 2e-5
    else:
        gb, g = si.bf16_normal(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))
        dout = bits_to_dev(gb)
        tol = 1e-2
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0)
    o = torch.from_numpy(ro.astype(np.float32)).cuda().to(dev["q"].dtype)
    lse = torch.from_numpy(rl.astype(np.float32)).cuda()
    dq, dk, dv = ea.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, dout, w.scale, w.causal, w.rope_base, w.q_pos0,
                             grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], g, w.scale, w.causal, w.rope_base, w.q_pos0)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        gh = got.cpu().numpy().astype(np.float64)
        err = float(np.max(np.abs(gh - ref)) / max(1.0, float(np.max(np.abs(ref)))))
        assert err <= tol, (w.name, name, err)


def test_odd_head_dim_and_plain_attn_fwd_are_rejected():
    lib = ea.load_library()
    w = P("d37", "bf16", 1, 2, 2, 16, 16, 38, True, 0.2, seed=309)
    x, dev = make_prefill(w)
    o = torch.empty_like(dev["q"])
    # attn_fwd has no workspace: padded dims are refused with a clear status
    import ctypes
    st = lib.attn_fwd(ctypes.c_void_p(dev["q"].data_ptr()), ctypes.c_void_p(dev["k"].data_ptr()),
                      ctypes.c_void_p(dev["v"].data_ptr()), ctypes.c_void_p(o.data_ptr()), None, 1, 2, 2, 16, 16, 38,
                      0.2, 1, 0, None)
    assert st == 4 and b"workspace" in lib.attn_last_error()
    assert lib.attn_fwd_ex_workspace_size(1, 2, 2, 16, 16, 37, 0, 0.0, 0) == 0      # odd: unsupported
