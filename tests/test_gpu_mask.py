"""attn_fwd_masked (additive mask on the scaled scores) against the fp64 oracle: shared, per-batch
and per-head masks, -inf key padding, rows masked everywhere, RoPE, D=128, fp32 and a padded
head dim."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, TOL_F32, compare, make_prefill, to_host_f64

pytestmark = pytest.mark.gpu

P = si.Prefill
CASES = [
    (P("shared_causal", "bf16", 2, 4, 4, 200, 200, 64, True, 0.125, seed=401), "shared"),
    (P("per_head_gqa", "bf16", 1, 8, 2, 150, 260, 64, False, 0.125, seed=402), "per_head"),
    (P("key_padding", "bf16", 3, 4, 4, 130, 170, 64, False, 0.125, seed=403), "key_padding"),
    (P("rope_d128", "bf16", 1, 4, 2, 140, 140, 128, True, 0.0884, rope_base=10000.0, seed=404), "shared"),
    # D=64 with RoPE: P in TMEM columns of its own, two MMA issuers, exponentiation turns
    (P("rope_d64_gqa_per_head", "bf16", 1, 8, 2, 300, 420, 64, True, 0.125, rope_base=10000.0, seed=408), "per_head"),
    (P("rows_all_inf", "bf16", 1, 2, 2, 90, 90, 64, False, 0.125, seed=405), "dead_rows"),
    (P("fp32_shared", "fp32", 1, 2, 2, 100, 120, 64, True, 0.125, seed=406), "shared"),
    (P("padded_d40", "bf16", 1, 4, 4, 110, 110, 40, True, 0.158, seed=407), "per_batch"),
    # more query tiles than SMs: two query tiles per CTA (row tiles of one head, or two heads of a
    # GQA pair), the mask boxes loaded by TMA (Skv a multiple of 4)
    (P("two_tile_shared_causal", "bf16", 2, 8, 8, 1300, 1300, 64, True, 0.125, seed=409), "shared"),
    (P("two_tile_per_head_gqa", "bf16", 1, 16, 8, 1200, 1240, 64, False, 0.125, seed=410), "per_head"),
]


def _mask(kind, w):
    rng = np.random.default_rng(w.seed)
    if kind == "shared":
        return rng.standard_normal((w.Sq, w.Skv)).astype(np.float32)
    if kind == "per_batch":
        return rng.standard_normal((w.B, w.Sq, w.Skv)).astype(np.float32)
    if kind == "per_head":
        return rng.standard_normal((w.B, w.Hq, w.Sq, w.Skv)).astype(np.float32)
    if kind == "key_padding":
        m = np.zeros((w.B, w.Sq, w.Skv), np.float32)
        for b in range(w.B):
            m[b, :, w.Skv - 17 * (b + 1):] = -np.inf      # the last keys of each sequence are padding
        return m
    if kind == "dead_rows":
        m = rng.standard_normal((w.Sq, w.Skv)).astype(np.float32)
        m[[0, 5, 64, 89], :] = -np.inf
        return m
    raise ValueError(kind)


@pytest.mark.parametrize("w,kind", CASES, ids=lambda c: c.name if hasattr(c, "name") else c)
def test_masked_forward_matches_oracle(w, kind):
    x, dev = make_prefill(w)
    m = _mask(kind, w)
    o, lse = ea.attn_fwd_masked(dev["q"], dev["k"], dev["v"], torch.from_numpy(m).cuda(), w.scale, w.causal,
                                w.rope_base, w.q_pos0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    ro, rl = oracle.attn_fwd_masked(x["q"], x["k"], x["v"], m, w.scale, w.causal, w.rope_base, w.q_pos0)
    tol_o, tol_l = (TOL_F32, TOL_F32) if w.dtype == "fp32" else (TOL_BF16_O, TOL_BF16_LSE)
    og, lg = to_host_f64(o), to_host_f64(lse)
    if kind == "dead_rows":
        assert np.all(og[:, [0, 5, 64, 89]] == 0.0) and np.all(lg[:, :, [0, 5, 64, 89]] == -np.inf)
    compare(og, ro, lg, rl, tol_o, tol_l, w.name)


def test_expanded_head_broadcast_mask():
    """A [B, 1, Sq, Skv] mask expanded over the heads (head stride 0) equals the per-batch mask."""
    w = P("expand", "bf16", 2, 4, 4, 96, 96, 64, True, 0.125, seed=408)
    x, dev = make_prefill(w)
    m = np.random.default_rng(3).standard_normal((w.B, 1, w.Sq, w.Skv)).astype(np.float32)
    md = torch.from_numpy(m).cuda().expand(w.B, w.Hq, w.Sq, w.Skv)
    o, lse = ea.attn_fwd_masked(dev["q"], dev["k"], dev["v"], md, w.scale, w.causal, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd_masked(x["q"], x["k"], x["v"], m[:, 0], w.scale, w.causal)
    compare(to_host_f64(o), ro, to_host_f64(lse), rl, TOL_BF16_O, TOL_BF16_LSE, "expanded mask")


BWD_CASES = [CASES[0], CASES[1], CASES[2], CASES[4], CASES[5], CASES[6]]


@pytest.mark.parametrize("w,kind", BWD_CASES, ids=lambda c: c.name if hasattr(c, "name") else c)
def test_masked_backward_matches_oracle(w, kind):
    """attn_bwd_masked with o and lse of the oracle's masked forward (bf16: 1e-2, fp32: 2e-5 of the
    largest reference gradient, as in tests/test_gpu_backward.py)."""
    x, dev = make_prefill(w)
    m = _mask(kind, w)
    if w.dtype == "fp32":
        g = si.normal_f32(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))
        dout = torch.from_numpy(g).cuda()
        tol = 2e-5
    else:
        gb, g = si.bf16_normal(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))
        dout = torch.from_numpy(np.ascontiguousarray(gb).view(np.int16)).view(torch.bfloat16).cuda()
        tol = 1e-2
    ro, rl = oracle.attn_fwd_masked(x["q"], x["k"], x["v"], m, w.scale, w.causal, w.rope_base, w.q_pos0)
    o = torch.from_numpy(ro.astype(np.float32)).cuda().to(dev["q"].dtype)
    lse = torch.from_numpy(rl.astype(np.float32)).cuda()
    dq, dk, dv = ea.attn_bwd_masked(dev["q"], dev["k"], dev["v"], torch.from_numpy(m).cuda(), o, lse, dout, w.scale,
                                    w.causal, w.rope_base, w.q_pos0, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    rq, rk, rv = oracle.attn_bwd_masked(x["q"], x["k"], x["v"], g, m, w.scale, w.causal, w.rope_base, w.q_pos0)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        gh = got.cpu().numpy().astype(np.float64)
        assert np.isfinite(gh).all(), name
        err = float(np.max(np.abs(gh - ref)) / max(1.0, float(np.max(np.abs(ref)))))
        assert err <= tol, (w.name, name, err)
