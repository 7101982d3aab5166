"""attn_bwd against the fp64 oracle backward (gradients by definition, pinned by finite
differences of the forward oracle).

Tolerances, as a fraction of the largest reference gradient of each tensor:
  * fp32 inputs, o and lse exact to fp32: 2e-5 (fp32 accumulation over <= a few thousand keys);
  * bf16 inputs (tensor-core products): o is stored in bf16, so D_i = dout . o carries o's
    rounding (2^-9 relative per element) into every dS of the row, and P and dS are rounded to
    bf16 as MMA operands: 1e-2;
  * the whole chain (the library's bf16 forward, then its backward): 2e-2.
"""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import bits_to_dev

pytestmark = pytest.mark.gpu


def _rel_err(got, ref):
    return float(np.max(np.abs(got - ref)) / max(1.0, float(np.max(np.abs(ref)))))


def _inputs(w, seed_g=7):
    x = si.prefill_inputs(w)
    if w.dtype == "fp32":
        g = si.normal_f32(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))
        gb = None
    else:
        gb, g = si.bf16_normal(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))
    return x, g, gb


def _dev(x, name, w):
    if w.dtype == "fp32":
        return torch.from_numpy(np.ascontiguousarray(x[name])).cuda()
    return bits_to_dev(x[name + "_bits"])


P = si.Prefill
CASES = [
    P("mha_causal_ragged", "fp32", 1, 2, 2, 130, 130, 64, True, 0.125, seed=201),
    P("gqa_bottom_right", "fp32", 2, 8, 2, 200, 260, 64, True, 0.125, seed=202),
    P("rope_offset_d128", "fp32", 1, 4, 2, 100, 150, 128, True, 0.0884, rope_base=10000.0, q_pos0=50, seed=203),
    P("noncausal_mqa", "fp32", 1, 4, 1, 90, 70, 64, False, 0.125, seed=204),
    P("masked_rows", "fp32", 1, 2, 2, 150, 100, 64, True, 0.125, seed=205),
    P("bf16_gqa_rope", "bf16", 1, 8, 2, 160, 160, 64, True, 0.125, rope_base=10000.0, seed=206),
    P("bf16_d128", "bf16", 2, 2, 2, 140, 140, 128, True, 0.0884, seed=207),
    P("bf16_d128_rope_offset_gqa", "bf16", 1, 4, 2, 100, 170, 128, True, 0.0884, rope_base=500000.0, q_pos0=70,
      seed=209),
    P("bf16_noncausal_masked_mqa", "bf16", 2, 4, 1, 77, 200, 64, False, 0.125, seed=210),
    P("bf16_causal_sq_gt_skv", "bf16", 1, 2, 2, 150, 90, 64, True, 0.125, seed=211),
    # shapes the tcgen05 backward takes (unmasked, Sq a multiple of 4): rows with no visible key,
    # several key and query tiles with ragged ends, MQA, GQA at D=128 with RoPE
    P("tc_bf16_sq_gt_skv", "bf16", 1, 2, 2, 300, 170, 64, True, 0.125, seed=212),
    P("tc_bf16_noncausal_mqa", "bf16", 2, 4, 1, 260, 330, 64, False, 0.125, seed=213),
    P("tc_bf16_d128_gqa_rope", "bf16", 1, 8, 2, 384, 384, 128, True, 0.0884, rope_base=10000.0, seed=214),
    P("tc_bf16_d64_bottom_right", "bf16", 2, 6, 3, 196, 452, 64, True, 0.125, seed=215),
    # D=64 with RoPE over several query and key tiles: the overlapped dq (dS double buffer) and
    # dk/dv (P^T, dS^T buffers of their own) pipelines run many iterations per CTA
    P("tc_bf16_d64_gqa_rope_multi_tile", "bf16", 1, 8, 2, 520, 520, 64, True, 0.125, rope_base=10000.0, seed=216),
    P("tc_bf16_d64_noncausal_ragged", "bf16", 1, 4, 4, 388, 611, 64, False, 0.125, seed=217),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(w):
    x, g, gb = _inputs(w)
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0)
    dq_r, dk_r, dv_r = oracle.attn_bwd(x["q"], x["k"], x["v"], g, w.scale, w.causal, w.rope_base, w.q_pos0)
    q, k, v = (_dev(x, n, w) for n in ("q", "k", "v"))
    lse = torch.from_numpy(lse_ref.astype(np.float32)).cuda()
    if w.dtype == "fp32":
        o = torch.from_numpy(o_ref.astype(np.float32)).cuda()
        dout = torch.from_numpy(g).cuda()
        tol = 2e-5
    else:
        o = torch.from_numpy(o_ref.astype(np.float32)).cuda().to(torch.bfloat16)
        dout = bits_to_dev(gb)
        tol = 1e-2
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, dout, w.scale, w.causal, w.rope_base, w.q_pos0,
                             grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    for name, got, ref in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        gh = got.cpu().numpy().astype(np.float64)
        assert np.isfinite(gh).all(), name
        err = _rel_err(gh, ref)
        assert err <= tol, (w.name, name, err)


def test_backward_after_library_forward_and_bf16_gradients():
    """The chain a training step runs: the library's bf16 forward (o, lse), then its backward, with
    gradients taken in bf16 and in fp32."""
    w = P("chain", "bf16", 2, 8, 4, 256, 256, 64, True, 0.125, rope_base=10000.0, seed=208)
    x, g, gb = _inputs(w)
    q, k, v = (_dev(x, n, w) for n in ("q", "k", "v"))
    o, lse = ea.attn_fwd_ex(q, k, v, w.scale, w.causal, w.rope_base, w.q_pos0)     # bf16 o
    dout = bits_to_dev(gb)
    dq_r, dk_r, dv_r = oracle.attn_bwd(x["q"], x["k"], x["v"], g, w.scale, w.causal, w.rope_base, w.q_pos0)
    for gd in (torch.float32, torch.bfloat16):
        dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, dout, w.scale, w.causal, w.rope_base, w.q_pos0, grad_dtype=gd)
        torch.cuda.synchronize()
        assert ea.read_device_status() == 0
        for name, got, ref in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
            err = _rel_err(got.float().cpu().numpy().astype(np.float64), ref)
            assert err <= 2e-2, (str(gd), name, err)


def test_backward_full_size_c2():
    """C2 (B=4, H=8, S=2048, D=64, causal) in the configuration bench.py times: bf16 inputs, the
    library's forward, fp32 gradients; against the oracle backward on every element."""
    w = si.C2
    x, g, gb = _inputs(w)
    q, k, v = (_dev(x, n, w) for n in ("q", "k", "v"))
    o, lse = ea.attn_fwd(q, k, v, w.scale, w.causal)
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, bits_to_dev(gb), w.scale, w.causal, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    dq_r, dk_r, dv_r = oracle.attn_bwd(x["q"], x["k"], x["v"], g, w.scale, w.causal)
    for name, got, ref in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        err = _rel_err(got.cpu().numpy().astype(np.float64), ref)
        assert err <= 2e-2, (name, err)


@pytest.mark.parametrize("w", [si.C3, si.C5], ids=["c3_gqa_rope", "c5_d128_peaked"])
def test_backward_full_size_sampled(w):
    """Full-size GQA 32/8 causal with RoPE (B2 S4096 D64) and long-context D=128 with peaked scores
    (B1 H16 S16384): the library's bf16 forward and its backward with fp32 gradients, in the
    configuration bench.py times, against the oracle's exact backward of two (batch, kv head)
    groups at sampled query rows (first, tile edges, last, random) and keys -- every q head of
    the group at those rows."""
    x, g, gb = _inputs(w)
    q, k, v = (_dev(x, n, w) for n in ("q", "k", "v"))
    ws = None
    if w.rope_base > 0:
        ws = torch.empty(ea.fwd_workspace_bytes(q, k, w.rope_base, w.q_pos0), dtype=torch.uint8, device="cuda")
    o, lse = ea.attn_fwd_ex(q, k, v, w.scale, w.causal, w.rope_base, w.q_pos0, workspace=ws)
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, bits_to_dev(gb), w.scale, w.causal, w.rope_base, w.q_pos0,
                             grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    dq, dk, dv = (t.cpu().numpy().astype(np.float64) for t in (dq, dk, dv))
    rng = np.random.default_rng(w.seed)
    G = w.Hq // w.Hkv
    for b, kvh in ((0, 0), (w.B - 1, w.Hkv - 1)):
        rows = np.unique(np.concatenate([[0, 1, 127, 128, w.Sq // 2, w.Sq - 1], rng.integers(0, w.Sq, 6)]))
        keys = np.unique(np.concatenate([[0, 1, 127, 128, w.Skv // 2, w.Skv - 1], rng.integers(0, w.Skv, 6)]))
        rq, rk, rv = oracle.attn_bwd_sampled(x["q"], x["k"], x["v"], g, w.scale, w.causal, w.rope_base, w.q_pos0,
                                             b, kvh, rows, keys)
        for hg in range(G):
            err = _rel_err(dq[b, rows, kvh * G + hg], rq[hg])
            assert err <= 1e-2, ("dq", b, kvh * G + hg, err)
        assert _rel_err(dk[b, keys, kvh], rk) <= 1e-2, ("dk", b, kvh)
        assert _rel_err(dv[b, keys, kvh], rv) <= 1e-2, ("dv", b, kvh)
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()


def test_backward_rejects_bad_workspace():
    w = CASES[0]
    x, g, _ = _inputs(w)
    q, k, v = (_dev(x, n, w) for n in ("q", "k", "v"))
    o = torch.zeros_like(q)
    lse = torch.zeros((w.B, w.Hq, w.Sq), device="cuda")
    with pytest.raises(ea.AttnError):
        ea.attn_bwd(q, k, v, o, lse, o, w.scale, w.causal, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
