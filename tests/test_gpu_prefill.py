"""Prefill parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element,
on seeded inputs that span several tiles with ragged tails, plus the method's edge cases."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, TOL_F32, compare, make_prefill, to_host_f64

pytestmark = pytest.mark.gpu


def run_case(w: si.Prefill, want_lse=True, out_dtype=torch.float32):
    """bf16 problems take O in fp32 (bf16 storage alone has a 2^-6 spacing at |O| >= 2)."""
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                            want_lse=want_lse, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0)
    tol_o, tol_l = (TOL_F32, TOL_F32) if w.dtype == "fp32" else (TOL_BF16_O, TOL_BF16_LSE)
    return compare(to_host_f64(o), o_ref, None if lse is None else to_host_f64(lse), lse_ref, tol_o, tol_l,
                   w.name)


def P(name, dtype, B, Hq, Hkv, Sq, Skv, D, causal, **kw):
    scale = kw.pop("scale", 1.0 / np.sqrt(D))
    return si.Prefill(name, dtype, B, Hq, Hkv, Sq, Skv, D, causal, scale, seed=kw.pop("seed", 77), **kw)


BF16_CASES = [
    P("one_tile_mha", "bf16", 1, 1, 1, 128, 128, 64, False),
    P("ragged_causal_mha", "bf16", 2, 2, 2, 300, 300, 64, True),
    P("ragged_noncausal", "bf16", 1, 3, 3, 200, 333, 64, False),
    P("gqa4_causal_pairs_heads", "bf16", 1, 8, 2, 384, 384, 64, True),
    P("gqa3_odd_group", "bf16", 1, 6, 2, 260, 260, 64, True),
    P("mqa", "bf16", 2, 4, 1, 130, 130, 64, True),
    P("chunked_prefill_sq_lt_skv", "bf16", 1, 4, 2, 100, 333, 64, True),
    P("sq_gt_skv_masked_rows", "bf16", 1, 2, 2, 300, 130, 64, True),
    P("single_key", "bf16", 1, 2, 2, 5, 1, 64, False),
    P("single_row", "bf16", 1, 2, 1, 1, 77, 64, True),
    P("d128_causal", "bf16", 1, 2, 2, 257, 257, 128, True),
    P("d128_gqa_noncausal", "bf16", 1, 4, 2, 130, 200, 128, False),
    P("d128_peaked_scores", "bf16", 1, 2, 2, 600, 600, 128, True, qk_std=3.0),
    P("d64_peaked_scores", "bf16", 1, 2, 2, 520, 520, 64, True, qk_std=3.0),
    P("long_rows_many_tiles", "bf16", 1, 1, 1, 1100, 1100, 64, True),
    P("rope_gqa_causal", "bf16", 1, 8, 2, 300, 300, 64, True, rope_base=10000.0),
    P("rope_mha_chunked", "bf16", 1, 2, 2, 90, 400, 64, True, rope_base=10000.0, q_pos0=310),
    P("rope_d128", "bf16", 1, 2, 2, 140, 140, 128, True, rope_base=500000.0),
    # Whisper encoder self-attention shape (whisper-apr attention_generated.rs: 1500 frames,
    # 6 heads of 64, non-causal)
    P("whisper_encoder_s1500_h6", "bf16", 1, 6, 6, 1500, 1500, 64, False),
]

F32_CASES = [
    P("c1_shape", "fp32", 1, 1, 1, 128, 128, 64, False, scale=1.0 / 8.0, seed=1001),
    P("f32_ragged_causal_gqa", "fp32", 2, 4, 2, 150, 150, 64, True),
    P("f32_chunked", "fp32", 1, 2, 1, 70, 200, 128, True),
    P("f32_masked_rows", "fp32", 1, 1, 1, 100, 30, 64, True),
    P("f32_rope", "fp32", 1, 4, 2, 140, 140, 64, True, rope_base=10000.0),
]


@pytest.mark.parametrize("w", BF16_CASES, ids=[c.name for c in BF16_CASES])
def test_bf16_prefill_matches_oracle(w):
    run_case(w)


@pytest.mark.parametrize("w", F32_CASES, ids=[c.name for c in F32_CASES])
def test_fp32_prefill_matches_oracle(w):
    run_case(w)


def test_config1_exact_workload():
    w = si.C1
    err_o, err_l = run_case(w)
    assert err_o <= TOL_F32 and err_l <= TOL_F32


BF16_OUT_CASES = [c for c in BF16_CASES if "peaked" not in c.name and "rope" not in c.name][:6]


@pytest.mark.parametrize("w", BF16_OUT_CASES, ids=[c.name for c in BF16_OUT_CASES])
def test_bf16_output_matches_oracle(w):
    # O stored as bf16: the same kernel with the bf16 epilogue (unit-variance scores)
    run_case(w, out_dtype=torch.bfloat16)


def test_lse_pointer_may_be_null():
    w = P("no_lse", "bf16", 1, 2, 2, 200, 200, 64, True)
    run_case(w, want_lse=False)


def test_gqa_equals_repeated_kv_on_gpu():
    w = P("gqa_rep", "bf16", 1, 8, 2, 256, 256, 64, True)
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd(dev["q"], dev["k"], dev["v"], w.scale, True)
    kr = dev["k"].repeat_interleave(4, dim=2).contiguous()
    vr = dev["v"].repeat_interleave(4, dim=2).contiguous()
    o2, lse2 = ea.attn_fwd(dev["q"], kr, vr, w.scale, True)
    torch.cuda.synchronize()
    # same math on the same bytes: MHA with repeated heads pairs rows, GQA pairs heads
    assert torch.allclose(o.float(), o2.float(), atol=1e-2)
    assert torch.allclose(lse, lse2, atol=1e-4)


def test_outputs_do_not_touch_neighbouring_memory():
    w = P("guard", "bf16", 1, 2, 2, 200, 200, 64, True)
    x, dev = make_prefill(w)
    n = w.B * w.Sq * w.Hq * w.D
    buf = torch.full((n + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    o = buf[:n].view(w.B, w.Sq, w.Hq, w.D)
    lbuf = torch.full((w.B * w.Hq * w.Sq + 1024,), 5.0, dtype=torch.float32, device="cuda")
    lse = lbuf[: w.B * w.Hq * w.Sq].view(w.B, w.Hq, w.Sq)
    ea.attn_fwd(dev["q"], dev["k"], dev["v"], w.scale, True, o=o, lse=lse)
    torch.cuda.synchronize()
    assert (buf[n:] == 7.0).all()
    assert (lbuf[w.B * w.Hq * w.Sq:] == 5.0).all()


def test_repeated_calls_are_deterministic():
    w = P("det", "bf16", 1, 4, 2, 333, 333, 64, True)
    x, dev = make_prefill(w)
    o1, l1 = ea.attn_fwd(dev["q"], dev["k"], dev["v"], w.scale, True)
    o2, l2 = ea.attn_fwd(dev["q"], dev["k"], dev["v"], w.scale, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# Problems whose single query tiles would exceed 148 CTAs run two query tiles per CTA; smaller
# ones one tile per CTA.  The cases below are sized to stay in the paired decomposition (row pairs of one head for
# odd groups, head pairs for even groups) while keeping ragged tails, offsets and RoPE.
PAIRED_CASES = [
    P("paired_rows_odd_group_ragged", "bf16", 4, 40, 8, 300, 300, 64, True, seed=91),       # 2 x 4 x 40 = 320 pairs
    P("paired_heads_gqa8_rope_offset", "bf16", 5, 32, 4, 200, 330, 64, True, rope_base=10000.0, q_pos0=130,
      seed=92),                                                                              # 2 x 5 x 16 = 160
    P("paired_heads_d128_noncausal", "bf16", 3, 64, 32, 130, 150, 128, False, seed=93),   # 2 x 3 x 32 = 192
]


@pytest.mark.parametrize("w", PAIRED_CASES, ids=[c.name for c in PAIRED_CASES])
def test_paired_decomposition_matches_oracle(w):
    """Sampled rows of every (batch, head) plus tile edges, against the oracle."""
    from attn_cases import gather_rows, sample_rows
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    rows = sample_rows(w, 1500, seed=5)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0, rows=rows)
    go, gl = gather_rows(to_host_f64(o), to_host_f64(lse), rows, w)
    compare(go, ro, gl, rl, TOL_BF16_O, TOL_BF16_LSE, w.name)
