"""Parity at the full workload sizes, in the launch configuration bench.py times (bf16 inputs,
fp32 accumulation, O taken in fp32): sampled rows against the fp64 oracle, plus properties that
hold for every row (finite outputs; query row 0 sees exactly key 0 in a causal problem)."""
import math

import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import (TOL_BF16_LSE, TOL_BF16_O, bits_to_dev, compare, gather_rows, make_prefill,
                        sample_rows, to_host_f64)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [si.C2, si.C3, si.C5], ids=lambda w: w.name)
def test_full_size_prefill(w):
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    og, lg = to_host_f64(o), to_host_f64(lse)
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    rows = sample_rows(w, 300 if w.D == 128 else 600, seed=1)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0, rows=rows)
    go, gl = gather_rows(og, lg, rows, w)
    compare(go, ro, gl, rl, TOL_BF16_O, TOL_BF16_LSE, w.name)
    # every (batch, head): causal row 0 attends to key 0 only -> O = v0, LSE = its score
    g = w.Hq // w.Hkv
    v0 = x["v"][:, 0].astype(np.float64)                                   # [B, Hkv, D]
    assert np.max(np.abs(og[:, 0] - np.repeat(v0, g, axis=1))) <= TOL_BF16_O
    q0 = x["q"][:, 0].astype(np.float64)
    k0 = np.repeat(x["k"][:, 0].astype(np.float64), g, axis=1)
    s0 = w.scale * np.sum(q0 * k0, axis=-1)                                # RoPE at position 0 is the identity
    assert np.max(np.abs(lg[:, :, 0] - s0)) <= TOL_BF16_LSE


@pytest.mark.parametrize("w", [si.F2_WHISPER, si.F2_CHUNK], ids=lambda w: w.name)
def test_full_size_f2_prefill(w):
    """Whisper-encoder shape (non-causal) and chunked prefill (Sq < Skv, bottom-right causal,
    RoPE at the cache offset): sampled rows against the oracle, every output finite."""
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    og, lg = to_host_f64(o), to_host_f64(lse)
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    rows = sample_rows(w, 400, seed=2)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0, rows=rows)
    go, gl = gather_rows(og, lg, rows, w)
    compare(go, ro, gl, rl, TOL_BF16_O, TOL_BF16_LSE, w.name)


def test_full_size_decode():
    w = si.C4
    d = si.decode_inputs(w)      # rows past each length hold NaN
    q, kc, vc = bits_to_dev(d["q_bits"]), bits_to_dev(d["k_bits"]), bits_to_dev(d["v_bits"])
    sl = torch.from_numpy(d["seqlens"]).cuda()
    o, lse = ea.attn_decode(q, kc, vc, sl, w.scale, w.num_splits, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    og, lg = to_host_f64(o), to_host_f64(lse)
    del kc, vc
    o_ref = np.empty_like(og)
    l_ref = np.empty_like(lg)
    for b in range(w.B):
        L = int(d["seqlens"][b])
        ob, lb = oracle.decode(d["q"][b:b + 1], si.bf16_bits_to_f32(d["k_bits"][b:b + 1, :L]),
                               si.bf16_bits_to_f32(d["v_bits"][b:b + 1, :L]), np.array([L], np.int32),
                               w.scale)
        o_ref[b], l_ref[b] = ob[0], lb[0]
    compare(og, o_ref, lg, l_ref, TOL_BF16_O, TOL_BF16_LSE, w.name)
