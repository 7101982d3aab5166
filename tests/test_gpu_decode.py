"""Split-KV decode parity against the fp64 oracle (unsplit definition), for several split counts,
group sizes and head dims; cache rows past each sequence's length hold NaN and must not be read."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, bits_to_dev, compare, to_host_f64

pytestmark = pytest.mark.gpu


def run_decode(w: si.Decode, num_splits=None, seqlens=None, out_dtype=torch.float32):
    d = si.decode_inputs(w, seqlens=seqlens)
    q = bits_to_dev(d["q_bits"])
    kc = bits_to_dev(d["k_bits"])
    vc = bits_to_dev(d["v_bits"])
    sl = torch.from_numpy(d["seqlens"]).cuda()
    o, lse = ea.attn_decode(q, kc, vc, sl, w.scale, num_splits or w.num_splits, out_dtype=out_dtype)
    torch.cuda.synchronize()
    status = ea.read_device_status()
    og, lg = to_host_f64(o), to_host_f64(lse)
    o_ref = np.empty_like(og)
    l_ref = np.empty_like(lg)
    for b in range(w.B):
        L = int(min(max(d["seqlens"][b], 1), w.Smax))
        kf = si.bf16_bits_to_f32(d["k_bits"][b:b + 1, :L])
        vf = si.bf16_bits_to_f32(d["v_bits"][b:b + 1, :L])
        ob, lb = oracle.decode(d["q"][b:b + 1], kf, vf, np.array([L], np.int32), w.scale)
        o_ref[b], l_ref[b] = ob[0], lb[0]
    compare(og, o_ref, lg, l_ref, TOL_BF16_O, TOL_BF16_LSE, w.name)
    return status


def D(name, B, Hq, Hkv, Dh, Smax, lo, hi, ns, seed=5):
    return si.Decode(name, B, Hq, Hkv, Dh, Smax, lo, hi, 1.0 / np.sqrt(Dh), ns, seed=seed)


CASES = [
    D("gqa4_d64", 3, 8, 2, 64, 3000, 1, 3000, 8),
    D("gqa4_d64_many_splits", 4, 8, 2, 64, 5000, 1000, 5000, 64),
    D("mha_d64", 2, 4, 4, 64, 1500, 1, 1500, 4),
    D("gqa2_d128", 2, 4, 2, 128, 2100, 600, 2100, 16),
    D("gqa8_d64_two_blocks", 2, 16, 2, 64, 1200, 1, 1200, 4),
    D("gqa3_d64", 2, 6, 2, 64, 900, 1, 900, 2),
    D("mqa_d128", 2, 8, 1, 128, 1100, 1, 1100, 3),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_decode_matches_oracle(w):
    assert run_decode(w) == 0


def test_decode_bf16_output():
    w = D("bf16_out", 3, 8, 2, 64, 2000, 1, 2000, 8, seed=21)
    assert run_decode(w, out_dtype=torch.bfloat16) == 0


@pytest.mark.parametrize("ns", [1, 2, 3, 7, 64])
def test_any_split_count_matches_unsplit(ns):
    w = D("splits", 3, 8, 2, 64, 4100, 1, 4100, ns, seed=9)
    assert run_decode(w, num_splits=ns, seqlens=[1, 513, 4100]) == 0


def test_tiny_sequences_and_single_key():
    w = D("tiny", 4, 8, 2, 64, 40, 1, 40, 64, seed=11)
    assert run_decode(w, seqlens=[1, 2, 31, 40]) == 0


def test_out_of_range_lengths_are_clamped_and_flagged():
    # lengths 0 and Smax+5 are outside [1, Smax]: clamped to 1 and Smax, status bit 2 set
    w = D("clamp", 2, 4, 2, 64, 300, 1, 300, 4, seed=13)
    d = si.decode_inputs(w, fill_tail_nan=False)
    q, kc, vc = bits_to_dev(d["q_bits"]), bits_to_dev(d["k_bits"]), bits_to_dev(d["v_bits"])
    sl = torch.tensor([0, 305], dtype=torch.int32, device="cuda")
    o, lse = ea.attn_decode(q, kc, vc, sl, w.scale, 4)
    torch.cuda.synchronize()
    assert ea.read_device_status() & 2
    assert torch.isfinite(o.float()).all()
    assert ea.read_device_status() == 0      # the read clears the word


def test_decode_equals_last_row_of_causal_prefill():
    # cached decode == full forward (whisper-apr lfm2 gqa.rs test of cached vs full attention)
    w = D("cached_vs_full", 1, 8, 2, 64, 700, 700, 700, 4, seed=15)
    d = si.decode_inputs(w)
    L = 700
    q = bits_to_dev(d["q_bits"])
    kc, vc = bits_to_dev(d["k_bits"]), bits_to_dev(d["v_bits"])
    o, lse = ea.attn_decode(q, kc, vc, torch.tensor([L], dtype=torch.int32, device="cuda"), w.scale, 4)
    qf = torch.zeros((1, L, 8, 64), dtype=torch.bfloat16, device="cuda")
    qf[0, L - 1] = q[0]
    of, lf = ea.attn_fwd(qf, kc[:, :L].contiguous(), vc[:, :L].contiguous(), w.scale, True)
    torch.cuda.synchronize()
    assert (o[0].float() - of[0, L - 1].float()).abs().max().item() <= 1e-2
    assert (lse[0] - lf[0, :, L - 1]).abs().max().item() <= 1e-3
