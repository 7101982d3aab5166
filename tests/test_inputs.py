"""The seeded input generator: determinism, bf16 rounding, workload shapes (CPU only)."""
import numpy as np
import torch

import seeded_inputs as si


def test_bf16_rounding_matches_torch():
    x = np.concatenate([si.normal_f32(1, 0, (100000,), 3.0),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.4e38, -1e-40,
                                  np.inf, -np.inf], dtype=np.float32)])
    bits = si.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (bits == ref).all()
    back = si.bf16_bits_to_f32(bits)
    assert (back == torch.from_numpy(x).to(torch.bfloat16).float().numpy()).all()
    assert si.f32_to_bf16_bits(np.array([np.nan], np.float32))[0] == si.BF16_NAN_BITS


def test_streams_deterministic_and_independent():
    a = si.normal_f32(5, 0, (64,))
    assert (a == si.normal_f32(5, 0, (64,))).all()
    assert not (a == si.normal_f32(5, 1, (64,))).all()
    assert not (a == si.normal_f32(6, 0, (64,))).all()


def test_workload_shapes_and_counts():
    c2 = si.C2
    assert c2.unmasked_pairs == 2048 * 2049 // 2
    assert abs(c2.flops - 17.19e9) / 17.19e9 < 1e-3
    assert abs(si.C3.flops - 137.47e9) / 137.47e9 < 1e-3
    assert abs(si.C5.flops - 1099.6e9) / 1099.6e9 < 1e-3
    assert si.C1.flops == 4 * 64 * 128 * 128
    sl = si.C4.seqlens()
    assert sl.shape == (16,) and sl.min() >= 1024 and sl.max() <= 32768
    assert (sl == si.C4.seqlens()).all()


def test_decode_inputs_tail_is_nan():
    w = si.Decode("tiny", 2, 4, 2, 8, 16, 3, 9, 0.3, 4, seed=77)
    d = si.decode_inputs(w)
    for b in range(2):
        L = int(d["seqlens"][b])
        assert (d["k_bits"][b, L:] == si.BF16_NAN_BITS).all()
        assert not np.isnan(si.bf16_bits_to_f32(d["k_bits"][b, :L])).any()
