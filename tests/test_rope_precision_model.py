"""CPU error model of the tensor-core operand precision for attention with RoPE.

RoPE (scirs2-neural 0.4.4 grouped_query_attention.rs, RotaryPositionEmbedding::apply) rotates q
and k in double; the rotated values are no longer bf16 numbers, so the tensor-core forward has to
choose how to feed them to a bf16/fp16/tf32 MMA.  This model takes GQA-prefill-shaped data (D=64,
keys at positions 0..4095, queries at random positions, bf16 N(0,1) inputs, causal rows, scale
1/8), rotates in double, and compares the logsumexp of each row against the exact one for every
operand scheme the kernel could use:

  bf16 single                   one MMA, rotated q and k rounded to bf16
  fp16 single / tf32 single     one MMA (tf32: at half the bf16 rate), 11-bit significands
  bf16 hi/lo, 3 chains          q = qh + ql, k = kh + kl (bf16 each): qh.kh + qh.kl + ql.kh
  bf16 hi/lo, 2 chains          either cross term dropped

The kernel uses the 3-chain scheme.  The assertions pin why: a single bf16 product, and either
2-chain form, exceed the 1e-3 LSE tolerance on this data; the 3-chain form stays three orders of
magnitude below it.  fp16 and tf32 single products pass here, but their error grows with |q| |k|
(inputs of a few times unit scale exceed 1e-3 -- checked below), and fp16 overflows past 65504.
"""
import numpy as np
import pytest

D, S, BASE, SCALE, NQ = 64, 4096, 10000.0, 1.0 / 8.0, 256


def _round_bits(x, drop):
    """Round float32 values to nearest-even, keeping 23 - drop significand bits."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    half = (1 << (drop - 1)) - 1
    b = ((b + half + ((b >> drop) & 1)) >> drop) << drop
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def bf16(x):
    return _round_bits(x, 16)


def tf32(x):
    return _round_bits(x, 13)


def f16(x):
    return np.asarray(x, np.float16).astype(np.float64)


def rope(x, pos):
    i = np.arange(D // 2)
    th = pos[:, None] / BASE ** (2 * i / D)
    c, s = np.cos(th), np.sin(th)
    y = np.empty_like(x)
    y[:, 0::2] = x[:, 0::2] * c - x[:, 1::2] * s
    y[:, 1::2] = x[:, 0::2] * s + x[:, 1::2] * c
    return y


def lse_rows(sc):
    m = sc.max(1, keepdims=True)
    return m[:, 0] + np.log(np.exp(sc - m).sum(1))


def errors(std=1.0, seed=5):
    rng = np.random.default_rng(seed)
    q = bf16(std * rng.standard_normal((NQ, D)))
    k = bf16(std * rng.standard_normal((S, D)))
    qpos = rng.integers(0, S, NQ).astype(np.float64)
    qr, kr = rope(q, qpos), rope(k, np.arange(S, dtype=np.float64))
    # the kernel rotates in fp32 (double angles, fp32 table and arithmetic), then splits
    qr32, kr32 = (np.asarray(a, np.float32).astype(np.float64) for a in (qr, kr))
    masked = np.arange(S)[None, :] > qpos[:, None]
    exact = lse_rows(np.where(masked, -np.inf, SCALE * qr @ kr.T))
    qh, kh = bf16(qr32), bf16(kr32)
    ql, kl = bf16(qr32 - qh), bf16(kr32 - kh)
    schemes = {
        "bf16 single": qh @ kh.T,
        "fp16 single": f16(qr32) @ f16(kr32).T,
        "tf32 single": tf32(qr32) @ tf32(kr32).T,
        "bf16 hi/lo 3 chains": qh @ kh.T + qh @ kl.T + ql @ kh.T,
        "bf16 hi/lo without ql.kh": qh @ kh.T + qh @ kl.T,
        "bf16 hi/lo without qh.kl": qh @ kh.T + ql @ kh.T,
    }
    return {n: float(np.max(np.abs(lse_rows(np.where(masked, -np.inf, SCALE * sc)) - exact)))
            for n, sc in schemes.items()}


def test_three_chain_scheme_is_far_inside_the_tolerance_and_cheaper_ones_are_not():
    e = errors()
    tol = 1e-3
    assert e["bf16 hi/lo 3 chains"] < 1e-5, e
    assert e["bf16 single"] > tol, e
    assert e["bf16 hi/lo without ql.kh"] > tol and e["bf16 hi/lo without qh.kl"] > tol, e
    # 11-bit products: inside the tolerance at unit scale ...
    assert e["fp16 single"] < tol / 4 and e["tf32 single"] < tol / 4, e


@pytest.mark.parametrize("std", [3.0])
def test_single_11_bit_products_leave_the_tolerance_at_larger_input_scale(std):
    # ... but not at three times that scale, where the 3-chain form still has ample room
    e = errors(std=std)
    assert e["tf32 single"] > 1e-3 and e["fp16 single"] > 1e-3, e
    assert e["bf16 hi/lo 3 chains"] < 2.5e-4, e
