"""Prefill parity past one wave of CTAs: D = 64 problems with more than 148 query tiles of 128
rows, against the fp64 oracle, element by element.

The cases cover MHA and GQA groups of 2, 3 and 4, ragged row and key tails, causal alignment
with Sq != Skv (fully masked rows included), peaked scores (many rescales), RoPE (hi/lo split
products), bf16 and fp32 outputs and an fp32-input problem of the same size."""
import numpy as np
import pytest
import torch

from test_gpu_prefill import P, run_case

pytestmark = pytest.mark.gpu


def n_query_tiles(w):
    return w.B * w.Hq * ((w.Sq + 127) // 128)


CASES = [
    # ragged last row tile
    P("large_mha_causal_ragged", "bf16", 1, 9, 9, 2200, 2200, 64, True),
    # G = 2, non-causal with a ragged key tail
    P("large_gqa2_noncausal", "bf16", 1, 10, 5, 2000, 2100, 64, False),
    # G = 4
    P("large_gqa4_causal", "bf16", 1, 8, 2, 2400, 2400, 64, True),
    # G = 3 (odd group)
    P("large_gqa3_causal", "bf16", 2, 6, 2, 1700, 1700, 64, True),
    # chunked prefill: Sq < Skv, bottom-right causal alignment
    P("large_chunked", "bf16", 1, 4, 4, 4800, 5000, 64, True),
    # Sq > Skv: the first Sq - Skv rows see no key (O = 0, LSE = -inf)
    P("large_sq_gt_skv", "bf16", 1, 16, 16, 1200, 700, 64, True),
    # large score range: many online-softmax rescales
    P("large_peaked", "bf16", 1, 8, 8, 2500, 2500, 64, True, qk_std=3.0),
    # RoPE: Q rotated in shared memory, K rotated by the pre-pass into hi + lo halves
    P("large_rope_gqa4", "bf16", 1, 8, 2, 2400, 2400, 64, True, rope_base=10000.0),
    P("large_rope_chunked_mha", "bf16", 1, 6, 6, 3100, 3300, 64, True, rope_base=10000.0, q_pos0=200),
    # fp32 inputs take the FFMA kernel
    P("large_size_fp32_inputs", "fp32", 1, 8, 8, 2400, 2400, 64, True),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_large_prefill_matches_oracle(w):
    assert n_query_tiles(w) > 148
    run_case(w)


@pytest.mark.parametrize("w", CASES[:3], ids=[c.name for c in CASES[:3]])
def test_large_prefill_bf16_output(w):
    run_case(w, out_dtype=torch.bfloat16)


def test_large_prefill_without_lse():
    run_case(CASES[2], want_lse=False)
