"""Interleaved keys against the fp64 oracle.

A query-tile count that fits one wave of the SMs runs one 128-row query tile per CTA; at D = 64
the CTA's two softmax warpgroups then take alternate key tiles of that one tile, each with its own
online-softmax state (m, l, O), and the epilogue merges the two states by their maxima.  The cases
pin the merge where it can go wrong: one group with no key tile at all, query tiles that see no
key (with RoPE, whose in-place rotation of Q must be complete before the merge reuses its slot),
odd and even key-tile counts, peaked scores (the two halves' maxima far apart), key splits on
top, and a bf16 output."""
import pytest
import torch

from test_gpu_prefill import P, run_case

pytestmark = pytest.mark.gpu

CASES = [
    P("ilv_even_key_tiles", "bf16", 1, 2, 2, 256, 1024, 64, False),
    P("ilv_odd_key_tiles_ragged", "bf16", 1, 3, 3, 200, 520, 64, False),
    # causal, Sq = Skv: the first query tile has one key tile, so the second group has none
    P("ilv_causal_one_key_tile", "bf16", 1, 2, 2, 300, 300, 64, True),
    # Sq > Skv, causal: the first query tiles see no key at all; with RoPE and an offset
    P("ilv_rope_tiles_without_keys", "bf16", 2, 4, 1, 300, 64, 64, True, rope_base=10000.0, q_pos0=380),
    P("ilv_rope_gqa_chunk", "bf16", 1, 8, 2, 128, 1100, 64, True, rope_base=10000.0, q_pos0=972),
    P("ilv_peaked_scores", "bf16", 1, 2, 2, 128, 1024, 64, False, qk_std=3.0),
    P("ilv_peaked_scores_causal", "bf16", 1, 2, 2, 600, 600, 64, True, qk_std=3.0),
    # a query-tile count small enough for key splits too: each split's chunk is interleaved
    P("ilv_with_key_splits", "bf16", 1, 2, 2, 1500, 1500, 64, False),
    P("ilv_padded_head_dim", "bf16", 1, 4, 2, 140, 700, 48, True),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_interleaved_keys_match_oracle(w):
    run_case(w)


@pytest.mark.parametrize("w", [CASES[0], CASES[2], CASES[7]], ids=["even", "one_key", "splits"])
def test_interleaved_keys_bf16_output(w):
    run_case(w, out_dtype=torch.bfloat16)
