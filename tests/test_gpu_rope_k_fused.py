"""The in-kernel form of RoPE on K (ATTN_ROPE_K_FORM=fused) against the fp64 oracle.

By default the bf16 forward rotates K once into hi + lo halves before the prefill kernel; with
ATTN_ROPE_K_FORM=fused each CTA loads K as it is and two of its warps rotate every K tile in
shared memory before the tensor core reads it.  Both forms must give the oracle's result within
the same tolerances; they also agree closely with each other (same rotation arithmetic)."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
from attn_cases import make_prefill, to_host_f64
from test_gpu_prefill import P, run_case

pytestmark = pytest.mark.gpu

CASES = [
    P("fused_rope_gqa_causal", "bf16", 1, 8, 2, 300, 300, 64, True, rope_base=10000.0),
    P("fused_rope_mha_chunked", "bf16", 1, 2, 2, 90, 400, 64, True, rope_base=10000.0, q_pos0=310),
    P("fused_rope_ragged_keys_noncausal", "bf16", 2, 4, 4, 200, 333, 64, False, rope_base=10000.0),
    P("fused_rope_d128", "bf16", 1, 2, 2, 140, 140, 128, True, rope_base=500000.0),
    P("fused_rope_large_gqa4", "bf16", 1, 8, 2, 2400, 2400, 64, True, rope_base=10000.0),
    # key splits (a small problem): every split rotates its own chunk of key tiles
    P("fused_rope_key_splits", "bf16", 1, 8, 2, 256, 2048, 64, True, rope_base=10000.0, q_pos0=1792),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fused_k_rope_matches_oracle(w, monkeypatch):
    monkeypatch.setenv("ATTN_ROPE_K_FORM", "fused")
    run_case(w)


def test_fused_and_prepass_forms_agree(monkeypatch):
    w = CASES[0]
    x, dev = make_prefill(w)
    outs = []
    for form in ("prepass", "fused"):
        monkeypatch.setenv("ATTN_ROPE_K_FORM", form)
        o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                                out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert ea.read_device_status() == 0
        outs.append((to_host_f64(o), to_host_f64(lse)))
    # the same rotation arithmetic feeds the same MMAs; only the fp32 rounding of the rotation
    # (contraction into FMAs may differ between the two kernels) can move a bit of K lo
    assert np.max(np.abs(outs[0][0] - outs[1][0])) <= 1e-4
    assert np.max(np.abs(outs[0][1] - outs[1][1])) <= 1e-5
