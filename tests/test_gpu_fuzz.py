"""Seeded random shapes (batch, head grouping, ragged Sq and Skv down to 1, native and padded head
dims, causal or not, RoPE with offsets) for the forward and the backward, each against the fp64
oracle.  The draws are fixed by the seed, so a failure names a reproducible case."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, bits_to_dev, compare, make_prefill, to_host_f64

pytestmark = pytest.mark.gpu


def _draw(n, seed=777):
    rng = np.random.default_rng(seed)
    out = []
    for t in range(n):
        Hkv = int(rng.choice([1, 2, 4]))
        G = int(rng.choice([1, 2, 3, 4, 8]))
        D = int(rng.choice([64, 64, 128, 32, 48, 96]))
        Sq = int(rng.choice([1, 2, 17, 127, 128, 129, 200, 300]))
        Skv = int(rng.choice([1, 3, 64, 128, 130, 257, 300]))
        causal = bool(rng.integers(0, 2))
        rope = bool(rng.integers(0, 2))
        q_pos0 = int(rng.integers(0, 500)) if rope else 0
        B = int(rng.integers(1, 3))
        out.append(si.Prefill(f"fuzz{t}_B{B}_Hq{Hkv * G}_Hkv{Hkv}_Sq{Sq}_Skv{Skv}_D{D}_{'c' if causal else 'n'}"
                              f"{'_rope' if rope else ''}", "bf16", B, Hkv * G, Hkv, Sq, Skv, D, causal,
                              float(1.0 / np.sqrt(D)), rope_base=10000.0 if rope else 0.0, q_pos0=q_pos0,
                              seed=900 + t))
    return out


CASES = _draw(24)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fuzz_forward(w):
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0)
    compare(to_host_f64(o), ro, to_host_f64(lse), rl, TOL_BF16_O, TOL_BF16_LSE, w.name)


@pytest.mark.parametrize("w", CASES[::3], ids=lambda w: w.name)
def test_fuzz_backward(w):
    x, dev = make_prefill(w)
    gb, g = si.bf16_normal(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0)
    o = torch.from_numpy(ro.astype(np.float32)).cuda().to(torch.bfloat16)
    lse = torch.from_numpy(rl.astype(np.float32)).cuda()
    dq, dk, dv = ea.attn_bwd(dev["q"], dev["k"], dev["v"], o, lse, bits_to_dev(gb), w.scale, w.causal, w.rope_base,
                             w.q_pos0, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], g, w.scale, w.causal, w.rope_base, w.q_pos0)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        gh = got.cpu().numpy().astype(np.float64)
        err = float(np.max(np.abs(gh - ref)) / max(1.0, float(np.max(np.abs(ref)))))
        assert err <= 1e-2, (w.name, name, err)
