"""Key-split forward: a bf16 problem whose query tiles fill at most half of the SMs divides each
tile's key tiles among several CTAs and merges their partials by logsumexp.  Parity with the
fp64 oracle for the split path and (through the C attn_fwd, no workspace) the unsplit path on
the same inputs, including chunks in which a row sees no key, rows masked everywhere, GQA,
RoPE with a position offset, D=128, a padded head dim and an additive mask."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, compare, make_prefill, to_host_f64

pytestmark = pytest.mark.gpu


def P(name, B, Hq, Hkv, Sq, Skv, D, causal, **kw):
    scale = kw.pop("scale", 1.0 / np.sqrt(D))
    return si.Prefill(name, "bf16", B, Hq, Hkv, Sq, Skv, D, causal, scale, seed=kw.pop("seed", 501), **kw)


# (workload, splits): n = min(148 // tiles, nkv // 2, 16) with tiles = ceil(Sq/128) * B * Hq <= 74
# and nkv = ceil(Skv/128), taken when nkv - ceil(nkv / n) >= 8
CASES = [
    (P("noncausal_ragged", 1, 4, 4, 700, 2100, 64, False), 6),             # 24 tiles, 17 key tiles
    (P("causal_empty_chunks", 1, 1, 1, 2048, 2048, 64, True), 8),          # row tile 0: 7 empty chunks
    (P("decode_like_gqa", 1, 8, 2, 128, 4096, 64, True, seed=502), 16),    # 8 tiles, 32 key tiles
    # offset 64: rows 0..63 of tile 0 see no key of its second chunk (partial lse = -inf)
    (P("offset64_masked_partials", 1, 1, 1, 1984, 2048, 64, True, seed=503), 8),
    (P("rope_gqa_offset", 1, 8, 2, 256, 2048, 64, True, rope_base=10000.0, q_pos0=1792, seed=504), 8),
    (P("d128_peaked", 1, 2, 2, 2048, 2048, 128, True, qk_std=3.0, seed=505), 4),
    (P("d128_noncausal_gqa", 2, 4, 2, 130, 1200, 128, False, seed=506), 5),
    # Sq > Skv, causal: rows 0..179 see no key at all (O = 0, LSE = -inf in every partial)
    (P("sq_gt_skv_dead_rows", 1, 1, 1, 2200, 2020, 64, True, seed=507), 8),
    (P("padded_d80", 1, 2, 2, 300, 2100, 80, False, seed=508), 8),
    # the Whisper-encoder shape (12 key tiles) runs unsplit: two chunks would spare only 6
    (P("whisper_shape_unsplit", 1, 6, 6, 1500, 1500, 64, False, seed=510), 1),
]


def _run(w, **kw):
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.rope_base, w.q_pos0,
                            out_dtype=kw.pop("out_dtype", torch.float32), **kw)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    return x, dev, o, lse


@pytest.mark.parametrize("w,splits", CASES, ids=[c[0].name for c in CASES])
def test_split_and_unsplit_match_oracle(w, splits):
    x, dev, o, lse = _run(w)
    assert ea.fwd_kv_splits(dev["q"], dev["k"], torch.float32) == splits
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0)
    compare(to_host_f64(o), ro, to_host_f64(lse), rl, TOL_BF16_O, TOL_BF16_LSE, w.name + " split")
    if w.rope_base <= 0 and w.D in (64, 128):
        _, _, o1, l1 = _run(w, kv_split=False)
        compare(to_host_f64(o1), ro, to_host_f64(l1), rl, TOL_BF16_O, TOL_BF16_LSE, w.name + " unsplit")


def test_split_bf16_output_and_null_lse():
    w = CASES[0][0]
    x, dev, o, lse = _run(w, out_dtype=torch.bfloat16, want_lse=False)
    assert lse is None and o.dtype == torch.bfloat16
    ro, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal)
    compare(to_host_f64(o), ro, None, None, TOL_BF16_O, TOL_BF16_LSE, w.name + " bf16 out")


def test_split_is_deterministic_and_stays_in_bounds():
    w = CASES[1][0]
    x, dev = make_prefill(w)
    n = w.B * w.Sq * w.Hq * w.D
    buf = torch.full((n + 4096,), 7.0, dtype=torch.float32, device="cuda")
    o = buf[:n].view(w.B, w.Sq, w.Hq, w.D)
    lbuf = torch.full((w.B * w.Hq * w.Sq + 1024,), 5.0, dtype=torch.float32, device="cuda")
    lse = lbuf[: w.B * w.Hq * w.Sq].view(w.B, w.Hq, w.Sq)
    ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, True, 0.0, 0, o=o, lse=lse)
    o2, l2 = ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, True, 0.0, 0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (buf[n:] == 7.0).all() and (lbuf[w.B * w.Hq * w.Sq:] == 5.0).all()
    assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_split_with_additive_mask():
    w = P("masked_split", 1, 4, 4, 300, 2200, 64, False, seed=509)
    x, dev = make_prefill(w)
    assert ea.fwd_kv_splits(dev["q"], dev["k"], torch.float32) == 9     # 12 tiles, 18 key tiles
    rng = np.random.default_rng(w.seed)
    m = rng.standard_normal((w.Sq, w.Skv)).astype(np.float32)
    m[:, 1500:] = -np.inf      # the last key tiles masked out: whole chunks without a visible key
    m[[3, 200], :] = -np.inf   # rows masked everywhere
    o, lse = ea.attn_fwd_masked(dev["q"], dev["k"], dev["v"], torch.from_numpy(m).cuda(), w.scale, False,
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    ro, rl = oracle.attn_fwd_masked(x["q"], x["k"], x["v"], m, w.scale, False)
    og, lg = to_host_f64(o), to_host_f64(lse)
    assert np.all(og[:, [3, 200]] == 0.0) and np.all(lg[:, :, [3, 200]] == -np.inf)
    compare(og, ro, lg, rl, TOL_BF16_O, TOL_BF16_LSE, w.name)


def test_non_null_workspace_too_small_is_refused():
    w = CASES[0][0]
    x, dev = make_prefill(w)
    need = ea.fwd_workspace_bytes(dev["q"], dev["k"], 0.0, 0, torch.float32)
    assert need > 0
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ea.AttnError):
        ea.attn_fwd_ex(dev["q"], dev["k"], dev["v"], w.scale, w.causal, 0.0, 0, workspace=ws,
                       out_dtype=torch.float32)
