"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a value
printed on a page (golden fixtures under tests/golden/), a closed form, an invariant,
or a brute-force evaluation written independently here in pure Python.  They are
collected by ``test_oracle_pins.py`` and re-run against deliberately broken builds of
the oracle by ``test_oracle_mutants.py`` (every planted mistake must trip at least one).
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle
from seeded_inputs import normal_f32

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
EXACT = 1e-12


def load_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = np.array([float(x) for x in val.split(",")], dtype=np.float64)
    return out


def _close(a, b, tol, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol, f"{what}: max abs error {err:.3e} > {tol:.1e}"


# ------------------------------------------------------------------------------------------
# Independent brute force (pure Python, log-domain, different algebra from the oracle)
# ------------------------------------------------------------------------------------------

def _exp(x: float) -> float:
    return math.exp(x) if x < 709.0 else math.inf


def brute_attention(q, k, v, scale, causal, rope_base=0.0, q_pos0=0):
    """Exact attention evaluated as weights w_j = 1 / sum_k exp(s_k - s_j) over the visible
    keys, with LSE = s_j + ln(sum_k exp(s_k - s_j)) for any visible j.  Pure Python floats.
    RoPE here rotates complex numbers z = x_{2i} + i x_{2i+1} by e^{i theta}."""
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    o = np.zeros((B, Sq, Hq, D))
    lse = np.zeros((B, Hq, Sq))

    def rot(vec, pos):
        if rope_base <= 0:
            return [float(x) for x in vec]
        out = []
        for i in range(D // 2):
            th = pos * rope_base ** (-(2.0 * i) / D)
            z = complex(float(vec[2 * i]), float(vec[2 * i + 1])) * complex(math.cos(th), math.sin(th))
            out += [z.real, z.imag]
        return out

    for b in range(B):
        for h in range(Hq):
            kh = h // g
            keys = [rot(k[b, j, kh], j) for j in range(Skv)]
            for i in range(Sq):
                qi = rot(q[b, i, h], q_pos0 + i)
                vis = [j for j in range(Skv) if not (causal and j > i + (Skv - Sq))]
                if not vis:
                    lse[b, h, i] = -math.inf
                    continue
                s = {j: scale * math.fsum(qi[d] * keys[j][d] for d in range(D)) for j in vis}
                j0 = max(vis, key=lambda j: s[j])
                lse[b, h, i] = s[j0] + math.log(math.fsum(_exp(s[kk] - s[j0]) for kk in vis))
                for d in range(D):
                    o[b, i, h, d] = math.fsum(
                        float(v[b, j, kh, d]) / math.fsum(_exp(s[kk] - s[j]) for kk in vis)
                        for j in vis)
    return o, lse


# ------------------------------------------------------------------------------------------
# Golden fixtures from the pages
# ------------------------------------------------------------------------------------------

def pin_golden_sdpa_basic():
    g = load_golden("p3_sdpa_basic.txt")
    q = g["q"].reshape(1, 2, 1, 4)
    k = g["k"].reshape(1, 2, 1, 4)
    v = g["v"].reshape(1, 2, 1, 4)
    o, lse = oracle.attn_fwd(q, k, v, float(g["scale"][0]), causal=False)
    _close(o.reshape(-1), g["expected_o"], 1e-6, "P3 basic O (fixture, 7 decimals)")
    _close(lse.reshape(-1), g["expected_lse"], 1e-6, "P3 basic LSE (fixture)")
    # the same values from the closed form sigma(1/2)
    s = 1.0 / (1.0 + math.exp(-0.5))
    o0 = [s * a + (1 - s) * b for a, b in zip((1, 2, 3, 4), (5, 6, 7, 8))]
    o1 = [(1 - s) * a + s * b for a, b in zip((1, 2, 3, 4), (5, 6, 7, 8))]
    _close(o.reshape(2, 4), np.array([o0, o1]), EXACT, "P3 basic O (closed form)")
    _close(lse.reshape(-1), [math.log1p(math.exp(0.5))] * 2, EXACT, "P3 basic LSE (closed form)")


def pin_golden_causal_first_row():
    g = load_golden("p3_flash_attention_causal_first_row.txt")
    q = g["q"].reshape(1, 2, 1, 4)
    k = g["k"].reshape(1, 2, 1, 4)
    v = g["v"].reshape(1, 2, 1, 4)
    o, lse = oracle.attn_fwd(q, k, v, float(g["scale"][0]), causal=True)
    _close(o[0, 0, 0], g["expected_o_row0"], EXACT, "P3 causal row 0")
    # row 0 has one visible key: LSE = its score = 0.5 * (q0 . k0) = 0.5
    _close(lse[0, 0, 0], 0.5, EXACT, "P3 causal row 0 LSE")
    # row 1 sees both keys with equal scores: mean of v0, v1; LSE = 0.5 + ln 2
    _close(o[0, 1, 0], 0.5 * (g["v"][:4] + g["v"][4:]), EXACT, "P3 causal row 1")
    _close(lse[0, 0, 1], 0.5 + math.log(2.0), EXACT, "P3 causal row 1 LSE")


def _decode_case(g):
    D = int(g["head_dim"][0])
    L = int(g["seq_len"][0])
    q = g["q"].reshape(1, 1, D)
    k = g["k"].reshape(1, L, 1, D)
    v = g["v"].reshape(1, L, 1, D)
    return q, k, v, np.array([L], dtype=np.int32), float(g["scale"][0])


def pin_golden_decode_single_token():
    g = load_golden("p4_flash_decode_single_token.txt")
    q, k, v, sl, scale = _decode_case(g)
    for o, lse in (oracle.decode(q, k, v, sl, scale), oracle.decode_split(q, k, v, sl, scale, 4)):
        _close(o.reshape(-1), g["expected_o"], EXACT, "P4 single token")
        _close(lse.reshape(-1), [scale * 0.5], EXACT, "P4 single token LSE = its score")


def pin_golden_decode_uniform_keys():
    g = load_golden("p4_flash_decode_uniform_keys.txt")
    q, k, v, sl, scale = _decode_case(g)
    s = scale * 4 * float(np.float32(0.1)) ** 2      # every score equal
    for nt in (1, 2, 3, 4, 7):
        o, lse = oracle.decode_split(q, k, v, sl, scale, nt)
        _close(o.reshape(-1), g["expected_o"], EXACT, f"P4 uniform keys, {nt} tiles")
        _close(lse.reshape(-1), [s + math.log(4.0)], EXACT, "P4 uniform keys LSE = s + ln n")
    o, lse = oracle.decode(q, k, v, sl, scale)
    _close(o.reshape(-1), g["expected_o"], EXACT, "P4 uniform keys, unsplit")


def pin_golden_rope_position_zero():
    g = load_golden("p2_rope_position_zero.txt")
    D, T, H = int(g["head_dim"][0]), int(g["seq_len"][0]), int(g["num_heads"][0])
    x = np.ones((T, H, D), dtype=np.float32)
    y = oracle.rope(x, np.arange(T), float(g["base"][0]))
    _close(y[0, 0], g["expected_pos0"], 1e-10, "P2 RoPE position 0 is the identity")
    assert np.max(np.abs(y[1, 0] - y[0, 0])) > 1e-10, "P2: position 1 must differ from position 0"


# ------------------------------------------------------------------------------------------
# Closed forms and invariants
# ------------------------------------------------------------------------------------------

def pin_softmax_rows_sum_to_one():
    # V = identity basis (Skv == D): O row i is the probability row p_i itself.
    D = 8
    q = normal_f32(7, 0, (1, 5, 2, D))
    k = normal_f32(7, 1, (1, D, 2, D))
    v = np.tile(np.eye(D, dtype=np.float32)[None, :, None, :], (1, 1, 2, 1))
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.3, causal)
        p = o.transpose(0, 2, 1, 3)                      # [B,H,Sq,Skv]
        _close(p.sum(-1), np.ones(p.shape[:-1]), EXACT, "rows of P sum to 1")
        assert (p >= 0).all()
        # ratios p_ij / p_ik = exp(s_ij - s_ik) computed here independently
        for h in range(2):
            for i in range(5):
                vis = [j for j in range(D) if not (causal and j > i + D - 5)]
                s = [0.3 * math.fsum(float(q[0, i, h, d]) * float(k[0, j, h, d]) for d in range(D))
                     for j in range(D)]
                for j in vis:
                    _close(p[0, h, i, j] / p[0, h, i, vis[0]], math.exp(s[j] - s[vis[0]]), 1e-10,
                           "p ratio")
                for j in range(D):
                    if j not in vis:
                        assert p[0, h, i, j] == 0.0, "masked key must get zero weight"
    # V all ones: O = 1 exactly (up to rounding)
    o, _ = oracle.attn_fwd(q, k, np.ones_like(k), 1.7, True)
    _close(o, np.ones_like(o), EXACT, "V = 1 gives O = 1")


def pin_single_key():
    q = normal_f32(11, 0, (2, 3, 4, 6))
    k = normal_f32(11, 1, (2, 1, 2, 6))
    v = normal_f32(11, 2, (2, 1, 2, 6))
    o, lse = oracle.attn_fwd(q, k, v, 0.7, causal=False)
    for b in range(2):
        for i in range(3):
            for h in range(4):
                _close(o[b, i, h], v[b, 0, h // 2], EXACT, "single key returns V")
                s = 0.7 * math.fsum(float(q[b, i, h, d]) * float(k[b, 0, h // 2, d]) for d in range(6))
                _close(lse[b, h, i], s, EXACT, "single key LSE = its score")


def pin_equal_scores_mean_of_v():
    # identical keys: every score equal, O = mean of visible V rows, LSE = s + ln n
    D, S = 5, 6
    q = normal_f32(13, 0, (1, S, 1, D))
    k = np.tile(normal_f32(13, 1, (1, 1, 1, D)), (1, S, 1, 1))
    v = normal_f32(13, 2, (1, S, 1, D))
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.4, causal)
        for i in range(S):
            n = i + 1 if causal else S
            _close(o[0, i, 0], v[0, :n, 0].astype(np.float64).mean(0), EXACT, "mean of V")
            s = 0.4 * math.fsum(float(q[0, i, 0, d]) * float(k[0, 0, 0, d]) for d in range(D))
            _close(lse[0, 0, i], s + math.log(n), EXACT, "LSE = s + ln n")


def pin_scale_two_keys():
    # two keys whose dot products with q differ by exactly 2: p0 = sigmoid(2 * scale)
    q = np.array([1, 0, 0, 0], dtype=np.float32).reshape(1, 1, 1, 4)
    k = np.array([[2, 0, 0, 0], [0, 3, 0, 0]], dtype=np.float32).reshape(1, 2, 1, 4)
    v = np.array([[1, 0, 0, 0], [0, 1, 0, 0]], dtype=np.float32).reshape(1, 2, 1, 4)
    for scale in (0.125, 0.5, 1.0, 3.0):
        o, lse = oracle.attn_fwd(q, k, v, scale, False)
        p0 = 1.0 / (1.0 + math.exp(-2.0 * scale))
        _close(o.reshape(-1), [p0, 1 - p0, 0, 0], EXACT, f"scale {scale}")
        _close(lse.reshape(-1), [2 * scale + math.log1p(math.exp(-2 * scale))], EXACT, "LSE")


def pin_large_scores_stable():
    # scores of order 1e3: no overflow, rows still sum to 1 (whisper-apr softmax stability test)
    q = (normal_f32(17, 0, (1, 4, 1, 8)) * 40).astype(np.float32)
    k = (normal_f32(17, 1, (1, 9, 1, 8)) * 40).astype(np.float32)
    v = np.ones((1, 9, 1, 8), dtype=np.float32)
    o, lse = oracle.attn_fwd(q, k, v, 1.0, False)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    _close(o, np.ones_like(o), EXACT, "large scores: O = 1 for V = 1")
    ob, lb = brute_attention(q, k, v, 1.0, False)
    _close(lse, lb, 1e-9, "large-score LSE vs brute force")


def pin_brute_force_tiny():
    cases = [
        # B, Sq, Skv, Hq, Hkv, D, causal, scale
        (1, 3, 3, 1, 1, 4, False, 0.5),
        (2, 4, 4, 2, 2, 3, True, 0.8),
        (1, 2, 5, 4, 2, 6, True, 0.35),     # Sq < Skv: bottom-right causal
        (1, 5, 3, 3, 1, 2, True, 1.1),      # Sq > Skv: first rows fully masked
        (2, 3, 4, 4, 1, 5, False, 0.2),     # MQA
        (1, 4, 4, 2, 1, 4, True, 0.9),
    ]
    for n, (B, Sq, Skv, Hq, Hkv, D, causal, scale) in enumerate(cases):
        q = normal_f32(100 + n, 0, (B, Sq, Hq, D))
        k = normal_f32(100 + n, 1, (B, Skv, Hkv, D))
        v = normal_f32(100 + n, 2, (B, Skv, Hkv, D))
        o, lse = oracle.attn_fwd(q, k, v, scale, causal)
        ob, lb = brute_attention(q, k, v, scale, causal)
        _close(o, ob, 1e-12, f"brute force O case {n}")
        fin = np.isfinite(lb)
        assert (np.isfinite(lse) == fin).all(), f"case {n}: masked rows"
        _close(lse[fin], lb[fin], 1e-12, f"brute force LSE case {n}")


def pin_brute_force_rope():
    for n, (Sq, Skv, D, base, p0) in enumerate([(3, 3, 4, 10000.0, 0), (2, 4, 6, 500.0, 2),
                                                (4, 4, 8, 10.0, 0)]):
        q = normal_f32(200 + n, 0, (1, Sq, 2, D))
        k = normal_f32(200 + n, 1, (1, Skv, 1, D))
        v = normal_f32(200 + n, 2, (1, Skv, 1, D))
        o, lse = oracle.attn_fwd(q, k, v, 0.6, True, rope_base=base, q_pos0=p0)
        ob, lb = brute_attention(q, k, v, 0.6, True, rope_base=base, q_pos0=p0)
        _close(o, ob, 1e-12, f"RoPE brute force O case {n}")
        fin = np.isfinite(lb)
        _close(lse[fin], lb[fin], 1e-12, f"RoPE brute force LSE case {n}")


def pin_fully_masked_rows():
    # Sq > Skv with causal bottom-right alignment: rows i < Sq - Skv see no key.
    q = normal_f32(19, 0, (1, 6, 1, 4))
    k = normal_f32(19, 1, (1, 2, 1, 4))
    v = normal_f32(19, 2, (1, 2, 1, 4))
    o, lse = oracle.attn_fwd(q, k, v, 0.5, True)
    for i in range(4):
        assert (o[0, i, 0] == 0.0).all(), "fully masked row -> O = 0"
        assert lse[0, 0, i] == -math.inf, "fully masked row -> LSE = -inf"
    _close(o[0, 4, 0], v[0, 0, 0], EXACT, "row Sq-Skv sees exactly key 0")
    on, ln = oracle.attn_fwd(q, k, v, 0.5, False)
    _close(o[0, 5, 0], on[0, 5, 0], EXACT, "last row sees every key")


def pin_causal_alignment():
    # Sq == Skv: causal row i equals non-causal attention over keys 0..i;
    # Sq < Skv: the last query row sees every key (bottom-right).
    q = normal_f32(23, 0, (1, 5, 1, 4))
    k = normal_f32(23, 1, (1, 5, 1, 4))
    v = normal_f32(23, 2, (1, 5, 1, 4))
    o, lse = oracle.attn_fwd(q, k, v, 0.9, True)
    for i in range(5):
        oi, li = oracle.attn_fwd(q[:, i:i + 1], k[:, :i + 1], v[:, :i + 1], 0.9, False)
        _close(o[0, i, 0], oi[0, 0, 0], EXACT, f"causal row {i} = prefix attention")
        _close(lse[0, 0, i], li[0, 0, 0], EXACT, "causal LSE")
    o2, _ = oracle.attn_fwd(q[:, 3:], k, v, 0.9, True)     # Sq=2, Skv=5
    _close(o2[0, 0, 0], o[0, 3, 0], EXACT, "bottom-right: chunk row 0 = full row 3")
    _close(o2[0, 1, 0], o[0, 4, 0], EXACT, "bottom-right: chunk row 1 = full row 4")


def pin_gqa_equals_repeated_mha():
    B, S, Hq, Hkv, D = 2, 7, 6, 2, 5
    q = normal_f32(29, 0, (B, S, Hq, D))
    k = normal_f32(29, 1, (B, S, Hkv, D))
    v = normal_f32(29, 2, (B, S, Hkv, D))
    g = Hq // Hkv
    kr = np.repeat(k, g, axis=2)
    vr = np.repeat(v, g, axis=2)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.45, causal)
        om, lm = oracle.attn_fwd(q, kr, vr, 0.45, causal)
        _close(o, om, EXACT, "GQA == MHA with repeated KV heads")
        _close(lse, lm, EXACT, "GQA LSE")
    # MQA: Hkv = 1, each q head equals a single-head problem
    o, lse = oracle.attn_fwd(q, k[:, :, :1], v[:, :, :1], 0.45, True)
    for h in range(Hq):
        oh, lh = oracle.attn_fwd(q[:, :, h:h + 1], k[:, :, :1], v[:, :, :1], 0.45, True)
        _close(o[:, :, h], oh[:, :, 0], EXACT, "MQA head")


def pin_tiled_equals_three_pass():
    # the online-softmax recurrence (any block sizes) reaches the three-pass definition
    B, Sq, Skv, Hq, Hkv, D = 1, 37, 45, 4, 2, 8
    q = normal_f32(31, 0, (B, Sq, Hq, D), 2.5)
    k = normal_f32(31, 1, (B, Skv, Hkv, D), 2.5)
    v = normal_f32(31, 2, (B, Skv, Hkv, D))
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.7, causal)
        for bq, bkv in ((1, 1), (4, 8), (16, 16), (64, 5), (37, 45)):
            ot, lt = oracle.attn_fwd_tiled(q, k, v, 0.7, causal, bq, bkv)
            _close(ot, o, EXACT, f"tiled O ({bq},{bkv}) causal={causal}")
            _close(lt, lse, EXACT, f"tiled LSE ({bq},{bkv})")
    # with fully masked rows (Sq > Skv)
    o, lse = oracle.attn_fwd(q, k[:, :20], v[:, :20], 0.7, True)
    ot, lt = oracle.attn_fwd_tiled(q, k[:, :20], v[:, :20], 0.7, True, 8, 8)
    _close(ot, o, EXACT, "tiled O, masked rows")
    assert (np.isneginf(lt) == np.isneginf(lse)).all()


def pin_decode_split_equals_unsplit():
    B, Hq, Hkv, Smax, D = 3, 4, 2, 40, 6
    q = normal_f32(37, 0, (B, Hq, D), 2.0)
    kc = normal_f32(37, 1, (B, Smax, Hkv, D), 2.0)
    vc = normal_f32(37, 2, (B, Smax, Hkv, D))
    sl = np.array([1, 17, 40], dtype=np.int32)
    o, lse = oracle.decode(q, kc, vc, sl, 0.5)
    for nt in (1, 2, 3, 5, 16, 40, 64):
        os_, ls = oracle.decode_split(q, kc, vc, sl, 0.5, nt)
        _close(os_, o, EXACT, f"split decode, {nt} tiles")
        _close(ls, lse, EXACT, f"split decode LSE, {nt} tiles")
    # decode == the last row of a causal prefill over the cache (cached decode == full forward)
    for b in range(B):
        L = int(sl[b])
        qf = np.zeros((1, L, Hq, D), dtype=np.float32)
        qf[0, L - 1] = q[b]
        of, lf = oracle.attn_fwd(qf, kc[b:b + 1, :L], vc[b:b + 1, :L], 0.5, True)
        _close(of[0, L - 1], o[b], EXACT, "decode == last causal row")
        _close(lf[0, :, L - 1], lse[b], EXACT, "decode LSE == last causal row")


def pin_rope_rotation():
    # D = 2: the single pair rotates by exactly pos radians, counter-clockwise
    for pos in (1, 2, 5, -3):
        y = oracle.rope(np.array([[[1.0, 0.0]], [[0.0, 1.0]]], dtype=np.float32), [pos, pos], 123.0)
        _close(y[0, 0], [math.cos(pos), math.sin(pos)], EXACT, "e0 -> (cos, sin)")
        _close(y[1, 0], [-math.sin(pos), math.cos(pos)], EXACT, "e1 -> (-sin, cos)")
    # D = 4, base 10^4: pair 1 has frequency 10^4^(-2/4) = 1/100; at pos 100 the angle is 1
    y = oracle.rope(np.array([[[0, 0, 1, 0]]], dtype=np.float32), [100], 10000.0)
    _close(y[0, 0], [0, 0, math.cos(1.0), math.sin(1.0)], EXACT, "pair frequency base^(-2i/D)")
    y = oracle.rope(np.array([[[1, 0, 0, 0]]], dtype=np.float32), [100], 10000.0)
    _close(y[0, 0], [math.cos(100.0), math.sin(100.0), 0, 0], EXACT, "pair 0 frequency 1")


def pin_rope_invariants():
    T, H, D = 9, 3, 16
    x = normal_f32(41, 0, (T, H, D))
    pos = np.array([0, 1, 2, 7, 100, 511, 4095, 30000, -5], dtype=np.int32)
    y = oracle.rope(x, pos, 10000.0)
    _close(np.linalg.norm(y, axis=-1), np.linalg.norm(x.astype(np.float64), axis=-1), 1e-12,
           "norm preserved")
    # inverse: rotating the rotated vector by -pos returns x (RoPE inverse = negated angle)
    back = oracle.rope(y.astype(np.float32), -pos, 10000.0)
    _close(back, x, 2e-6, "R(-p) R(p) = I (up to the float32 re-rounding of y)")
    # relative position: <R(m) a, R(n) b> depends only on n - m
    a = normal_f32(43, 0, (1, 1, D))
    b = normal_f32(43, 1, (1, 1, D))
    dots = []
    for m in (0, 3, 50, 1000):
        ra = oracle.rope(a, [m], 10000.0)[0, 0]
        rb = oracle.rope(b, [m + 17], 10000.0)[0, 0]
        dots.append(float(np.dot(ra, rb)))
    _close(dots, [dots[0]] * len(dots), 1e-10, "q.k after RoPE depends only on the offset")
    # different offsets give different results (scirs2-neural test_rope_position_offset)
    x1 = np.full((4, 1, 4), 0.5, dtype=np.float32)
    assert np.max(np.abs(oracle.rope(x1, np.arange(4), 1e4) - oracle.rope(x1, np.arange(2, 6), 1e4))) > 1e-10


def pin_error_paths():
    q = np.zeros((1, 2, 3, 4), dtype=np.float32)
    k = np.zeros((1, 2, 2, 4), dtype=np.float32)
    try:
        oracle.attn_fwd(q, k, k, 1.0, False)       # Hq = 3 not a multiple of Hkv = 2
        raise AssertionError("Hq % Hkv != 0 must be rejected")
    except oracle.OracleError:
        pass
    try:
        oracle.rope(np.zeros((1, 1, 7), dtype=np.float32), [0], 1e4)   # odd head dim
        raise AssertionError("odd RoPE head dim must be rejected")
    except oracle.OracleError:
        pass
    try:
        oracle.attn_fwd(q[:, :, :2], np.zeros((1, 0, 2, 4), np.float32),
                        np.zeros((1, 0, 2, 4), np.float32), 1.0, False)
        raise AssertionError("empty KV must be rejected")
    except oracle.OracleError:
        pass


def pin_sampled_rows_match_full():
    B, Sq, Hq, Hkv, D = 2, 9, 4, 2, 6
    q = normal_f32(47, 0, (B, Sq, Hq, D))
    k = normal_f32(47, 1, (B, Sq, Hkv, D))
    v = normal_f32(47, 2, (B, Sq, Hkv, D))
    o, lse = oracle.attn_fwd(q, k, v, 0.3, True, rope_base=100.0, q_pos0=0)
    rows = np.array([0, 5, 17, 40, 71, 3, 8], dtype=np.int64)   # (b*Hq + h)*Sq + i
    os_, ls = oracle.attn_fwd(q, k, v, 0.3, True, rope_base=100.0, q_pos0=0, rows=rows)
    for r, row in enumerate(rows):
        b, h, i = row // (Hq * Sq), (row // Sq) % Hq, row % Sq
        _close(os_[r], o[b, i, h], 0.0, "sampled row")
        _close(ls[r], lse[b, h, i], 0.0, "sampled LSE")


def _append_case(seed, B=3, Smax=12, Hkv=2, G=2, D=8, T=3):
    kc = normal_f32(seed, 0, (B, Smax, Hkv, D))
    vc = normal_f32(seed, 1, (B, Smax, Hkv, D))
    kn = normal_f32(seed, 2, (B, T, Hkv, D))
    vn = normal_f32(seed, 3, (B, T, Hkv, D))
    q = normal_f32(seed, 4, (B, T, Hkv * G, D))
    return kc, vc, kn, vn, q


def pin_kv_append_positions_and_copy():
    """Rows [L, L+T) receive the new tokens; a token at cache position 0 is unrotated (RoPE at
    position 0 is the identity); values and untouched rows are copied exactly; lengths advance."""
    kc, vc, kn, vn, q = _append_case(61)
    sl = np.array([0, 4, 9], dtype=np.int32)
    k2, v2, s2, q2, ovf = oracle.kv_append(kc, vc, sl, kn, vn, q, rope_base=10000.0)
    assert not ovf.any() and list(s2) == [3, 7, 12]
    _close(k2[0, 0], kn[0, 0], 0.0, "position 0 is the identity")
    _close(q2[0, 0], q[0, 0], 0.0, "query at position 0 unrotated")
    for b, L in enumerate(sl):
        _close(v2[b, L:L + 3], vn[b], 0.0, "values copied to rows [L, L+T)")
        _close(np.delete(v2[b], range(L, L + 3), axis=0), np.delete(vc[b], range(L, L + 3), axis=0), 0.0,
               "other rows untouched")
        _close(np.delete(k2[b], range(L, L + 3), axis=0), np.delete(kc[b], range(L, L + 3), axis=0), 0.0,
               "other key rows untouched")
    # without RoPE the keys are copied too and q is left alone
    k3, _, _, q3, _ = oracle.kv_append(kc, vc, sl, kn, vn, q, rope_base=0.0)
    _close(k3[1, 4:7], kn[1], 0.0, "plain append")
    _close(q3, q, 0.0, "q untouched without RoPE")


def pin_kv_append_same_position_dot():
    """Query and key of the same new token are rotated by the same angles: their dot product is
    the unrotated one (closed form, any position)."""
    kc, vc, kn, vn, q = _append_case(62, G=1)
    sl = np.array([0, 5, 8], dtype=np.int32)
    k2, _, _, q2, _ = oracle.kv_append(kc, vc, sl, kn, vn, q, rope_base=500.0)
    for b, L in enumerate(sl):
        for t in range(3):
            got = np.sum(q2[b, t] * k2[b, L + t], axis=-1)
            ref = np.sum(q[b, t].astype(np.float64) * kn[b, t].astype(np.float64), axis=-1)
            _close(got, ref, 1e-12, "same-position dot product")
    # and the rotation is not the identity away from position 0
    assert np.max(np.abs(k2[1, 5] - kn[1, 0])) > 1e-3


def pin_kv_append_chunks_compose():
    """Appending T tokens at once equals appending them in two chunks."""
    kc, vc, kn, vn, q = _append_case(63, T=5)
    sl = np.array([1, 0, 6], dtype=np.int32)
    a = oracle.kv_append(kc, vc, sl, kn, vn, q, rope_base=10000.0)
    k1, v1, s1, q1, _ = oracle.kv_append(kc, vc, sl, kn[:, :2], vn[:, :2], q[:, :2], rope_base=10000.0)
    k2, v2, s2, q2, _ = oracle.kv_append(k1.astype(np.float32), v1.astype(np.float32), s1, kn[:, 2:], vn[:, 2:],
                                         q[:, 2:], rope_base=10000.0)
    assert list(s2) == list(a[2])
    _close(k2, a[0], 2e-6, "keys (the first chunk's rows went through float32 once more)")
    _close(v2, a[1], 0.0, "values")
    _close(np.concatenate([q1, q2], axis=1), a[3], 0.0, "queries")


def pin_kv_append_then_decode_is_causal_prefill_row():
    """Append a whole sequence token by token into an empty cache (rotating each new q), decode
    the last query: equal to the last row of causal prefill with RoPE on the full sequence -- two
    independent paths of the oracle (append + decode against attn_fwd's own RoPE)."""
    B, S, Hkv, G, D, Smax = 2, 7, 2, 2, 8, 10
    kall = normal_f32(64, 0, (B, S, Hkv, D))
    vall = normal_f32(64, 1, (B, S, Hkv, D))
    qall = normal_f32(64, 2, (B, S, Hkv * G, D))
    kc = np.zeros((B, Smax, Hkv, D), dtype=np.float32)
    vc = np.zeros((B, Smax, Hkv, D), dtype=np.float32)
    sl = np.zeros(B, dtype=np.int32)
    for t in range(S):
        kc, vc, sl, qt, _ = oracle.kv_append(kc, vc, sl, kall[:, t:t + 1], vall[:, t:t + 1], qall[:, t:t + 1],
                                             rope_base=100.0)
        kc, vc = kc.astype(np.float32), vc.astype(np.float32)
    o_dec, l_dec = oracle.decode(qt[:, 0], kc, vc, sl, 0.4)
    o_pf, l_pf = oracle.attn_fwd(qall, kall, vall, 0.4, True, rope_base=100.0, q_pos0=0)
    _close(o_dec, o_pf[:, S - 1], 1e-6, "decode after append = last causal row (O)")
    _close(l_dec, l_pf[:, :, S - 1], 1e-6, "decode after append = last causal row (LSE)")


def pin_kv_append_overflow():
    """A sequence whose append would pass Smax (or with a negative length) is left untouched and
    reported; the others are appended."""
    kc, vc, kn, vn, q = _append_case(65)
    sl = np.array([9, 10, -1], dtype=np.int32)          # Smax 12, T 3: 9 fits, 10 and -1 do not
    k2, v2, s2, q2, ovf = oracle.kv_append(kc, vc, sl, kn, vn, q, rope_base=10000.0)
    assert list(ovf) == [False, True, True] and list(s2) == [12, 10, -1]
    for b in (1, 2):
        _close(k2[b], kc[b], 0.0, "overflowing sequence keys untouched")
        _close(v2[b], vc[b], 0.0, "overflowing sequence values untouched")
        _close(q2[b], q[b], 0.0, "overflowing sequence queries untouched")


def _grid(x, step=2.0 ** -12):
    """Round to a 2^-12 grid so that x +- 2^-10 is exact in float32 (finite differences)."""
    return (np.round(np.asarray(x, dtype=np.float64) / step) * step).astype(np.float32)


def _fd_grads(q, k, v, g, scale, causal, rope_base=0.0, q_pos0=0, eps=2.0 ** -10):
    """Central differences of L = sum(o * g) through the forward oracle, every input element."""
    def loss(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, scale, causal, rope_base, q_pos0)
        return float(np.sum(o * g.astype(np.float64)))
    out = []
    for which in range(3):
        xs = [q.copy(), k.copy(), v.copy()]
        grad = np.zeros(xs[which].shape, dtype=np.float64)
        flat = xs[which].reshape(-1)
        for idx in range(flat.size):
            x0 = flat[idx]
            flat[idx] = x0 + np.float32(eps)
            lp = loss(*xs)
            flat[idx] = x0 - np.float32(eps)
            lm = loss(*xs)
            flat[idx] = x0
            grad.reshape(-1)[idx] = (lp - lm) / (2 * eps)
        out.append(grad)
    return out


def pin_backward_matches_finite_differences():
    """dq, dk, dv of the backward oracle equal central differences of the *forward* oracle's
    L = sum(o * dout) -- non-causal MHA, bottom-right causal GQA with Sq < Skv and a fully
    masked row (Sq > Skv), and RoPE with a query offset."""
    cases = [
        dict(B=1, Sq=4, Skv=5, Hq=2, Hkv=2, D=4, scale=0.7, causal=False),
        dict(B=2, Sq=3, Skv=5, Hq=4, Hkv=2, D=4, scale=0.5, causal=True),
        dict(B=1, Sq=5, Skv=3, Hq=2, Hkv=1, D=4, scale=0.9, causal=True),       # row 0, 1 fully masked
        dict(B=1, Sq=3, Skv=4, Hq=2, Hkv=1, D=6, scale=0.6, causal=True, rope_base=50.0, q_pos0=1),
    ]
    for n, c in enumerate(cases):
        q = _grid(normal_f32(81 + n, 0, (c["B"], c["Sq"], c["Hq"], c["D"])))
        k = _grid(normal_f32(81 + n, 1, (c["B"], c["Skv"], c["Hkv"], c["D"])))
        v = _grid(normal_f32(81 + n, 2, (c["B"], c["Skv"], c["Hkv"], c["D"])))
        g = _grid(normal_f32(81 + n, 3, (c["B"], c["Sq"], c["Hq"], c["D"])))
        rb, qp = c.get("rope_base", 0.0), c.get("q_pos0", 0)
        dq, dk, dv = oracle.attn_bwd(q, k, v, g, c["scale"], c["causal"], rb, qp)
        fq, fk, fv = _fd_grads(q, k, v, g, c["scale"], c["causal"], rb, qp)
        for name, a, b in (("dq", dq, fq), ("dk", dk, fk), ("dv", dv, fv)):
            _close(a, b, 2e-6 * max(1.0, float(np.max(np.abs(b)))), f"case {n} {name} vs finite differences")


def pin_masked_backward_matches_finite_differences():
    """The masked backward equals central differences of the masked *forward* oracle (per-head
    mask with -inf entries, causal, GQA), and a zero mask gives the unmasked backward."""
    B, Sq, Skv, Hq, Hkv, D = 1, 4, 5, 2, 1, 4
    q = _grid(normal_f32(97, 0, (B, Sq, Hq, D)))
    k = _grid(normal_f32(97, 1, (B, Skv, Hkv, D)))
    v = _grid(normal_f32(97, 2, (B, Skv, Hkv, D)))
    g = _grid(normal_f32(97, 3, (B, Sq, Hq, D)))
    m = _grid(normal_f32(97, 4, (B, Hq, Sq, Skv)))
    m[0, 1, 2, 0] = -np.inf
    m[0, 0, 3, :] = -np.inf                               # a row masked everywhere
    dq, dk, dv = oracle.attn_bwd_masked(q, k, v, g, m, 0.6, True)

    def loss(qq, kk, vv):
        o, _ = oracle.attn_fwd_masked(qq, kk, vv, m, 0.6, True)
        return float(np.sum(o * g.astype(np.float64)))
    eps = 2.0 ** -10
    for which, ref in enumerate((dq, dk, dv)):
        xs = [q.copy(), k.copy(), v.copy()]
        flat = xs[which].reshape(-1)
        fd = np.zeros(flat.size)
        for idx in range(flat.size):
            x0 = flat[idx]
            flat[idx] = x0 + np.float32(eps)
            lp = loss(*xs)
            flat[idx] = x0 - np.float32(eps)
            lm = loss(*xs)
            flat[idx] = x0
            fd[idx] = (lp - lm) / (2 * eps)
        _close(ref.reshape(-1), fd, 2e-6 * max(1.0, float(np.max(np.abs(fd)))), f"masked backward {which}")
    z = oracle.attn_bwd_masked(q, k, v, g, np.zeros((Sq, Skv), np.float32), 0.6, True)
    for a, b in zip(z, oracle.attn_bwd(q, k, v, g, 0.6, True)):
        _close(a, b, 1e-15, "zero mask backward")


def pin_backward_invariants():
    """Without RoPE each row's dS sums to zero, so the key gradients of a (b, kv head) sum to
    zero; each row's probabilities sum to one, so the value gradients sum to the sum of dout over
    rows with a visible key; GQA gradients equal MHA gradients on repeated kv heads, with the
    kv-head gradients summed over the group."""
    B, Sq, Skv, Hq, Hkv, D = 2, 7, 9, 4, 2, 8
    q = normal_f32(91, 0, (B, Sq, Hq, D))
    k = normal_f32(91, 1, (B, Skv, Hkv, D))
    v = normal_f32(91, 2, (B, Skv, Hkv, D))
    g = normal_f32(91, 3, (B, Sq, Hq, D))
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, 0.4, True)
    _close(np.sum(dk, axis=1), np.zeros((B, Hkv, D)), 1e-12, "sum over keys of dk")
    G = Hq // Hkv
    gsum = np.sum(g.astype(np.float64).reshape(B, Sq, Hkv, G, D), axis=(1, 3))
    _close(np.sum(dv, axis=1), gsum, 1e-12, "sum over keys of dv = sum of dout")
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    mq, mk, mv = oracle.attn_bwd(q, kr, vr, g, 0.4, True)
    _close(dq, mq, 1e-12, "GQA dq = MHA dq")
    _close(dk, mk.reshape(B, Skv, Hkv, G, D).sum(axis=3), 1e-12, "GQA dk = summed MHA dk")
    _close(dv, mv.reshape(B, Skv, Hkv, G, D).sum(axis=3), 1e-12, "GQA dv = summed MHA dv")


def pin_sampled_backward_matches_full_backward():
    """The sampled backward of one (batch, kv head) group (used to check full-size problems)
    equals the full backward at its rows and keys: GQA with RoPE at a query offset and causal
    rows that see no key (Sq > Skv), and a non-causal MQA case."""
    for seed, (B, Hq, Hkv, Sq, Skv, D, causal, rb, qp) in ((93, (2, 4, 2, 37, 29, 16, True, 10000.0, 16)),
                                                            (94, (1, 3, 1, 40, 40, 8, False, 0.0, 0))):
        q = normal_f32(seed, 0, (B, Sq, Hq, D))
        k = normal_f32(seed, 1, (B, Skv, Hkv, D))
        v = normal_f32(seed, 2, (B, Skv, Hkv, D))
        g = normal_f32(seed, 3, (B, Sq, Hq, D))
        dq, dk, dv = oracle.attn_bwd(q, k, v, g, 0.3, causal, rb, qp)
        G = Hq // Hkv
        rows, keys = np.array([0, 5, Sq - 1]), np.array([0, 7, Skv - 1])
        for b in range(B):
            for kvh in range(Hkv):
                sq, sk, sv = oracle.attn_bwd_sampled(q, k, v, g, 0.3, causal, rb, qp, b, kvh, rows, keys)
                for hg in range(G):
                    _close(sq[hg], dq[b, rows, kvh * G + hg], 1e-12, "sampled dq")
                _close(sk, dk[b, keys, kvh], 1e-12, "sampled dk")
                _close(sv, dv[b, keys, kvh], 1e-12, "sampled dv")


def pin_additive_mask():
    """An additive mask of zeros changes nothing; -inf above the diagonal is the causal mask; a
    constant mask c leaves o unchanged and adds c to lse; -inf on one key equals attention
    without that key; a per-head mask [B, Hq, Sq, Skv] acts head by head; a row masked
    everywhere gives o = 0, lse = -inf; and a tiny case against the pure-Python brute force."""
    B, Sq, Skv, Hq, Hkv, D = 2, 6, 7, 4, 2, 8
    q = normal_f32(95, 0, (B, Sq, Hq, D))
    k = normal_f32(95, 1, (B, Skv, Hkv, D))
    v = normal_f32(95, 2, (B, Skv, Hkv, D))
    o0, l0 = oracle.attn_fwd(q, k, v, 0.4, False)
    o, l = oracle.attn_fwd_masked(q, k, v, np.zeros((Sq, Skv), np.float32), 0.4, False)
    _close(o, o0, 1e-15, "zero mask")
    _close(l, l0, 1e-15, "zero mask lse")
    tri = np.where(np.arange(Skv)[None, :] > np.arange(Sq)[:, None] + (Skv - Sq), -np.inf, 0.0).astype(np.float32)
    oc, lc = oracle.attn_fwd(q, k, v, 0.4, True)
    o, l = oracle.attn_fwd_masked(q, k, v, tri, 0.4, False)
    _close(o, oc, 1e-14, "triangular -inf mask = causal")
    _close(l, lc, 1e-14, "triangular -inf mask = causal (lse)")
    o, l = oracle.attn_fwd_masked(q, k, v, np.full((B, Sq, Skv), 1.75, np.float32), 0.4, False)
    _close(o, o0, 1e-14, "constant mask leaves o")
    _close(l, l0 + 1.75, 1e-14, "constant mask shifts lse")
    mk = np.zeros((Sq, Skv), np.float32)
    mk[:, 3] = -np.inf
    keep = [j for j in range(Skv) if j != 3]
    o, l = oracle.attn_fwd_masked(q, k, v, mk, 0.4, False)
    ok_, lk = oracle.attn_fwd(q, k[:, keep], v[:, keep], 0.4, False)
    _close(o, ok_, 1e-14, "-inf on a key removes it")
    _close(l, lk, 1e-14, "-inf on a key removes it (lse)")
    mh = normal_f32(95, 3, (B, Hq, Sq, Skv))
    o, l = oracle.attn_fwd_masked(q, k, v, mh, 0.4, True)
    for h in range(Hq):
        oh, lh = oracle.attn_fwd_masked(q[:, :, h:h + 1], k[:, :, h // 2:h // 2 + 1], v[:, :, h // 2:h // 2 + 1],
                                        mh[:, h], 0.4, True)
        _close(o[:, :, h], oh[:, :, 0], 1e-14, "per-head mask")
        _close(l[:, h], lh[:, 0], 1e-14, "per-head mask lse")
    mrow = np.zeros((Sq, Skv), np.float32)
    mrow[2, :] = -np.inf
    o, l = oracle.attn_fwd_masked(q, k, v, mrow, 0.4, False)
    assert np.all(o[:, 2] == 0.0) and np.all(l[:, :, 2] == -np.inf)
    # brute force: the mask enters as an additive term on the scaled score
    q1, k1, v1 = q[:1, :3, :1], k[:1, :4, :1], v[:1, :4, :1]
    m1 = normal_f32(95, 4, (3, 4))
    o, l = oracle.attn_fwd_masked(q1, k1, v1, m1, 0.7, False)
    for i in range(3):
        s = [0.7 * float(np.dot(q1[0, i, 0].astype(np.float64), k1[0, j, 0].astype(np.float64))) + float(m1[i, j])
             for j in range(4)]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        ref = sum(wj * v1[0, j, 0].astype(np.float64) for j, wj in enumerate(w)) / sum(w)
        _close(o[0, i, 0], ref, 1e-12, "mask brute force")
        _close(l[0, 0, i], mx + math.log(sum(w)), 1e-12, "mask brute force lse")


ALL_PINS = [obj for name, obj in sorted(globals().items()) if name.startswith("pin_")]
