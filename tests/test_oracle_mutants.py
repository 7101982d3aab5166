"""Every plausible mistake planted in a copy of the oracle's C source must fail at least
one pin (CPU only).  The copy is compiled into a temporary library; the real oracle
source is never modified."""
import os
import subprocess

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

# (name, original text, planted text) -- each original must occur in the source.
# Dropping the tiled recurrence's "running max is -inf" guard is not listed: with prefix
# (causal) visibility a row meets an all-masked key block before a visible one only when it
# has no visible key at all, and then the final "l > 0" test already yields O = 0, LSE = -inf,
# so that mutant computes the same function.
MUTANTS = [
    ("rope_sign", "x[2 * i] = x0 * c - x1 * s;", "x[2 * i] = x0 * c + x1 * s;"),
    ("rope_frequency", "pow(base, 2.0 * (double)i / (double)D)", "pow(base, (double)i / (double)D)"),
    ("rope_q_offset", "(double)q_pos0 + (double)i", "(double)i"),
    ("rope_on_values", "gather_head(v, b, kvh, Skv, Hkv, D, 0.0, Vd);",
     "gather_head(v, b, kvh, Skv, Hkv, D, rope_base, Vd);"),
    ("drop_scale", "s[j] = scale * dot;", "s[j] = dot;"),
    ("causal_off_by_one", "(long)(Skv - Sq) + 1;", "(long)(Skv - Sq);"),
    ("causal_top_left", "long n = (long)i + (long)(Skv - Sq) + 1;", "long n = (long)i + 1;"),
    ("lse_without_max", "*lse = m + log(l);", "*lse = log(l);"),
    ("no_normalisation", "double p = exp(s[j] - m) / l;", "double p = exp(s[j] - m);"),
    ("values_from_keys", "o[d] += p * V[(long)j * D + d];", "o[d] += p * K[(long)j * D + d];"),
    ("gqa_head_zero", "gather_head(k, b, kvh, Skv, Hkv, D, rope_base, Kd);",
     "gather_head(k, b, 0, Skv, Hkv, D, rope_base, Kd);"),
    ("masked_row_lse_zero", "        *lse = -INFINITY;\n        return;\n    }\n    for (int j = 0; j < Skv",
     "        *lse = 0.0;\n        return;\n    }\n    for (int j = 0; j < Skv"),
    ("combine_weight_max", "double w = exp(lses[t] - L);", "double w = exp(lses[t] - gmax);"),
    ("split_drops_remainder", "int len = base + (t < rem ? 1 : 0);", "int len = base;"),
    ("tiled_no_correction", "for (int d = 0; d < D; ++d) acc[(long)i * D + d] *= c;", ""),
    ("decode_drops_last_key", "attn_row(qq, Kd, Vd, L, D, L, scale", "attn_row(qq, Kd, Vd, L, D, L - 1, scale"),
    # backward
    ("bwd_dq_no_scale", "dqr[d] += scale * dS * Kd[(long)j * D + d];", "dqr[d] += dS * Kd[(long)j * D + d];"),
    ("bwd_no_dsum", "const double dS = p[j] * (dP[j] - Dsum);", "const double dS = p[j] * dP[j];"),
    ("bwd_dv_from_ds", "dVa[(long)j * D + d] += p[j] * go[d];", "dVa[(long)j * D + d] += p[j] * dP[j] * go[d];"),
    ("bwd_dk_rope_not_undone", "if (rope_base > 0.0) rope_vec(dkr, -(double)j, D, rope_base);",
     "if (rope_base > 0.0) rope_vec(dkr, (double)j, D, rope_base);"),
    ("bwd_dq_rope_not_undone", "if (rope_base > 0.0) rope_vec(dqr, -((double)q_pos0 + (double)i), D, rope_base);", ""),
    ("mask_before_scale", "s[j] = scale * dot + (double)mrow[j];", "s[j] = scale * (dot + (double)mrow[j]);"),
    ("mask_head_stride_ignored", "(long)hq * mask_hstride", "(long)0 * mask_hstride"),
    ("mask_all_inf_row_nan", "if (m == -INFINITY) {\n                            *lrow = -INFINITY;",
     "if (0) {\n                            *lrow = -INFINITY;"),
    ("bwd_mask_dropped", "s[j] = scale * dot + (mrow ? (double)mrow[j] : 0.0);", "s[j] = scale * dot;"),
    ("bwd_dp_from_keys", "for (int d = 0; d < D; ++d) dot += go[d] * Vd[(long)j * D + d];",
     "for (int d = 0; d < D; ++d) dot += go[d] * Kd[(long)j * D + d];"),
]


@pytest.mark.parametrize("name,orig,planted", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_planted_mistake(name, orig, planted, tmp_path):
    src = open(SRC).read()
    assert src.count(orig) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(orig, planted, 1)
    c_path = tmp_path / f"oracle_{name}.c"
    so_path = tmp_path / f"liboracle_{name}.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(c_path),
                           "-o", str(so_path), "-lm"])
    failed = []
    oracle.swap_library(str(so_path))
    try:
        for pin in ALL_PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError, FloatingPointError, ValueError):
                failed.append(pin.__name__)
    finally:
        oracle.swap_library(None)
    assert failed, f"planted mistake {name!r} passed every pin"


# Planted mistakes in the Python-level cache append (oracle.kv_append): each is a source edit of
# the function, applied to a copy that temporarily replaces it.
import inspect
import textwrap

APPEND_MUTANTS = [
    ("append_position_off_by_one", "pos = np.arange(L, L + T, dtype=np.int32)",
     "pos = np.arange(L + 1, L + T + 1, dtype=np.int32)"),
    ("append_rows_shifted", "kc[b, L:L + T] = rope(", "kc[b, L + 1:L + T + 1] = rope("),
    ("append_length_not_advanced", "sl[b] = L + T", "sl[b] = L"),
    ("append_q_not_rotated", "qo[b] = rope(qo[b], pos, rope_base)", "pass"),
    ("append_overflow_ignored", "if L < 0 or L + T > Smax:", "if L < 0:"),
    ("append_positions_from_zero", "pos = np.arange(L, L + T, dtype=np.int32)",
     "pos = np.arange(0, T, dtype=np.int32)"),
]


@pytest.mark.parametrize("name,orig,planted", APPEND_MUTANTS, ids=[m[0] for m in APPEND_MUTANTS])
def test_pins_reject_planted_append_mistake(name, orig, planted):
    src = textwrap.dedent(inspect.getsource(oracle.kv_append))
    assert src.count(orig) == 1, f"mutation site for {name} not found"
    ns = dict(vars(oracle))
    exec(src.replace(orig, planted, 1), ns)
    real = oracle.kv_append
    oracle.kv_append = ns["kv_append"]
    failed = []
    try:
        for pin in ALL_PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError, FloatingPointError, ValueError, IndexError):
                failed.append(pin.__name__)
    finally:
        oracle.kv_append = real
    assert failed, f"planted mistake {name!r} passed every pin"
