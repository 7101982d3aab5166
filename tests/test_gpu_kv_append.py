"""attn_kv_append (fused decode-step cache update) against the fp64 oracle: cache rows and
rotated queries within one bf16 ulp of the oracle's rotation, values and lengths exact,
overflowing sequences untouched and flagged, and a decode after the append matching the oracle's
append + decode."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_BF16_LSE, TOL_BF16_O, bits_to_dev, compare, to_host_f64

pytestmark = pytest.mark.gpu


def _bf16(seed, stream, shape):
    bits, vals = si.bf16_normal(seed, stream, shape)
    return bits, vals


def _within_one_ulp(got, ref):
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    return (np.abs(got - ref) <= ulp + 1e-6).all(), np.max(np.abs(got - ref) / ulp)


def _case(seed, B, T, Hq, Hkv, D, Smax, lens):
    kc_b, kc = _bf16(seed, 0, (B, Smax, Hkv, D))
    vc_b, vc = _bf16(seed, 1, (B, Smax, Hkv, D))
    kn_b, kn = _bf16(seed, 2, (B, T, Hkv, D))
    vn_b, vn = _bf16(seed, 3, (B, T, Hkv, D))
    q_b, q = _bf16(seed, 4, (B, T, Hq, D))
    sl = np.array(lens, dtype=np.int32)
    return (kc_b, vc_b, kn_b, vn_b, q_b), (kc, vc, kn, vn, q), sl


@pytest.mark.parametrize("B,T,Hq,Hkv,D,Smax,lens,base", [
    (3, 1, 8, 2, 64, 40, [0, 17, 39], 10000.0),
    (2, 5, 32, 8, 64, 300, [123, 0], 10000.0),
    (4, 3, 16, 16, 128, 64, [5, 61, 30, 1], 500000.0),
    (2, 4, 4, 1, 64, 20, [3, 9], 0.0),
])
def test_kv_append_matches_oracle(B, T, Hq, Hkv, D, Smax, lens, base):
    bits, vals, sl = _case(7 + T + D, B, T, Hq, Hkv, D, Smax, lens)
    kc_d, vc_d, kn_d, vn_d, q_d = (bits_to_dev(x) for x in bits)
    sl_d = torch.from_numpy(sl).cuda()
    ea.kv_append(kc_d, vc_d, sl_d, kn_d, vn_d, q=q_d, rope_base=base)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    kc_r, vc_r, sl_r, q_r, ovf = oracle.kv_append(*vals[:2], sl, vals[2], vals[3], vals[4], rope_base=base)
    assert not ovf.any()
    assert (sl_d.cpu().numpy() == sl_r).all()
    # values are a copy: bit-exact; so are untouched key rows
    assert (vc_d.view(torch.int16).cpu().numpy().view(np.uint16) == si.f32_to_bf16_bits(vc_r.astype(np.float32))).all()
    ok, worst = _within_one_ulp(kc_d.float().cpu().numpy().astype(np.float64), kc_r)
    assert ok, worst
    ok, worst = _within_one_ulp(q_d.float().cpu().numpy().astype(np.float64), q_r)
    assert ok, worst


def test_kv_append_overflow_is_flagged_and_skipped():
    B, T, Hq, Hkv, D, Smax = 3, 4, 8, 2, 64, 32
    bits, vals, sl = _case(71, B, T, Hq, Hkv, D, Smax, [28, 29, 10])      # sequence 1 would pass Smax
    kc_d, vc_d, kn_d, vn_d, q_d = (bits_to_dev(x) for x in bits)
    sl_d = torch.from_numpy(sl).cuda()
    ea.kv_append(kc_d, vc_d, sl_d, kn_d, vn_d, q=q_d, rope_base=10000.0)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 8
    kc_r, vc_r, sl_r, q_r, ovf = oracle.kv_append(*vals[:2], sl, vals[2], vals[3], vals[4], rope_base=10000.0)
    assert list(ovf) == [False, True, False]
    assert list(sl_d.cpu().numpy()) == [32, 29, 14] == list(sl_r)
    # the skipped sequence keeps its cache rows and its queries bit for bit
    kc_g = kc_d.view(torch.int16).cpu().numpy().view(np.uint16)
    q_g = q_d.view(torch.int16).cpu().numpy().view(np.uint16)
    assert (kc_g[1] == bits[0][1]).all() and (q_g[1] == bits[4][1]).all()
    ok, _ = _within_one_ulp(kc_d.float().cpu().numpy().astype(np.float64), kc_r)
    assert ok


def test_decode_step_after_append_matches_oracle():
    """One decode step on a long ragged cache: rotate + append the new token, then split-KV decode
    with the advanced lengths, against the oracle's append (rounded to bf16 storage) + decode."""
    B, Hq, Hkv, D, Smax = 4, 32, 8, 64, 5000
    scale = 0.125
    lens = np.array([4000, 1, 2999, 4998], dtype=np.int32)
    w = si.Decode("append_step", B, Hq, Hkv, D, Smax, 1, Smax, scale, 16, seed=72)
    d = si.decode_inputs(w, fill_tail_nan=True, seqlens=lens)
    kn_b, kn = _bf16(73, 2, (B, 1, Hkv, D))
    vn_b, vn = _bf16(73, 3, (B, 1, Hkv, D))
    q_b, q = _bf16(73, 4, (B, 1, Hq, D))
    kc_d, vc_d = bits_to_dev(d["k_bits"]), bits_to_dev(d["v_bits"])
    kn_d, vn_d, q_d = bits_to_dev(kn_b), bits_to_dev(vn_b), bits_to_dev(q_b)
    sl_d = torch.from_numpy(lens.copy()).cuda()
    ea.kv_append(kc_d, vc_d, sl_d, kn_d, vn_d, q=q_d, rope_base=10000.0)
    o, lse = ea.attn_decode(q_d.view(B, Hq, D), kc_d, vc_d, sl_d, scale, w.num_splits, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.read_device_status() == 0
    # oracle: the cache as stored (bf16), the append in fp64, stored back as bf16
    kc = si.bf16_bits_to_f32(d["k_bits"])
    vc = si.bf16_bits_to_f32(d["v_bits"])
    kc_r, vc_r, sl_r, q_r, _ = oracle.kv_append(kc, vc, lens, kn, vn, q, rope_base=10000.0)
    to_bf16 = lambda a: si.bf16_bits_to_f32(si.f32_to_bf16_bits(a.astype(np.float32)))
    o_ref, l_ref = oracle.decode(to_bf16(q_r)[:, 0], to_bf16(kc_r), vc_r.astype(np.float32), sl_r, scale)
    compare(to_host_f64(o), o_ref, to_host_f64(lse), l_ref, TOL_BF16_O, TOL_BF16_LSE, "decode after append")
