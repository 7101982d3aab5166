"""rope_apply parity against the fp64 oracle rotation (bf16 and fp32, several head dims/bases)."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import oracle
import seeded_inputs as si
from attn_cases import TOL_F32, bits_to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [8, 64, 128])
@pytest.mark.parametrize("base", [10000.0, 500000.0])
def test_rope_fp32(D, base):
    T, H = 37, 3
    x = si.normal_f32(3, 0, (T, H, D))
    pos = np.array(list(range(30)) + [100, 1000, 4095, 8191, 16383, 32767, 40000], dtype=np.int32)
    xd = torch.from_numpy(x).cuda()
    ea.rope_apply(xd, torch.from_numpy(pos).cuda(), base)
    torch.cuda.synchronize()
    ref = oracle.rope(x, pos, base)
    err = np.max(np.abs(xd.cpu().numpy().astype(np.float64) - ref))
    assert err <= TOL_F32, err


@pytest.mark.parametrize("D", [64, 128])
def test_rope_bf16_within_one_ulp(D):
    T, H = 50, 4
    bits, vals = si.bf16_normal(4, 0, (T, H, D))
    pos = np.arange(T, dtype=np.int32) * 97
    xd = bits_to_dev(bits)
    ea.rope_apply(xd, torch.from_numpy(pos).cuda(), 10000.0)
    torch.cuda.synchronize()
    ref = oracle.rope(vals, pos, 10000.0)
    got = xd.float().cpu().numpy().astype(np.float64)
    # the result is rounded to bf16: allow one bf16 ulp of the reference value
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert (np.abs(got - ref) <= ulp + 1e-6).all(), np.max(np.abs(got - ref) / ulp)
