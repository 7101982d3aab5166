"""The Python binding checks what the C ABI cannot see (it takes pointers and sizes): shapes and
dtypes of the tensors it marshals.  These checks run before any device work, so they are tested
here with CPU tensors; well-formed CPU tensors get past them and stop at the CUDA-tensor check."""
import pytest
import torch

import exact_attention_160_b200 as ea

bf, f32 = torch.bfloat16, torch.float32


def t(*shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


@pytest.fixture(scope="module", autouse=True)
def lib():
    from exact_attention_160_b200 import build
    build.build()
    return ea.load_library()


def test_forward_checks_shapes_and_dtypes():
    q, k, v = t(1, 8, 4, 64), t(1, 16, 2, 64), t(1, 16, 2, 64)
    with pytest.raises(TypeError, match="share one dtype"):
        ea.attn_fwd(q, t(1, 16, 2, 64, dtype=f32), v, 0.125, True)
    with pytest.raises(ValueError, match="differ"):
        ea.attn_fwd(q, k, t(1, 15, 2, 64), 0.125, True)
    with pytest.raises(ValueError, match="batch or the head dim"):
        ea.attn_fwd(q, t(2, 16, 2, 64), t(2, 16, 2, 64), 0.125, True)
    with pytest.raises(ValueError, match="batch or the head dim"):
        ea.attn_fwd(q, t(1, 16, 2, 32), t(1, 16, 2, 32), 0.125, True)
    with pytest.raises(ValueError, match=r"\[B, S, H, D\]"):
        ea.attn_fwd(t(8, 4, 64), k, v, 0.125, True)
    with pytest.raises(ValueError, match="q's shape"):
        ea.attn_fwd(q, k, v, 0.125, True, o=t(1, 8, 4, 32))
    with pytest.raises(ValueError, match="lse must be float32"):
        ea.attn_fwd(q, k, v, 0.125, True, lse=t(1, 4, 8, dtype=bf))
    with pytest.raises(ValueError, match="lse must be float32"):
        ea.attn_fwd(q, k, v, 0.125, True, lse=t(1, 8, 4, dtype=f32))
    with pytest.raises(ValueError, match="CUDA tensors"):       # well formed: on to the device check
        ea.attn_fwd(q, k, v, 0.125, True, o=t(1, 8, 4, 64, dtype=f32), lse=t(1, 4, 8, dtype=f32))
    mask = t(8, 16, dtype=f32)
    with pytest.raises(TypeError, match="share one dtype"):
        ea.attn_fwd_masked(q, k, t(1, 16, 2, 64, dtype=f32), mask, 0.125, False)


def test_backward_checks_o_and_dout():
    q, k, v = t(1, 8, 4, 64), t(1, 16, 2, 64), t(1, 16, 2, 64)
    lse = t(1, 4, 8, dtype=f32)
    with pytest.raises(TypeError, match="q's dtype"):
        ea.attn_bwd(q, k, v, t(1, 8, 4, 64, dtype=f32), lse, t(1, 8, 4, 64), 0.125, True)
    with pytest.raises(TypeError, match="q's dtype"):
        ea.attn_bwd(q, k, v, t(1, 8, 4, 64), lse, t(1, 8, 4, 64, dtype=f32), 0.125, True)
    with pytest.raises(ValueError, match="q's shape"):
        ea.attn_bwd(q, k, v, t(1, 8, 4, 64), lse, t(1, 7, 4, 64), 0.125, True)
    with pytest.raises(ValueError, match="lse must be float32"):
        ea.attn_bwd(q, k, v, t(1, 8, 4, 64), t(1, 8, 4, dtype=f32), t(1, 8, 4, 64), 0.125, True)
    qf, kf, vf = (x.float() for x in (q, k, v))
    with pytest.raises(TypeError, match="fp32 gradients"):
        ea.attn_bwd_masked(qf, kf, vf, t(8, 16, dtype=f32), t(1, 8, 4, 64, dtype=f32), lse,
                           t(1, 8, 4, 64, dtype=f32), 0.125, True, grad_dtype=bf)


def test_decode_checks_shapes_and_dtypes():
    q, kc, vc = t(2, 8, 64), t(2, 100, 2, 64), t(2, 100, 2, 64)
    sl = t(2, dtype=torch.int32)
    with pytest.raises(ValueError, match=r"\[B, Hq, D\]"):
        ea.attn_decode(t(2, 1, 8, 64), kc, vc, sl, 0.125, 4)
    with pytest.raises(ValueError, match=r"\[B, Hq, D\]"):
        ea.attn_decode(q, kc, t(2, 99, 2, 64), sl, 0.125, 4)
    with pytest.raises(ValueError, match="batch or the head dim"):
        ea.attn_decode(t(3, 8, 64), kc, vc, t(3, dtype=torch.int32), 0.125, 4)
    with pytest.raises(TypeError, match="bf16"):
        ea.attn_decode(q.float(), kc.float(), vc.float(), sl, 0.125, 4)
    with pytest.raises(ValueError, match="seqlens must be int32"):
        ea.attn_decode(q, kc, vc, t(2, dtype=torch.int64), 0.125, 4)
    with pytest.raises(ValueError, match="seqlens must be int32"):
        ea.attn_decode(q, kc, vc, t(3, dtype=torch.int32), 0.125, 4)
    with pytest.raises(ValueError, match="lse must be float32"):
        ea.attn_decode(q, kc, vc, sl, 0.125, 4, lse=t(2, 8, 1, dtype=f32))
    with pytest.raises(ValueError, match="CUDA tensors"):
        ea.attn_decode(q, kc, vc, sl, 0.125, 4)


def test_rope_and_append_check_shapes():
    with pytest.raises(ValueError, match="pos int32"):
        ea.rope_apply(t(5, 2, 64, dtype=f32), t(5, dtype=torch.int64), 1e4)
    with pytest.raises(ValueError, match="pos int32"):
        ea.rope_apply(t(5, 2, 64, dtype=f32), t(4, dtype=torch.int32), 1e4)
    kc, vc, sl = t(2, 100, 2, 64), t(2, 100, 2, 64), t(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="do not fit"):
        ea.kv_append(kc, vc, sl, t(2, 1, 2, 32), t(2, 1, 2, 32))
    with pytest.raises(ValueError, match="one shape each"):
        ea.kv_append(kc, vc, sl, t(2, 1, 2, 64), t(2, 2, 2, 64))
    with pytest.raises(ValueError, match=r"q must be \[B, T, Hq, D\]"):
        ea.kv_append(kc, vc, sl, t(2, 1, 2, 64), t(2, 1, 2, 64), q=t(2, 2, 8, 64))
    with pytest.raises(ValueError, match="seqlens must be"):
        ea.kv_append(kc, vc, t(3, dtype=torch.int32), t(2, 1, 2, 64), t(2, 1, 2, 64))
