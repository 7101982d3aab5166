"""The C ABI under CUDA-graph capture: a decode step (fused cache append + split-KV decode with
its programmatic-dependent combine) and a prefill (RoPE table, rotated K, tensor-core forward;
and a key-split forward with its combine) are captured once and replayed; every replay must
equal, bit for bit, the same calls made eagerly on copies of the same buffers."""
import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea

pytestmark = pytest.mark.gpu


def _bf16(shape, gen, scale=1.0):
    return (torch.randn(shape, generator=gen, device="cuda") * scale).to(torch.bfloat16)


def test_decode_step_replays_from_a_graph():
    gen = torch.Generator(device="cuda").manual_seed(11)
    B, Hq, Hkv, D, Smax, splits, steps = 4, 8, 2, 64, 2048, 8, 5
    scale = 1.0 / np.sqrt(D)
    kc = _bf16((B, Smax, Hkv, D), gen)
    vc = _bf16((B, Smax, Hkv, D), gen)
    sl = torch.tensor([300, 1000, 17, 1500], dtype=torch.int32, device="cuda")
    tokens = [(_bf16((B, 1, Hkv, D), gen), _bf16((B, 1, Hkv, D), gen), _bf16((B, 1, Hq, D), gen))
              for _ in range(steps)]
    # graph side: static inputs, outputs and workspace
    kg, vg, sg = kc.clone(), vc.clone(), sl.clone()
    kn, vn, qn = (torch.empty_like(t) for t in tokens[0])
    og = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    lg = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(ea.decode_workspace_bytes(B, Hq, D, splits), dtype=torch.uint8, device="cuda")

    def step(k, v, s, kn_, vn_, qn_, o, lse, w):
        ea.kv_append(k, v, s, kn_, vn_, q=qn_, rope_base=10000.0)
        ea.attn_decode(qn_.view(B, Hq, D), k, v, s, scale, splits, o=o, lse=lse, workspace=w)

    # warm-up on scratch copies (kernel attributes set outside the capture)
    step(kc.clone(), vc.clone(), sl.clone(), *(t.clone() for t in tokens[0]), og, lg, ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            step(kg, vg, sg, kn, vn, qn, og, lg, ws)
    torch.cuda.current_stream().wait_stream(side)

    ke, ve, se = kc.clone(), vc.clone(), sl.clone()
    oe = torch.empty_like(og)
    le = torch.empty_like(lg)
    for kt, vt, qt in tokens:
        kn.copy_(kt), vn.copy_(vt), qn.copy_(qt)
        g.replay()
        qe = qt.clone()
        step(ke, ve, se, kt, vt, qe, oe, le, ws.clone())
        torch.cuda.synchronize()
        assert torch.equal(og, oe) and torch.equal(lg, le)
        assert torch.equal(qn, qe)                  # q rotated in place the same way
    assert torch.equal(sg, se) and torch.equal(sg, sl + steps)
    assert torch.equal(kg, ke) and torch.equal(vg, ve)
    assert ea.read_device_status() == 0
    del g


@pytest.mark.parametrize("shape", [
    # (B, Hq, Hkv, Sq, Skv, D, causal, rope_base, q_pos0): paired tiles with RoPE; key splits
    (4, 16, 4, 384, 384, 64, True, 10000.0, 0),       # 192 single tiles: paired heads
    (1, 4, 2, 128, 4096, 64, True, 0.0, 0),
    (1, 2, 2, 200, 1000, 128, False, 500000.0, 800),
], ids=["rope_paired", "key_split", "rope_key_split_d128"])
def test_prefill_replays_from_a_graph(shape):
    B, Hq, Hkv, Sq, Skv, D, causal, base, pos0 = shape
    gen = torch.Generator(device="cuda").manual_seed(12)
    scale = 1.0 / np.sqrt(D)
    q = _bf16((B, Sq, Hq, D), gen)
    k = _bf16((B, Skv, Hkv, D), gen)
    v = _bf16((B, Skv, Hkv, D), gen)
    need = ea.fwd_workspace_bytes(q, k, base, pos0, torch.float32)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    o = torch.empty((B, Sq, Hq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device="cuda")

    def fwd(o_, l_, w_):
        ea.attn_fwd_ex(q, k, v, scale, causal, base, pos0, o=o_, lse=l_, workspace=w_ if need > 0 else None)

    fwd(o, lse, ws)
    torch.cuda.synchronize()
    o_ref, l_ref = o.clone(), lse.clone()
    o.zero_(), lse.zero_()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fwd(o, lse, ws)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
        o.zero_(), lse.zero_()
    assert ea.read_device_status() == 0
    del g
