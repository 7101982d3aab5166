"""Failure detection without a GPU fault: a wait that can never complete ends, after its bound,
with a status bit the host reads -- the kernel returns, the context stays usable."""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_160_b200 as ea
import seeded_inputs as si
from attn_cases import make_prefill

pytestmark = pytest.mark.gpu


def test_unsatisfiable_wait_reports_timeout_and_context_survives():
    lib = ea.load_library()
    assert ea.read_device_status() == 0
    st = lib.attn_selftest_wait_timeout(10000, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert ea.read_device_status() == 1          # bit 1: a bounded wait gave up
    assert ea.read_device_status() == 0          # reading clears it
    # the context is still usable: a normal call runs and returns a clean status
    w = si.Prefill("after_timeout", "bf16", 1, 2, 2, 130, 130, 64, True, 0.125, seed=3)
    x, dev = make_prefill(w)
    o, lse = ea.attn_fwd(dev["q"], dev["k"], dev["v"], w.scale, True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert ea.read_device_status() == 0


def test_selftest_rejects_bad_bound():
    lib = ea.load_library()
    assert lib.attn_selftest_wait_timeout(0, None) == 1
    assert lib.attn_selftest_wait_timeout(2000000, None) == 1
