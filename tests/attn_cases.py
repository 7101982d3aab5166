"""Shared helpers for the GPU parity tests: seeded inputs -> device tensors, oracle references."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import seeded_inputs as si

# tolerances stated for the path: fp32 mode 1e-4 max abs; bf16 inputs with fp32 accumulation
# 1e-2 max abs on O and 1e-3 max abs on LSE
TOL_F32 = 1e-4
TOL_BF16_O = 1e-2
TOL_BF16_LSE = 1e-3


def bits_to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def make_prefill(w: si.Prefill):
    """Device q, k, v for workload w, plus the float32 host values the oracle reads."""
    x = si.prefill_inputs(w)
    if w.dtype == "fp32":
        dev = {n: torch.from_numpy(x[n]).cuda() for n in ("q", "k", "v")}
    else:
        dev = {n: bits_to_dev(x[n + "_bits"]) for n in ("q", "k", "v")}
    return x, dev


def compare(o_gpu: np.ndarray, o_ref: np.ndarray, lse_gpu, lse_ref, tol_o: float, tol_lse: float, what=""):
    """Element-wise comparison; rows with lse = -inf must match exactly (O = 0, LSE = -inf)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    err_o = np.max(np.abs(o_gpu - o_ref)) if o_ref.size else 0.0
    assert err_o <= tol_o, f"{what}: max |O - oracle| = {err_o:.3e} > {tol_o:.1e}"
    if lse_gpu is not None:
        lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
        ninf = np.isneginf(lse_ref)
        assert (np.isneginf(lse_gpu) == ninf).all(), f"{what}: -inf pattern of LSE differs"
        if (~ninf).any():
            err_l = np.max(np.abs(lse_gpu[~ninf] - lse_ref[~ninf]))
            assert err_l <= tol_lse, f"{what}: max |LSE - oracle| = {err_l:.3e} > {tol_lse:.1e}"
        return err_o, (np.max(np.abs(lse_gpu[~ninf] - lse_ref[~ninf])) if (~ninf).any() else 0.0)
    return err_o, None


def sample_rows(w: si.Prefill, n: int, seed: int = 0) -> np.ndarray:
    """Flat row ids (b*Hq + h)*Sq + i: random rows plus every tile's first/last rows and the ends."""
    rng = np.random.default_rng(seed)
    B, Hq, Sq = w.B, w.Hq, w.Sq
    rows = set(rng.integers(0, B * Hq * Sq, size=n).tolist())
    for b in (0, B - 1):
        for h in (0, Hq - 1, Hq // 2):
            for i in (0, 1, 127, 128, 255, 256, Sq // 2, Sq - 129, Sq - 128, Sq - 2, Sq - 1):
                if 0 <= i < Sq:
                    rows.add((b * Hq + h) * Sq + i)
    return np.array(sorted(rows), dtype=np.int64)


def gather_rows(o: np.ndarray, lse: np.ndarray, rows: np.ndarray, w: si.Prefill):
    b = rows // (w.Hq * w.Sq)
    h = (rows // w.Sq) % w.Hq
    i = rows % w.Sq
    return o[b, i, h], lse[b, h, i]


def to_host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)
