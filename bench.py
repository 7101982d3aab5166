"""Benchmark of the exact-attention hot path on B200.

Headline workload (one GPU, the largest single-GPU configuration): long-context causal prefill
with peaked scores, bf16 inputs / fp32 accumulation, B=1, Hq=Hkv=16, S=16384, D=128, scale
1/sqrt(128), q and k ~ N(0, 3^2), v ~ N(0, 1) (synthetic, seeded).  A step is one attn_fwd_ex
call over that batch; `value` is its prefill rate in TFLOP/s (4 D FLOP per unmasked pair).

The same JSON line carries every other configuration, each timed on its own with its own
roofline and oracle CPU baseline (`configs`): the fp32 single-head parity case, MHA causal
prefill (D=64), GQA 32/8 causal prefill with RoPE, the split-KV decode (B=16, Hq=32, Hkv=8,
Smax=32768, lengths uniform in [1024, 32768]) with its fused cache append, the Whisper-encoder
shape, a chunked prefill against a cache, and the masked forward; and the backward (`backward`)
of three of the prefill workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
                    [--headline-only] [--no-cpu-baseline]

--impl reference times the fp64 CPU oracle (the deliberately slow reference definition) on a
bounded sample of the same workload, on this machine's host cores.

Multi-GPU (launched by torch.distributed.run): the path has no exchange step, so each rank runs an
independent replica of the workload on its own GPU ("replicas only"); value = work of all ranks
divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import seeded_inputs as si  # noqa: E402

METRIC = "prefill attn TFLOP/s & decode KV-read GB/s, % of B200 roofline"
L2_FLUSH_BYTES = 256 << 20          # > 126 MB of L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------------
# ranks
# ------------------------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(x: float, dist, device) -> float:
    """Maximum of a per-rank scalar over all ranks (identity on one rank)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_rank: float, ms_max: float, world: int) -> float:
    """Units per second of the whole job: every rank (replica) did work_per_rank units, the
    slowest rank took ms_max milliseconds."""
    return world * work_per_rank / (ms_max * 1e-3)


def barrier(dist, device):
    if dist is not None:
        import torch
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons sampled every millisecond through NVML (read-only
    queries), so that even a timed region of a few milliseconds gets several samples; falls back
    to nvidia-smi every 200 ms where NVML is unavailable."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_s: float = 0.001):
        self.idx = gpu_index
        self.period = period_s
        self.samples = []          # (sm_mhz, max_mhz, set of reason names)
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._nvml = None
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(gpu_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self._nvml = pynvml
        except Exception:
            self._nvml = None

    def _query(self):
        if self._nvml is not None:
            n = self._nvml
            sm = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
            mx = n.nvmlDeviceGetMaxClockInfo(self._h, n.NVML_CLOCK_SM)
            bits = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            masks = (n.nvmlClocksEventReasonHwSlowdown, n.nvmlClocksEventReasonHwThermalSlowdown,
                     n.nvmlClocksEventReasonSwThermalSlowdown, n.nvmlClocksEventReasonSwPowerCap)
            return float(sm), float(mx), {name for name, m in zip(self.NAMES, masks) if bits & m}
        out = subprocess.run(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                              "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
        f = [x.strip() for x in out.stdout.strip().split(",")]
        return (float(f[0]), float(f[1]),
                {name for name, v in zip(self.NAMES, f[2:]) if v.lower() == "active"})

    def _run(self):
        period = self.period if self._nvml is not None else 0.2
        while not self._stop.is_set():
            try:
                self.samples.append(self._query())
            except Exception:
                pass
            self._stop.wait(period)

    def __enter__(self):
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)
        if not self.samples:
            try:
                self.samples.append(self._query())
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml" if self._nvml is not None else "nvidia-smi"}


# ------------------------------------------------------------------------------------------
# peaks and profile evidence
# ------------------------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profile_traffic(name: str):
    """Per-launch DRAM bytes recorded in profiles/<name>.md ('traffic_bytes_per_launch: N'), if the
    summary is current; None otherwise."""
    p = os.path.join(ROOT, "profiles", name + ".md")
    if not os.path.exists(p):
        return None
    for line in open(p):
        if line.strip().startswith("traffic_bytes_per_launch:"):
            v = line.split(":", 1)[1].strip()
            return None if v in ("null", "") else float(v)
    return None


# ------------------------------------------------------------------------------------------
# GPU measurement
# ------------------------------------------------------------------------------------------

def make_l2_flush(torch, device):
    """Cold-cache preparation run before every timed step, outside its events: write a buffer
    larger than L2 (evicting the step's inputs), then read another one of the same size so that
    L2 holds clean lines only and the step does not pay the write-back of the flush."""
    wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    rbuf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    sink = torch.empty((), dtype=torch.float32, device=device)

    def flush():
        wbuf.zero_()
        torch.sum(rbuf, dim=0, out=sink)
    return flush


L2_NOTE = "flushed before every timed step (256 MB written, then 256 MB of other data read)"


def dev_bf16(bits, torch):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def time_steps(fn, steps, warmup, flush, torch, dist, device):
    """W untimed warm-up steps, then K steps each bracketed by CUDA events on the launching
    stream, L2 flushed before each (outside the events).  Returns per-step ms (this rank)."""
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def time_e2e_pipelined(w, hq, hk, hv, o_like, lse_like, ws_like, steps, warmup, torch, ea, dist, device):
    """End to end through the public API, every step: pinned host q, k, v -> device, attn_fwd_ex,
    o and lse -> pinned host.  Consecutive steps alternate between two CUDA streams with their
    own buffers, so one step's device->host copy overlaps the next step's host->device copy
    (PCIe is full duplex) -- every byte of every step still crosses the bus inside the timed
    region.  Returns ms per step (this rank), CUDA events on the host-facing stream."""
    streams = [torch.cuda.Stream(device=device) for _ in range(2)]
    bufs = []
    for _ in range(2):
        bufs.append({
            "q": torch.empty(hq.shape, dtype=hq.dtype, device=device),
            "k": torch.empty(hk.shape, dtype=hk.dtype, device=device),
            "v": torch.empty(hv.shape, dtype=hv.dtype, device=device),
            "o": torch.empty(o_like.shape, dtype=o_like.dtype, device=device),
            "lse": torch.empty(lse_like.shape, dtype=lse_like.dtype, device=device),
            "ws": None if ws_like is None else torch.empty_like(ws_like),
            "ho": torch.empty(o_like.shape, dtype=o_like.dtype).pin_memory(),
            "hl": torch.empty(lse_like.shape, dtype=lse_like.dtype).pin_memory(),
        })

    def issue(i):
        st, b = streams[i % 2], bufs[i % 2]
        with torch.cuda.stream(st):
            b["q"].copy_(hq, non_blocking=True)
            b["k"].copy_(hk, non_blocking=True)
            b["v"].copy_(hv, non_blocking=True)
            ea.attn_fwd_ex(b["q"], b["k"], b["v"], w.scale, w.causal, w.rope_base, w.q_pos0, o=b["o"],
                           lse=b["lse"], workspace=b["ws"], stream=st)
            b["ho"].copy_(b["o"], non_blocking=True)
            b["hl"].copy_(b["lse"], non_blocking=True)

    for i in range(warmup):
        issue(i)
    torch.cuda.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    for st in streams:
        st.wait_event(a)
    for i in range(steps):
        issue(i)
    for st in streams:
        main.wait_stream(st)
    z.record(main)
    torch.cuda.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    return a.elapsed_time(z) / steps


def prefill_device_inputs(w: si.Prefill, torch):
    x = si.prefill_inputs(w)
    if w.dtype == "fp32":
        q, k, v = (torch.from_numpy(x[n]).cuda() for n in ("q", "k", "v"))
    else:
        q, k, v = (dev_bf16(x[n + "_bits"], torch) for n in ("q", "k", "v"))
    return x, q, k, v


def shared_mask(w: si.Prefill) -> np.ndarray:
    """The masked-forward workload's additive mask: one fp32 [Sq, Skv] array shared by every batch
    and head (the pages' compute_block_scores adds mask[q, k] to the scaled score), seeded N(0, 1)
    values on the visible keys."""
    return si.normal_f32(w.seed, 11, (w.Sq, w.Skv))


def bench_prefill_gpu(w: si.Prefill, args, torch, ea, dist, device, steps: int, e2e: bool = False,
                      mask: np.ndarray = None):
    """Times one attn_fwd_ex (or attn_fwd_masked) call over the workload, L2 flushed before every
    timed call.  bf16 inputs give fp32 O (the configuration the parity tests check)."""
    x, q, k, v = prefill_device_inputs(w, torch)
    o = torch.empty(q.shape, dtype=torch.float32, device=device)
    lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=device)
    # the workspace (RoPE table and rotated K, key-split partials) is allocated once, outside the
    # timed region
    ws_bytes = ea.fwd_workspace_bytes(q, k, w.rope_base, w.q_pos0, o.dtype)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device) if ws_bytes > 0 else None
    splits = ea.fwd_kv_splits(q, k, o.dtype)
    flush = make_l2_flush(torch, device)
    if mask is None:
        def step():
            ea.attn_fwd_ex(q, k, v, w.scale, w.causal, w.rope_base, w.q_pos0, o=o, lse=lse, workspace=ws)
    else:
        mt = torch.from_numpy(mask).to(device)

        def step():
            ea.attn_fwd_masked(q, k, v, mt, w.scale, w.causal, w.rope_base, w.q_pos0, o=o, lse=lse, workspace=ws)

    # rope: table + rotated K + prefill; key splits add the combine
    # RoPE: the cos/sin table and (unless K is rotated inside the prefill kernel) the K hi/lo pass
    rope_launches = 0 if w.rope_base <= 0 else (1 if os.environ.get("ATTN_ROPE_K_FORM") == "fused" else 2)
    launches_per_step = 1 + rope_launches + (1 if splits > 1 else 0)
    with ClockSampler(device.index) as clk:
        ms = time_steps(step, steps, args.warmup, flush, torch, dist, device)
    status = ea.read_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after timing {w.name}")
    r = {"ms": statistics.mean(ms), "ms_list": ms, "clocks": clk.summary(),
         "launches_per_step": launches_per_step, "kv_splits": splits}
    if e2e:
        # end to end through the public API: pinned host inputs -> device -> attn -> host output
        if w.dtype == "fp32":
            hq, hk, hv = (torch.from_numpy(x[n]).pin_memory() for n in ("q", "k", "v"))
        else:
            hq, hk, hv = (torch.from_numpy(np.ascontiguousarray(x[n + "_bits"]).view(np.int16)).view(torch.bfloat16)
                          .pin_memory() for n in ("q", "k", "v"))
        r["ms_e2e"] = time_e2e_pipelined(w, hq, hk, hv, o, lse, ws, max(3, steps // 4), args.warmup, torch, ea, dist,
                                         device)
        r["h2d"] = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        r["d2h"] = o.numel() * o.element_size() + lse.numel() * lse.element_size()
    return r


def bench_decode_gpu(w: si.Decode, args, torch, ea, dist, device, steps: int):
    d = si.decode_inputs(w, fill_tail_nan=False)
    q, kc, vc = (dev_bf16(d[n], torch) for n in ("q_bits", "k_bits", "v_bits"))
    sl = torch.from_numpy(d["seqlens"]).to(device)
    o = torch.empty(q.shape, dtype=torch.float32, device=device)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)
    ws = torch.empty(ea.decode_workspace_bytes(w.B, w.Hq, w.D, w.num_splits), dtype=torch.uint8, device=device)
    flush = make_l2_flush(torch, device)

    def step():
        ea.attn_decode(q, kc, vc, sl, w.scale, w.num_splits, o=o, lse=lse, workspace=ws)

    # the cache (~0.5 GB) is larger than L2, so decode calls run back to back without a flush
    with ClockSampler(device.index) as clk:
        ms = time_steps(step, steps, args.warmup, lambda: None, torch, dist, device)
    if ea.read_device_status() != 0:
        raise RuntimeError("device status set after decode timing")
    kv_bytes = si.decode_kv_bytes(d["seqlens"], w.Hkv, w.D)

    # the fused cache append of the same decode step (one new token per sequence, RoPE on the
    # new key and query): timed on its own, lengths kept below the capacity for every call
    n_app = steps + args.warmup
    sl_app = torch.from_numpy(np.minimum(d["seqlens"], w.Smax - n_app - 1).astype(np.int32)).to(device)
    kn = torch.zeros((w.B, 1, w.Hkv, w.D), dtype=torch.bfloat16, device=device)
    vn = torch.zeros_like(kn)
    qn = torch.zeros((w.B, 1, w.Hq, w.D), dtype=torch.bfloat16, device=device)

    def step_append():
        ea.kv_append(kc, vc, sl_app, kn, vn, q=qn, rope_base=10000.0)

    ms_app = time_steps(step_append, steps, args.warmup, flush, torch, dist, device)
    if ea.read_device_status() != 0:
        raise RuntimeError("device status set after the append timing")
    app_bytes = w.B * (2 * 2 * w.Hkv * w.D * 2 + 2 * w.Hq * w.D * 2)   # k,v read+write; q read+write
    return {"ms": statistics.mean(ms), "kv_bytes": kv_bytes, "clocks": clk.summary(), "inputs": d,
            "qo_bytes": 2 * w.B * w.Hq * w.D * 2 + 4 * w.B * w.Hq,
            "append": {"us_per_call": round(statistics.mean(ms_app) * 1e3, 2), "bytes_per_call": app_bytes,
                       "what": "attn_kv_append: one token per sequence, RoPE on k and q, cache write, length advance"}}


def bench_backward_gpu(w: si.Prefill, args, torch, ea, dist, device, steps: int):
    """attn_bwd on the workload: bf16 inputs, the forward's o and lse, fp32 gradients; L2 flushed
    before every call.  Algorithmic work: 10 D FLOP per unmasked (query, key) pair -- the method
    recomputes S (2D) and forms dP, dV, dQ, dK (2D each)."""
    x, q, k, v = prefill_device_inputs(w, torch)
    dout = dev_bf16(si.bf16_normal(w.seed, 7, (w.B, w.Sq, w.Hq, w.D))[0], torch)
    ws_f = None
    if w.rope_base > 0:
        ws_f = torch.empty(ea.fwd_workspace_bytes(q, k, w.rope_base, w.q_pos0), dtype=torch.uint8, device=device)
    o, lse = ea.attn_fwd_ex(q, k, v, w.scale, w.causal, w.rope_base, w.q_pos0, workspace=ws_f)
    ws = torch.empty(ea.bwd_workspace_bytes(q, k, w.rope_base, w.q_pos0), dtype=torch.uint8, device=device)
    flush = make_l2_flush(torch, device)

    def step():
        ea.attn_bwd(q, k, v, o, lse, dout, w.scale, w.causal, w.rope_base, w.q_pos0, grad_dtype=torch.float32,
                    workspace=ws)

    ms = time_steps(step, steps, args.warmup, flush, torch, dist, device)
    if ea.read_device_status() != 0:
        raise RuntimeError("device status set after the backward timing")
    return {"ms": statistics.mean(ms), "flop": 2.5 * w.flops}


# ------------------------------------------------------------------------------------------
# the oracle on the host cores (rank 0, one GPU only)
# ------------------------------------------------------------------------------------------

def _repeat_timed(fn, target_s: float, max_s: float):
    """Run fn until about target_s seconds have been timed (never past max_s); (runs, seconds)."""
    t0 = time.perf_counter()
    fn()
    dt = time.perf_counter() - t0
    reps, total = 1, dt
    while total < target_s and total + dt <= max_s:
        t0 = time.perf_counter()
        fn()
        total += time.perf_counter() - t0
        reps += 1
    return reps, total


def cpu_baseline_prefill(w: si.Prefill, target_s: float = 10.0, max_s: float = 30.0, threads: int = 0,
                         mask: np.ndarray = None):
    """The fp64 oracle on a bounded sample of the workload's rows (all (b, h), every r-th row);
    a masked workload runs the masked oracle over the whole problem."""
    import oracle
    x = si.prefill_inputs(w)
    prev = oracle.threads()
    if threads > 0:
        oracle.set_threads(threads)
    try:
        used = oracle.threads()
        if mask is not None:
            def run():
                oracle.attn_fwd_masked(x["q"], x["k"], x["v"], mask, w.scale, w.causal, w.rope_base, w.q_pos0)
            reps, total = _repeat_timed(run, target_s, max_s)
            flops = w.flops
            sample = f"the whole problem ({flops / 1e9:.2f} GFLOP fp64, masked oracle), {reps} runs in {total:.1f} s"
        else:
            stride = 1
            # size the sample so that one run takes at most about target_s / 2: start with 1/64 of
            # the rows and widen while it stays short
            for stride in (64, 16, 4, 1):
                rows = np.arange(0, w.B * w.Hq * w.Sq, stride, dtype=np.int64)
                t0 = time.perf_counter()
                oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0, rows=rows)
                dt = time.perf_counter() - t0
                if dt * 4 > target_s or stride == 1:
                    break

            def run():
                oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0, rows=rows)
            reps, total = _repeat_timed(run, target_s, max_s)
            i = rows % w.Sq
            off = w.Skv - w.Sq
            vis = np.clip(i + off + 1, 0, w.Skv) if w.causal else np.full_like(i, w.Skv)
            flops = float(np.sum(4.0 * w.D * vis))
            sample = (f"{len(rows)} of {w.B * w.Hq * w.Sq} query rows (every {stride}th row of every "
                      f"(batch, head)), {flops / 1e9:.3f} GFLOP fp64, {reps} runs in {total:.1f} s")
    finally:
        oracle.set_threads(prev)
    return {"value": flops * reps / total / 1e12, "unit": "TFLOP/s", "cores": used, "kind": "oracle",
            "sample": sample}


def cpu_baseline_decode(w: si.Decode, d, target_s: float = 5.0, max_s: float = 20.0):
    """The fp64 decode oracle (unsplit definition) on the first sequences of the batch, as many as
    fit in about target_s; KV-read GB/s of the sample."""
    import oracle
    sl = d["seqlens"]
    n, total = 0, 0.0
    for b in range(w.B):
        L = int(sl[b])
        kf = si.bf16_bits_to_f32(d["k_bits"][b:b + 1, :L])
        vf = si.bf16_bits_to_f32(d["v_bits"][b:b + 1, :L])
        t0 = time.perf_counter()
        oracle.decode(d["q"][b:b + 1], kf, vf, np.array([L], np.int32), w.scale)
        total += time.perf_counter() - t0
        n += 1
        if total > target_s or total > max_s:
            break
    kv = si.decode_kv_bytes(sl[:n], w.Hkv, w.D)
    return {"value": kv / total / 1e9, "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{n} of {w.B} sequences ({kv / 1e6:.1f} MB of K/V read in fp64), {total:.1f} s"}


# ------------------------------------------------------------------------------------------
# rooflines
# ------------------------------------------------------------------------------------------

def roofline_prefill(w: si.Prefill, ms: float, peaks, how: str, traffic, launches: int):
    achieved = w.flops / (ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    note = "one launch" if launches == 1 else f"the whole step of {launches} launches (a lower bound for the kernel)"
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": f"{how} bf16_tflops (burst, cuBLAS bf16 GEMM)",
            "kernel": "prefill_tc_kernel", "algorithmic_flop_per_launch": w.flops, "timed": note}


def fp32_peak_tflops(sm_max_mhz) -> float:
    """CUDA-core fp32 peak from the unit counts: 148 SMs x 128 FFMA lanes x 2 FLOP x the SM clock."""
    mhz = float(sm_max_mhz) if sm_max_mhz else 1965.0
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def roofline_fp32(w: si.Prefill, ms: float, clocks):
    achieved = w.flops / (ms * 1e-3) / 1e12
    peak = fp32_peak_tflops(clocks.get("sm_max_mhz"))
    return {"bound": "alu", "achieved": round(achieved, 4), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 5), "traffic": None,
            "peak_source": "derived: 148 SMs x 128 fp32 FFMA lanes x 2 FLOP x max SM clock",
            "kernel": "prefill_f32_kernel", "algorithmic_flop_per_launch": w.flops,
            "note": "4.2 MFLOP on 2 CTAs: launch- and latency-bound, a parity configuration"}


def roofline_decode(kv_bytes: int, ms: float, peaks, how: str, traffic=None):
    achieved = kv_bytes / (ms * 1e-3) / 1e9
    peak = float(peaks["hbm_gbs"])
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": f"{how} hbm_gbs (copy)",
            "kernel": "decode_split_kernel (+ decode_combine_kernel in the timed call)",
            "algorithmic_bytes_per_call": kv_bytes}


def roofline_backward(flop: float, ms: float, peaks, how: str):
    achieved = flop / (ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": None,
            "peak_source": how + " bf16_tflops (burst, cuBLAS bf16 GEMM)",
            "algorithmic_flop_per_call": flop}


def profile_name(w) -> str:
    return {si.C2.name: "prefill_tc_c2", si.C3.name: "prefill_tc_c3", si.C5.name: "prefill_tc_c5",
            si.C4.name: "decode_split_c4", si.F2_WHISPER.name: "prefill_tc_whisper"}.get(w.name, "")


# ------------------------------------------------------------------------------------------
# arms
# ------------------------------------------------------------------------------------------

def prefill_entry(w, r, peaks, how, world, cpu):
    """Per-configuration object of a prefill workload."""
    value = whole_job_rate(w.flops, r["ms"], world) / 1e12
    if w.dtype == "fp32":
        roof = roofline_fp32(w, r["ms"], r["clocks"])
    else:
        roof = roofline_prefill(w, r["ms"], peaks, how, profile_traffic(profile_name(w)), r["launches_per_step"])
    e = {"value": round(value, 4), "unit": "TFLOP/s", "ms_per_call": round(r["ms"], 5),
         "us_per_call": round(r["ms"] * 1e3, 2), "launches_per_call": r["launches_per_step"],
         "kv_splits": r["kv_splits"], "algorithmic_flop": w.flops, "roofline": roof, "clocks": r["clocks"],
         "shape": {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.Sq, "Skv": w.Skv, "D": w.D, "causal": w.causal,
                   "rope_base": w.rope_base, "q_pos0": w.q_pos0, "inputs": w.dtype}}
    if cpu is not None:
        e["cpu_baseline"] = cpu
    return e


def run_gpu(args):
    import torch
    rank, world, local = dist_env()
    assert torch.cuda.is_available(), "bench.py needs CUDA devices (use --impl reference for the CPU oracle)"
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    from exact_attention_160_b200 import build as b
    if rank == 0:
        b.build()
    barrier(dist, device)
    import exact_attention_160_b200 as ea
    ea.load_library()
    import oracle  # noqa: F401  (the CPU-baseline leg; built here before any timing)
    if rank == 0:
        oracle.build()
    barrier(dist, device)

    peaks, how = load_peaks()
    if args.backward_only:
        # the backward of the workload alone (a profiling aid): value = its TFLOP/s
        w = si.WORKLOADS[args.workload]
        br = bench_backward_gpu(w, args, torch, ea, dist, device, args.steps)
        bms = max_over_ranks(br["ms"], dist, device)
        out = {"metric": "attention backward TFLOP/s", "value": round(whole_job_rate(br["flop"], bms, world) / 1e12, 3),
               "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": round(bms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
               "dtype": "bf16", "data": "synthetic", "config": {"workload": w.name, "part": "backward"},
               "roofline": roofline_backward(br["flop"], bms, peaks, how)}
        if rank == 0:
            print(json.dumps(out), flush=True)
        if dist is not None:
            barrier(dist, device)
            dist.destroy_process_group()
        return
    cpu_on = rank == 0 and world == 1 and not args.no_cpu_baseline
    sec_steps = max(5, args.steps // 3)
    w = si.WORKLOADS[args.workload]
    configs = {}
    if isinstance(w, si.Prefill):
        r = bench_prefill_gpu(w, args, torch, ea, dist, device, args.steps, e2e=True)
        ms = max_over_ranks(r["ms"], dist, device)
        ms_e2e = max_over_ranks(r["ms_e2e"], dist, device)
        value = whole_job_rate(w.flops, ms, world) / 1e12
        value_e2e = whole_job_rate(w.flops, ms_e2e, world) / 1e12
        unit = "TFLOP/s"
        r["ms"] = ms
        roof = roofline_prefill(w, ms, peaks, how, profile_traffic(profile_name(w)), r["launches_per_step"])
        clocks = r["clocks"]
        e2e = {"how": "attn_fwd_ex from pinned host q, k, v to pinned host o, lse every step; two streams "
                      "alternate so one step's device->host copy overlaps the next step's host->device copy",
               "value": round(value_e2e, 3), "unit": unit, "h2d_bytes_per_step": r["h2d"],
               "d2h_bytes_per_step": r["d2h"], "ms_per_step": round(ms_e2e, 4)}
        launches = r["launches_per_step"] * args.steps
        config = {"workload": w.name, "global_batch": w.B * world, "seq_len": w.Sq, "heads_q": w.Hq,
                  "heads_kv": w.Hkv, "head_dim": w.D, "causal": w.causal, "rope_base": w.rope_base,
                  "kv_splits": r["kv_splits"], "parallelism": f"replicas{world}", "l2": L2_NOTE,
                  "inputs": f"seeded synthetic N(0,{w.qk_std:g}^2) q, k and N(0,1) v, rounded to bf16 "
                            "(seeded_inputs)"}
        cpu_head = cpu_baseline_prefill(w) if cpu_on else None
    else:
        dec = bench_decode_gpu(w, args, torch, ea, dist, device, args.steps)
        ms = max_over_ranks(dec["ms"], dist, device)
        value = whole_job_rate(dec["kv_bytes"], ms, world) / 1e9
        unit = "GB/s"
        roof = roofline_decode(dec["kv_bytes"], ms, peaks, how, profile_traffic(profile_name(w)))
        clocks = dec["clocks"]
        e2e = None
        launches = 2 * args.steps
        config = {"workload": w.name, "global_batch": w.B * world, "heads_q": w.Hq, "heads_kv": w.Hkv,
                  "head_dim": w.D, "smax": w.Smax, "num_splits": w.num_splits,
                  "parallelism": f"replicas{world}",
                  "l2": "not flushed: the cache is larger than L2 (the append timing flushes: " + L2_NOTE + ")"}
        cpu_head = cpu_baseline_decode(w, dec["inputs"]) if cpu_on else None

    if not args.headline_only:
        # every other configuration, each timed on its own with its roofline and CPU baseline
        for cw in (si.C1, si.C2, si.C3, si.C5, si.F2_WHISPER, si.F2_CHUNK):
            if cw.name == w.name:
                continue
            cr = bench_prefill_gpu(cw, args, torch, ea, dist, device, sec_steps)
            cr["ms"] = max_over_ranks(cr["ms"], dist, device)
            cpu = None
            if cpu_on:
                cpu = cpu_baseline_prefill(cw, target_s=3.0, max_s=10.0)
                if cw.dtype == "fp32":
                    cpu["single_thread"] = cpu_baseline_prefill(cw, 2.0, 6.0, threads=1)
            configs[cw.name] = prefill_entry(cw, cr, peaks, how, world, cpu)
        # the masked forward on C2's shapes (a shared [Sq, Skv] fp32 mask on top of the causal mask)
        mk = shared_mask(si.C2)
        cr = bench_prefill_gpu(si.C2, args, torch, ea, dist, device, sec_steps, mask=mk)
        cr["ms"] = max_over_ranks(cr["ms"], dist, device)
        cpu = cpu_baseline_prefill(si.C2, 3.0, 10.0, mask=mk) if cpu_on else None
        e = prefill_entry(si.C2, cr, peaks, how, world, cpu)
        e["what"] = "attn_fwd_masked on C2's shapes: shared fp32 [Sq, Skv] additive mask plus the causal mask"
        e["roofline"]["traffic"] = None
        configs["c2_masked_shared_mask"] = e
        # C3 with K rotated inside the prefill kernel instead of by the K hi/lo pre-pass (the two
        # RoPE forms side by side; the pre-pass is the library's default)
        prev = os.environ.get("ATTN_ROPE_K_FORM")
        os.environ["ATTN_ROPE_K_FORM"] = "fused"
        try:
            cr = bench_prefill_gpu(si.C3, args, torch, ea, dist, device, sec_steps)
        finally:
            if prev is None:
                del os.environ["ATTN_ROPE_K_FORM"]
            else:
                os.environ["ATTN_ROPE_K_FORM"] = prev
        cr["ms"] = max_over_ranks(cr["ms"], dist, device)
        e = prefill_entry(si.C3, cr, peaks, how, world, None)
        e["what"] = ("C3 with RoPE on K applied inside the prefill kernel (ATTN_ROPE_K_FORM=fused) instead of "
                     "the K hi/lo pre-pass; same oracle as C3")
        e["roofline"]["traffic"] = None
        configs["c3_rope_k_fused_form"] = e
        if w.name != si.C4.name:
            dec = bench_decode_gpu(si.C4, args, torch, ea, dist, device, max(5, args.steps // 2))
            dms = max_over_ranks(dec["ms"], dist, device)
            e = {"value": round(whole_job_rate(dec["kv_bytes"], dms, world) / 1e9, 1), "unit": "GB/s",
                 "ms_per_call": round(dms, 5), "launches_per_call": 2, "num_splits": si.C4.num_splits,
                 "l2": "not flushed: the cache is larger than L2",
                 "roofline": roofline_decode(dec["kv_bytes"], dms, peaks, how,
                                             profile_traffic(profile_name(si.C4))),
                 "append": dec["append"], "clocks": dec["clocks"]}
            if cpu_on:
                e["cpu_baseline"] = cpu_baseline_decode(si.C4, dec["inputs"], 3.0, 10.0)
            configs[si.C4.name] = e
        backward = {}
        for bw in (si.C2, si.C3, si.C5):
            br = bench_backward_gpu(bw, args, torch, ea, dist, device, max(4, args.steps // 4))
            bms = max_over_ranks(br["ms"], dist, device)
            backward[bw.name] = {
                "what": "attn_bwd: dq, dk, dv (fp32) from bf16 q, k, v, o, dout and lse",
                "value": round(whole_job_rate(br["flop"], bms, world) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_call": round(bms, 4), "algorithmic_flop_per_call": br["flop"],
                "roofline": roofline_backward(br["flop"], bms, peaks, how)}

    out = {"metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config, "roofline": roof,
           "clocks": clocks, "gpu_launches": launches}
    if e2e is not None:
        out["e2e"] = e2e
    if cpu_head is not None:
        out["cpu_baseline"] = cpu_head
    if configs:
        out["configs"] = configs
    if not args.headline_only:
        out["backward"] = backward
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        barrier(dist, device)
        dist.destroy_process_group()


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w = si.WORKLOADS[args.workload]
    if not isinstance(w, si.Prefill):
        raise SystemExit("the reference arm times prefill workloads")
    x = si.prefill_inputs(w)
    # each step: every r-th query row of every (batch, head), r chosen so that a step is at most
    # about 20 GFLOP of fp64 work (the whole workload when it is smaller) -- a bounded slice
    stride = max(1, int(np.ceil(w.flops / 20e9)))
    rows = np.arange(0, w.B * w.Hq * w.Sq, stride, dtype=np.int64)
    i = rows % w.Sq
    vis = np.clip(i + (w.Skv - w.Sq) + 1, 0, w.Skv) if w.causal else np.full_like(i, w.Skv)
    flops = float(np.sum(4.0 * w.D * vis))
    for _ in range(args.warmup):
        oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0, rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.rope_base, w.q_pos0, rows=rows)
    dt = (time.perf_counter() - t0) / args.steps
    value = flops / dt / 1e12
    threads = oracle.threads()
    sample = (f"{len(rows)} query rows per step (every {stride}th row of every (batch, head)), "
              f"{flops / 1e9:.3f} GFLOP fp64")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "global_batch": w.B, "seq_len": w.Sq, "heads_q": w.Hq,
                      "heads_kv": w.Hkv, "head_dim": w.D, "causal": w.causal, "rope_base": w.rope_base,
                      "parallelism": "cpu", "inputs": "seeded synthetic q, k, v rounded to bf16 (seeded_inputs)"},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=si.C5.name, choices=sorted(si.WORKLOADS))
    ap.add_argument("--headline-only", action="store_true",
                    help="time the headline workload only (no per-configuration objects)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only attn_bwd on the workload (a profiling aid; not the benchmark line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
