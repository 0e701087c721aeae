#!/usr/bin/env python
"""Benchmark of the Infini-attention forward on B200: tokens/s and roofline fraction.

One step = one full forward (every segment's local attention, memory retrieval, gate and
memory update) over one batch of the workload's synthetic inputs, through the C ABI.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                  [--tail T] [--decode]

``--tail T`` appends a final segment of T < N tokens to every head of the workload.
``--decode`` times the token-by-token decode step instead of the forward: one step is one
segment of N tokens fed one at a time (every batch row and head per call), the fold of
the segment into the memory included; tokens/s counts B * N tokens per step.

Prints ONE JSON line on rank 0.  Under torchrun (N > 1) every rank runs its own batch of
the workload on its own GPU (independent problems: no data-path collective, weak
scaling); step time is the max over ranks.

Timing: W untimed warm-up steps, then K steps each bracketed by CUDA events on the launch
stream, with a 256 MiB write (larger than the 126 MB L2) before every step, outside the
events, so each step starts with a cold L2.  The library's launch trace (CUDA events
around each of its kernels, on the same stream) gives the dominant kernel's device time
for the roofline and the launch count.  A launch-bound workload (one whose workspace fits
the allocation-free entry point's fixed array) is timed as replays of a CUDA graph of that
call, and its per-kernel times come from the same steps run eagerly with the trace on.
``e2e`` pipelines the steps as a serving loop would: step i + 1's inputs are copied in
while step i computes and step i - 1's results are copied out.  ``--impl reference`` times the fp64 CPU oracle
instead, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from compressive_memory_long_b200 import workloads as wl  # noqa: E402

METRIC = "Infini-attention fwd tokens/s at 1 B200; % of bf16 TC peak or HBM roofline"
DECODE_METRIC = "Infini-attention decode tokens/s at 1 B200 (one token per call, per sequence)"
BACKWARD_METRIC = "Infini-attention backward tokens/s at 1 B200 (all gradients of one forward)"
DEFAULT_WORKLOAD = "stream1m_n2048_delta"
FLUSH_BYTES = 256 << 20

# Measured roofline denominators of this GPU pool (measured copy bandwidth and
# cuBLAS bf16 GEMM); used when the measured-peaks file is absent.
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from an ncu
# capture, keyed by (workload, kernel), with a digest of the kernel's source files at the
# time of the capture: a kernel whose sources have changed since reports no traffic (the
# counters no longer describe it) until it is captured again.  The summaries with the
# commands are under profiles/.  The N = 64 bandwidth, batched and 1M-stream figures are
# captures of fewer segments scaled to the workload's (traffic grows with the units
# processed).
KERNEL_SOURCES = {
    "segment_tc": ("tc_segment_p.cuh", "tc_segment.cuh", "tc_common.cuh"),
    "small_pieces": ("tc_pieces.cuh", "tc_small.cuh", "tc_common.cuh"),
    "small_fused": ("tc_small.cuh", "tc_common.cuh"),
}
NCU_TRAFFIC_BYTES: dict = {
    ("hf_repro_n64", "small_fused"): (6364160, "b4076352787a7b26"),
    # 2048 of 16384 segments captured (x 8)
    ("n64_bandwidth", "small_pieces"): ((1032990976 + 268926464) * 8, "5c6fb8137091e762"),
    ("gqa8b_n2048_delta", "segment_tc"): (421691904 + 238313216, "e5dbc14c5524c01e"),
    # 4 of 8 segments captured (x 2) and 16 of 512 segments captured (x 32)
    ("batched_n1024_linear", "segment_tc"): ((1705369856 + 516162816) * 2, "e5dbc14c5524c01e"),
    ("stream1m_n2048_delta", "segment_tc"): ((412875264 + 113371136) * 32, "e5dbc14c5524c01e"),
}


def kernel_digest(kernel: str):
    """sha256 (first 16 hex digits) of the CUDA sources a kernel is compiled from, or None."""
    import hashlib
    files = KERNEL_SOURCES.get(kernel)
    if not files:
        return None
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "compressive_memory_long_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def captured_traffic(workload: str, kernel: str):
    """(bytes per launch or None, note): the captured DRAM traffic when it describes the
    kernel as built now."""
    entry = NCU_TRAFFIC_BYTES.get((workload, kernel))
    if entry is None:
        return None, "no ncu capture of this kernel on this workload"
    byts, digest = entry
    if kernel_digest(kernel) != digest:
        return None, "stale: the kernel's sources changed since the ncu capture"
    return byts, "ncu capture of the current kernel"


def fp32_fma_peak_tflops(sm_mhz=1965.0, sms=148):
    """CUDA-core fp32 peak: SMs x 128 FP32 lanes x 2 flops (one FMA) x the SM clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks: dict, clk: dict):
    """(peak TFLOP/s, kind) for a tensor-bound kernel: the sustained bf16 figure when the
    clock record of its timed region shows sw_power_cap active (the loop ran long enough for
    the power cap to lower the clock), else the burst one."""
    if "sw_power_cap" in ((clk or {}).get("reasons") or []) and peaks.get("bf16_tflops_sustained"):
        return peaks["bf16_tflops_sustained"], "sustained: sw_power_cap active in the timed region"
    return peaks["bf16_tflops"], "burst"


# ---- algorithmic work per kernel (flops and bytes; snapshots and re-reads excluded) ----

def algorithmic(w: wl.Workload, kernel: str):
    """(flops, bytes) one launch of ``kernel`` does on workload ``w``.

    segment kernel: local causal attention 2 d N (N + 1) + retrieval 2 N d^2 flops per
    (b, h, segment); bytes = q, k, v read once and out written once.
    memory increments (and the CUDA-core state kernels): update 2 N d^2 (linear) or 4 N d^2
    (delta) flops per (b, kv head, segment); bytes = k, v read once plus M/z read and written
    once.  The z sums, the prefix and the recurrence over the increments: state bytes only.
    """
    e = w.elem_bytes
    B, H, Hkv, L, N, d, S = w.B, w.H, w.Hkv, w.L, w.N, w.d, w.S
    state_bytes = 2 * B * Hkv * (d * d + d) * 4
    if kernel == "decode_attn":     # one token per (b, h): the cached rows once, M and z once
        rows = (N - 2) / 2.0            # average cached rows over offsets 0 .. N - 2
        byts = (B * Hkv * (2 * rows * d * e + (d * d + d) * 4) + 2 * B * H * d * e
                + 2 * B * Hkv * d * e)
        flops = B * H * (4 * d * (rows + 1) + 2 * d * d)
        return flops, byts
    if kernel in ("small_fused", "small_pieces"):     # the whole forward in one launch
        f1, b1 = algorithmic(w, "segment")
        f2, b2 = algorithmic(w, "linear_state")
        return f1 + f2, b1 + state_bytes
    if kernel.startswith("segment"):
        flops = B * H * S * (2 * d * N * (N + 1) + 2 * N * d * d)
        byts = (2 * H + 2 * Hkv) * B * L * d * e
    elif kernel.startswith(("linear_increments", "linear_state", "delta_chain", "mem_increments")):
        per = 2 if w.rule == "linear" else 4
        flops = B * Hkv * S * per * N * d * d
        byts = 2 * B * Hkv * L * d * e + state_bytes
    else:   # scan / init: pure state traffic
        flops = 0
        byts = state_bytes
    return flops, byts


# ---- clocks during the timed region (NVML) ----

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            uuid = torch.cuda.get_device_properties(device_index).uuid
            self._h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == str(uuid).replace("GPU-", ""):
                    self._h = h
            if self._h is None:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as ex:   # NVML missing: report no clocks rather than fail the run
            self._nv = None
            self.error = repr(ex)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._nv is not None:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---- distributed plumbing ----

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---- CPU oracle samples (the baseline leg and the reference arm) ----

def oracle_sample(w: wl.Workload, seconds: float):
    """Time the fp64 oracle on a bounded sample of ``w``.

    Small workloads: the whole workload, repeated until about ``seconds`` have passed.
    Large ones: chain (b=0, kv head 0) with its G query heads over the first n segments,
    n sized to about ``seconds`` of work (one query head of H covers 1/H of a token).
    Returns (token-equivalents per second, seconds timed, description).
    """
    import oracle
    st = wl.has_initial_state(w)

    if w.B * w.H * w.L * w.d <= (1 << 22):
        q, k, v, beta, M0, z0 = wl.host_inputs(w)
        reps, dt = 0, 0.0
        while reps == 0 or dt < seconds:
            t0 = time.perf_counter()
            oracle.infini_attn_fwd(q, k, v, beta, M0 if st else None, z0 if st else None,
                                   N=w.N, rule=w.rule)
            dt += time.perf_counter() - t0
            reps += 1
        return w.B * w.L * reps / dt, dt, f"whole workload x {reps}"

    def run(n_seg):
        rows = n_seg * w.N
        q, k, v, beta, M0, z0 = wl.host_slices(w, 0, 0, rows=rows)
        t0 = time.perf_counter()
        oracle.infini_attn_fwd(q, k, v, beta, M0 if st else None, z0 if st else None, N=w.N,
                               rule=w.rule)
        return rows * w.G / w.H, time.perf_counter() - t0

    n = 1
    tok, dt = run(n)
    if dt < 0.5 * seconds and w.S > 1:
        n = int(min(w.S, max(2, round(seconds / max(dt, 1e-6)))))
        tok, dt = run(n)
    desc = (f"chain (b=0, kv head 0) with its {w.G} query head(s) of {w.H}, first {n} of "
            f"{w.S} segments ({n * w.N} tokens)")
    return tok / dt, dt, desc


def run_reference(args, w: wl.Workload, metric: str = METRIC):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    per_step = min(20.0, max(2.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, per_step)
    vals, secs = [], 0.0
    desc = ""
    for _ in range(args.steps):
        v, dt, desc = oracle_sample(w, per_step)
        vals.append(v)
        secs += dt
    value = float(statistics.mean(vals))
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * secs / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w: wl.Workload):
    return {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "d": w.d, "N": w.N,
            "S": w.S, "tail": w.tail, "L": w.L, "rule": w.rule, "activations": w.dtype,
            "l2": "256 MiB write before every step (L2 flushed)",
            "description": w.description}


# ---- the decode step (our arm, --decode) ----

def run_decode(args, w: wl.Workload, world: int, rank: int, local: int, dev):
    """One step = the N tokens of one segment through infini_attn_decode_step, one call per
    token (all batch rows and heads at once); the call at offset N - 1 folds the segment.

    The N calls of a step are captured once in a CUDA graph (the calls allocate nothing),
    and the timed region replays it: device time without the host's per-call overhead.
    The decode kernel's own time comes from a second graph of the calls at offsets
    0 .. N - 2 (no fold).  ``e2e`` adds each token's copies to the graph: its q, k, v from
    pinned host memory before its call and its output back after it.
    """
    from compressive_memory_long_b200 import binding
    host = wl.torch_inputs(w, pin_memory=True)
    # per-token slabs [N, B, heads, d], contiguous per token
    tok = {n: host[n].permute(2, 0, 1, 3).contiguous().pin_memory() for n in ("q", "k", "v")}
    t = {n: x.to(dev, non_blocking=True) for n, x in tok.items()}
    beta = host["beta"].to(dev)
    dt = w.torch_dtype
    kc = torch.zeros((w.B, w.Hkv, w.N, w.d), dtype=dt, device=dev)
    vc = torch.zeros_like(kc)
    M = torch.zeros((w.B, w.Hkv, w.d, w.d), dtype=torch.float32, device=dev)
    z = torch.zeros((w.B, w.Hkv, w.d), dtype=torch.float32, device=dev)
    outs = torch.empty((w.N, w.B, w.H, w.d), dtype=dt, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def calls(n_pos):
        for p in range(n_pos):
            binding.decode_step(t["q"][p], t["k"][p], t["v"][p], beta, kc, vc, p, M, z,
                                rule=w.rule, out=outs[p])

    for _ in range(2):
        calls(w.N)
    torch.cuda.synchronize(dev)
    g_step, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        calls(w.N)
    with torch.cuda.graph(g_attn):
        calls(w.N - 1)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        g_step.replay()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            g_step.replay()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = max_over_ranks(float(sum(s.elapsed_time(e) for s, e in zip(starts, ends))),
                              world, dev)
    per_step = w.N + (1 if w.rule == "linear" else 2)     # decode calls + fold kernels
    launches = int(per_step * args.steps * world)
    tokens = w.B * w.N * args.steps * world
    value = tokens / (total_ms / 1000.0)

    # the decode kernel alone: graph of the calls at offsets 0 .. N - 2
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(1, args.steps)
    flush.zero_()
    a0.record(stream)
    for _ in range(reps):
        g_attn.replay()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    n_attn = (w.N - 1) * reps
    dom_ms = max_over_ranks(a0.elapsed_time(a1) / n_attn, world, dev)
    peaks, peak_src = load_peaks()
    flops, byts = algorithmic(w, "decode_attn")
    achieved = byts / (dom_ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel": "decode_attn",
            "kernel_ms": dom_ms, "peak_source": f"{peak_src} (burst)",
            "algorithmic_flops": flops, "algorithmic_bytes": byts,
            "kernel_share": dom_ms * w.N / (total_ms / args.steps)}
    kernels = {"decode_attn": {"launches": n_attn, "ms": a0.elapsed_time(a1)}}
    del g_step, g_attn

    out_h = torch.empty(outs.shape, dtype=dt, pin_memory=True)
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e):
        for p in range(w.N):
            for n in ("q", "k", "v"):
                t[n][p].copy_(tok[n][p], non_blocking=True)
            binding.decode_step(t["q"][p], t["k"][p], t["v"][p], beta, kc, vc, p, M, z,
                                rule=w.rule, out=outs[p])
            out_h[p].copy_(outs[p], non_blocking=True)
    for _ in range(args.warmup):
        g_e2e.replay()
    barrier(world)
    torch.cuda.synchronize(dev)
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        e_starts[i].record(stream)
        g_e2e.replay()
        e_ends[i].record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(float(sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends))),
                            world, dev)
    del g_e2e
    h2d = sum(x.numel() * x.element_size() for x in tok.values())
    d2h = out_h.numel() * out_h.element_size()

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        v, sec, desc = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": "oracle forward over the same segment (the outputs the decode "
                         f"reproduces): {desc}; {sec:.1f} s on 1 host core"}
    if rank == 0:
        line = {
            "metric": DECODE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": dict(config_of(w), timing="CUDA graph of one segment's calls"),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": w.B * w.N * args.steps * world / (e2e_ms / 1000.0),
                    "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches, "kernels": kernels, "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---- the backward pass (our arm, --backward) ----

def backward_flops(w: wl.Workload):
    """Algorithmic flops of one backward: the local attention's five N x N x d products over
    the causal half (recomputed scores, dP, dS K, dS^T Q, P^T dA) plus the retrieval's and
    the memory's d x d contractions (forward recompute and gradients, about four times the
    forward's)."""
    B, H, Hkv, N, d = w.B, w.H, w.Hkv, w.N, w.d
    S = -(-w.L // N)
    local = B * H * S * 5 * d * N * (N + 1)
    memory = B * H * S * 4 * 2 * N * d * d + B * Hkv * S * 4 * (4 if w.rule == "delta" else 2) * N * d * d
    return local + memory


def backward_roofline(w: wl.Workload, kernels: dict, steps: int, clk: dict) -> dict:
    """The backward's dominant kernel against its own ceiling.  Algorithmic flops per
    (b, h, segment), one causal product = d N (N + 1): the row statistics recompute S and P V
    (2) plus the retrieval's sigma(q) M and dout M^T (4 N d^2); the dq kernel S, dP and dS K
    (3); the dk/dv kernel S^T, dP^T, P^T dout and dS^T Q (4); G^M 2 N d^2; the update
    (per kv head) 8 N d^2 (delta) or 4 N d^2 (linear).  On the tensor cores (bf16 peak) for
    bf16 with d in {64, 128} and N % 128 == 0 except the update, else on CUDA cores (fp32 FMA
    peak)."""
    B, H, N, d = w.B, w.H, w.N, w.d
    S = -(-w.L // N)
    prod = B * H * S * d * N * (N + 1)
    # G^M_s: one N x d x d product per (b, h, segment); the update: 4 (delta) or 2 (linear)
    # N x d x d products per (b, kv head, segment)
    upd = (8 if w.rule == "delta" else 4) * N * d * d * B * w.Hkv * S
    flops = {"bwd_rows": 2 * prod + B * H * S * 4 * N * d * d, "bwd_dq": 3 * prod, "bwd_dkdv": 4 * prod,
             "bwd_gm": B * H * S * 2 * N * d * d, "bwd_update": upd}
    tensor = w.dtype == "bf16" and d in (64, 128) and N % 128 == 0
    on_tc = {"bwd_rows", "bwd_dq", "bwd_dkdv", "bwd_gm"} if tensor else set()
    cand = {k: v for k, v in kernels.items() if k in flops}
    if not cand:
        return None
    dom = max(cand, key=lambda k: cand[k]["ms"])
    ms = cand[dom]["ms"] / max(1, cand[dom]["launches"]) * (cand[dom]["launches"] / max(1, steps))
    achieved = flops[dom] / (ms / 1e3) / 1e12 if ms > 0 else 0.0
    frac_burst = None
    if dom in on_tc:
        peaks, src = load_peaks()
        frac_burst = achieved / peaks["bf16_tflops"]
        peak, kind = tensor_peak(peaks, clk)
        bound, psrc = "tensor", f"{src} ({kind})"
    else:
        peak, bound = fp32_fma_peak_tflops(clk["sm_mhz"] or 1965.0), "alu"
        psrc = "derived: 148 SMs x 128 fp32 lanes x 2 x SM clock"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "frac_of_burst_peak": frac_burst, "traffic": None,
            "kernel": dom, "kernel_ms": ms,
            "peak_source": psrc, "algorithmic_flops": flops[dom],
            "kernel_share": cand[dom]["ms"] / sum(v["ms"] for v in kernels.values())}


def run_backward(args, w: wl.Workload, world: int, rank: int, local: int, dev):
    """One step = all gradients of one forward of the workload (infini_attn_bwd), with a
    fixed random upstream gradient; inputs resident on the device, L2 flushed before each
    step.  The roofline is the dominant kernel's (backward_roofline)."""
    import ctypes
    from compressive_memory_long_b200 import binding
    host = wl.torch_inputs(w, pin_memory=True)
    t = {k: (None if x is None else x.to(dev, non_blocking=True)) for k, x in host.items()}
    g = torch.Generator(device=dev).manual_seed(w.seed + 7)
    dout = torch.randn(t["q"].shape, device=dev, generator=g).to(t["q"].dtype)
    dM = 0.1 * torch.randn((w.B, w.Hkv, w.d, w.d), device=dev, generator=g)
    dz = 0.01 * torch.randn((w.B, w.Hkv, w.d), device=dev, generator=g)
    outs = [torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"]),
            torch.empty((w.H,), device=dev), torch.empty_like(dM), torch.empty_like(dz)]
    fn = binding.LIB.infini_attn_bwd if w.dtype == "bf16" else binding.LIB.infini_attn_bwd_f32
    stream = torch.cuda.current_stream(dev)
    P = lambda x: None if x is None else ctypes.c_void_p(x.data_ptr())

    def step():
        rc = fn(P(t["q"]), P(t["k"]), P(t["v"]), P(t["beta"]), P(t["M0"]), P(t["z0"]), P(dout),
                P(dM), P(dz), *(P(x) for x in outs), w.B, w.H, w.Hkv, w.L, w.N, w.d,
                binding.RULES[w.rule], ctypes.c_void_p(stream.cuda_stream))
        if rc != 0:
            raise binding.InfiniError(rc, binding.infini_attn_status_string(rc))

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    binding.infini_attn_trace_enable(True)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    binding.infini_attn_trace_enable(False)
    barrier(world)
    kernels = {k: v for k, v in binding.infini_attn_trace_report().items() if isinstance(v, dict)}
    total_ms = max_over_ranks(float(sum(s_.elapsed_time(e) for s_, e in zip(starts, ends))), world, dev)
    value = w.tokens * args.steps * world / (total_ms / 1000.0)
    clk = clocks.summary()
    roof = backward_roofline(w, kernels, args.steps, clk)
    if rank == 0:
        line = {
            "metric": BACKWARD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": dict(config_of(w), pass_="backward"), "roofline": roof,
            "cpu_baseline": None, "e2e": None,
            "gpu_launches": int(sum(v["launches"] for v in kernels.values())),
            "kernels": kernels, "clocks": clk,
            "algorithmic_flops_total": backward_flops(w),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---- our arm ----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU-oracle sample size for cpu_baseline (0 disables)")
    ap.add_argument("--segment-len", type=int, default=0,
                    help="run the workload's tokens in segments of this length instead (other "
                         "kernels' profiles: N = 128 selects the one-tile segment kernel)")
    ap.add_argument("--tail", type=int, default=0,
                    help="append a final segment of this many (< N) tokens to every head")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (all gradients of one forward) instead")
    ap.add_argument("--decode", action="store_true",
                    help="time the token-by-token decode step over one segment instead")
    ap.add_argument("--segments", type=int, default=0,
                    help="run the workload with this many segments instead (small profiling "
                         "captures of a large workload's kernels); 0 keeps the workload's own")
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    if args.segments > 0:
        w = dataclasses.replace(w, name=f"{w.name}@S{args.segments}", S=args.segments)
    if args.segment_len:
        if args.segment_len <= 0 or args.segment_len % 64 or w.L % args.segment_len:
            ap.error("--segment-len must be a positive multiple of 64 dividing L")
        w = dataclasses.replace(w, name=f"{w.name}@N{args.segment_len}", N=args.segment_len,
                                S=w.L // args.segment_len)
    if args.tail:
        if not 0 < args.tail < w.N:
            ap.error("--tail must be in (0, N)")
        w = dataclasses.replace(w, name=f"{w.name}+T{args.tail}", tail=args.tail)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.decode:
        w = dataclasses.replace(w, name=f"{w.name}:decode", S=1, tail=0)

    if args.impl == "reference":
        return run_reference(args, w, DECODE_METRIC if args.decode else METRIC)

    world, rank, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    from compressive_memory_long_b200 import binding

    if args.decode:
        return run_decode(args, w, world, rank, local, dev)
    if args.backward:
        return run_backward(args, w, world, rank, local, dev)

    host = wl.torch_inputs(w, pin_memory=True)
    t = {k: (None if x is None else x.to(dev, non_blocking=True)) for k, x in host.items()}
    out = torch.empty_like(t["q"])
    M_out = torch.empty((w.B, w.Hkv, w.d, w.d), dtype=torch.float32, device=dev)
    z_out = torch.empty((w.B, w.Hkv, w.d), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    fwd = binding.infini_attn_fwd if w.dtype == "bf16" else binding.infini_attn_fwd_f32

    def step():
        fwd(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], out, M_out, z_out, w.N,
            w.rule, stream)

    # Launch-bound workloads (a workspace that fits the allocation-free entry point's fixed
    # array): the timed step replays a CUDA graph of that call, as a serving loop would; the
    # per-kernel times for the roofline come from an eager traced pass of the same steps.
    graph = None
    if w.dtype == "bf16" and binding.infini_attn_workspace_bytes(
            w.B, w.Hkv, w.L, w.N, w.d) <= binding.NOALLOC_SCRATCH_BYTES:
        def call_noalloc():
            binding.infini_attn_fwd_noalloc(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"],
                                            out, M_out, z_out, w.N, w.rule)
        call_noalloc()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call_noalloc()
        torch.cuda.synchronize(dev)

    def timed_step():
        if graph is not None:
            graph.replay()
        else:
            step()

    for _ in range(args.warmup):
        flush.zero_()
        timed_step()
    torch.cuda.synchronize(dev)

    # ---- timed region (device time; trace on for per-kernel events unless graphed) ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    binding.infini_attn_trace_enable(graph is None)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            timed_step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    binding.infini_attn_trace_enable(False)
    barrier(world)
    if graph is not None:       # the same steps eagerly, traced, for the per-kernel times
        binding.infini_attn_trace_enable(True)
        for i in range(args.steps):
            flush.zero_()
            step()
        torch.cuda.synchronize(dev)
        binding.infini_attn_trace_enable(False)
    trace = binding.infini_attn_trace_report()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(float(sum(step_ms)), world, dev)
    launches = int(sum_over_ranks(float(sum(v["launches"] for k, v in trace.items()
                                            if isinstance(v, dict))), world, dev))
    tokens = w.tokens * args.steps * world
    value = tokens / (total_ms / 1000.0)

    # ---- dominant kernel roofline ----
    peaks, peak_src = load_peaks()
    kernels = {k: v for k, v in trace.items() if isinstance(v, dict)}
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    dom_ms = kernels[dom]["ms"] / kernels[dom]["launches"]
    dom_ms = max_over_ranks(dom_ms, world, dev)
    flops, byts = algorithmic(w, dom)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    peak_kind = "burst"
    if flops > 0 and flops / byts > ridge:
        achieved = flops / (dom_ms / 1e3) / 1e12
        # a tensor-bound kernel timed inside a loop of steps long enough for the power cap to
        # act (sw_power_cap seen during the timed region) is held to the sustained figure, a
        # kernel that ran at full clock to the burst one; both fractions are reported
        burst = peaks["bf16_tflops"]
        peak, peak_kind = tensor_peak(peaks, clocks.summary())
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "frac_of_burst_peak": achieved / burst}
    else:
        achieved = byts / (dom_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    roof["traffic"], roof["traffic_source"] = captured_traffic(w.name, dom)
    roof.update({"kernel": dom, "kernel_ms": dom_ms, "peak_source": f"{peak_src} ({peak_kind})",
                 "algorithmic_flops": flops, "algorithmic_bytes": byts,
                 "kernel_share": kernels[dom]["ms"] / sum(v["ms"] for v in kernels.values())})

    # ---- end to end through the public call with host buffers ----
    # The steps run as a serving loop would run them: two device buffer sets, step i + 1's
    # inputs copied in from pinned host memory (copy-in stream) while step i computes and
    # step i - 1's out / M / z are copied back (copy-out stream).  Every step's copies are
    # inside the timed region, which runs from before the first copy-in to after the last
    # copy-out.  No L2 flush here: each step's inputs arrive through the copy itself.
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    M_h = torch.empty(M_out.shape, dtype=torch.float32, pin_memory=True)
    z_h = torch.empty(z_out.shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(x.numel() * x.element_size() for x in host.values() if x is not None)
    d2h = sum(x.numel() * x.element_size() for x in (out_h, M_h, z_h))
    t2 = {k: (None if x is None else torch.empty_like(x)) for k, x in t.items()}
    sets = [(t, out, M_out, z_out),
            (t2, torch.empty_like(out), torch.empty_like(M_out), torch.empty_like(z_out))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        for i in range(n):
            b = i % 2
            ti, oi, Mi, zi = sets[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[b])          # step i - 2 has read this input set
                for kname, x in host.items():
                    if x is not None:
                        ti[kname].copy_(x, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])          # step i - 2's results are copied out
            fwd(ti["q"], ti["k"], ti["v"], ti["beta"], ti["M0"], ti["z0"], oi, Mi, zi, w.N,
                w.rule, stream)
            ev_c[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[b])
                out_h.copy_(oi, non_blocking=True)
                M_h.copy_(Mi, non_blocking=True)
                z_h.copy_(zi, non_blocking=True)
                ev_out[b].record(s_out)

    e2e_run(args.warmup)
    barrier(world)
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(s_in)
    e2e_run(args.steps)
    e_end.record(s_out)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(float(e_start.elapsed_time(e_end)), world, dev)

    # ---- CPU oracle baseline (rank 0, single GPU only) ----
    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        v, dt, desc = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": desc + f"; {dt:.1f} s on 1 host core (fp64, single-threaded C)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic",
            "config": dict(config_of(w), launch="CUDA graph of infini_attn_fwd_noalloc"
                           if graph is not None else "eager infini_attn_fwd calls"),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": w.tokens * args.steps * world / (e2e_ms / 1000.0),
                    "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "pipelined": "copy-in, compute and copy-out streams overlap across steps"},
            "gpu_launches": launches, "kernels": kernels,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
