"""Benchmark: chunked causal linear attention forward + backward on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
lasp_fwd (states, prefix, output) then lasp_bwd (gradient states, suffix,
dQ/dK/dV), as a user calls them. The library's trace brackets each of its
kernel launches with CUDA events on the same stream, so every kernel's
duration is measured live inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Prints one JSON line (rank 0). With N > 1 (launched by torch.distributed.run)
every rank runs the same workload on its own GPU with no data exchange
(independent sequences: weak scaling); the step time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sequence_linear_attention_b200 import inputs as lasp_inputs  # noqa: E402

METRIC = "linear-attn fwd+bwd tokens/s (H16 d128 N64K bf16); % of bf16 tensor peak"
DEFAULT_WORKLOAD = "decayed_bf16_N64K"


# ------------------------------------------------------------ algorithmic work
def algorithmic_bytes(name: str, tokens_heads: int, d: int, C: int, G: int, elem: int) -> float:
    """Bytes a kernel must move per launch: each token tensor once, each state once.

    Per token-head, with e = element size, s = 4 d^2 (one fp32 state), C the
    chunk and G the segment length in tokens:
      chunk_states_* (M_c or dM_c):  read 2 token rows, write s/C        = 2de + s/C
      segment_states_tc:             read 2 token rows, write s/G        = 2de + s/G
      state_scan:                    read and write s/C                  = 2s/C
      segment_scan:                  read and write s/G                  = 2s/G
      state_total:  the decayed total of the segment (or chunk) states,
                    read only                                            = s/G
      chunk_out_*:                   read q, k, v and P, write o         = 4de + s/C
      fwd_walk_tc:  read q, k, v and the segment's P (s/G), write o and
                    the cache: for C <= 128 the bf16 operand tile of the state
                    entering each 128-token tile (s/256), for C > 128 fp32 P of
                    the other chunks (s/C - s/G)
                                               = 4de + s/G + s/256  (C <= 128)
                                               = 4de + s/C          (C > 128)
      chunk_bwd_*:  read q, k, v, dO, P and R, write dq, dk, dv          = 7de + 2s/C
      bwd_walk_tc:  read q, k, v, dO, the cached bf16 tiles (s/256) and the
                    segment's R (s/G), write dq, dk, dv            = 7de + s/256 + s/G
    Gated form (a log-gate per token and key feature, fp32: 4d bytes; the
    gla_*_exact launches count nothing: they return at once on these gates):
      gla_states_*: read 2 token rows and the gates, write s/C         = 2de + 4d + s/C
      gla_scan:     read and write s/C, read the chunk's gate totals   = 2s/C + 4d/C
      gla_out_simt: read q, k, v, the gates and P, write o             = 4de + 4d + s/C
      gla_bwd_simt: read q, k, v, dO, the gates, P and R, write dq, dk,
                    dv and the gate gradient                          = 7de + 8d + 2s/C
      gla_segment_states_tc: the forward's states per segment of G tokens
                    (read 2 token rows and the gates, write s/G) = 2de + 4d + s/G
      gla_segment_scan: read and write s/G, the segments' gate totals = 2s/G + 4d/G
      gla_out_tc:   the walk through each segment: read q, k, v, the gates
                    and the segment's P (s/G), write o and the bf16 tile of
                    diag(e^r) P per 128-token tile     = 4de + 4d + s/G + s/256
      gla_bwd_tc:   the walk back through each segment: read q, k, v, dO, the
                    gates, that bf16 tile and the segment's R (s/G; the states
                    it forms for the segment's other tiles stay in L2), write
                    dq, dk, dv and the gate gradient = 7de + 8d + s/256 + s/G
    """
    s = 4 * d * d
    de = d * elem
    per = {
        "chunk_states_tc": 2 * de + s / C, "chunk_states_simt": 2 * de + s / C,
        "segment_states_tc": 2 * de + s / G,
        "state_scan": 2 * s / C, "segment_scan": 2 * s / G, "state_total": s / G,
        "chunk_out_tc": 4 * de + s / C, "chunk_out_simt": 4 * de + s / C, "fwd_walk_tc": 4 * de + (s / G + s / 256 if C <= 128 else s / C),
        "chunk_bwd_tc": 7 * de + 2 * s / C, "chunk_bwd_simt": 7 * de + 2 * s / C,
        "bwd_walk_tc": 7 * de + s / 256 + s / G,
        # bidirectional form: the sum of the segment states (s/G; the total and
        # its tile per (b, h) are negligible), and one token tensor in, one out
        "bidir_total": s / G, "bidir_apply_tc": 2 * de,
        "gla_states_tc": 2 * de + 4 * d + s / C, "gla_states_simt": 2 * de + 4 * d + s / C,
        "gla_scan": 2 * s / C + 4 * d / C,
        "gla_segment_states_tc": 2 * de + 4 * d + s / G, "gla_segment_scan": 2 * s / G + 4 * d / G,
        "gla_out_tc": 4 * de + 4 * d + s / G + s / 256, "gla_out_simt": 4 * de + 4 * d + s / C,
        "gla_bwd_tc": 7 * de + 8 * d + s / 256 + s / G, "gla_bwd_simt": 7 * de + 8 * d + 2 * s / C,
        # the exact CUDA-core sequence a tensor-core gated call also launches;
        # it returns at once unless a tile's gates leave the factorized range
        "gla_states_exact": 0.0, "gla_scan_exact": 0.0, "gla_out_exact": 0.0, "gla_bwd_exact": 0.0,
    }[name]
    return per * tokens_heads


def cache_bytes(name: str, tokens_heads: int, d: int, C: int, G: int) -> float:
    """The part of :func:`algorithmic_bytes` that is state traffic of the walks'
    own making rather than the step's minimum (q, k, v, dO in; o, dq, dk, dv
    out): the segment-entering states they read and the per-tile state cache
    (LASP page, section 3.4, KV state caching) the forward writes and the
    backward reads back. The roofline's ``frac`` leaves it out; ``frac_with_cache``
    counts it."""
    s = 4 * d * d
    per = {
        "fwd_walk_tc": (s / G + s / 256) if C <= 128 else s / C,
        "bwd_walk_tc": s / 256 + s / G,
        "gla_out_tc": s / G + s / 256,
        "gla_bwd_tc": s / 256 + s / G,
    }.get(name, 0.0)
    return per * tokens_heads


def flops_per_step(tokens_heads: int, d: int, C: int) -> float:
    """fwd 2(2Cd + 2d^2) and bwd 2(5Cd + 4d^2) FLOPs per token-head."""
    return tokens_heads * (2 * (2 * C * d + 2 * d * d) + 2 * (5 * C * d + 4 * d * d))


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# each kernel on this workload, from the ncu capture summarised in profiles/,
# valid only while the kernel's sources hash to the recorded value.
MEASURED_TRAFFIC = {
    # DRAM bytes per launch at the workload's full size: twice the ncu capture of
    # the 32768-token case of the same workload (traffic grows with the tokens)
    "bwd_walk_tc": (["k_tc_bwd_walk.cu", "sm100.cuh", "lasp_common.cuh", "tma_host.h"], "a8458a2dda72b0b5",
                    2 * (723464448 + 365351168)),
    "fwd_walk_tc": (["k_tc_fwd_walk.cu", "sm100.cuh", "lasp_common.cuh", "tma_host.h"], "0ad0edd4699b890d",
                    2 * (437797120 + 226962944)),
    "segment_states_tc": (["k_tc_states.cu", "sm100.cuh", "lasp_common.cuh", "tma_host.h"], "48a5dd38bfe5a0ce",
                          2 * (268479488 + 8521472)),
    # the gated form (bench.py --gated): four times the capture of the 16384-token case
    "gla_bwd_tc": (["k_tc_gla.cu", "sm100.cuh", "lasp_common.cuh", "tma_host.h"], "0ccaa17fdf1decfe",
                   4 * (491264256 + 320168704)),
}


def measured_traffic(kernel: str, workload: str):
    """Recorded DRAM bytes per launch, or None if not captured for the current kernel sources."""
    import hashlib
    if workload != DEFAULT_WORKLOAD or kernel not in MEASURED_TRAFFIC:
        return None
    files, digest, nbytes = MEASURED_TRAFFIC[kernel]
    m = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "sequence_linear_attention_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return nbytes if m.hexdigest()[:16] == digest else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- distributed
def dist_setup():
    """(rank, world, local_rank). Initialises torch.distributed when WORLD_SIZE > 1."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = os.environ.get("LASP_BENCH_BACKEND", "nccl")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(units_per_rank: float, seconds_per_rank: float, world: int, device=None) -> tuple[float, float]:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    t = max_over_ranks(seconds_per_rank, world, device)
    return units_per_rank * world / t, t


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.15)  # the first sample is taken as the timed region starts
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons)}
        loaded = [x for x in sm if smax and x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, rank, world, local):
    import torch
    import sequence_linear_attention_b200 as lasp

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = lasp_inputs.WORKLOADS[args.workload]
    B, N, H, d, C = w["B"], w["N"], w["H"], w["d"], w["C"]
    if args.tokens is not None:
        if args.tokens <= 0 or args.tokens % C:
            raise ValueError(f"--tokens must be a positive multiple of C = {C}")
        N = args.tokens
    bf16 = w["bf16"]
    tdtype = torch.bfloat16 if bf16 else torch.float32
    elem = 2 if bf16 else 4
    T = N // C
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=w["seed"] + 7919 * rank, bf16=bf16, decayed=w["decayed"])

    def host_tensor(x):
        if bf16:
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))

    host = {n: host_tensor(inp[n]).pin_memory() for n in ("q", "k", "v", "do")}
    dv_ = {n: host[n].to(dev) for n in host}
    q, k, v, do = dv_["q"], dv_["k"], dv_["v"], dv_["do"]
    decay = None if inp["lam"] is None else torch.from_numpy(inp["lam"]).to(dev)
    o, dq, dk, dvv = (torch.empty_like(q) for _ in range(4))
    P = torch.empty((B, T, H, d, d), dtype=torch.float32, device=dev)
    R = torch.empty_like(P)
    stream = torch.cuda.current_stream(dev)
    G = lasp.lasp_segment_tokens(N, C, d, 1 if bf16 else 0)

    def step():
        lasp.lasp_fwd(q, k, v, decay, o, C, P)
        lasp.lasp_bwd(q, k, v, decay, do, dq, dk, dvv, C, P, R)

    for _ in range(args.warmup):
        step()
    st, site = lasp.lasp_check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {lasp.lasp_status_string(st)} at site {site}")

    # timed region: the steps as a user runs them (no per-kernel instrumentation)
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            events[i][0].record(stream)
            step()
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    total_ms = sum(a.elapsed_time(b) for a, b in events)
    tokens = B * N
    value, t_max = aggregate(tokens * args.steps, total_ms / 1e3, world, dev)
    ms_per_step = t_max * 1e3 / args.steps

    # kernel durations: a second timed pass in which the library brackets each of
    # its launches with CUDA events on this stream (the event records add about
    # 2 us between launches, so they stay out of the pass that gives `value`)
    ksteps = min(args.steps, 200)
    lasp.lasp_trace_enable(16 * ksteps + 16)
    torch.cuda.synchronize(dev)
    for _ in range(ksteps):
        step()
    torch.cuda.synchronize(dev)
    trace = lasp.lasp_trace_read(16 * ksteps + 16)
    lasp.lasp_trace_enable(0)
    per_kernel = {}
    for name, ms in trace:
        per_kernel.setdefault(name, []).append(ms)
    # the forward and backward separately: each step's launches are lasp_fwd's
    # followed by as many of lasp_bwd's
    per_step = len(trace) // ksteps
    fwd_ms = sum(ms for i, (_, ms) in enumerate(trace) if i % per_step < per_step // 2) / ksteps
    bwd_ms = sum(ms for i, (_, ms) in enumerate(trace) if i % per_step >= per_step // 2) / ksteps

    # end to end through the public API: every step copies its inputs (q, k, v,
    # dO) in from pinned host memory and its results (o, dq, dk, dv) back out.
    # The copies run on two copy streams, so that step i+1's inputs go in and
    # step i-1's results come out while step i's kernels run (PCIe is full
    # duplex); the device buffers alternate between two sets, ordered by events.
    outs_host = {n: torch.empty_like(host["q"]).pin_memory() for n in ("o", "dq", "dk", "dv")}
    # enough steps that the pipeline's fill and drain (the first step's inputs
    # and the last step's results cross alone) do not dominate
    e2e_steps = max(1, min(args.steps, 30))
    ins = [dv_, {n: torch.empty_like(dv_[n]) for n in dv_}]
    outs = [{"o": o, "dq": dq, "dk": dk, "dv": dvv}, {n: torch.empty_like(q) for n in ("o", "dq", "dk", "dv")}]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready, comp_done, out_free = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_issue(i):
        x, y = ins[i % 2], outs[i % 2]
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(comp_done[i % 2])  # step i-2's kernels have read this set
            for n in ("q", "k", "v", "do"):
                x[n].copy_(host[n], non_blocking=True)
            in_ready[i % 2].record(h2d)
        stream.wait_event(in_ready[i % 2])
        if i >= 2:
            stream.wait_event(out_free[i % 2])  # step i-2's results have left this set
        lasp.lasp_fwd(x["q"], x["k"], x["v"], decay, y["o"], C, P, stream=stream.cuda_stream)
        lasp.lasp_bwd(x["q"], x["k"], x["v"], decay, x["do"], y["dq"], y["dk"], y["dv"], C, P, R,
                      stream=stream.cuda_stream)
        comp_done[i % 2].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[i % 2])
            for n in ("o", "dq", "dk", "dv"):
                outs_host[n].copy_(y[n], non_blocking=True)
            out_free[i % 2].record(d2h)

    for i in range(2):
        e2e_issue(i)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d.wait_event(e0)
    for i in range(e2e_steps):
        e2e_issue(i)
    stream.wait_event(out_free[(e2e_steps - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_value, _ = aggregate(tokens * e2e_steps, e0.elapsed_time(e1) / 1e3, world, dev)
    st, site = lasp.lasp_check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {lasp.lasp_status_string(st)} at site {site}")

    # the per-chunk scan on its own (LASP Eq. 10; the prefix of the LASP-2
    # review): the chunk states of the workload, one d x d fp32 state per chunk
    # and head (B * T * H * d * d * 4 bytes, larger than L2), read once and
    # their prefix written once, out of place; L2 is flushed between launches
    scan = time_scan(lasp, k, v, decay, P, R, C, dev, stream)

    peaks = load_peaks()
    th = tokens * H
    names = list(per_kernel)
    top = max(names, key=lambda n: sum(per_kernel[n]))
    kernel_table = {}
    for n in names:
        mean = statistics.mean(per_kernel[n])
        full = algorithmic_bytes(n, th, d, C, G, elem)
        least = full - cache_bytes(n, th, d, C, G)
        kernel_table[n] = {"launches_per_step": len(per_kernel[n]) / ksteps, "ms": round(mean, 4),
                           "GBps": round(least / (mean / 1e3) / 1e9, 1),
                           "hbm_frac": round(least / (mean / 1e3) / 1e9 / peaks["hbm"], 4),
                           "hbm_frac_with_cache": round(full / (mean / 1e3) / 1e9 / peaks["hbm"], 4)}
    achieved = kernel_table[top]["GBps"]
    top_cache = cache_bytes(top, th, d, C, G)
    top_bytes = algorithmic_bytes(top, th, d, C, G, elem) - top_cache
    flops = flops_per_step(th, d, C)
    tflops = flops / (ms_per_step / 1e3) / 1e12
    # a timed region of under a second is a burst (the SMs hold their top
    # clock); longer runs reach the power cap
    burst = t_max < 1.0
    # the attainable rate of the step: min(tensor peak, arithmetic intensity x
    # HBM bandwidth), the intensity over the algorithmic bytes of all launches
    step_bytes = sum(algorithmic_bytes(n, th, d, C, G, elem) * len(per_kernel[n]) / ksteps for n in names)
    attainable = min(peaks["bf16_sustained"], flops / step_bytes * peaks["hbm"] / 1e3)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if bf16 else "f32", "data": "synthetic (seeded normal q,k,v,dO; no dataset)",
        "config": dict(workload_config(args.workload, w, N, world), segment=G),
        "tflops": round(tflops, 2),
        "tensor_peak_frac": round(tflops / (peaks["bf16"] if burst else peaks["bf16_sustained"]), 4),
        "tensor_peak_basis": "burst" if burst else "sustained",
        "tensor_peak_frac_burst": round(tflops / peaks["bf16"], 4),
        "tensor_peak_frac_sustained": round(tflops / peaks["bf16_sustained"], 4),
        "attainable_frac": round(tflops / attainable, 4),
        "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
        "roofline": {"bound": "hbm", "kernel": top, "achieved": round(achieved, 1), "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm"], 4),
                     "traffic": measured_traffic(top, args.workload) if args.tokens is None else None,
                     "algorithmic_bytes": top_bytes, "cache_bytes": top_cache,
                     "frac_with_cache": round((top_bytes + top_cache) / top_bytes * achieved / peaks["hbm"], 4),
                     "peak_source": peaks["source"]},
        "kernels": kernel_table,
        "scan": dict(scan, peak=peaks["hbm"], hbm_frac=round(scan["GBps"] / peaks["hbm"], 4)),
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": 4 * B * N * H * d * elem, "d2h_bytes_per_step": 4 * B * N * H * d * elem,
                "api": "lasp_fwd + lasp_bwd with pinned host buffers; copies overlap the neighbouring steps' kernels"},
        # launches in the timed region: the traced pass's launches per step x steps
        "gpu_launches": int(round(len(trace) / ksteps * args.steps)),
        "clocks": clk.summary(),
    }
    return line


def time_scan(lasp, k, v, decay, M, out, C, dev, stream, launches: int = 10):
    """lasp_state_prefix over the per-chunk states M (filled by
    lasp_chunk_states) into ``out``, timed launch by launch with CUDA events on
    the launching stream; a 256 MiB write between launches flushes L2."""
    import torch
    lasp.lasp_chunk_states(None, k, v, decay, M, C)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
    lasp.lasp_state_prefix(M, out, decay, C)  # warm-up
    for a, b in ev:
        flush.fill_(1)
        a.record(stream)
        lasp.lasp_state_prefix(M, out, decay, C)
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    nbytes = 2 * M.numel() * 4
    return {"kernel": "state_scan", "states_bytes": M.numel() * 4, "bytes_per_launch": nbytes,
            "ms": round(ms, 4), "GBps": round(nbytes / (ms / 1e3) / 1e9, 1), "launches": launches,
            "l2": "flushed between launches (256 MiB write)"}


def run_bidir(args, rank, world, local):
    """The bidirectional (unmasked) form on the workload's shapes (its decay is
    not used): a step is lasp_bidir_fwd + lasp_bidir_bwd. Printed as its own
    line, with its own metric; the default run does not include it."""
    import torch
    import sequence_linear_attention_b200 as lasp

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = lasp_inputs.WORKLOADS[args.workload]
    B, N, H, d = w["B"], (args.tokens or w["N"]), w["H"], w["d"]
    if not w["bf16"] or lasp.lasp_bidir_workspace_floats(B, H, N, d) == 0:
        raise ValueError("the bidirectional form needs a bf16 workload with d = 128 and N a multiple of 128")
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=w["seed"] + 7919 * rank, bf16=True, decayed=False)
    q, k, v, do = (torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16)).view(torch.bfloat16).to(dev)
                   for n in ("q", "k", "v", "do"))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    ws = torch.empty(lasp.lasp_bidir_workspace_floats(B, H, N, d), dtype=torch.float32, device=dev)
    dws = torch.empty_like(ws)
    stream = torch.cuda.current_stream(dev)
    G = lasp.lasp_segment_tokens(N, 128, d, 1)

    def step():
        lasp.lasp_bidir_fwd(q, k, v, o, ws)
        lasp.lasp_bidir_bwd(q, k, v, do, dq, dk, dv, ws, dws)

    for _ in range(args.warmup):
        step()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            events[i][0].record(stream)
            step()
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    tokens = B * N
    value, t_max = aggregate(tokens * args.steps, sum(a.elapsed_time(b) for a, b in events) / 1e3, world, dev)
    ksteps = min(args.steps, 200)
    lasp.lasp_trace_enable(16 * ksteps + 16)
    for _ in range(ksteps):
        step()
    torch.cuda.synchronize(dev)
    trace = lasp.lasp_trace_read(16 * ksteps + 16)
    lasp.lasp_trace_enable(0)
    st, site = lasp.lasp_check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {lasp.lasp_status_string(st)} at site {site}")
    per_kernel = {}
    for name, ms in trace:
        per_kernel.setdefault(name, []).append(ms)
    peaks = load_peaks()
    th = tokens * H
    kernel_table = {}
    for n, ms in per_kernel.items():
        mean = statistics.mean(ms)
        gbps = algorithmic_bytes(n, th, d, 128, G, 2) / (mean / 1e3) / 1e9
        kernel_table[n] = {"launches_per_step": len(ms) / ksteps, "ms": round(mean, 4), "GBps": round(gbps, 1),
                           "hbm_frac": round(gbps / peaks["hbm"], 4)}
    top = max(per_kernel, key=lambda n: sum(per_kernel[n]))
    return {
        "metric": "bidirectional linear-attn fwd+bwd tokens/s", "impl": "bidirectional",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_max * 1e3 / args.steps, 4), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded normal q,k,v,dO; no dataset)",
        "config": {"workload": args.workload, "B": B, "H": H, "N": N, "d": d, "segment": G, "decay": "none"},
        "roofline": {"bound": "hbm", "kernel": top, "achieved": kernel_table[top]["GBps"], "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": kernel_table[top]["hbm_frac"], "peak_source": peaks["source"]},
        "kernels": kernel_table,
        "gpu_launches": int(round(len(trace) / ksteps * args.steps)),
        "clocks": clk.summary(),
    }


def run_gated(args, rank, world, local):
    """The gated form (a log-gate per token and key feature) on the workload's
    shapes, C = 128: a step is lasp_gla_fwd + lasp_gla_bwd, gates
    log(sigmoid(x)) / 16. Printed as its own line, with its own metric; the
    default run does not include it."""
    import torch
    import sequence_linear_attention_b200 as lasp

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = lasp_inputs.WORKLOADS[args.workload]
    B, N, H, d, C = w["B"], (args.tokens or w["N"]), w["H"], w["d"], 128
    if not w["bf16"] or d != 128 or N % C:
        raise ValueError("the gated form is timed on a bf16 workload with d = 128 and N a multiple of 128")
    seed = w["seed"] + 7919 * rank
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=seed, bf16=True, decayed=False)
    q, k, v, do = (torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16)).view(torch.bfloat16).to(dev)
                   for n in ("q", "k", "v", "do"))
    g = torch.from_numpy(lasp_inputs.make_log_gates(B, N, H, d, seed=seed)).to(dev)
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    dg = torch.empty_like(g)
    cache = torch.empty(lasp.lasp_gla_cache_floats(B, H, N, d, C), dtype=torch.float32, device=dev)
    ws = torch.empty(B * (N // C) * H * d * d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lasp.lasp_gla_fwd(q, k, v, g, o, C, cache)
        lasp.lasp_gla_bwd(q, k, v, g, do, dq, dk, dv, dg, C, cache, ws)

    for _ in range(args.warmup):
        step()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            events[i][0].record(stream)
            step()
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    tokens = B * N
    value, t_max = aggregate(tokens * args.steps, sum(a.elapsed_time(b) for a, b in events) / 1e3, world, dev)
    ksteps = min(args.steps, 200)
    lasp.lasp_trace_enable(16 * ksteps + 16)
    for _ in range(ksteps):
        step()
    torch.cuda.synchronize(dev)
    trace = lasp.lasp_trace_read(16 * ksteps + 16)
    lasp.lasp_trace_enable(0)
    st, site = lasp.lasp_check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {lasp.lasp_status_string(st)} at site {site}")
    per_kernel = {}
    for name, ms in trace:
        per_kernel.setdefault(name, []).append(ms)
    peaks = load_peaks()
    th = tokens * H
    kernel_table = {}
    G = lasp.lasp_segment_tokens(N, C, d, lasp.LASP_BF16)  # the forward walk's segment
    for n, ms in per_kernel.items():
        mean = statistics.mean(ms)
        gbps = algorithmic_bytes(n, th, d, C, G, 2) / (mean / 1e3) / 1e9
        kernel_table[n] = {"launches_per_step": len(ms) / ksteps, "ms": round(mean, 4), "GBps": round(gbps, 1),
                           "hbm_frac": round(gbps / peaks["hbm"], 4)}
    top = max(per_kernel, key=lambda n: sum(per_kernel[n]))
    return {
        "metric": "gated linear-attn fwd+bwd tokens/s", "impl": "gated",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_max * 1e3 / args.steps, 4), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded normal q,k,v,dO; log-gates log(sigmoid(x))/16; no dataset)",
        "config": {"workload": args.workload, "B": B, "H": H, "N": N, "d": d, "C": C, "gates": "log(sigmoid(x))/16",
                   "l2": "inputs larger than L2"},
        "roofline": {"bound": "hbm", "kernel": top, "achieved": kernel_table[top]["GBps"], "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": kernel_table[top]["hbm_frac"],
                     "traffic": measured_traffic(top, args.workload) if N == w["N"] else None,
                     "algorithmic_bytes": algorithmic_bytes(top, th, d, C, G, 2), "peak_source": peaks["source"]},
        "kernels": kernel_table,
        "gpu_launches": int(round(len(trace) / ksteps * args.steps)),
        "clocks": clk.summary(),
    }


def softmax_flops(name: str, B: int, H: int, N: int, d: int) -> float:
    """Tensor-core FLOPs of one launch of the softmax-attention kernels over
    the causal pairs (j <= i: N (N + 1) / 2 per head), 2 d per pair and
    product: the forward computes S and P V (4 d per pair); the dK/dV kernel
    S^T, dP^T, dV and dK (8 d); the dQ kernel S, dP and dQ (6 d, of which S and
    dP repeat the dK/dV kernel's: the minimal backward is 10 d per pair)."""
    pairs = B * H * N * (N + 1) / 2
    return {"softmax_fwd_tc": 4, "softmax_dkdv_tc": 8, "softmax_dq_tc": 6, "softmax_delta": 0}[name] * d * pairs


def run_softmax(args, rank, world, local):
    """The softmax-attention layers of a hybrid model (LASP-2H) on the
    workload's shapes: a step is lasp_softmax_fwd + lasp_softmax_bwd over one
    whole sequence (causal, scale d^-1/2), inputs standard normal. Printed as
    its own line, with its own metric; the default run does not include it."""
    import torch
    import sequence_linear_attention_b200 as lasp

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = lasp_inputs.WORKLOADS[args.workload]
    B, N, H, d = w["B"], (args.tokens or w["N"]), w["H"], w["d"]
    if not w["bf16"] or d != 128:
        raise ValueError("softmax attention is timed on a bf16 workload with d = 128")
    inp = lasp_inputs.make_attention_inputs(B, N, N, H, d, seed=w["seed"] + 7919 * rank)
    q, k, v, do = (torch.from_numpy(np.ascontiguousarray(inp[n]).view(np.int16)).view(torch.bfloat16).to(dev)
                   for n in ("q", "k", "v", "do"))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    delta = torch.empty_like(lse)
    stream = torch.cuda.current_stream(dev)

    def step():
        lasp.lasp_softmax_fwd(q, k, v, o, lse)
        lasp.lasp_softmax_bwd(q, k, v, o, lse, do, dq, dk, dv, delta)

    for _ in range(args.warmup):
        step()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            events[i][0].record(stream)
            step()
            events[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    tokens = B * N
    value, t_max = aggregate(tokens * args.steps, sum(a.elapsed_time(b) for a, b in events) / 1e3, world, dev)
    ksteps = min(args.steps, 20)
    lasp.lasp_trace_enable(8 * ksteps + 8)
    for _ in range(ksteps):
        step()
    torch.cuda.synchronize(dev)
    trace = lasp.lasp_trace_read(8 * ksteps + 8)
    lasp.lasp_trace_enable(0)
    st, site = lasp.lasp_check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {lasp.lasp_status_string(st)} at site {site}")
    per_kernel = {}
    for name, ms in trace:
        per_kernel.setdefault(name, []).append(ms)
    peaks = load_peaks()
    burst = t_max < 1.0
    peak = peaks["bf16"] if burst else peaks["bf16_sustained"]
    kernel_table = {}
    for n, ms in per_kernel.items():
        mean = statistics.mean(ms)
        tf = softmax_flops(n, B, H, N, d) / (mean / 1e3) / 1e12
        kernel_table[n] = {"launches_per_step": len(ms) / ksteps, "ms": round(mean, 4), "TFLOPs": round(tf, 1),
                           "tensor_frac": round(tf / peak, 4)}
    top = max(per_kernel, key=lambda n: sum(per_kernel[n]))
    ms_step = t_max * 1e3 / args.steps
    # the step at the minimal count: forward 4 d and backward 10 d per causal pair
    step_tf = 14 * d * B * H * N * (N + 1) / 2 / (ms_step / 1e3) / 1e12
    return {
        "metric": "softmax-attention (LASP-2H layer) fwd+bwd tokens/s", "impl": "softmax",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded standard-normal q, k, v, dO; no dataset)",
        "config": {"workload": args.workload, "B": B, "H": H, "N": N, "d": d, "causal": True,
                   "scale": "d^-1/2", "l2": "inputs larger than L2" if 4 * B * N * H * d * 2 > (126 << 20)
                   else "inputs fit in L2"},
        "tflops": round(step_tf, 1), "tensor_peak_frac": round(step_tf / peak, 4),
        "tensor_peak_basis": "burst" if burst else "sustained",
        "roofline": {"bound": "tensor", "kernel": top, "achieved": kernel_table[top]["TFLOPs"], "peak": peak,
                     "unit": "TFLOP/s", "frac": kernel_table[top]["tensor_frac"], "traffic": None,
                     "algorithmic_flops": softmax_flops(top, B, H, N, d), "peak_source": peaks["source"]},
        "kernels": kernel_table,
        "gpu_launches": int(round(len(trace) / ksteps * args.steps)),
        "clocks": clk.summary(),
    }


def cpu_baseline_softmax(args):
    """The oracle's softmax attention fwd+bwd on a bounded sample: all heads,
    the first 4096 positions of batch 0. Its cost grows with the square of the
    length, so the value is the sample's time per token scaled by the ratio of
    the lengths (the workload's per-token work over the sample's)."""
    import oracle
    n = 4096
    w = lasp_inputs.WORKLOADS[args.workload]
    N = args.tokens or w["N"]
    inp = lasp_inputs.make_attention_inputs(1, n, n, w["H"], w["d"], seed=w["seed"], bf16=True)
    f = {x: lasp_inputs.as_f32(inp[x], True) for x in ("q", "k", "v", "do")}
    oracle.build()
    t0 = time.perf_counter()
    oracle.softmax_fwd(f["q"], f["k"], f["v"])
    oracle.softmax_bwd(f["q"], f["k"], f["v"], f["do"])
    dt = time.perf_counter() - t0
    value = 1.0 / (dt / n * (N / n))
    return {"value": round(value, 1), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"fp64 oracle softmax attention fwd+bwd, batch 0, all heads, first {n} positions "
                      f"({dt:.1f} s), per-token time scaled by {N}/{n} to the workload's length"}


def run_lasp2(args, rank, world, local):
    """LASP-2 sequence parallelism: one sequence of the workload split over the
    ranks, rank r holding tokens [r L, (r + 1) L) with L = N / world; a step is
    lasp2_fwd + lasp2_bwd, with one AllGather of shard states per direction
    (NCCL). The sequence is the same at every world size (strong scaling). At
    one rank the process group has one member and the gather is a copy. Printed
    as its own line; the default run does not include it."""
    import tempfile

    import torch
    import torch.distributed as dist

    import sequence_linear_attention_b200 as lasp
    from sequence_linear_attention_b200 import lasp2

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = lasp_inputs.WORKLOADS[args.workload]
    B, N, H, d, C = w["B"], (args.tokens or w["N"]), w["H"], w["d"], w["C"]
    if N % world or (N // world) % C:
        raise ValueError("the sequence must split into equal shards of whole chunks")
    L = N // world
    own_group = None
    if world == 1:
        fd, path = tempfile.mkstemp(prefix="lasp2_pg_")
        os.close(fd)
        dist.init_process_group("nccl", store=dist.FileStore(path, 1), rank=0, world_size=1)
        own_group = path
    inp = lasp_inputs.make_shard_inputs(B, N, H, d, seed=w["seed"], row0=rank * L, rows=L, bf16=w["bf16"],
                                        decayed=w["decayed"])
    elem = 2 if w["bf16"] else 4
    to_dev = ((lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev))
              if w["bf16"] else (lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)))
    q, k, v, do = (to_dev(inp[n]) for n in ("q", "k", "v", "do"))
    del inp["q"], inp["k"], inp["v"], inp["do"]
    decay = None if inp["lam"] is None else torch.from_numpy(inp["lam"]).to(dev)
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    cache = torch.empty((B, L // C, H, d, d), dtype=torch.float32, device=dev)
    ws = torch.empty_like(cache)
    stream = torch.cuda.current_stream(dev)

    parts = args.parts or lasp2.default_parts(q, C, world)

    def step():
        lasp2.lasp2_fwd(q, k, v, decay, o, C, cache, parts=parts)
        lasp2.lasp2_bwd(q, k, v, decay, do, dq, dk, dv, C, cache, ws, parts=parts)

    try:
        for _ in range(args.warmup):
            step()
        events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        with ClockSampler(local) as clk:
            for i in range(args.steps):
                events[i][0].record(stream)
                step()
                events[i][1].record(stream)
            torch.cuda.synchronize(dev)
        barrier(world, dev)
        value, t_max = aggregate(B * L * args.steps, sum(a.elapsed_time(b) for a, b in events) / 1e3, world, dev)
        ksteps = min(args.steps, 50)
        lasp.lasp_trace_enable(16 * ksteps + 16)
        for _ in range(ksteps):
            step()
        torch.cuda.synchronize(dev)
        trace = lasp.lasp_trace_read(16 * ksteps + 16)
        lasp.lasp_trace_enable(0)
        st, site = lasp.lasp_check_device_status()
        if st != 0:
            raise RuntimeError(f"device status {lasp.lasp_status_string(st)} at site {site}")
    finally:
        if own_group is not None:
            dist.destroy_process_group()
            if os.path.exists(own_group):  # the store may have removed it
                os.unlink(own_group)
    per_kernel = {}
    for name, ms in trace:
        per_kernel.setdefault(name, []).append(ms)
    peaks = load_peaks()
    th = B * L * H
    G = lasp.lasp_segment_tokens(L, C, d, lasp.LASP_BF16 if w["bf16"] else lasp.LASP_F32)

    def shard_bytes(name):
        # the scans over the W gathered shard states
        if name == "state_scan":
            return 2 * world * B * H * 4 * d * d
        return algorithmic_bytes(name, th, d, C, G, elem)

    kernel_table = {}
    for n, ms in per_kernel.items():
        mean = statistics.mean(ms)
        gbps = shard_bytes(n) / (mean / 1e3) / 1e9
        kernel_table[n] = {"launches_per_step": len(ms) / ksteps, "ms": round(mean, 4), "GBps": round(gbps, 1),
                           "hbm_frac": round(gbps / peaks["hbm"], 4)}
    top = max(per_kernel, key=lambda n: sum(per_kernel[n]))
    return {
        "metric": "LASP-2 sequence-parallel linear-attn fwd+bwd tokens/s", "impl": "lasp2",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_max * 1e3 / args.steps, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16" if w["bf16"] else "f32",
        "data": "synthetic (seeded normal q,k,v,dO; no dataset)",
        "config": {"workload": args.workload, "B": B, "H": H, "N": N, "d": d, "C": C, "shard_tokens": L,
                   "segment": G, "parts": parts,
                   "parallelism": f"sequence x{world} (AllGathers of shard states per direction, one per part of "
                                  f"the (b, h) pairs, each overlapping the next part's work)",
                   "l2": "inputs larger than L2"},
        "roofline": {"bound": "hbm", "kernel": top, "achieved": kernel_table[top]["GBps"], "peak": peaks["hbm"],
                     "unit": "GB/s", "frac": kernel_table[top]["hbm_frac"], "traffic": None,
                     "algorithmic_bytes": shard_bytes(top), "peak_source": peaks["source"]},
        "kernels": kernel_table,
        "gpu_launches": int(round(len(trace) / ksteps * args.steps)),
        "clocks": clk.summary(),
    }


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(args, tokens: int):
    """A bounded sample of the workload for the fp64 oracle: all heads, the
    first `tokens` positions of batch 0 (per-token work does not depend on N)."""
    w = lasp_inputs.WORKLOADS[args.workload]
    inp = lasp_inputs.make_inputs(1, tokens, w["H"], w["d"], seed=w["seed"], bf16=w["bf16"], decayed=w["decayed"])
    return [lasp_inputs.as_f32(inp[n], w["bf16"]) for n in ("q", "k", "v", "do")] + [inp["lam"]]


def time_oracle(args, tokens: int, reps: int = 1):
    import oracle
    q, k, v, do, lam = oracle_sample(args, tokens)
    oracle.build()
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.fwd(q, k, v, lam)
        oracle.bwd(q, k, v, do, lam)
    return tokens * reps / (time.perf_counter() - t0), oracle.num_threads()


def cpu_baseline(args):
    # about 10-30 s of host work: all heads over 32768 positions of the workload
    tokens = 32768
    value, cores = time_oracle(args, tokens)
    return {"value": round(value, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle fwd+bwd, batch 0, all heads, first {tokens} positions"}


def cpu_baseline_bidir(args):
    """The oracle's bidirectional fwd+bwd on a bounded sample (all heads, the
    first 32768 positions of batch 0), for the --bidir line."""
    import oracle
    tokens = 32768
    w = lasp_inputs.WORKLOADS[args.workload]
    inp = lasp_inputs.make_inputs(1, tokens, w["H"], w["d"], seed=w["seed"], bf16=w["bf16"], decayed=False)
    q, k, v, do = (lasp_inputs.as_f32(inp[n], w["bf16"]) for n in ("q", "k", "v", "do"))
    oracle.build()
    t0 = time.perf_counter()
    oracle.bidir_fwd(q, k, v)
    oracle.bidir_bwd(q, k, v, do)
    value = tokens / (time.perf_counter() - t0)
    return {"value": round(value, 1), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"fp64 oracle bidirectional fwd+bwd, batch 0, all heads, first {tokens} positions"}


def cpu_baseline_gated(args):
    """The oracle's gated fwd+bwd on a bounded sample (all heads, the first
    32768 positions of batch 0, the bench's gates), for the --gated line."""
    import oracle
    tokens = 32768
    w = lasp_inputs.WORKLOADS[args.workload]
    inp = lasp_inputs.make_inputs(1, tokens, w["H"], w["d"], seed=w["seed"], bf16=w["bf16"], decayed=False)
    q, k, v, do = (lasp_inputs.as_f32(inp[n], w["bf16"]) for n in ("q", "k", "v", "do"))
    g = lasp_inputs.make_log_gates(1, tokens, w["H"], w["d"], seed=w["seed"])
    oracle.build()
    t0 = time.perf_counter()
    oracle.gla_fwd(q, k, v, g)
    oracle.gla_bwd(q, k, v, g, do)
    value = tokens / (time.perf_counter() - t0)
    return {"value": round(value, 1), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"fp64 oracle gated fwd+bwd, batch 0, all heads, first {tokens} positions"}


def workload_config(name: str, w: dict, N: int, world: int) -> dict:
    """The `config` of the main line and of the reference arm: the workload,
    its shape and decay, how the inputs relate to L2, and the multi-GPU mode."""
    elem = 2 if w["bf16"] else 4
    return {"workload": name, "B": w["B"], "H": w["H"], "N": N, "d": w["d"], "C": w["C"],
            "decay": "per-head 1-2^-(5+8h/H)" if w["decayed"] else "none",
            "l2": "inputs larger than L2 (q, k, v, dO are 4 x %d MiB)" % (w["B"] * N * w["H"] * w["d"] * elem >> 20),
            "parallelism": f"replicas x{world} (independent sequences, no collective)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    tokens = 2048
    import oracle
    q, k, v, do, lam = oracle_sample(args, tokens)
    oracle.build()
    for _ in range(args.warmup):
        oracle.fwd(q, k, v, lam)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.fwd(q, k, v, lam)
        oracle.bwd(q, k, v, do, lam)
    dt = time.perf_counter() - t0
    value = tokens * args.steps / dt
    w = lasp_inputs.WORKLOADS[args.workload]
    sample = f"fp64 oracle fwd+bwd, batch 0, all heads, first {tokens} positions per step"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(args.workload, w, w["N"], world),
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "kind": "oracle",
                         "cores": __import__("oracle").num_threads(), "sample": sample},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=None, choices=sorted(lasp_inputs.WORKLOADS),
                    help=f"workload (default {DEFAULT_WORKLOAD}; with --lasp2, shards_bf16_N2M)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bidir", action="store_true",
                    help="time the bidirectional (unmasked) form instead (its own metric and line)")
    ap.add_argument("--gated", action="store_true",
                    help="time the gated form (a log-gate per token and key feature) instead (its own metric and line)")
    ap.add_argument("--softmax", action="store_true",
                    help="time the softmax-attention layers of the hybrid model (LASP-2H) instead "
                         "(its own metric and line)")
    ap.add_argument("--lasp2", action="store_true",
                    help="time LASP-2 sequence parallelism instead: one sequence split over the ranks "
                         "(its own metric and line)")
    ap.add_argument("--parts", type=int, default=None,
                    help="with --lasp2: parts of the (b, h) pairs whose exchanges overlap (default: the library's)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="sequence length N instead of the workload's (a smaller case of the same shape, for "
                         "profiling); the line is then not the workload's headline number")
    args = ap.parse_args(argv)
    if args.workload is None:
        args.workload = "shards_bf16_N2M" if args.lasp2 else DEFAULT_WORKLOAD
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        elif args.bidir:
            line = run_bidir(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline_bidir(args)
        elif args.lasp2:
            line = run_lasp2(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(args)
        elif args.softmax:
            line = run_softmax(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline_softmax(args)
        elif args.gated:
            line = run_gated(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline_gated(args)
        else:
            line = run_gpu(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(args)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
