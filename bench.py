#!/usr/bin/env python
"""Benchmark of the looped GDN mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the looped-prefill workload: T = 4 loops of (q/k/v projection ->
GDN chunkwise prefill with in-kernel q/k L2 norm -> loop residual) over one
sequence of 4096 tokens, d = 2048 (16 heads x 128).  Inputs are resident in
HBM when the timed region starts; L2 is flushed between steps (256 MiB write).
`value` is whole-job tokens/s (sequence tokens through all T loops).  The same
JSON line carries the roofline of the prefill kernel, the CPU oracle baseline,
the end-to-end figure through host buffers, and the other workloads (long
prefill, variable-length prefill, decode state streaming) measured on their
own.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of
the workload (weak scaling, no collective on the data path); the timed region
is bracketed by a barrier + synchronize and the time is the max over ranks.

--impl reference times the CPU oracle (rank 0 only) on the same workload:
every step is the whole 4096-token sequence through all 4 loops.
"""
from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "looped GDN prefill tokens/s (T=4) and decode state-HBM GB/s vs B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the prefill kernel sources (the kernels, their shared device code
    and their tensor-map setup): ncu traffic figures are reported only while
    they were taken on the kernel as it stands."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "looped_linear_attention_b200", "csrc")
    for name in ("common.cuh", "tma_host.h", "gdn_prefill_tc.cu"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """Per-launch DRAM traffic of the prefill kernel from the committed ncu summary,
    if it was captured on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "gdn_prefill_tc_looped_prefill.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel_source_hash") == kernel_source_hash():
            return d.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clock and clock-event reasons sampled during a timed region.

    NVML is polled every `period_s` from a background thread (the timed regions
    here last milliseconds, too short for nvidia-smi's start-up); the device is
    matched to the CUDA device by PCI location.  nvidia-smi -lms is the fallback
    when NVML is unavailable."""

    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    _NVML_NAMES = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
                   "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
                   "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
                   "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index: int, period_s: float = 0.002):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []      # (sm_mhz, reason bitmask or set of names)
        self.max_mhz = None
        self.proc = None
        self.thread = None

    def _nvml_handle(self, nv):
        import torch
        props = torch.cuda.get_device_properties(self.cuda_index)
        want = (getattr(props, "pci_domain_id", None), getattr(props, "pci_bus_id", None),
                getattr(props, "pci_device_id", None))
        for i in range(nv.nvmlDeviceGetCount()):
            h = nv.nvmlDeviceGetHandleByIndex(i)
            pci = nv.nvmlDeviceGetPciInfo(h)
            if (pci.domain, pci.bus, pci.device) == want:
                return h
        return None

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._nvml_handle(nv)
            if h is None:
                raise RuntimeError("no NVML device matches the CUDA device")
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            masks = {n: getattr(nv, a) for n, a in self._NVML_NAMES.items()}
            self.stop = threading.Event()

            def poll():
                while not self.stop.is_set():
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(sm), {n for n, m in masks.items() if r & m}))
                    self.stop.wait(self.period)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            for line in out.splitlines():
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, self.max_mhz = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                self.samples.append((sm, {n for n, v in zip(self.REASONS, parts[5:9])
                                          if v.lower() == "active"}))

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ byte / flop accounting
def prefill_bytes_per_token_head(dk, dv, io_bytes=2, residual=False):
    """Algorithmic HBM bytes of one token of one head in one prefill launch:
    q, k (dk each), v and o (dv each) in the io dtype, a and b in fp32; with the
    loop residual fused into the output, also h_prev (dv, io dtype)."""
    return io_bytes * (2 * dk + 2 * dv + (dv if residual else 0)) + 8


def prefill_state_bytes(n_seq, H, dk, dv, s0, st):
    return n_seq * H * dk * dv * 4 * ((1 if s0 else 0) + (1 if st else 0))


def decode_bytes_per_head_state(dk, dv, io_bytes=2):
    """State read + write (fp32) plus q, k, v, o and a, b."""
    return 2 * dk * dv * 4 + io_bytes * (2 * dk + 2 * dv) + 8


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local):
    import numpy as np
    import torch

    import looped_linear_attention_b200 as lla
    from looped_linear_attention_b200 import build as lib_build
    from looped_linear_attention_b200 import workloads as W

    if rank == 0 and not os.path.exists(lib_build.LIB_PATH):
        lib_build.build()
    barrier(world)
    lla.library()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream()

    wl = W.WORKLOADS["looped_prefill"]
    inp = W.looped_inputs(wl, dev)
    L, d = inp["L"], inp["d"]
    runner = lla.LoopedPrefill(L, wl.H, wl.dk, wl.dv, wl.loops, dev, time_mixer=True)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    out = torch.empty(L, d, dtype=torch.bfloat16, device=dev)

    def step():
        runner.run(inp["h0"], inp["Wq"], inp["Wk"], inp["Wv"], inp["a"], inp["b"], inp["rho"],
                   out=out)

    def timed(one_step, sampler=None):
        """W warm-up steps, then K steps between CUDA events on the launching
        stream (L2 flushed before each); returns the per-step milliseconds."""
        for _ in range(args.warmup):
            flush.zero_()
            one_step()
        torch.cuda.synchronize()
        events = []
        barrier(world)
        torch.cuda.synchronize()
        with (sampler if sampler is not None else contextlib.nullcontext()):
            for _ in range(args.steps):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                one_step()
                e1.record(stream)
                events.append((e0, e1))
            torch.cuda.synchronize()
        barrier(world)
        return [a.elapsed_time(b) for a, b in events]

    # stream-launched steps: per-mixer-call CUDA events for the roofline
    step_ms_stream = timed(step)
    gdn_events = list(runner.mixer_events)[-args.steps * wl.loops:]
    runner.time_mixer = False
    # the step as one CUDA-graph replay (every launch of the T loops, no host
    # work between them): the headline value
    runner_g = lla.LoopedPrefill(L, wl.H, wl.dk, wl.dv, wl.loops, dev)
    out_g = torch.empty(L, d, dtype=torch.bfloat16, device=dev)
    graph, _ = runner_g.capture(inp["h0"], inp["Wq"], inp["Wk"], inp["Wv"], inp["a"], inp["b"],
                                inp["rho"], out=out_g)
    clocks = ClockSampler(local)
    step_ms = timed(graph.replay, clocks)
    total_s = max_over_ranks(sum(step_ms) / 1e3, world)
    tokens_per_step = L
    value = world * tokens_per_step * args.steps / total_s
    gdn_ms = [a.elapsed_time(b) for a, b in gdn_events]
    gdn_avg_s = statistics.mean(gdn_ms) / 1e3
    gdn_bytes = prefill_bytes_per_token_head(wl.dk, wl.dv, residual=runner.fused_residual) * L * wl.H
    achieved = gdn_bytes / gdn_avg_s / 1e9
    hbm_peak = peaks["hbm_gbs"]
    # this library's kernels per loop: the mixer (one launch per pass, plus the
    # combine on the segmented schedule) and the loop residual
    sched = lla.prefill_schedule(1, L, wl.H, wl.dk, wl.dv)
    mixer_launches = sched["launches"]
    launches = args.steps * wl.loops * runner_g.launches_per_loop()

    # ---- end to end through host buffers (pinned), same step
    e2e = run_e2e(args, runner, inp, wl, dev, stream, world)

    # ---- other workloads, each on its own
    extras = {}
    if not args.no_extras:
        del flush
        torch.cuda.empty_cache()
        extras["long_prefill"] = bench_prefill_workload(W.WORKLOADS["long_prefill"], dev, args,
                                                        peaks, world)
        torch.cuda.empty_cache()
        extras["decode"] = bench_decode(W.WORKLOADS["decode"], dev, args, peaks, world)
        torch.cuda.empty_cache()
        extras["varlen"] = bench_prefill_workload(W.WORKLOADS["varlen"], dev, args, peaks, world)
        torch.cuda.empty_cache()
        extras["backward"] = bench_backward(dev, args, peaks, world)
        torch.cuda.empty_cache()
        extras["swa"] = bench_swa(dev, args, peaks, world)
        torch.cuda.empty_cache()
        extras["kda"] = bench_kda(dev, args, peaks, world)
        torch.cuda.empty_cache()

    st = lla.gdn_get_device_status()
    if st != lla.GDN_OK:
        raise RuntimeError(f"device status after the benchmark: {lla.status_string(st)}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)
        # each workload's oracle beside its GPU figure
        for name in ("long_prefill", "varlen"):
            if name in extras:
                extras[name]["cpu_baseline"] = cpu_baseline_prefill(name)
        if "decode" in extras:
            extras["decode"]["cpu_baseline"] = cpu_baseline_decode()
        if "backward" in extras:
            extras["backward"]["cpu_baseline"] = cpu_baseline_backward()
        if "swa" in extras:
            extras["swa"]["cpu_baseline"] = cpu_baseline_swa()
        if "kda" in extras:
            extras["kda"]["cpu_baseline"] = cpu_baseline_kda()

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_s * 1e3 / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; random-init projection weights)",
        "step_launch": "one CUDA-graph replay per step (all T loops; LoopedPrefill.capture)",
        "ms_per_step_stream": max_over_ranks(sum(step_ms_stream) / 1e3, world) * 1e3 / args.steps,
        "config": {"workload": "looped_prefill", "batch": 1, "seq_len": L, "d_model": d,
                   "heads": wl.H, "dk": wl.dk, "dv": wl.dv, "loops": wl.loops, "chunk": 64,
                   "parallelism": f"replicas x{world}", "l2": "flushed between steps (256 MiB write)"},
        "roofline": {"kernel": "gdn_prefill_tc", "bound": "hbm", "achieved": achieved,
                     "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                     "peak_source": peak_kind, "traffic": profiled_traffic(),
                     "algorithmic_bytes_per_launch": gdn_bytes,
                     "avg_launch_ms": gdn_avg_s * 1e3,
                     "schedule": (f"segmented: segment 0 of {sched['seg0_tok']} tokens in full "
                                  f"beside the state pass of {sched['n_segs'] - 1} segments of "
                                  f"{sched['seg_tok']} tokens, combine, output pass "
                                  f"({mixer_launches} launches per mixer call, timed together)"
                                  if sched["n_segs"] > 1
                                  else "one pass per chain (1 launch per mixer call)")},
        "gpu_launches": launches,
        "e2e": e2e,
        "clocks": clocks.summary(),
        "workloads": extras,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, runner, inp, wl, dev, stream, world):
    """Same step through the public API with the inputs in pinned host memory:
    every step copies h0, a, b in and h^(T) out inside the timed region;
    HostPipeline overlaps one step's copies with its neighbours' compute."""
    import torch
    import looped_linear_attention_b200 as lla
    h_host = inp["h0"].cpu().pin_memory()
    a_host = inp["a"].cpu().pin_memory()
    b_host = inp["b"].cpu().pin_memory()
    out_host = [torch.empty(inp["L"], inp["d"], dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    pipe = lla.HostPipeline(runner, dev)

    def step(i):
        pipe.submit(h_host, a_host, b_host, out_host[i % 2], inp["Wq"], inp["Wk"], inp["Wv"],
                    inp["rho"])

    for i in range(args.warmup):
        step(i)
    pipe.join()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.start_after(stream)              # the first copy-in starts after e0
    for i in range(args.steps):
        step(i)
    pipe.join(stream)                     # e1 after the last copy-out
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    h2d = h_host.numel() * 2 + a_host.numel() * 4 + b_host.numel() * 4
    d2h = out_host[0].numel() * 2
    return {"value": world * inp["L"] * args.steps / t, "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "copies of each step overlap the neighbouring steps' compute (HostPipeline)"}


def bench_prefill_workload(wl, dev, args, peaks, world):
    """T = wl.loops prefill launches per step over the same inputs (each loop from
    its S0); returns tokens/s, GB/s and fraction of the HBM roof."""
    import torch
    import looped_linear_attention_b200 as lla
    from looped_linear_attention_b200 import workloads as W
    inp = W.prefill_inputs(wl, dev)
    cu = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).to(dev)
    o = torch.empty(inp["total_tokens"], wl.H, wl.dv, dtype=wl.dtype, device=dev)
    ST = torch.empty(inp["n_seq"], wl.H, wl.dk, wl.dv, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        for _ in range(wl.loops):
            lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], cu,
                              n_seq=inp["n_seq"], o=o, S_T=ST)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n = max(1, args.steps)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record(stream)
        for _ in range(n):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world) / n
    tokens = inp["total_tokens"]
    bytes_launch = (prefill_bytes_per_token_head(wl.dk, wl.dv) * tokens * wl.H
                    + prefill_state_bytes(inp["n_seq"], wl.H, wl.dk, wl.dv, inp["S0"] is not None, True))
    launch_s = t / wl.loops
    gbs = bytes_launch / launch_s / 1e9
    res = {"tokens_per_s": world * tokens / t, "ms_per_step": t * 1e3, "loops": wl.loops,
           "tokens": tokens, "heads": wl.H, "dk": wl.dk, "dv": wl.dv,
           "achieved_gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
           "algorithmic_bytes_per_launch": bytes_launch, "clocks": clocks.summary()}
    del inp, o, ST
    return res


def bench_decode(wl, dev, args, peaks, world):
    """One decode launch over every (slot, head) state per step, in place."""
    import torch
    import looped_linear_attention_b200 as lla
    from looped_linear_attention_b200 import workloads as W
    inp = W.decode_inputs(wl, dev)
    o = torch.empty(wl.n_seq, wl.H, wl.dv, dtype=wl.dtype, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        lla.gdn_decode_step(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S"], o=o)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    n = max(1, args.steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record(stream)
        for _ in range(n):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world) / n
    nbytes = decode_bytes_per_head_state(wl.dk, wl.dv) * wl.n_seq * wl.H
    gbs = nbytes / t / 1e9
    res = {"state_gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"], "ms_per_step": t * 1e3,
           "seq_tokens_per_s": world * 256 / t * 1.0, "slots": wl.n_seq, "heads": wl.H,
           "bytes_per_step": nbytes, "clocks": clocks.summary(),
           "note": "one step = one token for 256 sequences x 24 layers x 4 loops (all slots)"}
    del inp, o
    return res


def swa_flops(lengths, window, H, d=128, dv=128):
    """Algorithmic FLOPs of sliding-window attention: for every query, 2 d
    (q . k) and 2 dv (p v) per key in its window."""
    import numpy as np
    keys = 0
    for L in lengths:
        t = np.arange(L)
        keys += int(np.minimum(t + 1, window).sum())
    return keys * H * (2 * d + 2 * dv)


def bench_swa(dev, args, peaks, world, window=2048, L=4096, H=16):
    """Sliding-window attention of the hybrid loops at the 1.3B setting
    (w = 2048) on the looped workload's shape (L = 4096, 16 heads of 128),
    T = 4 loops per step; tensor-bound: achieved algorithmic TFLOP/s against
    the measured bf16 peak."""
    import torch
    import looped_linear_attention_b200 as lla
    from looped_linear_attention_b200 import workloads as W
    q, k, v = W.qkv(L, H, 128, 128, torch.bfloat16, False, dev, "bench", "swa")
    o = torch.empty_like(v)
    loops = 4

    def step():
        for _ in range(loops):
            lla.swa_fwd(q, k, v, window, o=o)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    n = max(1, args.steps)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record()
        for _ in range(n):
            step()
        e1.record()
        torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world) / n
    flops = swa_flops([L], window, H)
    tflops = flops * loops / t / 1e12
    return {"tokens_per_s": world * L / t, "ms_per_step": t * 1e3, "loops": loops, "window": window,
            "tokens": L, "heads": H, "d": 128, "achieved_tflops": tflops,
            "frac_of_bf16_peak": tflops / peaks["bf16_tflops"], "peak_kind": "burst (kernel timed alone)",
            "algorithmic_flops_per_launch": flops, "clocks": clocks.summary(),
            "kernel": "swa_fwd_kernel (tcgen05 S = Q K^T and O += P V, windowed online softmax)"}


def bench_kda(dev, args, peaks, world, L=4096, H=16):
    """The per-channel (diagonal) gate variant, KDA, on the looped workload's
    mixer shape (L = 4096, 16 heads, dk = dv = 128, bf16, in-kernel q/k norm),
    T = 4 loops per step; HBM roofline as the scalar-gate prefill, with a at
    dk floats per token and head."""
    import dataclasses
    import torch
    import looped_linear_attention_b200 as lla
    from looped_linear_attention_b200 import workloads as W
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], name="kda")
    inp = W.prefill_inputs(wl, dev)
    a, b = W.channel_gates(L, H, 128, dev, "bench", "kda")
    o = torch.empty(L, H, 128, dtype=torch.bfloat16, device=dev)
    loops = 4
    fl = lla.GDN_QK_L2NORM | lla.GDN_CHANNEL_GATE

    def step():
        for _ in range(loops):
            lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], a, b, None, flags=fl, o=o, return_state=False)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    n = max(1, min(args.steps, 5))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record()
        for _ in range(n):
            step()
        e1.record()
        torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world) / n
    nbytes = (prefill_bytes_per_token_head(128, 128) + 4 * 127) * L * H   # a: dk floats, not one
    gbs = nbytes / (t / loops) / 1e9
    return {"tokens_per_s": world * L / t, "ms_per_step": t * 1e3, "loops": loops, "tokens": L, "heads": H,
            "achieved_gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
            "clocks": clocks.summary(),
            "kernel": "gdn_prefill_kda_prep_kernel (one CTA per chunk and head: decayed operands, T, W, Q', "
                      "U~, O~; fp32 CUDA cores) + gdn_prefill_kda_chain_kernel (one CTA per (sequence, head, "
                      "16 columns); 3xTF32 warp MMAs)"}


def bench_backward(dev, args, peaks, world):
    """One reverse-mode call (gdn_chunk_bwd) on 8 sequences x 1024 tokens x 16
    heads, dk = dv = 128, bf16 inputs, with a final-state gradient.  Algorithmic
    bytes per (token, head): q, k, v and grad_o in bf16 (8 dk), a and b, and the
    fp32 gradients of q, k, v, a and b (12 dk + 8); plus S0, grad_S_T, grad_S0
    per chain."""
    import dataclasses
    import torch
    import looped_linear_attention_b200 as lla
    from looped_linear_attention_b200 import workloads as W
    wl = dataclasses.replace(W.WORKLOADS["long_prefill"], name="backward", n_seq=8, seq_len=1024,
                             random_s0=True)
    inp = W.prefill_inputs(wl, dev)
    g = torch.Generator(device=dev).manual_seed(W.seed_for("bench", "backward"))
    go = torch.randn(inp["v"].shape, generator=g, device=dev).to(wl.dtype)
    gST = torch.randn(wl.n_seq, wl.H, wl.dk, wl.dv, generator=g, device=dev)
    stream = torch.cuda.current_stream()

    def step(flags=0):
        return lla.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], go, inp["S0"], gST,
                                 n_seq=wl.n_seq, flags=flags)

    for _ in range(max(1, min(args.warmup, 2))):
        step()
    torch.cuda.synchronize()
    barrier(world)
    n = 2
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record(stream)
        for _ in range(n):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3, world) / n
    # the token-by-token path (GDN_PRECISE), one call, for comparison
    step(lla.GDN_PRECISE)
    torch.cuda.synchronize()
    e0.record(stream)
    step(lla.GDN_PRECISE)
    e1.record(stream)
    torch.cuda.synchronize()
    t_tok = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    tokens = wl.n_seq * wl.seq_len
    nbytes = tokens * wl.H * (8 * wl.dk + 12 * wl.dk + 8 + 8) + 3 * wl.n_seq * wl.H * wl.dk * wl.dv * 4
    gbs = nbytes / t / 1e9
    return {"tokens_per_s": world * tokens / t, "ms_per_call": t * 1e3, "achieved_gbs": gbs,
            "frac_of_hbm": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_call": nbytes,
            "tokens": tokens, "heads": wl.H, "dk": wl.dk, "dv": wl.dv, "clocks": clocks.summary(),
            "kernel": "chunkwise: gdn_bwd_prep_kernel, gdn_bwd_states_kernel, gdn_bwd_dstates_kernel, "
                      "gdn_bwd_grads_kernel (fp32 CUDA cores)",
            "token_path_ms_per_call": t_tok * 1e3}


# ------------------------------------------------------------------ CPU oracle
def cpu_baseline(seconds_target: float = 15.0, sample_tokens: int = 4096):
    """The oracle as it stands, on the first `sample_tokens` tokens of the
    looped-prefill workload (all 4 loops, full width; by default the whole
    4096-token sequence), repeated until about `seconds_target` seconds of CPU
    work have run, on this host's cores."""
    import torch
    import oracle
    from looped_linear_attention_b200 import workloads as W
    wl = W.WORKLOADS["looped_prefill"]
    inp = W.looped_inputs(wl, "cpu")
    Ls = sample_tokens
    t0 = time.perf_counter()
    runs = 0
    while True:
        oracle.looped_forward(inp["h0"][:Ls], inp["Wq"], inp["Wk"], inp["Wv"],
                              inp["a"][:, :Ls], inp["b"][:, :Ls], inp["rho"], wl.H, wl.dk, wl.dv)
        runs += 1
        el = time.perf_counter() - t0
        if el > seconds_target or runs >= 50:
            break
    value = Ls * runs / el
    try:
        model = next(l.split(":", 1)[1].strip() for l in open("/proc/cpuinfo") if "model name" in l)
    except Exception:
        model = "unknown"
    return {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {Ls} of {wl.seq_len} tokens, all {wl.loops} loops, d={wl.H * wl.dk}, "
                      f"{runs} run(s), {el:.1f} s; fp64 C oracle (OpenMP) + numpy projections",
            "cpu": model}


def cpu_baseline_backward(seconds_target: float = 3.0, sample_tokens: int = 256):
    """The oracle's reverse mode beside the GPU one: the first `sample_tokens`
    tokens of each of the 16 heads of one sequence of the backward workload
    (dk = dv = 128, with a final-state gradient), repeated for about
    `seconds_target` seconds on this host's cores."""
    import dataclasses
    import torch
    import oracle
    from looped_linear_attention_b200 import workloads as W
    wl = dataclasses.replace(W.WORKLOADS["long_prefill"], name="backward", n_seq=1,
                             seq_len=sample_tokens, random_s0=True)
    inp = W.prefill_inputs(wl, "cpu")
    g = torch.Generator().manual_seed(W.seed_for("bench", "backward", "cpu"))
    go = torch.randn(inp["v"].shape, generator=g).to(wl.dtype)
    gST = torch.randn(1, wl.H, wl.dk, wl.dv, generator=g)
    t0 = time.perf_counter()
    runs = 0
    while True:
        oracle.gdn_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], go, inp["S0"], gST)
        runs += 1
        el = time.perf_counter() - t0
        if el > seconds_target or runs >= 20:
            break
    return {"value": sample_tokens * runs / el, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{sample_tokens} tokens x {wl.H} heads, dk = dv = {wl.dk}, "
                                        f"{runs} run(s), {el:.1f} s; fp64 C oracle (OpenMP)"}


def cpu_baseline_prefill(name: str, seconds_target: float = 4.0):
    """The oracle on a sample of a prefill workload: one whole sequence (every
    head) of the long-prefill workload, or the varlen sequence of median
    length, one loop, repeated for about `seconds_target` seconds on this
    host's cores; scaled to the workload's T loops (T calls over the same
    inputs), so the figure reads like the GPU's tokens/s."""
    import dataclasses
    import numpy as np
    import oracle
    from looped_linear_attention_b200 import workloads as W
    wl = W.WORKLOADS[name]
    if wl.varlen:
        lens = W.varlen_lengths(wl)
        s = int(np.argsort(lens)[len(lens) // 2])
        L = int(lens[s])
        inp = W.prefill_inputs(dataclasses.replace(wl, name=wl.name), "cpu", lengths=[L])
        what = f"sequence {s} of {wl.n_seq} (median length {L}), all {wl.H} heads, dv = {wl.dv}"
    else:
        L = wl.seq_len
        inp = W.prefill_inputs(wl, "cpu", n_seq=1)
        what = f"sequence 0 of {wl.n_seq} ({L} tokens), all {wl.H} heads"
    cu = np.array([0, L], dtype=np.int32)
    t0 = time.perf_counter()
    runs = 0
    while True:
        oracle.gdn_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], cu)
        runs += 1
        el = time.perf_counter() - t0
        if el > seconds_target or runs >= 20:
            break
    per_loop = el / runs
    return {"value": L / (wl.loops * per_loop), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{what}, one loop, {runs} run(s), {el:.1f} s; scaled to {wl.loops} loops "
                      f"(tokens / (loops x time per loop)); fp64 C oracle (OpenMP over heads)"}


def cpu_baseline_decode(seconds_target: float = 4.0, n_slots: int = 256):
    """The oracle's decode step on `n_slots` of the decode workload's 24576
    slots (all 16 heads), repeated for about `seconds_target` seconds; scaled to
    the whole step (all slots) as sequence-tokens/s and state GB/s."""
    import oracle
    from looped_linear_attention_b200 import workloads as W
    wl = W.WORKLOADS["decode"]
    inp = W.decode_inputs(wl, "cpu", n_slots=n_slots)
    t0 = time.perf_counter()
    runs = 0
    while True:
        oracle.gdn_decode(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S"])
        runs += 1
        el = time.perf_counter() - t0
        if el > seconds_target or runs >= 50:
            break
    step_s = el / runs * wl.n_seq / n_slots
    nbytes = decode_bytes_per_head_state(wl.dk, wl.dv) * wl.n_seq * wl.H
    return {"value": 256 / step_s, "unit": "seq-tokens/s", "state_gbs": nbytes / step_s / 1e9,
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n_slots} of {wl.n_seq} slots x {wl.H} heads, {runs} run(s), {el:.1f} s; "
                      f"scaled to the whole step (x {wl.n_seq // n_slots}); fp64 C oracle (OpenMP)"}


def cpu_baseline_swa(seconds_target: float = 3.0, window: int = 2048, L: int = 4096, heads: int = 2):
    """The oracle's sliding-window attention on `heads` of the 16 heads of the
    swa workload (L = 4096, w = 2048), scaled to all heads and T = 4 loops."""
    import torch
    import oracle
    from looped_linear_attention_b200 import workloads as W
    q, k, v = W.qkv(L, heads, 128, 128, torch.bfloat16, False, "cpu", "bench", "swa", "cpu")
    t0 = time.perf_counter()
    runs = 0
    while True:
        oracle.swa_fwd(q, k, v, window)
        runs += 1
        el = time.perf_counter() - t0
        if el > seconds_target or runs >= 20:
            break
    step_s = el / runs * (16 / heads) * 4
    return {"value": L / step_s, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{heads} of 16 heads, L = {L}, w = {window}, {runs} run(s), {el:.1f} s; scaled to "
                      f"16 heads and 4 loops; fp64 C oracle (OpenMP)"}


def cpu_baseline_kda(seconds_target: float = 3.0, L: int = 4096):
    """The oracle's per-channel gate variant on the kda workload (all 16
    heads, L = 4096), one loop, scaled to T = 4 loops."""
    import dataclasses
    import numpy as np
    import oracle
    from looped_linear_attention_b200 import workloads as W
    wl = dataclasses.replace(W.WORKLOADS["looped_prefill"], name="kda")
    inp = W.prefill_inputs(wl, "cpu")
    a, b = W.channel_gates(L, 16, 128, "cpu", "bench", "kda")
    q, k = oracle.qk_l2norm(inp["q"]), oracle.qk_l2norm(inp["k"])
    t0 = time.perf_counter()
    runs = 0
    while True:
        oracle.kda_fwd(q, k, inp["v"], a, b)
        runs += 1
        el = time.perf_counter() - t0
        if el > seconds_target or runs >= 20:
            break
    return {"value": L / (4 * el / runs), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{L} tokens x 16 heads, one loop, {runs} run(s), {el:.1f} s; scaled to 4 loops; "
                      f"fp64 C oracle (OpenMP)"}


def run_reference(args, rank, world):
    """CPU oracle arm: rank 0 only; every step is the whole looped-prefill
    configuration (the 4096-token sequence, all 4 loops), as in cpu_baseline."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    for _ in range(max(0, min(args.warmup, 1))):
        cpu_baseline(0.0)
    times = []
    Ls = 4096
    for _ in range(args.steps):
        r = cpu_baseline(0.0, sample_tokens=Ls)
        times.append(Ls / r["value"])
    total = sum(times)
    value = Ls * args.steps / total
    from looped_linear_attention_b200 import workloads as W
    wl = W.WORKLOADS["looped_prefill"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": "looped_prefill", "batch": 1, "seq_len": wl.seq_len,
                   "d_model": wl.H * wl.dk, "heads": wl.H, "dk": wl.dk, "dv": wl.dv,
                   "loops": wl.loops, "parallelism": "cpu oracle, rank 0"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"each step: all {Ls} of {wl.seq_len} tokens, all {wl.loops} loops "
                                   f"(the whole configuration)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Small fixed case for profiler captures: `--profile WORKLOAD` runs only that
    workload's kernel (warm-up + steps launches) with `--n-seq` sequences/slots."""
    import torch
    import looped_linear_attention_b200 as lla
    from looped_linear_attention_b200 import workloads as W
    import dataclasses
    torch.cuda.set_device(0)
    wl = W.WORKLOADS.get(args.profile, W.WORKLOADS["looped_prefill"])
    if args.n_seq:
        wl = dataclasses.replace(wl, n_seq=args.n_seq)
    dev = torch.device("cuda", 0)
    if args.profile == "kda":
        # the per-channel gate prefill on the looped mixer shape
        inp = W.prefill_inputs(dataclasses.replace(W.WORKLOADS["looped_prefill"], name="kda"), dev)
        a, b = W.channel_gates(4096, 16, 128, dev, "bench", "kda")
        o = torch.empty(4096, 16, 128, dtype=torch.bfloat16, device=dev)
        fl = lla.GDN_QK_L2NORM | lla.GDN_CHANNEL_GATE
        run = lambda: lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], a, b, None, flags=fl, o=o,
                                        return_state=False)
        wl = W.WORKLOADS["looped_prefill"]
    elif args.profile == "backward":
        # the chunkwise reverse mode on the timed backward workload (8 x 1024 tokens)
        wl = dataclasses.replace(W.WORKLOADS["long_prefill"], name="backward", n_seq=args.n_seq or 8,
                                 seq_len=1024, random_s0=True)
        inp = W.prefill_inputs(wl, dev)
        g = torch.Generator(device=dev).manual_seed(W.seed_for("bench", "backward"))
        go = torch.randn(inp["v"].shape, generator=g, device=dev).to(wl.dtype)
        gST = torch.randn(wl.n_seq, wl.H, wl.dk, wl.dv, generator=g, device=dev)
        run = lambda: lla.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], go, inp["S0"],
                                        gST, n_seq=wl.n_seq)
    elif args.profile == "swa":
        # sliding-window attention, w = 2048, on the looped workload's shape
        q, k, v = W.qkv(4096, 16, 128, 128, torch.bfloat16, False, dev, "bench", "swa")
        o = torch.empty_like(v)
        run = lambda: lla.swa_fwd(q, k, v, 2048, o=o)
        wl = W.WORKLOADS["looped_prefill"]
    elif args.profile == "decode":
        inp = W.decode_inputs(wl, dev)
        run = lambda: lla.gdn_decode_step(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S"])
    elif args.profile == "looped_prefill":
        # the looped step's mixer call: in-kernel q/k norm, the loop residual
        # fused into the output, no final state
        inp = W.prefill_inputs(wl, dev)
        g = torch.Generator(device=dev).manual_seed(W.seed_for("profile", "h_prev"))
        d = wl.H * wl.dv
        hp = torch.randn(inp["total_tokens"], d, generator=g, device=dev).to(wl.dtype)
        rho = 0.5 * torch.rand(d, generator=g, device=dev)
        out = torch.empty_like(hp)
        fl = lla.GDN_QK_L2NORM | (lla.GDN_SINGLE_PASS if args.single_pass else 0)
        run = lambda: lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], None, None,
                                        n_seq=inp["n_seq"], flags=fl, o=out, return_state=False,
                                        h_prev=hp, rho=rho)
    else:
        inp = W.prefill_inputs(wl, dev)
        cu = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).to(dev)
        fl = lla.GDN_SINGLE_PASS if args.single_pass else 0
        run = lambda: lla.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], cu,
                                        n_seq=inp["n_seq"], flags=fl)
    for _ in range(args.warmup + args.steps):
        run()
    torch.cuda.synchronize()
    st = lla.gdn_get_device_status()
    print(json.dumps({"profile_case": args.profile, "n_seq": wl.n_seq, "launches": args.warmup + args.steps,
                      "status": lla.status_string(st)}))
    if st != lla.GDN_OK:
        sys.exit(1)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile", choices=["tiny", "looped_prefill", "long_prefill", "varlen", "decode", "swa",
                                          "kda", "backward"],
                    default=None,
                    help="run only this workload's kernel (for profiler captures)")
    ap.add_argument("--n-seq", type=int, default=0, help="sequences (or decode slots) for --profile")
    ap.add_argument("--single-pass", action="store_true",
                    help="--profile: force the one-pass prefill schedule (GDN_SINGLE_PASS)")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        # the CPU oracle arm: rank 0 alone, no process group
        run_reference(args, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
