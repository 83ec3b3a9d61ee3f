#!/usr/bin/env python
"""Benchmark of the Dynamic Mask Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the forward hot path on the prefill workload (B=1, H=16, Hkv=8,
N=4096, d=128, w=1024, bf16, seed 1): gate -> causal top-w mask -> masked
attention forward, all in libdma's kernels, inputs resident in HBM.  The
headline metric is kept-pair TFLOP/s: 4 d sum_t min(t+1, w) per (b, h) divided
by the step time.  L2 is flushed (256 MiB written, then 256 MiB read) before every
step, outside the timed intervals.  The step is captured in two CUDA graphs
(gate + mask, then attention) so that the attention kernel's own duration is
measured with CUDA events on the launching stream (the roofline figure).

Extra legs in the same JSON line: decode (B=8, H=32, Hkv=8, L=65536, w=2048;
selected-KV GB/s against HBM bandwidth) and the training step (B=2, H=16,
Hkv=8, N=8192, w=2048; forward + backward kept-pair TFLOP/s).

With N > 1 (torchrun) every rank runs the same workload on its own GPU
(independent replicas, weak scaling; the path has no exchange step), the time
is the max over ranks and the value the sum over ranks.

--impl reference times the CPU oracle (the only reference this method has:
no implementation ships with the pages) on a bounded sample of the same
workload on the host cores; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DMA fwd kept-pair TFLOP/s & % bf16 peak; decode selected-KV GB/s vs HBM"
# The pages' own speed claim, quoted beside our figures (context, not a target): page 1 (HF blog
# "dmattn"), section "Practical Speed Improvements"; the pages name no hardware.
PAGES_CLAIM = {"claim": "training: up to 10x speedup over standard attention for longer sequences; "
                        "inference: gains compounding as sequence length increases",
               "source": "Trainable Dynamic Mask Sparse Attention (HF blog dmattn), Practical Speed Improvements",
               "hardware": "not stated"}
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Empties L2 between timed steps: writes a buffer twice the size of L2, then reads another one
    as large, so that the write-backs of the dirty lines the write leaves happen here, untimed, and
    the timed step starts on an L2 that holds nothing of its own data (and nothing dirty)."""

    def __init__(self, torch):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device="cuda")
        self.sink = torch.zeros((), dtype=torch.int64, device="cuda")
        self.torch = torch

    def __call__(self):
        self.w.zero_()
        self.sink = self.r.sum()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "of measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "of fallback"}


def _traffic(kernel: str, source_file: str):
    """DRAM bytes per launch from a committed ncu summary, null if the kernel's
    source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        src = open(os.path.join(ROOT, "trainable_dynamic_mask_b200", "csrc", source_file), "rb").read()
        if hashlib.sha256(src).hexdigest()[:16] != rec["source_sha256_16"]:
            return None
        return float(rec["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, torch_device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception as e:  # pragma: no cover - reported in the JSON line
            self.error = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def mark(self):
        """Start of the timed region: samples from here on are also counted on their own."""
        self._mark = len(self.samples)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = get(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "nvml")}
        reasons = sorted(self.reasons - {"gpu_idle"})
        timed = self.samples[getattr(self, "_mark", 0):]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "samples_in_timed_region": len(timed),
                "sm_mhz_timed_region": statistics.median(timed) if timed else None,
                "window": "the same step replayed untimed for --clock-soak seconds immediately before the "
                          "timed region, then the timed region"}


# ---------------------------------------------------------------- helpers

def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _to_dev_bf16(bits, torch):
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _max_over_ranks(x: float, world: int, torch) -> float:
    """The maximum of x over the ranks (the device timings of a step are reported as the slowest
    rank's).  The reduction runs on the process group's device: CUDA for NCCL, the host for gloo."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _barrier(world, torch):
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


# ---------------------------------------------------------------- our arm

def run_ours(args, world, rank):
    import numpy as np
    import torch

    import trainable_dynamic_mask_b200 as dma
    from workloads import get, make_inputs

    torch.cuda.set_device(_dist()[2])
    dma.load()
    peaks = _peaks()
    if args.no_main:
        # a profiling aid: only the selected legs, each in its own JSON object (no bench line)
        legs = [x for x in args.legs.split(",") if x]
        run = {"decode": leg_decode, "train": leg_train, "chunk": leg_chunk, "long": leg_long, "cp": leg_cp}
        return {"legs_only": {name: run[name](args, world, torch, dma, peaks) for name in legs}}
    wl = get("prefill")
    I = make_inputs(wl)
    # an inference prefill: no backward follows, so the forward keeps nothing for one
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype="bf16", forward_only=True)
    Q, K, V = (_to_dev_bf16(I.bits[n], torch) for n in ("Q", "K", "V"))
    Dl = _to_dev_bf16(I.bits["Delta"], torch)
    A = torch.from_numpy(I.A).cuda()
    ws = dma.alloc_workspace(p)
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    evict = torch.empty((wl.B, wl.H, wl.N), dtype=torch.int32, device="cuda")
    O = torch.empty((wl.B, wl.H, wl.N, wl.d), dtype=torch.bfloat16, device="cuda")
    LSE = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    flush = L2Flush(torch)
    flops = 4.0 * wl.d * wl.kept_pairs()

    stream = torch.cuda.Stream()
    s_ptr = stream.cuda_stream

    def part_a():
        dma.gate(p, V, Dl, A, delta, None, ws, s_ptr)
        dma.topk_mask(p, delta, evict, ws, s_ptr)

    def part_b():
        dma.attn_fwd(p, Q, K, V, delta, evict, ws, O, LSE, s_ptr)

    with torch.cuda.stream(stream):
        part_a(); part_b()
        stream.synchronize()
        ga, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(ga, stream=stream):
            part_a()
        with torch.cuda.graph(gb, stream=stream):
            part_b()
    # gate; top-w: segment sort, ranks, (thresholds: rows longer than 4096 keys only; shorter rows'
    # eviction kernel finds them itself), eviction, lists; attention
    launches_per_step = 7 if wl.N > 4096 else 6

    def timed(n, sampler=None):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        with torch.cuda.stream(stream):
            for e0, e1, e2 in evs:
                flush()
                e0.record(stream)
                ga.replay()
                e1.record(stream)
                gb.replay()
                e2.record(stream)
        stream.synchronize()
        step = [e0.elapsed_time(e2) for e0, e1, e2 in evs]
        attn = [e1.elapsed_time(e2) for e0, e1, e2 in evs]
        return step, attn

    def soak(seconds):
        # the same step, untimed, in batches until `seconds` have passed: the clock sampler needs a
        # window longer than its sampling period, which a short timed region alone does not give
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            while time.perf_counter() - t0 < seconds:
                for _ in range(200):
                    flush()
                    ga.replay()
                    gb.replay()
                stream.synchronize()

    timed(args.warmup)
    _barrier(world, torch)
    with ClockSampler(torch.cuda.current_device()) as clk:
        soak(args.clock_soak)
        _barrier(world, torch)
        clk.mark()
        step_ms, attn_ms = timed(args.steps)
    _barrier(world, torch)
    total_ms = _max_over_ranks(sum(step_ms), world, torch)
    ms_per_step = total_ms / args.steps
    value = world * flops * args.steps / (total_ms * 1e-3) / 1e12
    attn_avg = sum(attn_ms) / len(attn_ms)
    achieved = flops / (attn_avg * 1e-3) / 1e12
    traffic = _traffic("attn_fwd_prefill", "attn_fwd_tc.cu")
    torch.cuda.synchronize()
    density = _pair_density(evict.cpu().numpy(), wl, np)

    # the same kernels with w = N (dense causal attention), timed the same way
    wl_d = wl.with_(w=wl.N)
    p_d = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.N, dtype="bf16", forward_only=True)
    ws_d = dma.alloc_workspace(p_d)
    O_d, LSE_d = torch.empty_like(O), torch.empty_like(LSE)
    with torch.cuda.stream(stream):
        dma.gate(p_d, V, Dl, A, delta, None, ws_d, s_ptr)
        dma.topk_mask(p_d, delta, evict, ws_d, s_ptr)
        dma.attn_fwd(p_d, Q, K, V, delta, evict, ws_d, O_d, LSE_d, s_ptr)
        stream.synchronize()
        gda, gdb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gda, stream=stream):
            dma.gate(p_d, V, Dl, A, delta, None, ws_d, s_ptr)
            dma.topk_mask(p_d, delta, evict, ws_d, s_ptr)
        with torch.cuda.graph(gdb, stream=stream):
            dma.attn_fwd(p_d, Q, K, V, delta, evict, ws_d, O_d, LSE_d, s_ptr)
    ga_s, gb_s = ga, gb
    ga, gb = gda, gdb
    timed(args.warmup)
    n_d = max(5, min(args.steps, 100))
    step_d, attn_d = timed(n_d)
    ga, gb = ga_s, gb_s
    step_d = _max_over_ranks(sum(step_d), world, torch) / n_d
    attn_d = _max_over_ranks(sum(attn_d), world, torch) / n_d
    flops_d = 4.0 * wl.d * wl_d.kept_pairs()
    dense = {"w": wl.N, "kept_pairs": wl_d.kept_pairs(), "step_us": round(step_d * 1e3, 2),
             "attn_us": round(attn_d * 1e3, 2), "attn_tflops": round(flops_d / (attn_d * 1e-3) / 1e12, 2),
             "speedup_attn": round(attn_d / attn_avg, 3), "speedup_step": round(step_d / ms_per_step, 3),
             "steps": n_d}
    del ws_d, O_d, LSE_d

    # end to end through the public API: pinned host inputs in, O and LSE back to the host
    host = {n: torch.from_numpy(np.ascontiguousarray(I.bits[n]).view(np.int16)).view(torch.bfloat16).pin_memory()
            for n in ("Q", "K", "V", "Delta")}
    host["A"] = torch.from_numpy(I.A).pin_memory()
    out_O = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
    out_L = torch.empty(LSE.shape, dtype=torch.float32).pin_memory()
    dev_in = {n: torch.empty(t.shape, dtype=t.dtype, device="cuda") for n, t in host.items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_O.numel() * 2 + out_L.numel() * 4

    def e2e_step():
        for n, t in host.items():
            dev_in[n].copy_(t, non_blocking=True)
        r = dma.forward(p, dev_in["Q"], dev_in["K"], dev_in["V"], dev_in["Delta"], dev_in["A"], workspace=ws)
        out_O.copy_(r["O"], non_blocking=True)
        out_L.copy_(r["LSE"], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            e2e_step()
        stream.synchronize()
        _barrier(world, torch)
        n_e2e = max(10, min(args.steps, 200))
        e2e_ms = 0.0
        for _ in range(n_e2e):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step()
            b.record(stream)
            b.synchronize()
            e2e_ms += a.elapsed_time(b)
    e2e_ms = _max_over_ranks(e2e_ms, world, torch) / n_e2e
    e2e_value = world * flops / (e2e_ms * 1e-3) / 1e12

    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, Delta ~ N(0, 0.02^2), A ~ U(-1, 0))",
        "config": {"workload": "prefill", "quoted_on": "the prefill configuration (the metric's own); the long "
                   "prefill configuration is reported in legs.long",
                   "B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "N": wl.N, "d": wl.d, "w": wl.w,
                   "kept_pairs": wl.kept_pairs(), "step": "gate + top-w mask + attention forward",
                   "forward_only": True,
                   "parallelism": f"replicas{world}", "l2": "flushed before every step (256 MiB written, then 256 MiB read: no dirty lines left)"},
        "roofline": {"kernel": "attn_fwd", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4), "peak_kind": "burst " + peaks["source"],
                     "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "traffic": traffic, "avg_launch_us": round(attn_avg * 1e3, 2),
                     "per_launch_flops": flops, "tile_density": density},
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "api": "trainable_dynamic_mask_b200.forward"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "dense_causal": dense,
        "pages_claim": PAGES_CLAIM,
    }
    legs = [] if args.no_legs else [x for x in args.legs.split(",") if x]
    if legs:
        run = {"decode": leg_decode, "train": leg_train, "chunk": leg_chunk, "long": leg_long, "cp": leg_cp}
        line["legs"] = {name: run[name](args, world, torch, dma, peaks) for name in legs}
        line["gpu_launches"] += sum(leg["gpu_launches"] for leg in line["legs"].values())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    return line


def leg_decode(args, world, torch, dma, peaks):
    """Single-query decode over a 65536-row cache: selected-KV bytes / kernel time."""
    import numpy as np

    from workloads import get, make_inputs
    wl = get("decode")
    I = make_inputs(wl)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, Nq=1, dtype="bf16")
    Q = _to_dev_bf16(I.bits["Q"], torch)
    K = _to_dev_bf16(I.bits["K"], torch)
    V = _to_dev_bf16(I.bits["V"], torch)
    Dl = _to_dev_bf16(I.bits["Delta"], torch)
    A = torch.from_numpy(I.A).cuda()
    del I
    ws = dma.alloc_workspace(p)
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    O = torch.empty((wl.B, wl.H, 1, wl.d), dtype=torch.bfloat16, device="cuda")
    LSE = torch.empty((wl.B, wl.H, 1), dtype=torch.float32, device="cuda")
    flush = L2Flush(torch)
    dma.gate(p, V, Dl, A, delta)        # the cache's gate values are precomputed (untimed)
    dma.topk_mask(p, delta, None, ws)
    torch.cuda.synchronize()
    lay = dma.workspace_layout(p)
    sel = ws[lay.off_sel: lay.off_sel + wl.B * wl.H * lay.sel_len * 4].cpu().numpy().view(np.int32)
    sel = sel.reshape(wl.B, wl.Hkv, wl.G * lay.sel_len)
    unique_rows = sum(len(np.unique(sel[b, g])) for b in range(wl.B) for g in range(wl.Hkv))
    bytes_unique = unique_rows * 2 * wl.d * 2
    bytes_per_head = wl.B * wl.H * lay.sel_len * 2 * wl.d * 2
    n = max(5, min(args.steps, 200))
    t_sel, t_att = 0.0, 0.0
    for i in range(args.warmup + n):
        flush()
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record()
        dma.topk_mask(p, delta, None, ws)
        b.record()
        flush()
        b2 = torch.cuda.Event(enable_timing=True)
        b2.record()
        dma.attn_fwd(p, Q, K, V, delta, None, ws, O, LSE)
        c.record()
        c.synchronize()
        if i >= args.warmup:
            t_sel += a.elapsed_time(b)
            t_att += b2.elapsed_time(c)
    t_sel = _max_over_ranks(t_sel, world, torch) / n
    t_att = _max_over_ranks(t_att, world, torch) / n
    gbs = bytes_unique / (t_att * 1e-3) / 1e9
    # the incremental selection: one key appended to a cache of L - 1 keys (the selection over L - 1
    # keys is restored before every timed call; the result must equal the full selection)
    sel_bytes = wl.B * wl.H * lay.sel_len * 4
    full_sel = ws[lay.off_sel: lay.off_sel + sel_bytes].clone()
    p_prev = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N - 1, wl.d, wl.w, Nq=1, dtype="bf16")
    dma.topk_mask(p_prev, delta[:, :, :wl.N - 1].contiguous(), None, ws)
    prev_sel = ws[lay.off_sel: lay.off_sel + sel_bytes].clone()
    t_app = 0.0
    for i in range(args.warmup + n):
        ws[lay.off_sel: lay.off_sel + sel_bytes].copy_(prev_sel)
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dma.topk_append(p, delta, ws)
        b.record()
        b.synchronize()
        if i >= args.warmup:
            t_app += a.elapsed_time(b)
    t_app = _max_over_ranks(t_app, world, torch) / n
    append_ok = bool(torch.equal(ws[lay.off_sel: lay.off_sel + sel_bytes], full_sel))
    # the same kernels with w = L (every cached row attended), timed the same way
    p_d = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.N, Nq=1, dtype="bf16")
    ws_d = dma.alloc_workspace(p_d)
    dma.topk_mask(p_d, delta, None, ws_d)
    td = 0.0
    n_d = 5
    for i in range(2 + n_d):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dma.attn_fwd(p_d, Q, K, V, delta, None, ws_d, O, LSE)
        b.record()
        b.synchronize()
        if i >= 2:
            td += a.elapsed_time(b)
    del ws_d
    td = _max_over_ranks(td, world, torch) / n_d
    bytes_d = wl.B * wl.Hkv * wl.N * 2 * wl.d * 2
    dense = {"w": wl.N, "attn_us": round(td * 1e3, 2), "gbs": round(bytes_d / (td * 1e-3) / 1e9, 2),
             "speedup_attn": round(td / t_att, 3), "steps": n_d}
    return {"metric": "decode selected-KV GB/s", "value": round(world * gbs, 2), "unit": "GB/s",
            "config": {"workload": "decode", "B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "L": wl.N, "d": wl.d, "w": wl.w},
            "attn_us": round(t_att * 1e3, 2), "select_us": round(t_sel * 1e3, 2),
            "select_append_us": round(t_app * 1e3, 2), "append_equals_full_selection": append_ok,
            "roofline": {"kernel": "decode_split+combine", "bound": "hbm", "achieved": round(gbs, 2),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "peak_kind": peaks["source"], "traffic": _traffic("decode_split", "attn_fwd.cu"),
                         "traffic_kernel": "decode_split_kernel (the combine reads 1 MB more)",
                         "algorithmic_bytes": bytes_unique, "bytes_if_per_head": bytes_per_head},
            "dense_causal": dense,
            "gpu_launches": 4 * n}


def leg_chunk(args, world, torch, dma, peaks):
    """Chunked prefill: the last 2048 query positions of a 16384-key sequence (the long workload's
    heads, window and seed), with the selection over all keys; kept-pair TFLOP/s of the attention."""
    import numpy as np

    from workloads import get, make_inputs
    wl = get("long").with_(Nq=2048)
    I = make_inputs(wl)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, Nq=wl.Nq, dtype="bf16")
    Q, K, V = (_to_dev_bf16(I.bits[n], torch) for n in ("Q", "K", "V"))
    Dl = _to_dev_bf16(I.bits["Delta"], torch)
    A = torch.from_numpy(I.A).cuda()
    del I
    ws = dma.alloc_workspace(p)
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    evict = torch.empty((wl.B, wl.H, wl.N), dtype=torch.int32, device="cuda")
    O = torch.empty((wl.B, wl.H, wl.Nq, wl.d), dtype=torch.bfloat16, device="cuda")
    LSE = torch.empty((wl.B, wl.H, wl.Nq), dtype=torch.float32, device="cuda")
    flush = L2Flush(torch)
    q0 = wl.N - wl.Nq
    pairs = wl.B * wl.H * sum(min(t + 1, wl.w) for t in range(q0, wl.N))
    flops = 4.0 * wl.d * pairs
    n = max(5, min(args.steps // 10, 50))
    t_step = t_att = 0.0
    for i in range(args.warmup + n):
        flush()
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record()
        dma.gate(p, V, Dl, A, delta)
        dma.topk_mask(p, delta, evict, ws)
        b.record()
        dma.attn_fwd(p, Q, K, V, delta, evict, ws, O, LSE)
        c.record()
        c.synchronize()
        if i >= args.warmup:
            t_step += a.elapsed_time(c)
            t_att += b.elapsed_time(c)
    t_step = _max_over_ranks(t_step, world, torch) / n
    t_att = _max_over_ranks(t_att, world, torch) / n
    tf = flops / (t_att * 1e-3) / 1e12
    return {"metric": "chunked prefill attention kept-pair TFLOP/s", "value": round(world * tf, 2), "unit": "TFLOP/s",
            "config": {"workload": "long with a chunk of queries", "B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "N": wl.N,
                       "Nq": wl.Nq, "q0": q0, "d": wl.d, "w": wl.w, "kept_pairs": pairs},
            "attn_us": round(t_att * 1e3, 2), "step_us": round(t_step * 1e3, 2),
            "roofline": {"kernel": "attn_fwd", "bound": "tensor", "achieved": round(tf, 2),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4)},
            "gpu_launches": 7 * n}   # gate, top-w 5 (16384-key rows), attention


def _pair_density(evict, wl, np):
    """Executed-tile density of the attention forward: kept-pair FLOPs over the FLOPs of the
    tensor-core tiles the kernel runs (each pair of 128-row blocks walks its live keys in tiles of
    128; a key is live for the pair [t0, t1) when j < t1 and e_j > max(j, t0)).  Computed on the
    host from the eviction indices the GPU wrote."""
    e = evict.reshape(-1, wl.N)
    j = np.arange(wl.N)
    tiles = 0
    for t0 in range(wl.q_pos0 // 256 * 256, wl.N, 256):
        t1 = min(t0 + 256, wl.N)
        live = ((j[None, :t1] < t1) & (e[:, :t1] > np.maximum(j[None, :t1], t0))).sum(axis=1)
        tiles += int(((live + 127) // 128).sum())
    executed = tiles * 128 * 256   # query rows x keys per tile
    return {"kept_pairs": wl.kept_pairs(), "executed_pairs": executed,
            "density": round(wl.kept_pairs() / executed, 4)}


def leg_long(args, world, torch, dma, peaks):
    """The long prefill workload (B=1, H=32, Hkv=8, N=16384, d=128, w=2048, 5% of key positions
    scaled by 4): gate -> top-w mask -> attention forward, replayed from two CUDA graphs with L2
    flushed before every step, the attention timed on its own for the roofline."""
    import numpy as np

    from workloads import get, make_inputs
    wl = get("long")
    I = make_inputs(wl)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype="bf16", forward_only=True)
    Q, K, V = (_to_dev_bf16(I.bits[n], torch) for n in ("Q", "K", "V"))
    Dl = _to_dev_bf16(I.bits["Delta"], torch)
    A = torch.from_numpy(I.A).cuda()
    ws = dma.alloc_workspace(p)
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    evict = torch.empty((wl.B, wl.H, wl.N), dtype=torch.int32, device="cuda")
    O = torch.empty((wl.B, wl.H, wl.N, wl.d), dtype=torch.bfloat16, device="cuda")
    LSE = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    flush = L2Flush(torch)
    flops = 4.0 * wl.d * wl.kept_pairs()
    stream = torch.cuda.Stream()
    s_ptr = stream.cuda_stream

    def graphs(pp, w_ws, o, lse):
        with torch.cuda.stream(stream):
            dma.gate(pp, V, Dl, A, delta, None, w_ws, s_ptr)
            dma.topk_mask(pp, delta, evict, w_ws, s_ptr)
            dma.attn_fwd(pp, Q, K, V, delta, evict, w_ws, o, lse, s_ptr)
            stream.synchronize()
            ga, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(ga, stream=stream):
                dma.gate(pp, V, Dl, A, delta, None, w_ws, s_ptr)
                dma.topk_mask(pp, delta, evict, w_ws, s_ptr)
            with torch.cuda.graph(gb, stream=stream):
                dma.attn_fwd(pp, Q, K, V, delta, evict, w_ws, o, lse, s_ptr)
        return ga, gb

    def timed(ga, gb, n):
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(n)]
        with torch.cuda.stream(stream):
            for e0, e1, e2 in evs:
                flush()
                e0.record(stream)
                ga.replay()
                e1.record(stream)
                gb.replay()
                e2.record(stream)
        stream.synchronize()
        return sum(e0.elapsed_time(e2) for e0, e1, e2 in evs) / n, sum(e1.elapsed_time(e2) for e0, e1, e2 in evs) / n

    ga, gb = graphs(p, ws, O, LSE)
    n = max(5, min(args.steps, 100))
    timed(ga, gb, args.warmup)
    step_ms, attn_ms = timed(ga, gb, n)
    step_ms = _max_over_ranks(step_ms, world, torch)
    attn_ms = _max_over_ranks(attn_ms, world, torch)
    torch.cuda.synchronize()
    dens = _pair_density(evict.cpu().numpy(), wl, np)
    achieved = flops / (attn_ms * 1e-3) / 1e12
    del ga, gb
    # the same kernels with w = N (dense causal), timed the same way
    p_d = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.N, dtype="bf16", forward_only=True)
    ws_d = dma.alloc_workspace(p_d)
    gda, gdb = graphs(p_d, ws_d, O, LSE)
    timed(gda, gdb, 2)
    n_d = 5
    step_d, attn_d = timed(gda, gdb, n_d)
    step_d = _max_over_ranks(step_d, world, torch)
    attn_d = _max_over_ranks(attn_d, world, torch)
    del gda, gdb, ws_d
    pairs_d = wl.with_(w=wl.N).kept_pairs()
    flops_d = 4.0 * wl.d * pairs_d
    dense = {"w": wl.N, "kept_pairs": pairs_d, "step_us": round(step_d * 1e3, 2), "attn_us": round(attn_d * 1e3, 2),
             "attn_tflops": round(flops_d / (attn_d * 1e-3) / 1e12, 2),
             "speedup_attn": round(attn_d / attn_ms, 3), "speedup_step": round(step_d / step_ms, 3), "steps": n_d}
    out = {"metric": "long prefill kept-pair TFLOP/s (gate + top-w mask + attention forward)",
           "value": round(world * flops / (step_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
           "config": {"workload": "long", "B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "N": wl.N, "d": wl.d, "w": wl.w,
                      "kept_pairs": wl.kept_pairs(), "scaled_key_positions": "5% x4", "forward_only": True,
                      "l2": "flushed before every step (256 MiB written, then 256 MiB read: no dirty lines left)"},
           "step_us": round(step_ms * 1e3, 2), "attn_us": round(attn_ms * 1e3, 2),
           "roofline": {"kernel": "attn_fwd", "bound": "tensor", "achieved": round(achieved, 2),
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                        "peak_kind": "burst " + peaks["source"],
                        "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                        "traffic": _traffic("attn_fwd_long", "attn_fwd_tc.cu"), "avg_launch_us": round(attn_ms * 1e3, 2),
                        "per_launch_flops": flops},
           "tile_density": dens,
           "dense_causal": dense,
           "gpu_launches": 7 * n}
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds / 2, workload="long")
    return out


def leg_cp(args, world, torch, dma, peaks):
    """Context-parallel prefill of the long workload over R = 2 shards, the ranks emulated one after
    another on this GPU: phase A per rank (gate on the shard, its candidates), the exchange (an
    all-gather of R candidate buffers: not run here, its bytes reported), phase B per rank (prefix
    stand-in, selection and attention of the shard's queries).  The step of R GPUs would take
    max_r A_r + exchange + max_r B_r."""
    import numpy as np

    from trainable_dynamic_mask_b200 import cp
    from workloads import get, make_inputs
    R = 2
    wl = get("long")
    I = make_inputs(wl)
    Q, K, V = (_to_dev_bf16(I.bits[n], torch) for n in ("Q", "K", "V"))
    Dl = _to_dev_bf16(I.bits["Delta"], torch)
    A = torch.from_numpy(I.A).cuda()
    del I
    flush = L2Flush(torch)
    ranks = []
    for r, (s0, s1) in enumerate(cp.shard_bounds(wl.N, R)):
        n = s1 - s0
        p = dma.make_params(wl.B, wl.H, wl.Hkv, n, wl.d, wl.w, dtype="bf16")
        lay = dma.cp_layout(p, s0, r)
        Pr = lay.prefix_rows
        Nc = Pr + n
        p2 = dma.make_params(wl.B, wl.H, wl.Hkv, Nc, wl.d, wl.w, Nq=n, dtype="bf16", forward_only=True)
        x = {"p": p, "p2": p2, "s0": s0, "n": n, "lay": lay, "Nc": Nc,
             "Q": Q[:, :, s0:s1].contiguous(), "K": K[:, :, s0:s1].contiguous(), "V": V[:, :, s0:s1].contiguous(),
             "delta": torch.empty((wl.B, wl.H, n), dtype=torch.float32, device="cuda"),
             "cand": torch.empty(lay.cand_bytes, dtype=torch.uint8, device="cuda"),
             "ws": torch.zeros(lay.ws_bytes, dtype=torch.uint8, device="cuda"),
             "dc": torch.empty((wl.B, wl.H, Nc), dtype=torch.float32, device="cuda"),
             "Kc": torch.empty((wl.B, wl.Hkv, Nc, wl.d), dtype=torch.bfloat16, device="cuda"),
             "Vc": torch.empty((wl.B, wl.Hkv, Nc, wl.d), dtype=torch.bfloat16, device="cuda"),
             "pc": torch.empty((wl.B, wl.Hkv, Nc), dtype=torch.int32, device="cuda"),
             "ws2": dma.alloc_workspace(p2),
             "ev": torch.empty((wl.B, wl.H, Nc), dtype=torch.int32, device="cuda"),
             "O": torch.empty((wl.B, wl.H, n, wl.d), dtype=torch.bfloat16, device="cuda"),
             "LSE": torch.empty((wl.B, wl.H, n), dtype=torch.float32, device="cuda")}
        ranks.append(x)
    allc = torch.empty((R, ranks[0]["lay"].cand_bytes), dtype=torch.uint8, device="cuda")

    def phase_a(x):
        dma.gate(x["p"], x["V"], Dl, A, x["delta"], None, None)
        dma.cp_candidates(x["p"], x["s0"], x["delta"], x["K"], x["V"], x["cand"], x["ws"])

    def phase_b(x, r):
        dma.cp_compact(x["p"], x["s0"], r, allc[:r] if r else None, x["delta"], x["K"], x["V"], x["dc"], x["Kc"],
                       x["Vc"], x["pc"], x["ws"])
        dma.topk_mask(x["p2"], x["dc"], x["ev"], x["ws2"])
        dma.attn_fwd(x["p2"], x["Q"], x["Kc"], x["Vc"], x["dc"], x["ev"], x["ws2"], x["O"], x["LSE"])

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush()
        a.record()
        fn()
        b.record()
        b.synchronize()
        return a.elapsed_time(b)

    n_rep = max(3, min(args.steps // 50, 10))
    ta = [[] for _ in range(R)]
    tb = [[] for _ in range(R)]
    for rep in range(2 + n_rep):
        for r, x in enumerate(ranks):
            t = timed(lambda: phase_a(x))
            allc[r].copy_(x["cand"])          # the exchange's result (an all-gather across GPUs)
            if rep >= 2:
                ta[r].append(t)
        torch.cuda.synchronize()
        for r, x in enumerate(ranks):
            t = timed(lambda: phase_b(x, r))
            if rep >= 2:
                tb[r].append(t)
    A_ms = [statistics.median(v) for v in ta]
    B_ms = [statistics.median(v) for v in tb]
    step_ms = max(A_ms) + max(B_ms)
    flops = 4.0 * wl.d * wl.kept_pairs()
    cb = ranks[0]["lay"].cand_bytes
    return {"metric": "context-parallel long prefill kept-pair TFLOP/s (R = 2 shards, ranks emulated on one GPU, "
                      "exchange not included)",
            "value": round(flops / (step_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "config": {"workload": "long", "shards": R, "B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "N": wl.N, "d": wl.d,
                       "w": wl.w, "compacted_keys_per_rank": [x["Nc"] for x in ranks]},
            "phase_a_us": [round(t * 1e3, 2) for t in A_ms], "phase_b_us": [round(t * 1e3, 2) for t in B_ms],
            "step_us_without_exchange": round(step_ms * 1e3, 2),
            "exchange_bytes_received_per_rank": R * cb, "candidate_buffer_bytes": cb,
            "exchange_us_at_measured_nvlink_770_GBps": round(R * cb / 770e9 * 1e6, 2),
            "note": "not measured across GPUs: both ranks run on one GPU, the exchange is not timed",
            # per timed repetition: phase A 3 kernels per rank; phase B 7 on rank 0 (copy of its own rows,
            # top-w 5, attention) and 10 on rank 1 (merged selection: gather, select, union, then the same)
            "gpu_launches": (3 + 7 + 3 + 10) * n_rep}


def leg_train(args, world, torch, dma, peaks):
    """Training step on the train workload: gate (saving x) + mask + attention
    forward + attention backward + gate backward.  kept-pair FLOPs = 14 d pairs
    (4 d forward, 10 d backward)."""
    from workloads import get, make_inputs
    wl = get("train")
    I = make_inputs(wl)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype="bf16")
    Q, K, V, Dl, dO = (_to_dev_bf16(I.bits[n], torch) for n in ("Q", "K", "V", "Delta", "dO"))
    A = torch.from_numpy(I.A).cuda()
    ws = dma.alloc_workspace(p)
    f32 = torch.float32
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=f32, device="cuda")
    x = torch.empty_like(delta)
    evict = torch.empty((wl.B, wl.H, wl.N), dtype=torch.int32, device="cuda")
    O = torch.empty_like(Q)
    LSE = torch.empty((wl.B, wl.H, wl.N), dtype=f32, device="cuda")
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    dd = torch.empty_like(delta)
    dDelta = torch.empty((wl.Hkv * wl.d, wl.H), dtype=f32, device="cuda")
    dA = torch.empty((wl.H,), dtype=f32, device="cuda")
    dVg = torch.empty(tuple(V.shape), dtype=f32, device="cuda")
    flush = L2Flush(torch)
    pairs = wl.kept_pairs()
    n = max(3, min(args.steps // 10, 30))
    t_f = t_b = 0.0
    for i in range(args.warmup + n):
        flush()
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record()
        dma.gate(p, V, Dl, A, delta, x, ws)
        dma.topk_mask(p, delta, evict, ws)
        dma.attn_fwd(p, Q, K, V, delta, evict, ws, O, LSE)
        b.record()
        dma.attn_bwd(p, Q, K, V, delta, evict, ws, O, LSE, dO, dQ, dK, dV, dd)
        dma.gate_bwd(p, V, Dl, A, x, delta, dd, dDelta, dA, dVg, ws)
        c.record()
        c.synchronize()
        if i >= args.warmup:
            t_f += a.elapsed_time(b)
            t_b += b.elapsed_time(c)
    t_f = _max_over_ranks(t_f, world, torch) / n
    t_b = _max_over_ranks(t_b, world, torch) / n
    ff, fb = 4.0 * wl.d * pairs, 10.0 * wl.d * pairs
    # the same kernels with w = N (dense causal), timed the same way
    p_d = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.N, dtype="bf16")
    ws_d = dma.alloc_workspace(p_d)
    td_f = td_b = 0.0
    n_d = 3
    for i in range(2 + n_d):
        flush()
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record()
        dma.gate(p_d, V, Dl, A, delta, x, ws_d)
        dma.topk_mask(p_d, delta, evict, ws_d)
        dma.attn_fwd(p_d, Q, K, V, delta, evict, ws_d, O, LSE)
        b.record()
        dma.attn_bwd(p_d, Q, K, V, delta, evict, ws_d, O, LSE, dO, dQ, dK, dV, dd)
        dma.gate_bwd(p_d, V, Dl, A, x, delta, dd, dDelta, dA, dVg, ws_d)
        c.record()
        c.synchronize()
        if i >= 2:
            td_f += a.elapsed_time(b)
            td_b += b.elapsed_time(c)
    del ws_d
    td_f = _max_over_ranks(td_f, world, torch) / n_d
    td_b = _max_over_ranks(td_b, world, torch) / n_d
    pairs_d = wl.with_(w=wl.N).kept_pairs()
    dense = {"w": wl.N, "kept_pairs": pairs_d, "fwd_ms": round(td_f, 4), "bwd_ms": round(td_b, 4),
             "tflops": round(14.0 * wl.d * pairs_d / ((td_f + td_b) * 1e-3) / 1e12, 3),
             "speedup_fwd_bwd": round((td_f + td_b) / (t_f + t_b), 3), "steps": n_d}
    return {"metric": "train fwd+bwd kept-pair TFLOP/s", "unit": "TFLOP/s",
            "value": round(world * (ff + fb) / ((t_f + t_b) * 1e-3) / 1e12, 3),
            "config": {"workload": "train", "B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "N": wl.N, "d": wl.d, "w": wl.w,
                       "kept_pairs": pairs},
            "fwd_ms": round(t_f, 4), "bwd_ms": round(t_b, 4),
            "fwd_tflops": round(ff / (t_f * 1e-3) / 1e12, 2), "bwd_tflops": round(fb / (t_b * 1e-3) / 1e12, 2),
            "bwd_frac_of_peak": round(fb / (t_b * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
            "dense_causal": dense,
            "gpu_launches": 17 * n}   # forward 7, attention backward 6, gate backward 4


# ---------------------------------------------------------------- the CPU oracle

def _cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _oracle_sample(n_rows, wl, I, d32, e_cache, oracle, np):
    """Oracle forward on the first n_rows query rows (over heads, in order) of
    a prefill-type workload; returns (seconds, kept-pair flops)."""
    t0 = time.perf_counter()
    rows_left, flops = n_rows, 0.0
    for h in range(wl.H):
        if rows_left <= 0:
            break
        if h not in e_cache:
            e_cache[h] = oracle.topw_eviction(d32[0, h], wl.w)
        r = np.arange(min(rows_left, wl.N))
        sl = (slice(0, 1), slice(h, h + 1))
        oracle.attn_fwd(I.Q[sl], I.K[:, h // wl.G: h // wl.G + 1], I.V[:, h // wl.G: h // wl.G + 1],
                        d32[sl].astype(np.float64), e_cache[h][None, None], rows=r)
        flops += 4.0 * wl.d * float(np.minimum(r + 1, wl.w).sum())
        rows_left -= r.size
    return time.perf_counter() - t0, flops


def cpu_baseline(budget_s=20.0, workload="prefill"):
    """The oracle, as it stands, on the host cores: gate on the whole workload
    plus masked attention forward on as many query rows as fit the time
    budget; kept-pair TFLOP/s of the rows processed."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle
    from workloads import get, make_inputs
    cores = _cpu_cores()
    wl = get(workload)
    I = make_inputs(wl)
    with threadpool_limits(limits=cores):
        t0 = time.perf_counter()
        _, d = oracle.gate(I.V, I.Delta, I.A)
        t_gate = time.perf_counter() - t0
        d32 = d.astype(np.float32)
        cache = {}
        t_small, _ = _oracle_sample(256, wl, I, d32, cache, oracle, np)
        n_rows = int(max(256, min(wl.N * wl.H, 256 * max(1.0, (budget_s - t_gate) / max(t_small, 1e-3)))))
        t_rows, flops = _oracle_sample(n_rows, wl, I, d32, cache, oracle, np)
    # scale the gate's cost to the sampled share of the workload
    share = flops / (4.0 * wl.d * wl.kept_pairs())
    secs = t_rows + t_gate * share
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{workload} workload: float64 gate on all of V (cost charged pro rata) + top-w and masked "
                      f"attention forward on the first {n_rows} query rows ({share * 100:.1f}% of kept pairs)",
            "seconds": round(secs, 3)}


def run_reference(args, world, rank):
    """The oracle timed as the reference arm, on the prefill workload's metric.
    Each step is a bounded sample sized so the whole run ends within minutes."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle
    from workloads import get, make_inputs
    cores = _cpu_cores()
    wl = get("prefill")
    I = make_inputs(wl)
    budget = float(args.ref_seconds)
    with threadpool_limits(limits=cores):
        _, d = oracle.gate(I.V, I.Delta, I.A)
        d32 = d.astype(np.float32)
        cache = {}
        t1, _ = _oracle_sample(128, wl, I, d32, cache, oracle, np)
        per_row = max(t1 / 128, 1e-5)
        rows = int(max(16, min(wl.N, budget / (args.steps + args.warmup) / per_row)))
        for _ in range(args.warmup):
            _oracle_sample(rows, wl, I, d32, cache, oracle, np)
        tot_t, tot_f = 0.0, 0.0
        for _ in range(args.steps):
            t, f = _oracle_sample(rows, wl, I, d32, cache, oracle, np)
            tot_t += t
            tot_f += f
    value = tot_f / tot_t / 1e12
    sample = f"prefill workload, first {rows} query rows of head 0 per step (oracle top-w + masked attention, float64)"
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "prefill", "B": wl.B, "H": wl.H, "Hkv": wl.Hkv, "N": wl.N, "d": wl.d, "w": wl.w},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-legs", action="store_true", help="skip the decode and training legs")
    ap.add_argument("--legs", default="long,decode,train,chunk,cp",
                    help="comma-separated legs to run: long, decode, train, chunk, cp")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-main", action="store_true",
                    help="profiling aid: run only the legs given by --legs and print them (no bench line)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--clock-soak", type=float, default=1.5,
                    help="seconds of untimed replays of the step, clock-sampled, before the timed region")
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    world, rank, local = _dist()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        line = run_ours(args, world, rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
