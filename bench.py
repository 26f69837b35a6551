#!/usr/bin/env python
"""Benchmark of the fused block-Hadamard rotate + FP4 quantize path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one fp4q_rotate_quantize call over the whole workload (rotation, amax, scale,
round, pack and store of every element).  The default workload is NVFP4 (group 16,
Hadamard block 16, static per-tensor scale) on a 4096 x 4096 bf16 activation matrix.
Inputs are resident in HBM when timing starts; successive steps cycle through enough
distinct input/output buffers that every step reads from HBM, not L2.  Steps are replayed
from CUDA graphs and timed with CUDA events on the launching stream.  Rank 0 prints one
JSON line.

Under torchrun (N > 1) every rank runs the same workload on its own GPU (rows are
independent: no collective on the data path); the elapsed time is the max over ranks.

--impl reference times the CPU oracle (as it stands) on a bounded sample of the same
workload on the host cores and prints the same line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from microscaling_fp4_quantization_b200 import workloads as W  # noqa: E402

METRIC = "fused rotate+FP4-quantize GB/s (bf16 in + packed out), % of B200 HBM peak"
KERNELS = {"auto": 0, "butterfly": 1, "tensor_core": 2}


def kernel_name(w, requested: str, signed: bool = False) -> str:
    """The kernel a plan with this request runs (auto: tensor core when b >= 16, b >= g and
    M*K >= 2^22, except MXFP4 with channel signs at b = 128 and M*K >= 3 * 2^26)."""
    if requested != "auto":
        return requested
    if signed and w.fmt == W.MXFP4 and w.block == 128 and w.numel >= (3 << 26):
        return "butterfly"
    return "tensor_core" if (w.block >= 16 and w.block >= w.group and w.numel >= (1 << 22)) else "butterfly"


L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "rotate_quantize_nvfp4_b16_4096x4096.md")
KERNEL_SOURCES = ["fp4q.cu", "fp4q_kernels.cuh", "fp4q_device.cuh", "fp4q_mma.cuh", "fp4q_launch.cuh"]


def kernel_source_hash() -> str:
    """Hash of the kernel sources with comments and blank lines removed (a comment edit does
    not change the kernel a profile was taken of)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "microscaling_fp4_quantization_b200", "csrc", f)) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, when
    it was taken on the current kernel sources; else None."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        line = line.strip().lstrip("-* ")
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU while running (NVML, every 5 ms)."""

    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "applications_clocks_setting": 0x2,
    }

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [k for k, v in self.REASONS.items() if self.reasons & v],
                "samples": len(self.samples)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(torch, ms: float, world: int, device) -> float:
    """The slowest rank's time.  Every rank calls it, in the same order (one all-reduce)."""
    if world == 1:
        return ms
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: int, steps: int, ms: float) -> float:
    """Weak scaling: every rank processes its own replica, so the job moves world x the bytes
    of one replica in the slowest rank's time."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def time_graph_steps(torch, launch, n_buf: int, steps: int, warmup: int, stream):
    """Capture `launch(i)` for i in 0..G-1 into a CUDA graph (i cycles the buffers) and time
    `steps` steps.  Returns (ms total, n_graph_launches)."""
    G = min(max(steps, 1), 256)
    G = max(n_buf, (G // n_buf) * n_buf) if G >= n_buf else G
    for i in range(max(warmup, 3)):
        launch(i % n_buf)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(G):
            launch(i % n_buf)
    rem = steps % G
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=stream):
            for i in range(rem):
                launch(i % n_buf)
    reps = steps // G
    # a short untimed soak so that the clocks settle under this load; every graph is launched
    # once here, so that no first launch (which uploads the graph) falls in a timed region
    g.replay()
    if g_rem is not None:
        g_rem.replay()
    torch.cuda.synchronize()
    return g, g_rem, reps


def time_replays(torch, g, g_rem, reps, stream) -> float:
    """Device milliseconds of `reps` replays of graph g (then g_rem once), between two CUDA
    events on `stream`.  One untimed replay of g is queued first: the host then submits the
    timed replays while the device is still busy, so the region starts with work queued
    behind the first event and no host submission gap lands inside it."""
    with torch.cuda.stream(stream):
        g.replay()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(reps):
            g.replay()
        if g_rem is not None:
            g_rem.replay()
        a1.record(stream)
    torch.cuda.synchronize()
    return a0.elapsed_time(a1)


def run_gpu(args):
    import torch
    from microscaling_fp4_quantization_b200 import fp4q as F

    world, rank, local = dist_setup()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload_for(args)
    M, K = w.M, w.K
    plan = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
    F.fp4q_plan_set_kernel(plan, KERNELS[args.kernel])
    x_np = w.generate()
    bytes_call = w.bytes_per_call()
    n_buf = max(1, math.ceil(3 * L2_BYTES / bytes_call)) if bytes_call < 2 * L2_BYTES else 1
    n_buf = min(n_buf, 16)
    x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    xs = [x_host.to(dev, non_blocking=True) for _ in range(n_buf)]
    codes = [torch.empty((M, K // 2), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    scales = [torch.empty((M, K // w.group), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    ts = torch.ones(1, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    extra = {}
    is_nv = w.fmt == W.NVFP4
    if is_nv:
        # static per-tensor scale from the library's own amax pass, before timing
        F.fp4q_amax(plan, xs[0], M, K, ts, stream=torch.cuda.current_stream())
        torch.cuda.synchronize()
        extra["tensor_scale"] = float(ts.item())

    def launch(i):
        F.fp4q_rotate_quantize(plan, xs[i], M, K, codes[i], scales[i], ts if is_nv else None,
                               stream=torch.cuda.current_stream())

    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, n_buf, args.steps, args.warmup, stream)
    sampler = ClockSampler(dev.index if world == 1 else local)
    sampler.start()
    # soak: about half a second of the same replays, untimed, so the clock samples mean something
    with torch.cuda.stream(stream):
        t_end = time.time() + 0.5
        while time.time() < t_end:
            g.replay()
            stream.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    ms_local = time_replays(torch, g, g_rem, reps, stream)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    sampler.stop()
    ms = max_over_ranks(torch, ms_local, world, dev)
    ms_step = ms / args.steps
    value = whole_job_gbs(world, bytes_call, args.steps, ms)
    kernel_us = ms_step * 1e3
    peak, peak_kind = measured_peak()

    # NVFP4: the amax pass and the dynamic mode (amax pass + quantize), timed on their own
    if is_nv and rank == 0:
        dyn = F.fp4q_plan_create(W.NVFP4, w.group, w.block, W.SCALE_NV_DYNAMIC)
        ts_d = torch.empty(1, dtype=torch.float32, device=dev)

        def launch_amax(i):
            F.fp4q_amax(plan, xs[i], M, K, ts_d, stream=torch.cuda.current_stream())

        def launch_dyn(i):
            F.fp4q_rotate_quantize(dyn, xs[i], M, K, codes[i], scales[i], ts_d, stream=torch.cuda.current_stream())

        for name, fn, nbytes in (("amax_pass", launch_amax, 2 * M * K), ("dynamic_mode", launch_dyn, bytes_call)):
            steps2 = max(50, min(args.steps, 400))
            with torch.cuda.stream(stream):
                g2, g2r, reps2 = time_graph_steps(torch, fn, n_buf, steps2, 3, stream)
                ms_ = time_replays(torch, g2, g2r, reps2, stream)
            torch.cuda.synchronize()
            us = ms_ * 1e3 / steps2
            extra[name] = {"us_per_call": round(us, 3), "GBps_algorithmic": round(nbytes / us / 1e3, 1),
                           "bytes_per_call": nbytes}
        extra["dynamic_mode"]["note"] = "reads X twice (amax pass, then quantize); bytes are the algorithmic ones"

    # context for the roofline at this size: a plain device copy that reads and writes the same
    # total bytes (half each way), timed the same way over as many rotating buffers
    if rank == 0:
        extra["copy_same_bytes"] = time_copy(torch, bytes_call, n_buf, stream, peak, steps=args.steps)

    # the randomised rotation (per-channel random signs) on the same workload, on the kernel the plan picks
    if rank == 0:
        extra["signed_rotation"] = time_signed(torch, F, w, xs, codes, scales, ts if is_nv else None, stream, peak,
                                               max(50, min(args.steps, 400)))

    # the quantization-error pass (signal / error energies and QSNR) on the same workload
    if rank == 0:
        extra["quant_error"] = time_quant_error(torch, F, w, plan, xs, ts if is_nv else None, stream, peak,
                                                max(50, min(args.steps, 400)))

    # e2e: the public API with host buffers, H2D of X and D2H of codes + scales inside the region.
    # Steps are pipelined as a user streaming batches would: copy-in, quantize and copy-out on
    # three streams over two buffer sets, so one step's copy-out overlaps the next step's
    # copy-in (the link is full duplex); events order the reuse of every buffer.
    e2e = None
    if rank == 0 or world > 1:
        nb = min(2, len(xs))
        codes_h = [torch.empty((M, K // 2), dtype=torch.uint8).pin_memory() for _ in range(nb)]
        scales_h = [torch.empty((M, K // w.group), dtype=torch.uint8).pin_memory() for _ in range(nb)]
        n_e2e = max(3, min(20, args.steps))
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        cur = torch.cuda.current_stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_q = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]
        started = [False] * nb

        def e2e_step(i):
            j = i % nb
            with torch.cuda.stream(s_in):
                if started[j]:
                    s_in.wait_event(ev_q[j])      # the quantize that last read xs[j] is done
                xs[j].copy_(x_host, non_blocking=True)
                ev_in[j].record(s_in)
            cur.wait_event(ev_in[j])
            if started[j]:
                cur.wait_event(ev_out[j])         # the copy-out that last read codes[j] is done
            F.fp4q_rotate_quantize(plan, xs[j], M, K, codes[j], scales[j], ts if is_nv else None, stream=cur)
            ev_q[j].record(cur)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_q[j])
                codes_h[j].copy_(codes[j], non_blocking=True)
                scales_h[j].copy_(scales[j], non_blocking=True)
                ev_out[j].record(s_out)
            started[j] = True

        for i in range(2 * nb):
            e2e_step(i)
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        s_out.wait_stream(cur)
        s_out.wait_stream(s_in)
        b1.record(s_out)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(torch, b0.elapsed_time(b1), world, dev)
        e2e = {"value": round(whole_job_gbs(world, bytes_call, n_e2e, e_ms), 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(x_host.numel() * 2),
               "d2h_bytes_per_step": int(codes_h[0].numel() + scales_h[0].numel()), "steps": n_e2e,
               "pipelined": f"{nb} buffer sets, copy-in / quantize / copy-out on three streams"}

    # the other target workloads, each timed like the headline (same step count, a lead-in
    # replay, clocks sampled through its region), on the kernel AUTO picks (rank 0)
    targets = {}
    if rank == 0 and not args.headline_only:
        cache = {}
        for tw in TARGET_WORKLOADS:
            if tw.name != w.name:
                targets[tw.name] = time_target(torch, F, tw, dev, stream, peak, args.steps, cache)
        del cache
        torch.cuda.empty_cache()

    # the other workloads' throughput, each timed the same way (rank 0, when asked)
    others = {}
    if rank == 0 and kernel_name(w, "auto") == "tensor_core" and args.kernel == "auto":
        # the measured alternative: the same workload on the butterfly kernel
        extra["butterfly_kernel"] = time_other(torch, F, w, dev, stream, peak, kernel="butterfly")
    if args.all_workloads and rank == 0:
        for ow in (W.SMALL_MX, W.MX_8K_FLOOR, W.MX_8K_CEIL, W.PREFILL_NV, W.PREFILL_MX) + W.DECODE:
            others[ow.name] = time_other(torch, F, ow, dev, stream, peak)
            if ow.block >= 16 and ow.block >= ow.group:
                alt = "butterfly" if kernel_name(ow, "auto") == "tensor_core" else "tensor_core"
                others[ow.name + f" [{alt} kernel]"] = time_other(torch, F, ow, dev, stream, peak, kernel=alt)
        for ow in (W.MX_8K_FLOOR, W.PREFILL_MX):
            others[ow.name + " [MBS-Static]"] = time_mbs(torch, F, ow, dev, stream, peak)
            for k in ("butterfly", "tensor_core"):
                others[ow.name + f" [MBS-Static, {k} kernel]"] = time_mbs(torch, F, ow, dev, stream, peak, kernel=k)
        gemms = {}
        for fmt, name in ((W.MXFP4, "mxfp4"), (W.NVFP4, "nvfp4")):
            for (M, N, K) in ((8192, 8192, 8192), (4096, 14336, 4096), (4096, 4096, 14336)):
                gemms[f"{name}_{M}x{N}x{K}"] = time_gemm(torch, F, fmt, M, N, K, stream)
        line_extra_gemm = gemms
        extra["fp4_gemm"] = line_extra_gemm

    if rank == 0:
        cpu = cpu_baseline(w, args) if world == 1 and not args.no_cpu_baseline else None
        traffic = profiled_traffic()
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 6),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded; N(0,1) rows with 0.5% outlier channels x50, bf16)",
            "config": {
                "workload": w.name, "M": M, "K": K,
                "format": "NVFP4" if is_nv else "MXFP4", "group": w.group, "hadamard_block": w.block,
                "scale_rule": W.RULE_NAMES[w.rule], "bytes_per_step": bytes_call,
                "kernel": kernel_name(w, args.kernel),
                "l2": f"inputs larger than L2 per step: {n_buf} rotating buffer sets "
                      f"({n_buf * bytes_call / 1e6:.0f} MB in total)" if n_buf > 1 else "input larger than L2",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            },
            "pct_of_hbm_peak": round(100 * value / world / peak, 2),
            "pct_of_spec_8TBps": round(100 * value / world / SPEC_HBM_GBS, 2),
            "elements_per_s": round(world * M * K / (ms_step * 1e-3), 1),
            "roofline": {
                "bound": "hbm",
                "achieved": round(bytes_call / (kernel_us * 1e-6) / 1e9, 2),
                "peak": peak,
                "unit": "GB/s",
                "frac": round(bytes_call / (kernel_us * 1e-6) / 1e9 / peak, 4),
                "traffic": traffic,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6650 GB/s",
                "kernel": ("rotate_quantize_mma_kernel" if kernel_name(w, args.kernel) == "tensor_core"
                           else "rotate_quantize_kernel"), "us_per_launch": round(kernel_us, 3),
            },
            "gpu_launches": args.steps,
            # the pages' own figures, for context only: end-to-end and layer-wise speedups of the
            # whole MR-GPTQ FP4 stack (quantized GEMMs in vLLM) over FP16, on other workloads
            "context": {
                "source": "Bridging the Gap Between Promise and Performance for Microscaling FP4 "
                          "Quantization: abstract; Technische Zusammenfassung, 3. Wichtige Ergebnisse",
                "speedup_vs_fp16_B200": {"layer_wise": "up to 3.6x", "end_to_end": "up to 2.2x"},
                "speedup_vs_fp16_RTX5090": {"layer_wise": "up to 6x", "end_to_end": "up to 4x"},
                "note": "not a measurement of this path, and not its target",
            },
            "clocks": sampler.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "extra": extra,
        }
        if targets:
            line["targets"] = targets
        if others:
            line["workloads"] = others
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def workload_for(args):
    w = W.BY_NAME[args.workload]
    return w.with_rows(args.rows) if args.rows else w


def run_kernel_only(args):
    """W + K back-to-back launches of the workload's kernel on cuda:0, nothing else timed."""
    import torch
    from microscaling_fp4_quantization_b200 import fp4q as F
    torch.cuda.set_device(0)
    w = workload_for(args)
    plan = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
    F.fp4q_plan_set_kernel(plan, KERNELS[args.kernel])
    if args.signs:
        mask = torch.from_numpy(W.random_sign_mask(w.K, 1234).view(np.int32)).cuda()
        F.fp4q_plan_set_signs(plan, mask, w.K)
    x = torch.from_numpy(w.generate().view(np.int16)).view(torch.bfloat16).cuda()
    codes = torch.empty((w.M, w.K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((w.M, w.K // w.group), dtype=torch.uint8, device="cuda")
    ts = torch.ones(1, dtype=torch.float32, device="cuda")
    if w.fmt == W.NVFP4:
        F.fp4q_amax(plan, x, w.M, w.K, ts)
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    for _ in range(args.warmup + args.steps):
        if args.op == "quant_error":
            F.fp4q_quant_error(plan, x, w.M, w.K, ts if w.fmt == W.NVFP4 else None, out)
        else:
            F.fp4q_rotate_quantize(plan, x, w.M, w.K, codes, scales, ts if w.fmt == W.NVFP4 else None)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    print(f"kernel-only: {args.op} {w.name} M={w.M} K={w.K} signs={args.signs} launches={args.warmup + args.steps}",
          flush=True)


def tensor_peak_fp4(sustained: bool = False):
    """Dense FP4 tensor peak: the measured bf16 figure times the nominal fp4 / bf16 ratio
    (9 / 2.25 = 4); the burst figure (a kernel timed alone), or the sustained one (a
    seconds-long loop under the power cap)."""
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 4.0 * float(json.load(f)[key]), f"measured {key} x 4 (nominal fp4/bf16)"
    except Exception:
        return 4.0 * (1400.0 if sustained else 1590.0), "fallback bf16 figure x 4"


def time_gemm(torch, F, fmt, M, N, K, stream, steps=200):
    """fp4q_gemm on operands quantized by the library (activations N(0,1) rows, Laplace
    weights), two rotating operand / output sets (more than L2 in total): TFLOP/s against the
    FP4 tensor peak."""
    g = 32 if fmt == W.MXFP4 else 16
    rule = W.SCALE_FLOOR_OCP if fmt == W.MXFP4 else W.SCALE_NV_DYNAMIC
    blk = 32 if fmt == W.MXFP4 else 16
    rng = np.random.default_rng(M + N + K)
    sets = []
    for i in range(2):
        xs_ = []
        for R, data in ((M, None), (N, None)):
            plan = F.fp4q_plan_create(fmt, g, blk, rule)
            x = torch.randn((R, K), dtype=torch.float32, device="cuda", generator=None).to(torch.bfloat16)
            c = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
            sc = torch.empty((R, K // g), dtype=torch.uint8, device="cuda")
            ts_ = torch.empty(1, dtype=torch.float32, device="cuda")
            F.fp4q_rotate_quantize(plan, x, R, K, c, sc, ts_ if fmt == W.NVFP4 else None)
            del x
            xs_.append((c, sc, ts_))
        d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        sets.append((xs_[0], xs_[1], d))
    torch.cuda.synchronize()
    nv = fmt == W.NVFP4

    def launch(i):
        a, bb, d = sets[i]
        F.fp4q_gemm(fmt, a[0], a[1], a[2] if nv else None, bb[0], bb[1], bb[2] if nv else None, M, N, K, d,
                    stream=torch.cuda.current_stream())

    sampler = ClockSampler(torch.cuda.current_device())
    with torch.cuda.stream(stream):
        gph, g_rem, reps = time_graph_steps(torch, launch, 2, steps, 3, stream)
        # a short untimed soak so that the clocks settle under this load (dense FP4 work can
        # meet the power cap), then clocks sampled through the timed region
        t_end = time.time() + 0.3
        while time.time() < t_end:
            gph.replay()
            stream.synchronize()
        sampler.start()
        ms_ = time_replays(torch, gph, g_rem, reps, stream)
    torch.cuda.synchronize()
    sampler.stop()
    us = ms_ * 1e3 / steps
    tflops = 2.0 * M * N * K / (us * 1e-6) / 1e12
    peak, kind = tensor_peak_fp4()
    peak_s, _ = tensor_peak_fp4(sustained=True)
    del sets
    torch.cuda.empty_cache()
    return {"M": M, "N": N, "K": K, "us_per_call": round(us, 2), "TFLOPs": round(tflops, 1),
            "frac_of_fp4_peak": round(tflops / peak, 4), "fp4_peak_TFLOPs": round(peak, 1), "peak_source": kind,
            "frac_of_fp4_peak_sustained": round(tflops / peak_s, 4), "fp4_peak_sustained_TFLOPs": round(peak_s, 1),
            "bound": "tensor", "steps": steps, "clocks": sampler.summary()}


def time_copy(torch, nbytes, n_buf, stream, peak, steps=2000):
    """A device-to-device copy of nbytes / 2 bytes (so nbytes move through HBM), over n_buf
    rotating buffer pairs, replayed from a CUDA graph and timed with CUDA events: what a plain
    copy achieves at the size of one call.  A reference point, not part of the path."""
    half = nbytes // 2 // 16 * 16
    srcs = [torch.empty(half, dtype=torch.uint8, device="cuda").fill_(1) for _ in range(n_buf)]
    dsts = [torch.empty(half, dtype=torch.uint8, device="cuda") for _ in range(n_buf)]

    def launch(i):
        dsts[i].copy_(srcs[i], non_blocking=True)

    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, n_buf, steps, 3, stream)
        ms_ = time_replays(torch, g, g_rem, reps, stream)
    torch.cuda.synchronize()
    us = ms_ * 1e3 / steps
    gbs = 2 * half / us / 1e3
    del srcs, dsts
    return {"bytes_per_call": 2 * half, "us_per_call": round(us, 3), "GBps": round(gbs, 1),
            "pct_of_hbm_peak": round(100 * gbs / peak, 2), "buffers": n_buf}


def time_plan(torch, F, plan, w, xs, codes, scales, ts, stream, steps):
    """Device microseconds per fp4q_rotate_quantize call of `plan` over the buffers in turn
    (CUDA graph replays, CUDA events on the launching stream)."""
    M, K = w.M, w.K

    def launch(i):
        F.fp4q_rotate_quantize(plan, xs[i], M, K, codes[i], scales[i], ts, stream=torch.cuda.current_stream())

    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, len(xs), steps, 3, stream)
        ms_ = time_replays(torch, g, g_rem, reps, stream)
    torch.cuda.synchronize()
    return ms_ * 1e3 / steps


def time_signed(torch, F, w, xs, codes, scales, ts, stream, peak, steps, kernel="auto"):
    """fp4q_rotate_quantize with a plan carrying per-channel random signs (seeded mask): the
    same bytes as the plain call, on the kernel the plan picks."""
    K = w.K
    plan = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
    F.fp4q_plan_set_kernel(plan, KERNELS[kernel])
    mask = torch.from_numpy(W.random_sign_mask(K, 1234).view(np.int32)).to(xs[0].device)
    F.fp4q_plan_set_signs(plan, mask, K)
    us = time_plan(torch, F, plan, w, xs, codes, scales, ts, stream, steps)
    nbytes = w.bytes_per_call()
    gbs = nbytes / us / 1e3
    return {"us_per_call": round(us, 3), "GBps": round(gbs, 1), "pct_of_hbm_peak": round(100 * gbs / peak, 2),
            "bytes_per_call": nbytes, "kernel": kernel_name(w, kernel, signed=True)}


def run_gemm_only(args):
    """W + K launches of fp4q_gemm (a case for profilers): N(0, 1) activations [M][K] and weights
    [N][K] quantized by the library (block 32 floor for MXFP4, 16 dynamic for NVFP4)."""
    import torch
    from microscaling_fp4_quantization_b200 import fp4q as F
    torch.cuda.set_device(0)
    M, N, K = args.gemm
    fmt = W.MXFP4 if args.gemm_format == "mxfp4" else W.NVFP4
    g = 32 if fmt == W.MXFP4 else 16
    rule = W.SCALE_FLOOR_OCP if fmt == W.MXFP4 else W.SCALE_NV_DYNAMIC
    ops = []
    for R in (M, N):
        plan = F.fp4q_plan_create(fmt, g, g, rule)
        x = torch.randn((R, K), device="cuda").to(torch.bfloat16)
        c = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
        sc = torch.empty((R, K // g), dtype=torch.uint8, device="cuda")
        t = torch.empty(1, dtype=torch.float32, device="cuda")
        F.fp4q_rotate_quantize(plan, x, R, K, c, sc, t if fmt == W.NVFP4 else None)
        ops.append((c, sc, t))
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    nv = fmt == W.NVFP4
    for _ in range(args.warmup + args.steps):
        F.fp4q_gemm(fmt, ops[0][0], ops[0][1], ops[0][2] if nv else None, ops[1][0], ops[1][1],
                    ops[1][2] if nv else None, M, N, K, d)
    torch.cuda.synchronize()
    assert F.fp4q_device_status() == F.FP4Q_OK
    print(f"gemm-only: {args.gemm_format} {M}x{N}x{K} launches={args.warmup + args.steps}", flush=True)


def time_quant_error(torch, F, w, plan, xs, ts, stream, peak, steps):
    """fp4q_quant_error on the workload's rotating inputs: device time per call (one kernel),
    GB/s on its algorithmic bytes (X read once, 24 bytes out) and the QSNR."""
    M, K = w.M, w.K
    out = torch.empty(3, dtype=torch.float64, device=xs[0].device)

    def launch(i):
        F.fp4q_quant_error(plan, xs[i], M, K, ts, out, stream=torch.cuda.current_stream())

    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, len(xs), steps, 3, stream)
        ms_ = time_replays(torch, g, g_rem, reps, stream)
    torch.cuda.synchronize()
    us = ms_ * 1e3 / steps
    launch(0)
    torch.cuda.synchronize()
    sig, err, q = out.tolist()
    nbytes = 2 * M * K + 24
    gbs = nbytes / us / 1e3
    return {"us_per_call": round(us, 3), "GBps": round(gbs, 1), "pct_of_hbm_peak": round(100 * gbs / peak, 2),
            "bytes_per_call": nbytes, "launches_per_call": 1, "qsnr_db": round(q, 4), "signal": sig, "error": err,
            "mse": err / (M * K)}


def time_mbs(torch, F, w, dev, stream, peak, kernel="auto"):
    """MBS-Static (MXFP4 with 128-element macro scales) on an MX workload's input: GB/s on its
    algorithmic bytes (bf16 in; codes, E8M0 group scales and macro bytes out), and the QSNR
    against plain MXFP4 with the same rule."""
    M, K = w.M, w.K
    plan = F.fp4q_plan_create(F.FP4Q_MXFP4_MBS, 32, w.block, w.rule)
    F.fp4q_plan_set_kernel(plan, KERNELS[kernel])
    x_np = w.generate()
    nbytes = M * K * 2 + M * K // 2 + M * K // 32 + M * K // 128
    n_buf = max(1, math.ceil(3 * L2_BYTES / nbytes)) if nbytes < 2 * L2_BYTES else 1
    xh = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16)
    xs = [xh.to(dev) for _ in range(n_buf)]
    del x_np, xh
    codes = [torch.empty((M, K // 2), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    scales = [torch.empty((M, K // 32), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    macro = [torch.empty((M, K // 128), dtype=torch.uint8, device=dev) for _ in range(n_buf)]

    def launch(i):
        F.fp4q_rotate_quantize_mbs(plan, xs[i], M, K, codes[i], scales[i], macro[i], stream=torch.cuda.current_stream())

    steps = 200 if nbytes > 1e8 else 2000
    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, n_buf, steps, 5, stream)
        ms_ = time_replays(torch, g, g_rem, reps, stream)
    torch.cuda.synchronize()
    us = ms_ * 1e3 / steps
    gbs = nbytes / us / 1e3
    qe_mbs = time_quant_error(torch, F, w, plan, xs, None, stream, peak, 20)
    plain = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
    F.fp4q_plan_set_kernel(plain, KERNELS[kernel])
    qe_plain = time_quant_error(torch, F, w, plain, xs, None, stream, peak, 20)
    used = kernel_name(w, kernel)   # MBS plans choose as MXFP4 plans do (group 32)
    out = {"GBps": round(gbs, 1), "pct_of_hbm_peak": round(100 * gbs / peak, 2), "us_per_call": round(us, 3),
           "bytes_per_call": nbytes, "buffers": n_buf, "kernel": used,
           "qsnr_db": qe_mbs["qsnr_db"], "qsnr_db_plain_mxfp4": qe_plain["qsnr_db"],
           "quant_error": {k: qe_mbs[k] for k in ("us_per_call", "GBps", "pct_of_hbm_peak")}}
    del xs, codes, scales, macro
    torch.cuda.empty_cache()
    return out


# The workloads the fused kernel is graded on besides the headline (8192 x 8192 MXFP4 b128 under
# both rules, and the 32768 x 14336 prefill under NVFP4 and MXFP4 b128), then the small one and
# the decode rows (latency: microseconds per call).
TARGET_WORKLOADS = (W.MX_8K_FLOOR, W.MX_8K_CEIL, W.PREFILL_NV, W.PREFILL_MX, W.SMALL_MX) + W.DECODE


def time_target(torch, F, w, dev, stream, peak, steps, cache):
    """One target workload on the kernel AUTO picks: `steps` calls over rotating buffers (more
    than L2 in total, or one buffer larger than L2), replayed from a CUDA graph after a short
    untimed soak, timed with CUDA events, SM clocks sampled through the timed region.  Inputs
    with the same seed and shape are generated once (`cache`)."""
    M, K = w.M, w.K
    key = (w.seed, M, K)
    if key not in cache:
        cache.clear()
        cache[key] = torch.from_numpy(w.generate().view(np.int16)).view(torch.bfloat16)
    xh = cache[key]
    plan = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
    bytes_call = w.bytes_per_call()
    n_buf = max(1, math.ceil(3 * L2_BYTES / bytes_call)) if bytes_call < 2 * L2_BYTES else 1
    n_buf = min(n_buf, 64)
    xs = [xh.to(dev) for _ in range(n_buf)]
    codes = [torch.empty((M, K // 2), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    scales = [torch.empty((M, K // w.group), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    ts = torch.ones(1, dtype=torch.float32, device=dev)
    nv = w.fmt == W.NVFP4
    if nv:
        F.fp4q_amax(plan, xs[0], M, K, ts, stream=torch.cuda.current_stream())

    def launch(i):
        F.fp4q_rotate_quantize(plan, xs[i], M, K, codes[i], scales[i], ts if nv else None,
                               stream=torch.cuda.current_stream())

    sampler = ClockSampler(dev.index)
    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, n_buf, steps, 3, stream)
        # the samples cover the soak (the same replays) and the timed region
        sampler.start()
        t_end = time.time() + 0.2
        while time.time() < t_end:
            g.replay()
            stream.synchronize()
    ms = time_replays(torch, g, g_rem, reps, stream)
    sampler.stop()
    assert F.fp4q_device_status() == F.FP4Q_OK
    us = ms * 1e3 / steps
    gbs = bytes_call / us / 1e3
    del g, g_rem
    out = {"GBps": round(gbs, 1), "pct_of_hbm_peak": round(100 * gbs / peak, 2), "us_per_call": round(us, 3),
           "elements_per_s": round(M * K / (us * 1e-6), 1), "bytes_per_call": bytes_call, "steps": steps,
           "buffers": n_buf, "kernel": kernel_name(w, "auto"), "format": "NVFP4" if nv else "MXFP4",
           "hadamard_block": w.block, "scale_rule": W.RULE_NAMES[w.rule], "clocks": sampler.summary()}
    if kernel_name(w, "auto") == "tensor_core":
        # the randomised rotation (per-channel random signs) on the same buffers and kernel
        out["signed"] = time_signed(torch, F, w, xs, codes, scales, ts if nv else None, stream, peak, steps)
    if w.block == 128:
        # the error pass, and (MXFP4) MBS-Static, on the same inputs
        out["quant_error"] = time_quant_error(torch, F, w, plan, xs, ts if nv else None, stream, peak, steps)
        if not nv:
            out["mbs_static"] = time_mbs_on(torch, F, w, xs, stream, peak, steps)
    del xs, codes, scales
    return out


def time_mbs_on(torch, F, w, xs, stream, peak, steps):
    """MBS-Static (MXFP4 with 128-element macro scales, the workload's block and rule) on the
    given input buffers: device time per call, GB/s on its algorithmic bytes (bf16 in; codes,
    E8M0 group scales and macro bytes out)."""
    M, K = w.M, w.K
    plan = F.fp4q_plan_create(F.FP4Q_MXFP4_MBS, 32, w.block, w.rule)
    dev = xs[0].device
    codes = [torch.empty((M, K // 2), dtype=torch.uint8, device=dev) for _ in xs]
    scales = [torch.empty((M, K // 32), dtype=torch.uint8, device=dev) for _ in xs]
    macro = [torch.empty((M, K // 128), dtype=torch.uint8, device=dev) for _ in xs]

    def launch(i):
        F.fp4q_rotate_quantize_mbs(plan, xs[i], M, K, codes[i], scales[i], macro[i], stream=torch.cuda.current_stream())

    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, len(xs), steps, 3, stream)
    us = time_replays(torch, g, g_rem, reps, stream) * 1e3 / steps
    nbytes = M * K * 2 + M * K // 2 + M * K // 32 + M * K // 128
    gbs = nbytes / us / 1e3
    del g, g_rem, codes, scales, macro
    return {"us_per_call": round(us, 3), "GBps": round(gbs, 1), "pct_of_hbm_peak": round(100 * gbs / peak, 2),
            "bytes_per_call": nbytes, "kernel": kernel_name(w, "auto")}


def time_other(torch, F, w, dev, stream, peak, kernel="auto"):
    M, K = w.M, w.K
    plan = F.fp4q_plan_create(w.fmt, w.group, w.block, w.rule)
    F.fp4q_plan_set_kernel(plan, KERNELS[kernel])
    x_np = w.generate()
    bytes_call = w.bytes_per_call()
    n_buf = max(1, math.ceil(3 * L2_BYTES / bytes_call)) if bytes_call < 2 * L2_BYTES else 1
    n_buf = min(n_buf, 64)
    xh = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16)
    xs = [xh.to(dev) for _ in range(n_buf)]
    del x_np, xh
    codes = [torch.empty((M, K // 2), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    scales = [torch.empty((M, K // w.group), dtype=torch.uint8, device=dev) for _ in range(n_buf)]
    ts = torch.ones(1, dtype=torch.float32, device=dev)
    if w.fmt == W.NVFP4:
        F.fp4q_amax(plan, xs[0], M, K, ts, stream=torch.cuda.current_stream())

    def launch(i):
        F.fp4q_rotate_quantize(plan, xs[i], M, K, codes[i], scales[i], ts if w.fmt == W.NVFP4 else None,
                               stream=torch.cuda.current_stream())

    steps = 200 if bytes_call > 1e8 else 2000
    with torch.cuda.stream(stream):
        g, g_rem, reps = time_graph_steps(torch, launch, n_buf, steps, 5, stream)
        ms_ = time_replays(torch, g, g_rem, reps, stream)
    torch.cuda.synchronize()
    us = ms_ * 1e3 / steps
    gbs = bytes_call / us / 1e3
    out = {"GBps": round(gbs, 1), "pct_of_hbm_peak": round(100 * gbs / peak, 2), "us_per_call": round(us, 3),
           "bytes_per_call": bytes_call, "buffers": n_buf, "kernel": kernel_name(w, kernel)}
    out["signed"] = time_signed(torch, F, w, xs, codes, scales, ts if w.fmt == W.NVFP4 else None, stream, peak,
                                steps, kernel)
    if kernel == "auto":
        out["quant_error"] = time_quant_error(torch, F, w, plan, xs, ts if w.fmt == W.NVFP4 else None, stream, peak,
                                              steps // 2)
    del xs, codes, scales
    torch.cuda.empty_cache()
    return out


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def _oracle_batch(job):
    """One batch of the oracle in a pool process (rows of X through rotate_quantize)."""
    import oracle
    x, fmt, group, block, rule, ts = job
    oracle.rotate_quantize(x, fmt, group, block, rule, tensor_scale=ts)
    return x.shape[0]


def oracle_pool(n: int):
    """A pool of n host processes for the oracle, one BLAS thread each, started with `spawn`
    (the parent has initialised CUDA; a process forked after that can hang)."""
    import multiprocessing as mp
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    try:
        return mp.get_context("spawn").Pool(n)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def oracle_sample(w, rows: int):
    """The first `rows` rows of the workload and, for NVFP4, the oracle's tensor scale of them."""
    import oracle
    x = next(iter(w.row_chunks(chunk_rows=rows)))
    ts = oracle.nv_tensor_scale(oracle.rotated_amax(x, w.block)) if w.fmt == W.NVFP4 else None
    return x, ts


def cpu_baseline(w, args, seconds: float = 8.0):
    """The oracle, as it stands, on bounded samples of the workload's rows: once on one host
    thread, then on every host core (one process per core, each running the oracle on its own
    batches of rows; rows are independent).  GB/s on the samples' algorithmic bytes.  The
    line's value is the all-cores figure, with the single-thread one beside it."""
    import oracle
    from threadpoolctl import threadpool_limits

    rows_per_batch = max(1, (1 << 20) // w.K)
    x, ts = oracle_sample(w, rows_per_batch)
    done_rows = 0
    t0 = time.perf_counter()
    with threadpool_limits(limits=1):
        while True:
            oracle.rotate_quantize(x, w.fmt, w.group, w.block, w.rule, tensor_scale=ts)
            done_rows += x.shape[0]
            if time.perf_counter() - t0 >= seconds:
                break
    dt1 = time.perf_counter() - t0
    single = {"value": round(w.with_rows(done_rows).bytes_per_call() / dt1 / 1e9, 5), "unit": "GB/s", "cores": 1,
              "sample": f"{done_rows} rows x {w.K} ({x.shape[0]}-row batches), {dt1:.1f} s wall on 1 host thread"}

    n = min(host_cores(), 128)
    job = (x, w.fmt, w.group, w.block, w.rule, ts)
    with oracle_pool(n) as pool:
        pool.map(_oracle_batch, [job] * n, chunksize=1)          # start-up and imports, untimed
        done_rows = 0
        pending = []
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            while len(pending) < 2 * n:
                pending.append(pool.apply_async(_oracle_batch, (job,)))
            done_rows += pending.pop(0).get()
        for p in pending:
            done_rows += p.get()
        dtn = time.perf_counter() - t0
    value = w.with_rows(done_rows).bytes_per_call() / dtn / 1e9
    return {"value": round(value, 5), "unit": "GB/s", "cores": n, "kind": "oracle",
            "sample": f"{done_rows} rows x {w.K} ({x.shape[0]}-row batches of the same workload, one process per "
                      f"core, one BLAS thread each), {dtn:.1f} s wall on {n} host cores",
            "cpu_model": cpu_model(), "host_cores": host_cores(), "single_thread": single}


def run_reference(args):
    """The reference arm: the oracle, as it stands, on every host core.  One step is one
    bounded sample of the workload: one batch of rows per core, run in parallel."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    w = W.BY_NAME[args.workload]
    rows = max(1, (1 << 18) // w.K)
    x, ts = oracle_sample(w, rows)
    n = min(host_cores(), 128)
    job = (x, w.fmt, w.group, w.block, w.rule, ts)
    with oracle_pool(n) as pool:
        pool.map(_oracle_batch, [job] * n, chunksize=1)
        for _ in range(args.warmup):
            pool.map(_oracle_batch, [job] * n, chunksize=1)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            pool.map(_oracle_batch, [job] * n, chunksize=1)
        dt = time.perf_counter() - t0
    sb = w.with_rows(x.shape[0] * n).bytes_per_call()
    value = sb * args.steps / dt / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 5), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "sample_rows_per_step": x.shape[0] * n},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": n, "kind": "oracle",
                         "sample": f"{x.shape[0]} rows x {w.K} per core per step, {n} host cores",
                         "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=W.NV_4K.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--impl", default="fp4q", choices=["fp4q", "reference"])
    ap.add_argument("--all-workloads", action="store_true",
                    help="also time every workload's variants (other kernel, signs, error pass, MBS) and the FP4 GEMM")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other target workloads (the 'targets' entry of the line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rows", type=int, default=0, help="override the workload's row count M")
    ap.add_argument("--kernel", default="auto", choices=["auto", "butterfly", "tensor_core"],
                    help="which rotate + quantize kernel the plan uses")
    ap.add_argument("--kernel-only", action="store_true",
                    help="only W + K plain launches of the workload (a case for profilers), no JSON line")
    ap.add_argument("--op", default="rotate_quantize", choices=["rotate_quantize", "quant_error"],
                    help="with --kernel-only: the call to launch")
    ap.add_argument("--signs", action="store_true",
                    help="with --kernel-only: the plan carries per-channel random signs (seeded mask)")
    ap.add_argument("--gemm", type=int, nargs=3, metavar=("M", "N", "K"), default=None,
                    help="with --kernel-only: W + K launches of fp4q_gemm on operands the library quantized")
    ap.add_argument("--gemm-format", default="nvfp4", choices=["mxfp4", "nvfp4"])
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.kernel_only and args.gemm:
        run_gemm_only(args)
    elif args.kernel_only:
        run_kernel_only(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
