#!/usr/bin/env python
"""Throughput of the Multi-Token Attention forward on B200.

`python bench.py --gpus N --steps K --warmup W` runs W untimed and K timed
steps of the MTA forward on the long-context workload (B2 H16 d128 T4096,
(c_q, c_k, c_h) = (6, 11, 2), bf16) on each of N GPUs (one process per GPU,
independent replicas: weak scaling), and rank 0 prints one JSON line.

Timing: device time from CUDA events on the stream the library launches on,
with the L2 cache flushed (a 256 MiB write, untimed) before every timed step;
barrier + synchronize on both sides of the timed region; max over ranks.
Per-kernel times come from the library's traced entry point (events recorded
around each of its launches).  SM clocks and throttle reasons are sampled
through NVML during the timed region.  `e2e` repeats the measurement through
the public API with pinned host buffers, copies included.  `cpu_baseline`
times the fp64 oracle on a bounded sample of the same workload on the host.

`--compose NAME` times one composition of "Putting Everything Together: The
Full MTA Module" (e.g. `repeat`: the MTA convolution repeated after the
softmax) through mta_forward_composed, with FLOPs counted for the steps it
has.

`--impl reference` times that oracle (the only reference implementation of
this method: the pages ship no code) on the host cores instead.
"""
import argparse
import ctypes
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from convolved_logit_attention_b200.workloads import (COMPOSITIONS, WORKLOADS,  # noqa: E402
                                                      composed_inputs, make_inputs)

METRIC = "MTA fwd TFLOP/s and tokens/s at T=4096 bf16; % of B200 bf16 tensor peak"
L2_FLUSH_BYTES = 256 << 20
# FP32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1965 MHz.
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["mta", "reference"], default="mta")
    p.add_argument("--workload", default="longctx_4k", choices=sorted(WORKLOADS))
    p.add_argument("--path", choices=["forward", "unfused"], default="forward",
                   help="forward: mta_forward (the fused path where supported); "
                        "unfused: mta_forward_unfused (materialised maps)")
    p.add_argument("--batch", type=int, default=None,
                   help="override the workload's batch size (smaller cases for profiler captures)")
    p.add_argument("--gate", action="store_true",
                   help="time mta_forward_gated (sigmoid-gated output, fixed gate values) "
                        "instead of mta_forward")
    p.add_argument("--compose", choices=sorted(COMPOSITIONS), default=None,
                   help="time mta_forward_composed on this composition of the module")
    p.add_argument("--backward", action="store_true",
                   help="time mta_backward (gradients of the default composition for a seeded "
                        "upstream gradient) instead of the forward")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, device_index, period_s=0.005):
        self.samples = []
        self.reasons = set()
        self.period = period_s
        self._stop = threading.Event()
        self._ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as exc:   # no NVML: report the absence
            self.error = repr(exc)

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self._t.join()
        return False

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons - {"gpu_idle"})}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if args.impl == "mta" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif args.impl == "mta":
        torch.cuda.set_device(local)
    return world, rank, local


def dist_max(x, world, device):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tflops(world, flops_per_step, steps, max_total_ms):
    """Whole-job throughput of `world` independent replicas, each doing
    `steps` steps of `flops_per_step`, timed by the slowest rank."""
    return world * flops_per_step * steps / (max_total_ms / 1e3) / 1e12


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


WEIGHTS = ("w_kq", "w_head", "w_kq_post", "w_head_post")   # positional order of the call


def compose_kw(args, d):
    """Keyword arguments of mta_forward_composed beyond the four positional
    weights: the logit mix, the 3-D kernel and the exact-mask flag."""
    return {"w_head_pre": d.get("w_head_pre"), "w_kq_3d": d.get("w_kq_3d"),
            "exact_mask": bool(COMPOSITIONS[args.compose].get("exact_mask"))}


def device_inputs(x, io, device):
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    d = {n: torch.from_numpy(x[n]).to(device).to(dt) for n in ("q", "k", "v")}
    for n in WEIGHTS + ("w_head_pre", "w_kq_3d", "gn_weight", "gn_bias"):
        d[n] = torch.from_numpy(x[n]).to(device) if x.get(n) is not None else None
    return d


def step_flops(args, w):
    return w.composition_flops(COMPOSITIONS[args.compose]) if args.compose \
        else w.algorithmic_flops()


def conv_heads_per_launch(comp):
    """Input heads per k_conv launch, averaged over a composition's k_conv
    launches: c_h for the 3-D kernel, 1 for every 2-D one."""
    if not comp:
        return 1.0
    per = [comp["c_h"]] if comp.get("w_kq_3d") else ([1] if comp.get("w_kq") else [])
    per += [1] if comp.get("w_kq_post") else []
    return sum(per) / len(per) if per else 1.0


def kernel_units(name, w, comp=None):
    """(bound, algorithmic amount per launch, unit) for each kernel the
    library launches on workload w (comp: the composition's steps, with
    c_h, when one is timed).  L = T(T+1)/2 live logits per (b, h)."""
    logits = w.B * w.H * w.live_logits()
    io_bytes = 2 if w.io == "bf16" else 4
    conv = logits * 2 * w.c_q * w.c_k * conv_heads_per_launch(comp)
    table = {
        "k_logits": ("alu", logits * 2 * w.d, "FLOP"),
        "k_conv": ("alu", conv, "FLOP"),
        "k_softmax_mix": ("hbm", logits * 8, "B"),            # read C, write A_new (fp32)
        "k_head_mix": ("hbm", logits * 8, "B"),               # read and write one fp32 map
        "k_pv_groupnorm": ("alu", logits * 2 * w.d, "FLOP"),
        # tensor-core forms: write (read) the fp32 map, read q and k (v, write out)
        "k_logits_tc": ("hbm", logits * 4 + w.B * w.H * w.T * w.d * 2 * io_bytes, "B"),
        "k_pv_groupnorm_tc": ("hbm", logits * 4 + w.B * w.H * w.T * w.d * 2 * io_bytes, "B"),
        # the prologue: read k, write the c_q folded-key copies (fp16); read q
        # and k, write the permuted q (fp16) and the 16-entry correction rows
        "k_fold": ("hbm", w.B * w.H * w.T * (w.d * 2 * (1 + w.c_q) + w.d * 2 * 3 + 64), "B"),
        "k_mta_fused": ("tensor", w.algorithmic_flops(), "FLOP"),
        # read the fp16 partial outputs (c_h per output head), write out
        "k_mix_groupnorm": ("hbm", w.B * w.T * w.H * w.d * (2 * w.c_h + io_bytes), "B"),
        # backward: causal products of a map with a [T, d] operand, 2d FLOP per live logit
        "k_causal_mm": ("alu", logits * 2 * w.d, "FLOP"),
        # the same products and dA = dO V^T as 3xTF32 MMAs: read (or write) the
        # fp32 map, read the [T, d] operand, write (or read) an fp32 [T, d] array
        "k_mm_tf32": ("hbm", logits * 4 + w.B * w.H * w.T * w.d * (4 + 4), "B"),
        # read O and dout, write dO (fp32)
        "k_gn_bwd": ("hbm", w.B * w.H * w.T * w.d * (4 + io_bytes + 4), "B"),
        # read dA and P twice, write dC (fp32 maps)
        "k_mix_softmax_bwd": ("hbm", logits * 20, "B"),
        "k_conv_adj": ("alu", logits * 2 * w.c_q * w.c_k, "FLOP"),
        "k_dtheta": ("alu", logits * 2 * w.c_q * w.c_k, "FLOP"),
    }
    return table.get(name, ("unknown", 0, "FLOP"))


def load_traffic():
    """Per-launch DRAM traffic from committed ncu summaries, valid only while
    the kernel source they were taken on is unchanged."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return {}
    out = {}
    for name, rec in table.items():
        src = os.path.join(ROOT, rec.get("source", ""))
        try:
            digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        except OSError:
            continue
        if digest == rec.get("source_sha256_16"):
            out[name] = rec
    return out


def roofline(name, w, avg_ms, peaks, peak_src, comp=None):
    bound, amount, unit = kernel_units(name, w, comp)
    secs = avg_ms / 1e3
    traffic = load_traffic().get(name)
    tr_bytes = None
    if traffic is not None and traffic.get("workload") == w.name:
        tr_bytes = traffic.get("dram_bytes_per_launch")
    if bound == "hbm":
        achieved, peak, u = amount / secs / 1e9, peaks["hbm_gbs"], "GB/s"
        src = peak_src
    elif bound == "tensor":
        achieved, peak, u = amount / secs / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        src = peak_src
    else:
        achieved, peak, u = amount / secs / 1e12, FP32_ALU_TFLOPS, "TFLOP/s"
        src = "derived: 148 SM x 128 FP32 lanes x 2 x 1965 MHz"
    return {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak, "unit": u,
            "frac": achieved / peak, "traffic": tr_bytes, "peak_source": src,
            "algorithmic_per_launch": amount, "algorithmic_unit": unit,
            "avg_launch_ms": avg_ms}


def time_mta(args, w, d, world, device):
    import convolved_logit_attention_b200 as mta
    unfused = args.path == "unfused"
    if args.compose:
        kw = compose_kw(args, d)
        shape = mta.composed_shape(d["q"], *(d[n] for n in WEIGHTS), gn_eps=w.gn_eps,
                                   w_head_pre=kw["w_head_pre"], w_kq_3d=kw["w_kq_3d"])
        comp = mta.composition(*(d[n] for n in WEIGHTS), **kw)
        names = mta.mta_composed_kernel_names(shape, comp)
        nk = len(names)
        fused = "k_mta_fused" in names
        ws_bytes = mta.lib().mta_composed_workspace_size(ctypes.byref(shape), ctypes.byref(comp))
    else:
        shape = mta.shape_of(d["q"], d["w_kq"], d["w_head"], w.gn_eps)
        nk = mta.mta_kernel_count(shape, unfused)
        names = [mta.mta_kernel_name(shape, i, unfused) for i in range(nk)]
        fused = not unfused and mta.mta_forward_path(shape) == mta.MTA_PATH_FUSED_TC
        ws_bytes = (mta.mta_unfused_workspace_size(shape) if unfused
                    else mta.mta_workspace_size(shape))
    path = "fused_tc" if fused else "materialised"
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    out = torch.empty((w.B, w.T, w.H * w.d), dtype=d["q"].dtype, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    gate = torch.linspace(-2.0, 2.0, w.H, dtype=torch.float32, device=device)

    # The timed steps are plain public calls (mta_forward / mta_forward_unfused /
    # mta_forward_gated): events recorded between the kernels would add their
    # own cost to the step.  Traced steps just before and just after the timed
    # region give each kernel's time for the roofline.
    def composed(events=None):
        mta.mta_forward_composed(d["q"], d["k"], d["v"], *(d[n] for n in WEIGHTS),
                                 gn_weight=d["gn_weight"], gn_bias=d["gn_bias"],
                                 depth_scale=w.depth_scale, gate=gate if args.gate else None,
                                 out=out, workspace=ws, stream=stream, gn_eps=w.gn_eps,
                                 events=events, **compose_kw(args, d))

    def step():
        if args.compose:
            composed()
        elif args.gate:
            mta.mta_forward_gated(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                                  d["gn_bias"], gate, out=out, workspace=ws, stream=stream,
                                  gn_eps=w.gn_eps)
        else:
            fn = mta.mta_forward_unfused if unfused else mta.mta_forward
            fn(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"], d["gn_bias"],
               w.depth_scale, out=out, workspace=ws, stream=stream, gn_eps=w.gn_eps)

    def traced_step(events):
        if args.compose:
            composed(events)
            return
        mta.mta_forward_traced(unfused, events, d["q"], d["k"], d["v"], d["w_kq"], d["w_head"],
                               d["gn_weight"], d["gn_bias"], w.depth_scale, out=out,
                               workspace=ws, stream=stream, gn_eps=w.gn_eps)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    mta.mta_sync_status(stream, device)
    # per-kernel breakdown: traced steps bracketing the timed region, half just
    # before it and half just after, so that their average sees the clock and
    # power state the timed steps ran in (the gated call shares the kernels of
    # mta_forward)
    n_tr = min(args.steps, 10)
    kern_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)] for _ in range(n_tr)]
    for s in range(n_tr // 2):
        flush.zero_()
        traced_step(kern_ev[s])
    torch.cuda.synchronize(device)
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(device)
    with sampler:
        for s in range(args.steps):
            flush.zero_()
            step_ev[s][0].record(stream)
            step()
            step_ev[s][1].record(stream)
        torch.cuda.synchronize(device)
    barrier(world)
    mta.mta_sync_status(stream, device)
    total_ms = sum(a.elapsed_time(b) for a, b in step_ev)
    for s in range(n_tr // 2, n_tr):
        flush.zero_()
        traced_step(kern_ev[s])
    torch.cuda.synchronize(device)
    mta.mta_sync_status(stream, device)
    per_kernel = {}          # average ms per launch (a name may launch twice per step)
    for i, name in enumerate(names):
        per_kernel[name] = per_kernel.get(name, 0.0) + sum(
            kern_ev[s][2 * i].elapsed_time(kern_ev[s][2 * i + 1]) for s in range(n_tr)) / n_tr
    for name in per_kernel:
        per_kernel[name] /= names.count(name)
    return {"total_ms": total_ms, "per_kernel_ms": per_kernel, "names": names,
            "launches": nk * args.steps, "clocks": sampler.summary(), "path": path}


def backward_flops(w):
    """Algorithmic FLOPs of the gradients (the forward's recompute excluded):
    per live logit dA = dO V^T and dV = A^T dO (2d each), the mix backward
    and the dw sums (c_h MACs each), the adjoint convolution and the kernel
    gradient (c_q c_k MACs each), dQ and dK (2d each): twice the forward's
    4d + 2 c_q c_k + 2 c_h."""
    return 2 * w.algorithmic_flops()


def time_backward(args, w, x, d, world, device):
    """K timed mta_backward calls (L2 flushed before each), bracketed by traced
    calls for the per-kernel breakdown."""
    import convolved_logit_attention_b200 as mta
    dt = torch.bfloat16 if w.io == "bf16" else torch.float32
    rng = np.random.default_rng(w.seed + 1000)
    dout = torch.from_numpy(rng.standard_normal((w.B, w.T, w.H * w.d)).astype(np.float32))
    dout = dout.to(device).to(dt)
    shape = mta.shape_of(d["q"], d["w_kq"], d["w_head"], w.gn_eps)
    names = mta.mta_backward_kernel_names(shape)
    ws = torch.empty(mta.mta_backward_workspace_size(shape), dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step(events=None):
        mta.mta_backward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                         d["gn_bias"], w.depth_scale, dout, workspace=ws, stream=stream,
                         gn_eps=w.gn_eps, events=events)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    mta.mta_sync_status(stream, device)
    # traced calls bracketing the timed region (one before, the rest after)
    n_tr = min(args.steps, 3)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
           for _ in range(n_tr)]
    flush.zero_()
    step(kev[0])
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(device)
    with sampler:
        for s in range(args.steps):
            flush.zero_()
            ev[s][0].record(stream)
            step()
            ev[s][1].record(stream)
        torch.cuda.synchronize(device)
    barrier(world)
    mta.mta_sync_status(stream, device)
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    for s in range(1, n_tr):
        flush.zero_()
        step(kev[s])
    torch.cuda.synchronize(device)
    per_kernel = {}
    for i, name in enumerate(names):
        per_kernel[name] = per_kernel.get(name, 0.0) + sum(
            kev[s][2 * i].elapsed_time(kev[s][2 * i + 1]) for s in range(n_tr)) / n_tr
    for name in per_kernel:
        per_kernel[name] /= names.count(name)
    return {"total_ms": total_ms, "per_kernel_ms": per_kernel, "names": names,
            "launches": len(names) * args.steps, "clocks": sampler.summary()}


def backward_line(args, w, x, d, world, rank, device):
    peaks, peak_src = load_peaks()
    res = time_backward(args, w, x, d, world, device)
    total_ms = dist_max(res["total_ms"], world, device)
    flops = backward_flops(w)
    value = replica_tflops(world, flops, args.steps, total_ms)
    kernels = res["per_kernel_ms"]
    dom = max(kernels, key=lambda n: kernels[n] * res["names"].count(n))
    rl = roofline(dom, w, kernels[dom], peaks, peak_src)
    line = {"metric": "MTA bwd TFLOP/s at T=4096 (gradient FLOPs, 2x the forward's; the "
                      "forward recompute excluded)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": dict(workload_config(w, "materialised backward"), **{"pass": "backward"}),
            "tokens_per_s": world * w.tokens() * args.steps / (total_ms / 1e3),
            "peaks": dict(peaks, source=peak_src),
            "roofline": {k: rl[k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                             "traffic")},
            "kernels": [dict(roofline(n, w, kernels[n], peaks, peak_src),
                             launches_per_step=res["names"].count(n))
                        for n in dict.fromkeys(res["names"])],
            "gpu_launches": res["launches"], "clocks": res["clocks"]}
    return line if rank == 0 else None


def time_e2e(args, w, x, device):
    """The public API with host buffers: every step copies all of its inputs
    from pinned host memory to the device, calls mta_forward and copies the
    output back to pinned host memory.  Steps are pipelined the way a serving
    loop would drive the library: two device buffer sets, with step s+1's
    input copy (copy-in stream) overlapping step s's compute (compute stream)
    and step s-1's output copy (copy-out stream).  The time runs from the
    first input copy of the timed steps to the end of their last output copy."""
    import convolved_logit_attention_b200 as mta
    dt = torch.bfloat16 if w.io == "bf16" else torch.float32
    names = tuple(n for n in ("q", "k", "v") + WEIGHTS + ("w_head_pre", "w_kq_3d", "gn_weight",
                                                         "gn_bias")
                  if x.get(n) is not None)
    host = {n: torch.from_numpy(x[n]).to(dt).pin_memory() for n in ("q", "k", "v")}
    for n in names[3:]:
        host[n] = torch.from_numpy(x[n]).pin_memory()
    nbuf = 2
    dev = [{n: torch.empty_like(host[n], device=device) for n in names} for _ in range(nbuf)]
    out = [torch.empty((w.B, w.T, w.H * w.d), dtype=dt, device=device) for _ in range(nbuf)]
    out_host = [torch.empty(out[0].shape, dtype=dt).pin_memory() for _ in range(nbuf)]
    if args.compose:
        wts = [dev[0].get(n) for n in WEIGHTS]
        kw = compose_kw(args, dev[0])
        shape = mta.composed_shape(dev[0]["q"], *wts, gn_eps=w.gn_eps, w_head_pre=kw["w_head_pre"],
                                   w_kq_3d=kw["w_kq_3d"])
        ws_bytes = mta.lib().mta_composed_workspace_size(
            ctypes.byref(shape), ctypes.byref(mta.composition(*wts, **kw)))
    else:
        shape = mta.shape_of(dev[0]["q"], dev[0]["w_kq"], dev[0]["w_head"], w.gn_eps)
        ws_bytes = mta.mta_workspace_size(shape)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out[0].numel() * out[0].element_size()

    def run(n_steps, first=None, last=None):
        copied = [None] * n_steps
        computed = [None] * n_steps
        drained = [None] * n_steps
        for st in range(n_steps):
            bi = st % nbuf
            with torch.cuda.stream(s_in):
                if st >= nbuf:
                    s_in.wait_event(computed[st - nbuf])      # buffer set free again
                if st == 0 and first is not None:
                    first.record(s_in)
                for n in names:
                    dev[bi][n].copy_(host[n], non_blocking=True)
                copied[st] = torch.cuda.Event()
                copied[st].record(s_in)
            s_comp.wait_event(copied[st])
            if st >= nbuf:
                s_comp.wait_event(drained[st - nbuf])         # output buffer read back
            d = dev[bi]
            if args.compose:
                mta.mta_forward_composed(d["q"], d["k"], d["v"], *(d.get(n) for n in WEIGHTS),
                                         gn_weight=d["gn_weight"], gn_bias=d["gn_bias"],
                                         depth_scale=w.depth_scale, out=out[bi], workspace=ws,
                                         stream=s_comp, gn_eps=w.gn_eps, **compose_kw(args, d))
            else:
                mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                                d["gn_bias"], w.depth_scale, out=out[bi], workspace=ws,
                                stream=s_comp, gn_eps=w.gn_eps)
            computed[st] = torch.cuda.Event()
            computed[st].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[st])
                out_host[bi].copy_(out[bi], non_blocking=True)
                drained[st] = torch.cuda.Event()
                drained[st].record(s_out)
        if last is not None:
            s_out.wait_event(drained[n_steps - 1])
            last.record(s_out)

    run(max(1, args.warmup))
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(args.steps, t0, t1)
    torch.cuda.synchronize(device)
    mta.mta_sync_status(s_comp, device)
    return t0.elapsed_time(t1), h2d, d2h


def oracle_sample(w, x, n_units, flops_per_step):
    """The first n_units (batch, head-group) units of the workload at full T,
    as separate B=1, H=c_h problems (dicts of arrays; weights a composition
    leaves out stay None), with their algorithmic FLOPs."""
    def part(name, sl):
        return x[name][sl] if x.get(name) is not None else None
    units = []
    for u in range(min(n_units, w.B * w.G)):
        b, g = divmod(u, w.G)
        hs = slice(g * w.c_h, (g + 1) * w.c_h)
        cs = slice(g * w.c_h * w.d, (g + 1) * w.c_h * w.d)
        gs = slice(g, g + 1)
        units.append({"q": x["q"][b:b + 1, hs], "k": x["k"][b:b + 1, hs],
                      "v": x["v"][b:b + 1, hs], "w_kq": part("w_kq", hs),
                      "w_head_pre": part("w_head_pre", gs), "w_head": part("w_head", gs),
                      "w_kq_post": part("w_kq_post", hs), "w_head_post": part("w_head_post", gs),
                      "w_kq_3d": part("w_kq_3d", gs),
                      "gn_weight": x["gn_weight"][cs], "gn_bias": x["gn_bias"][cs],
                      "exact_mask": bool(x.get("exact_mask"))})
    flops = len(units) * flops_per_step // (w.B * w.G)
    return units, flops


def run_oracle_unit(u, w, nthreads=1):
    import oracle
    default = (u["w_kq"] is not None and u["w_head"] is not None and u["w_head_pre"] is None
               and u["w_kq_post"] is None and u["w_head_post"] is None and not u["exact_mask"]
               and u["w_kq_3d"] is None)
    if default:
        return oracle.forward(u["q"], u["k"], u["v"], u["w_kq"], u["w_head"], u["gn_weight"],
                              u["gn_bias"], w.depth_scale, gn_eps=w.gn_eps, nthreads=nthreads)
    return oracle.forward_composed(u["q"], u["k"], u["v"], u["w_kq"], u["w_head"], u["w_kq_post"],
                                   u["w_head_post"], u["gn_weight"], u["gn_bias"], w.depth_scale,
                                   gn_eps=w.gn_eps, nthreads=nthreads,
                                   w_head_pre=u["w_head_pre"], exact_mask=u["exact_mask"],
                                   w_kq_3d=u["w_kq_3d"])


def run_oracle_units(units, w, nthreads):
    """Runs the oracle forward on every unit, one unit per host thread (the
    ctypes call releases the GIL); returns the wall time in seconds."""
    import concurrent.futures as cf

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=nthreads) as ex:
        list(ex.map(lambda u: run_oracle_unit(u, w), units))
    return time.perf_counter() - t0


def cpu_baseline(w, x, flops_per_step):
    cores = os.cpu_count() or 1
    n_units = min(cores, w.B * w.G)
    units, flops = oracle_sample(w, x, n_units, flops_per_step)
    secs = run_oracle_units(units, w, n_units)
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": n_units, "kind": "oracle",
            "seconds": secs,
            "sample": "%d of %d (batch, head-group) units of %s at full T=%d, one unit per "
                      "host thread" % (len(units), w.B * w.G, w.name, w.T)}


def reference_arm(args, w, world, rank):
    """The fp64 oracle on the host cores, timed like a step: each step is a
    bounded sample (one unit per host thread, full T) of the workload."""
    if rank != 0:
        return None
    x = composed_inputs(w, args.compose) if args.compose else make_inputs(w)
    cores = os.cpu_count() or 1
    n_units = min(cores, w.B * w.G)
    units, flops = oracle_sample(w, x, n_units, step_flops(args, w))
    for _ in range(args.warmup):
        run_oracle_units(units[:1], w, 1)
    total = sum(run_oracle_units(units, w, n_units) for _ in range(args.steps))
    value = flops * args.steps / total / 1e12
    sample = ("%d of %d (batch, head-group) units of %s at full T=%d per step, one unit per host "
              "thread" % (len(units), w.B * w.G, w.name, w.T))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(w, "oracle (host)"),
                           composition=args.compose or "default"),
            "tokens_per_s": n_units * w.T * args.steps / total,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": n_units, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def workload_config(w, path):
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "c_q": w.c_q,
            "c_k": w.c_k, "c_h": w.c_h, "io": w.io, "path": path,
            "l2": "flushed before every timed step (256 MiB write, untimed)",
            "parallelism": "independent replicas, one per GPU"}


def mta_arm(args, w, world, rank, local):
    device = torch.device("cuda", local)
    from convolved_logit_attention_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier(world)
    x = (composed_inputs(w, args.compose, seed=w.seed + rank) if args.compose
         else make_inputs(w, seed=w.seed + rank))
    d = device_inputs(x, w.io, device)
    if args.backward:
        return backward_line(args, w, x, d, world, rank, device)
    peaks, peak_src = load_peaks()
    res = time_mta(args, w, d, world, device)
    bad = [r for r in res["clocks"]["reasons"] if r in BAD_REASONS]
    if bad:   # one re-measurement after a throttled run
        res = time_mta(args, w, d, world, device)
    total_ms = dist_max(res["total_ms"], world, device)
    per_step_ms = total_ms / args.steps
    flops = step_flops(args, w)
    value = replica_tflops(world, flops, args.steps, total_ms)
    kernels = dict(res["per_kernel_ms"])   # average ms per launch, traced pass
    # the dominant kernel by device time per step (a name may launch twice)
    dom = max(kernels, key=lambda n: kernels[n] * res["names"].count(n))
    comp = dict(COMPOSITIONS[args.compose], c_h=w.c_h) if args.compose else None
    rl = roofline(dom, w, kernels[dom], peaks, peak_src, comp)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if (w.io == "bf16" and res["path"] == "fused_tc") else "f32",
            "data": "synthetic",
            "config": dict(workload_config(w, res["path"]),
                           output_scale="sigmoid gate" if args.gate else "depth scale",
                           composition=args.compose or "default"),
            "tokens_per_s": world * w.tokens() * args.steps / (total_ms / 1e3),
            "pct_of_bf16_peak": 100.0 * value / world / peaks["bf16_tflops"],
            "peaks": dict(peaks, source=peak_src),
            "roofline": {k: rl[k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                             "traffic")},
            "roofline_detail": rl,
            "kernels": [dict(roofline(n, w, kernels[n], peaks, peak_src, comp),
                             launches_per_step=res["names"].count(n))
                        for n in dict.fromkeys(res["names"])],
            "gpu_launches": res["launches"], "clocks": res["clocks"]}
    if not args.no_e2e and not args.gate:     # e2e follows --compose when given
        e2e_ms, h2d, d2h = time_e2e(args, w, x, device)
        e2e_ms = dist_max(e2e_ms, world, device)
        line["e2e"] = {"value": world * flops * args.steps / (e2e_ms / 1e3) / 1e12,
                       "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e2e_ms / args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, x, flops)
    return line if rank == 0 else None


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_setup(args)
    w = WORKLOADS[args.workload]
    if args.batch is not None:
        from dataclasses import replace
        w = replace(w, B=args.batch, name="%s_b%d" % (w.name, args.batch))
    try:
        if args.impl == "reference":
            line = reference_arm(args, w, world, rank)
        else:
            line = mta_arm(args, w, world, rank, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
