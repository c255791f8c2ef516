#!/usr/bin/env python3
"""Benchmark of the depthwise conv2d hot path (forward + input gradient).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mobilenet|large|conformer|tiny]

One step = forward and input gradient of every shape of the workload (the
default is the MobileNet-style NHWC set: 1x112x112x32 3x3 SAME, 1x56x56x128
5x5 SAME, 32x56x56x144 3x3 stride 2 pad 1).  Inputs are seeded synthetic
tensors resident in HBM and rotated over enough buffer sets that every step
reads data that is not in L2.  Steps are replayed from CUDA graphs of the
C-ABI calls and timed with CUDA events on the launching stream; with N > 1
ranks (torchrun) every rank runs its own replica (no data-path collective:
every (n, c) slice of a depthwise convolution is independent) and the time is
the max over ranks.

Prints one JSON line (rank 0).  `value` is achieved HBM throughput in GB/s:
algorithmic bytes of all ranks' steps (every input element read once, every
output element written once, plus filters and bias) divided by the time.
`--impl reference` times the float64 CPU oracle instead, on the same metric,
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "depthwise conv fwd+bwd_input µs/call and achieved HBM GB/s (% of B200 roofline)"
FALLBACK_HBM_GBS = 6650.0
L2_FALLBACK = 126 * 1024 * 1024


# ------------------------------------------------------------------ helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_cases(name):
    from depthwise_convolution_fwd_b200 import workloads as wl
    if name == "mobilenet":
        return wl.mobilenet(), ("MobileNet-style NHWC f32: 1x112x112x32 3x3 SAME, 1x56x56x128 "
                                "5x5 SAME, 32x56x56x144 3x3 stride 2 pad 1")
    if name == "large":
        return [c for c in wl.large() if c.H == 512], \
            "Large bandwidth case: 1x512x512x256 3x3 SAME, NHWC and NCHW f32"
    if name == "conformer":
        return [c for c in wl.conformer() if c.W == 512], \
            "Conformer-style 1-D: 16x1x512x512 1x31 SAME, NHWC and NCHW f32"
    if name == "tiny":
        return wl.tiny(), "Tiny: 1x8x8x4 3x3 SAME NHWC f32"
    if name == "multiplier":
        return [c for c in wl.multiplier() if c.H == 512], \
            "Channel multiplier 2: 1x512x512x128 -> 256 channels 3x3 SAME, NHWC and NCHW f32"
    raise ValueError(name)


def algorithmic_bytes(case, Ho, Wo, op, esz=4):
    """Bytes one call must move at minimum: read the input once, write the
    output once, read the filters (and the bias for the forward); esz is the
    activation element size (4 for float32, 2 for float16 / bfloat16)."""
    Co = case.C * case.multiplier  # output channels
    n_in = case.N * case.C * case.H * case.W
    n_out = case.N * Co * Ho * Wo
    wbytes = Co * case.kH * case.kW * (2 if case.wtype == "f16" else 4)
    if op == "fwd":
        return esz * (n_in + n_out) + wbytes + (4 * Co if case.bias else 0)
    if op == "fused":  # forward + four [Co] batch-norm statistics
        return esz * (n_in + n_out) + wbytes + (4 * Co if case.bias else 0) + 16 * Co
    if op == "wgrad":  # read x and dy, write dW [Co,kH,kW] and db [Co] (f32)
        return esz * (n_in + n_out) + 4 * Co * case.kH * case.kW + 4 * Co
    return esz * (n_out + n_in) + wbytes


# the sources the NHWC tiled kernels (the MobileNet step's dominant launches)
# are compiled from: a change to any of them voids the committed counters
DIGEST_FILES = ("dw_common.cuh", "dw_tiled_nhwc.cuh", "dw_tiled_nhwc.cu", "dw_tiled_nhwc_bwd.cu")


def src_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "depthwise_convolution_fwd_b200", "csrc")
    for fn in DIGEST_FILES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return {}
    if d.get("src_digest") != src_digest():
        return {}
    return d.get("kernels", {})


def reduce_max(value, device):
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, bytes_per_step, steps, ms):
    """Algorithmic bytes of every rank's steps over the (max-over-ranks) time."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.nv = None
            self.error = repr(e)

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:  # noqa: BLE001
            bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in self.REASONS.items():
            if bits & bit and bit != 0x1:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def start(self):
        if self.nv:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        self._thread.join()
        self._sample()
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(self.reasons)}


# --------------------------------------------------------------- GPU arm --

class Shape:
    """One workload shape with its buffer sets and prepared C-ABI calls."""

    def __init__(self, case, dw, torch, device, sets, atype="f32"):
        from depthwise_convolution_fwd_b200.workloads import make_inputs
        self.case = case
        desc = dw.make_desc(case.N, case.H, case.W, case.C, case.kH, case.kW,
                            stride=case.stride, dilation=case.dilation, padding=case.padding,
                            layout=case.layout, wtype=case.wtype, multiplier=case.multiplier,
                            atype=atype)
        self.desc = desc
        self.Ho, self.Wo = dw.dwconv2d_out_shape(desc)
        dt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[atype]
        self.esz = 4 if atype == "f32" else 2
        host = make_inputs(case, (self.Ho, self.Wo))
        host["x"], host["dy"] = host["x"].to(dt), host["dy"].to(dt)
        self.host = host
        self.bytes = {op: algorithmic_bytes(case, self.Ho, self.Wo, op, self.esz)
                      for op in ("fwd", "bwd")}
        self.w = self.host["w"].to(device)
        self.b = None if self.host["b"] is None else self.host["b"].to(device)
        out_shape = case.out_shape(self.Ho, self.Wo)
        self.sets = []
        for _ in range(sets):
            self.sets.append({
                "x": self.host["x"].to(device), "dy": self.host["dy"].to(device),
                "y": torch.empty(out_shape, device=device, dtype=dt),
                "dx": torch.empty(case.in_shape(), device=device, dtype=dt)})
        self.set_bytes = sum(t.numel() * t.element_size() for t in self.sets[0].values())

    def prepare_next_rows(self, dw, torch, device, act):
        """Buffers of the calls measured beside the step: the weight gradient
        and the forward with the fused batch-norm / activation epilogue."""
        from depthwise_convolution_fwd_b200.workloads import make_bn
        c = self.case
        self.act = act
        self.bn = [t.to(device) for t in make_bn(c.Co, c.seed + 500)[:4]]
        self.ws_bytes = dw.dwconv2d_bwd_weight_workspace_size(self.desc)
        self.ws = torch.empty(max(1, self.ws_bytes), dtype=torch.uint8, device=device)
        self.dW = torch.empty(c.Co * c.kH * c.kW, device=device)
        self.db = torch.empty(c.Co, device=device)
        for op in ("fused", "wgrad"):
            self.bytes[op] = algorithmic_bytes(c, self.Ho, self.Wo, op, self.esz)

    def call(self, dw, op, r, stream):
        s = self.sets[r % len(self.sets)]
        if op == "fused":
            acts = {"relu": dw.DW_ACT_RELU, "relu6": dw.DW_ACT_RELU6, "silu": dw.DW_ACT_SILU}
            st = dw.fwd_bn_act_raw(self.desc, s["x"].data_ptr(), self.w.data_ptr(),
                                   None if self.b is None else self.b.data_ptr(),
                                   [t.data_ptr() for t in self.bn], 1e-5, acts[self.act],
                                   s["y"].data_ptr(), stream)
        elif op == "wgrad":
            st = dw.bwd_weight_raw(self.desc, s["x"].data_ptr(), s["dy"].data_ptr(),
                                   self.dW.data_ptr(), self.db.data_ptr(), self.ws.data_ptr(),
                                   self.ws_bytes, stream)
        elif op == "fwd":
            st = dw.fwd_raw(self.desc, s["x"].data_ptr(), self.w.data_ptr(),
                            None if self.b is None else self.b.data_ptr(), s["y"].data_ptr(), stream)
        else:
            st = dw.bwd_input_raw(self.desc, s["dy"].data_ptr(), self.w.data_ptr(),
                                  s["dx"].data_ptr(), stream)
        if st != dw.DW_OK:
            raise dw.DwError(st, f"{self.case.name} {op}")


def time_graph(torch, graph, reps, stream):
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        graph.replay()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(reps):
            graph.replay()
        end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import depthwise_convolution_fwd_b200 as dw
    from depthwise_convolution_fwd_b200 import build as dwbuild

    dwbuild.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 0) or L2_FALLBACK
    cases, workload_desc = workload_cases(args.workload)

    # enough buffer sets that a set is evicted from L2 before it is reused
    probe = [Shape(c, dw, torch, device, 1) for c in cases]
    per_set = sum(s.set_bytes for s in probe)
    sets = max(2, -(-int(2.2 * l2) // per_set) + 1)
    del probe
    shapes = [Shape(c, dw, torch, device, sets) for c in cases]
    ops = [(sh, op) for sh in shapes for op in ("fwd", "bwd")]
    step_bytes = sum(sh.bytes[op] for sh, op in ops)

    stream = torch.cuda.Stream(device)
    sptr = stream.cuda_stream
    # one eager pass per shape/op sets per-kernel attributes outside capture
    with torch.cuda.stream(stream):
        for sh, op in ops:
            sh.call(dw, op, 0, sptr)
    torch.cuda.synchronize()

    graphs = []
    for r in range(sets):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for sh, op in ops:
                sh.call(dw, op, r, stream.cuda_stream)
        graphs.append(g)

    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            graphs[k % sets].replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    with torch.cuda.stream(stream):
        start.record(stream)
        for k in range(args.steps):
            graphs[k % sets].replay()
        end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms = reduce_max(start.elapsed_time(end), device)
    ms_per_step = ms / args.steps
    value = whole_job_gbs(world, step_bytes, args.steps, ms)

    # per-kernel launch durations: a CUDA graph of back-to-back launches of
    # one kernel over enough buffer copies that its inputs come from HBM
    kernels = {}
    for sh, op in ops:
        kernels[f"{sh.case.name}:{op}"] = time_kernel(torch, dw, sh, op, l2, stream)
    total_us = sum(v["us"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = v["us"] / total_us
    dom_key = max(kernels, key=lambda k: kernels[k]["us"])
    dom = kernels[dom_key]
    peak, peak_kind = load_peaks()
    traffic = load_traffic(args.workload).get(dom_key)

    # the rows measured beside the step (not part of it): weight gradient, and
    # the forward with the fused batch-norm + activation epilogue
    next_rows = {}
    if not args.no_next_rows:
        act = "silu" if args.workload == "conformer" else "relu6"
        for sh in shapes:
            sh.prepare_next_rows(dw, torch, device, act)
            with torch.cuda.stream(stream):
                for op in ("fused", "wgrad"):
                    sh.call(dw, op, 0, sptr)
            torch.cuda.synchronize()
            for op in ("fused", "wgrad"):
                k = time_kernel(torch, dw, sh, op, l2, stream)
                k["frac"] = k["gbs"] / peak
                if op == "fused":
                    k["epilogue"] = f"inference batch norm + {act}"
                next_rows[f"{sh.case.name}:{op}"] = k
        # 16-bit activations: the same calls moving half the bytes
        for c in cases:
            for at in ("f16", "bf16"):
                sh16 = Shape(c, dw, torch, device, 1, atype=at)
                sh16.prepare_next_rows(dw, torch, device, act)
                with torch.cuda.stream(stream):
                    for op in ("fwd", "bwd", "wgrad"):
                        sh16.call(dw, op, 0, sptr)
                torch.cuda.synchronize()
                for op in ("fwd", "bwd", "wgrad"):
                    k = time_kernel(torch, dw, sh16, op, l2, stream)
                    k["frac"] = k["gbs"] / peak
                    next_rows[f"{c.name}:{op}_{at}"] = k
                del sh16

    # end to end through the public tensor API: pinned host inputs -> device,
    # forward + input gradient, outputs -> pinned host, every step
    e2e = run_e2e(args, torch, dw, shapes, device, stream, world)

    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded U(-1,1) activations, N(0,1/(kH*kW)) filters, U(-0.1,0.1) bias)",
        "config": {"workload": workload_desc, "global_batch": sum(c.N for c in cases) * world,
                   "layouts": sorted({c.layout for c in cases}),
                   "step": "forward + input gradient of every shape (" + str(len(ops)) + " launches)",
                   "l2": f"inputs larger than L2: rotated over {sets} buffer sets "
                         f"({sets * per_set / 1e6:.0f} MB vs L2 {l2 / 1e6:.0f} MB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "timing": "CUDA events around CUDA-graph replays on the launching stream"},
        "us_per_call": {"step_fwd_plus_bwd_input": ms_per_step * 1e3,
                        **{k: v["us"] for k, v in kernels.items()}},
        "roofline": {"bound": "hbm", "kernel": dom_key, "achieved": dom["gbs"], "peak": peak,
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS hbm_gbs, copy read+write)"
                     if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "unit": "GB/s", "frac": dom["gbs"] / peak,
                     "traffic": traffic,
                     "timing": "avg launch of a CUDA graph of back-to-back launches, inputs "
                               "rotated over buffer copies > 3x L2, CUDA events"},
        "kernels": kernels,
        "next_rows": next_rows,
        "e2e": e2e,
        "gpu_launches": len(ops) * args.steps,
        "clocks": clocks,
        "achieved_step_frac_of_peak": value / world / peak,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cases, budget_s=args.cpu_budget)
    for g in graphs:
        del g
    return result


def time_kernel(torch, dw, sh, op, l2, stream):
    """Average launch time of one call: a CUDA graph of back-to-back launches
    over enough buffer copies (> 3x L2) that its inputs come from HBM."""
    per = sh.bytes[op]
    reuse = max(len(sh.sets), -(-int(3 * l2) // max(1, per)))
    extra = []
    if reuse > len(sh.sets):
        for _ in range(reuse - len(sh.sets)):
            extra.append({k: torch.empty_like(v).copy_(v) for k, v in sh.sets[0].items()})
    pool = sh.sets + extra
    saved = sh.sets
    sh.sets = pool
    launches = len(pool)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for r in range(launches):
            sh.call(dw, op, r, stream.cuda_stream)
    reps = max(3, int(60e-3 / max(1e-6, per / 6e12) / launches))
    ms_k = time_graph(torch, g, reps, stream) / (reps * launches)
    sh.sets = saved
    del g, extra, pool
    return {"us": ms_k * 1e3, "bytes": per, "gbs": per / (ms_k * 1e-3) / 1e9}


def run_e2e(args, torch, dw, shapes, device, stream, world):
    """Whole-job throughput through the public tensor API with host buffers:
    every step copies its inputs from pinned host memory, runs the forward and
    the input gradient of every shape, and copies both results back.  Steps
    are pipelined two deep on three streams (host-to-device copies, compute,
    device-to-host copies), so one step's uploads overlap the previous step's
    downloads (PCIe is full duplex); each step still moves all of its bytes."""
    steps = max(1, min(args.steps, args.e2e_steps))
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    slots = 2
    jobs = []
    h2d = d2h = 0
    for sh in shapes:
        c = sh.case
        host = {k: (None if v is None else v.pin_memory()) for k, v in sh.host.items() if k != "w32"}
        dev = [{k: (None if v is None else torch.empty_like(v, device=device)) for k, v in host.items()}
               for _ in range(slots)]
        res = [{"y": torch.empty(c.out_shape(sh.Ho, sh.Wo), device=device, dtype=host["x"].dtype),
                "dx": torch.empty(c.in_shape(), device=device, dtype=host["x"].dtype)}
               for _ in range(slots)]
        outs = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in r.items()} for r in res]
        jobs.append((c, host, dev, res, outs))
        h2d += sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        d2h += sum(v.numel() * v.element_size() for v in res[0].values())
    ev = {n: [torch.cuda.Event() for _ in range(slots)] for n in ("in", "cmp", "out")}
    used = [False] * slots

    def step(k):
        j = k % slots
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(ev["cmp"][j])  # slot j's inputs are free again
            for c, host, dev, res, outs in jobs:
                for key, v in host.items():
                    if v is not None:
                        dev[j][key].copy_(v, non_blocking=True)
            ev["in"][j].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev["in"][j])
            if used[j]:
                s_cmp.wait_event(ev["out"][j])  # slot j's results were copied out
            for c, host, dev, res, outs in jobs:
                d = dev[j]
                dw.dwconv2d_fwd(d["x"], d["w"], d["b"], stride=c.stride, dilation=c.dilation,
                                padding=c.padding, layout=c.layout, out=res[j]["y"])
                dw.dwconv2d_bwd_input(d["dy"], d["w"], (c.H, c.W), stride=c.stride,
                                      dilation=c.dilation, padding=c.padding, layout=c.layout,
                                      multiplier=c.multiplier, out=res[j]["dx"])
            ev["cmp"][j].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["cmp"][j])
            for c, host, dev, res, outs in jobs:
                outs[j]["y"].copy_(res[j]["y"], non_blocking=True)
                outs[j]["dx"].copy_(res[j]["dx"], non_blocking=True)
            ev["out"][j].record(s_out)
        used[j] = True

    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    s_cmp.wait_event(start)
    s_out.wait_event(start)
    for k in range(steps):
        step(k)
    end.record(s_out)  # the last download depends on every earlier operation
    torch.cuda.synchronize()
    ms = reduce_max(start.elapsed_time(end), device)
    step_bytes = sum(sh.bytes["fwd"] + sh.bytes["bwd"] for sh in shapes)
    return {"value": whole_job_gbs(world, step_bytes, steps, ms), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / steps, "steps": steps, "pipelined": "2 steps in flight",
            "api": "depthwise_convolution_fwd_b200.dwconv2d_fwd / dwconv2d_bwd_input"}


def run_profile(args, local_rank):
    """Launch one kernel of the workload `--steps` times (no timing, no other
    kernels), so a profiler capture sees only that kernel."""
    import torch

    import depthwise_convolution_fwd_b200 as dw
    from depthwise_convolution_fwd_b200 import build as dwbuild
    dwbuild.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    # SHAPE:OP with OP fwd, bwd, fused or wgrad, optionally suffixed _f16 / _bf16
    name, op = args.profile.split(":")
    op, _, atype = op.partition("_")
    cases, _ = workload_cases(args.workload)
    match = [c for c in cases if c.name == name]
    if not match or op not in ("fwd", "bwd", "fused", "wgrad") or atype not in ("", "f16", "bf16"):
        raise SystemExit(f"unknown kernel {args.profile!r}; shapes: {[c.name for c in cases]}")
    sh = Shape(match[0], dw, torch, device, 1, atype=atype or "f32")
    if op in ("fused", "wgrad"):
        sh.prepare_next_rows(dw, torch, device, "silu" if args.workload == "conformer" else "relu6")
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            sh.call(dw, op, 0, stream.cuda_stream)
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "launches": args.steps,
                      "algo": dw.dwconv2d_query_algo(sh.desc, {"fwd": 0, "fused": 0, "bwd": 1,
                                                              "wgrad": 2}[op],
                                                     sh.sets[0]["x"].data_ptr(), sh.w.data_ptr(),
                                                     sh.sets[0]["y"].data_ptr())}), flush=True)
    return 0


# --------------------------------------------------------------- CPU arms --

def oracle_step(cases, fraction, oracle, np, torch):
    """Prepare one oracle pass over a channel slice of every shape (channels
    are independent, so a slice is an exact share of the work)."""
    from depthwise_convolution_fwd_b200.workloads import make_inputs
    jobs = []
    total_bytes = 0
    for c in cases:
        M = c.multiplier
        p = oracle.problem(c.in_shape(), c.kH, c.kW, c.stride, c.dilation, c.padding, c.layout,
                           multiplier=M)
        o = oracle.out_shape(p)
        Ho, Wo = (o[1], o[2]) if c.layout == "nhwc" else (o[2], o[3])
        inp = make_inputs(c, (Ho, Wo))
        keep = max(1, int(round(c.C * fraction)))
        cax = 3 if c.layout == "nhwc" else 1
        sl = [slice(None)] * 4
        sl[cax] = slice(0, keep)
        x = np.ascontiguousarray(inp["x"].numpy()[tuple(sl)], dtype=np.float64)
        sl[cax] = slice(0, keep * M)  # the kept input channels' output channels
        dy = np.ascontiguousarray(inp["dy"].numpy()[tuple(sl)], dtype=np.float64)
        w = np.ascontiguousarray(inp["w32"].numpy()[:keep * M], dtype=np.float64)
        b = None if inp["b"] is None else np.ascontiguousarray(inp["b"].numpy()[:keep * M],
                                                               dtype=np.float64)
        shape = list(c.in_shape())
        shape[cax] = keep
        ps = oracle.problem(tuple(shape), c.kH, c.kW, c.stride, c.dilation, c.padding, c.layout,
                            multiplier=M)
        sub = c.with_(C=keep)
        total_bytes += algorithmic_bytes(sub, Ho, Wo, "fwd") + algorithmic_bytes(sub, Ho, Wo, "bwd")
        jobs.append((ps, x, w, b, dy))
    return jobs, total_bytes


def run_oracle_jobs(jobs, oracle):
    for ps, x, w, b, dy in jobs:
        oracle.fwd(ps, x, w, b)
        oracle.bwd_input(ps, dy, w)


def cpu_baseline(cases, budget_s=8.0):
    import numpy as np
    import torch

    import oracle
    oracle.build()
    jobs, nbytes = oracle_step(cases, 1.0, oracle, np, torch)
    t0 = time.perf_counter()
    run_oracle_jobs(jobs, oracle)
    one = time.perf_counter() - t0
    reps = max(1, int(budget_s / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        run_oracle_jobs(jobs, oracle)
    dt = time.perf_counter() - t0
    return {"value": reps * nbytes / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{reps} full passes (forward + input gradient of every shape), "
                      f"{dt:.1f} s wall; float64 C oracle, OpenMP over (n, c)"}


def run_reference(args, rank, world):
    import numpy as np
    import torch

    import oracle
    oracle.build()
    cases, workload_desc = workload_cases(args.workload)
    jobs, nbytes = oracle_step(cases, 1.0, oracle, np, torch)
    t0 = time.perf_counter()
    run_oracle_jobs(jobs, oracle)
    full = time.perf_counter() - t0
    # bounded sample: the whole K + W run fits the time budget
    frac = min(1.0, args.ref_budget / max(1e-9, full * (args.steps + args.warmup)))
    if frac < 1.0:
        jobs, nbytes = oracle_step(cases, frac, oracle, np, torch)
    for _ in range(args.warmup):
        run_oracle_jobs(jobs, oracle)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_jobs(jobs, oracle)
    dt = time.perf_counter() - t0
    value = nbytes * args.steps / dt / 1e9
    sample = (f"channel fraction {frac:.4f} of every shape per step" if frac < 1.0
              else "the whole workload per step")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload_desc},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# -------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["mobilenet", "large", "conformer", "tiny", "multiplier"],
                    default="mobilenet")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=8.0)
    ap.add_argument("--ref-budget", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the weight-gradient and fused-epilogue measurements")
    ap.add_argument("--profile", metavar="SHAPE:OP", default=None,
                    help="launch only this kernel (e.g. mobilenet_32x56x56x144_3x3_s2:fwd) "
                         "--steps times on one buffer set, untimed; for ncu captures")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.profile:
        return run_profile(args, local_rank)

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        result = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
