#!/usr/bin/env python
"""Benchmark of S2-Attn forward + backward on B200 GPUs (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: s2attn_forward (one
kernel) then s2attn_backward (preprocess, dK/dV, dQ kernels), through the C ABI.
The headline is effective fwd+bwd TFLOP/s, FLOPs counted as
4*B*H*N*G*D/2 forward and 2.5x that backward.  Rank 0 prints one JSON line.

Under torchrun (N > 1) every rank runs the same workload on its own batch
(weak scaling, no collective on the data path); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference there is) on a
bounded sample of the same workload, on this machine's host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_attention_attn_b200 import inputs as I  # noqa: E402

METRIC = "S2-Attn fwd+bwd TFLOP/s & tokens/s on 1 B200; % of BF16 tensor peak"
KERNEL_NAMES = {0: "s2_fwd_kernel", 1: "s2_bwd_pre_kernel", 2: "s2_bwd_dkdv_kernel", 3: "s2_bwd_dq_kernel",
                4: "s2_bwd_fused_kernel", 5: "s2_bwd_dq_post_kernel", 6: "s2_rope_apply_kernel",
                7: "s2_nf4_qkv_kernel", 8: "s2_nf4_dequant_kernel", 9: "s2_bwd_dq_ds_kernel"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def effective_flops(s: I.Shape):
    fwd = 4.0 * s.B * s.H * s.N * s.G * s.D * 0.5
    return fwd, 2.5 * fwd


def kernel_algorithmic(s: I.Shape, fused: bool = False):
    """Algorithmic work of each kernel per step (per launch where the kernel
    launches once a step, as every kernel does at the LLaMA2-7B shape).  The UMMA kernels are
    credited the GEMMs they must issue on the causal half of every group
    (2*B*H*N*G*D/2 FLOPs per GEMM): forward 2 (S, O); split backward dK/dV 4
    (S, dP, dV, dK) and dQ 3 (S, dP, dQ); fused backward 5 (S, dP, dV, dK, dQ).
    The preprocess moves bytes: O and dO read, Delta and lse*log2(e) written,
    lse read, and on the fused path the fp32 dq accumulator zeroed; the dq
    conversion reads the accumulator and writes bf16 dq.  On the split-dS path
    the dQ GEMM (one GEMM-unit, 0.04 ms of tensor work at the LLaMA2-7B shape)
    is bound by its bytes: the dS blocks read (B H (N/G) T (T+1)/2 blocks of
    128 x 128 bf16, T = G/128), K read once and bf16 dq written."""
    gemm = 2.0 * s.B * s.H * s.N * s.G * s.D * 0.5
    rows = s.B * s.H * s.N
    acc = rows * s.D * 4.0
    T = s.G // 128
    ds_bytes = s.B * s.H * (s.N // s.G) * (T * (T + 1) // 2) * 128 * 128 * 2.0
    return {0: ("tensor", 2 * gemm), 2: ("tensor", 4 * gemm), 3: ("tensor", 3 * gemm), 4: ("tensor", 5 * gemm),
            1: ("hbm", 2.0 * rows * s.D * 2 + rows * 4 * 3 + (acc if fused else 0.0)),
            5: ("hbm", acc + rows * s.D * 2.0),
            9: ("hbm", ds_bytes + s.B * s.N * s.Hkv * s.D * 2.0 + rows * s.D * 2.0)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_digest(names, csrc: str):
    """sha256 over the code of the named sources with comments and whitespace
    removed, so a record stays valid across comment-only edits."""
    import re
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(csrc, name)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(name.encode())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str, root: str = ROOT):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    record (profiles/dram_traffic_<workload>.txt), or None when there is no
    record or the kernel's sources changed since it was taken."""
    path = os.path.join(root, "profiles", f"dram_traffic_{workload}.txt")
    if not os.path.exists(path):
        return None
    csrc = os.path.join(root, "sparse_attention_attn_b200", "csrc")
    with open(path) as fh:
        for line in fh:
            f = line.split()
            if not f or f[0].startswith("#") or f[0] != kernel or f[1] != workload:
                continue
            if not all(os.path.exists(os.path.join(csrc, name)) for name in f[5:]):
                return None
            return int(f[2]) + int(f[3]) if source_digest(f[5:], csrc) == f[4] else None
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, csv_dir=None):
        """The raw samples go to `csv_dir`/clocks_rank<gpu>.csv when a directory
        is given, else to a temporary file removed once summarised."""
        self.proc = None
        self.gpu = gpu_index
        self.keep = csv_dir is not None
        if self.keep:
            self.path = os.path.join(csv_dir, f"clocks_rank{gpu_index}.csv")
        else:
            fd, self.path = tempfile.mkstemp(prefix=f"s2attn_clocks{gpu_index}_", suffix=".csv")
            os.close(fd)

    def start(self):
        try:
            os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            if not self.keep and os.path.exists(self.path):
                os.remove(self.path)
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            lines = fh.readlines()
        if not self.keep:
            os.remove(self.path)
        for line in lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


WATCHDOG_S = 120.0


def device_sync(limit_s: float = None, poll_s: float = 0.0005):
    """torch.cuda.synchronize() behind a host-side watchdog: an event recorded
    on the current stream is polled (cudaEventQuery) until it completes; if
    the device has not finished within limit_s seconds the run stops with an
    error instead of blocking forever.  The kernels' own waits are bounded,
    so this only catches what they cannot (a stuck copy, a driver stall)."""
    limit_s = WATCHDOG_S if limit_s is None else limit_s
    ev = torch.cuda.Event()
    ev.record()
    t0 = time.monotonic()
    while not ev.query():
        if time.monotonic() - t0 > limit_s:
            raise RuntimeError(f"watchdog: the device did not finish its work within {limit_s:.0f} s")
        time.sleep(poll_s)
    torch.cuda.synchronize()


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def oracle_sample(shape: I.Shape, budget_s: float, seed_offset: int = 0):
    """Time the fp64 oracle on whole (b, h, group) units of the workload until
    `budget_s` seconds have passed (at least one unit).  Returns
    (seconds, units, effective flops done, threads)."""
    import oracle.s2_ref as ref
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    g = torch.Generator().manual_seed(1234 + seed_offset)
    # one unit's inputs: the group's rows of one head (same distribution as the workload)
    fwd_unit = 4.0 * shape.G * shape.G * shape.D * 0.5
    t0 = time.perf_counter()
    units = 0
    while True:
        qg, kg, vg, dog = (torch.randn(shape.G, shape.D, generator=g).to(torch.bfloat16).double().numpy()
                           for _ in range(4))
        scale = 1.0 / np.sqrt(shape.D)
        ref.group_causal_attention(qg, kg, vg, scale)
        ref.group_causal_attention_grad(qg, kg, vg, dog, scale)
        units += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return el, units, units * fwd_unit * 3.5, threads


def workload_config(shape: I.Shape, world: int):
    """The `config` object of the JSON line; both arms print the same one."""
    q_bytes = shape.B * shape.N * shape.H * shape.D * 2
    kv_bytes = shape.B * shape.N * shape.Hkv * shape.D * 2
    return {"workload": shape.name, "B": shape.B, "H": shape.H, "Hkv": shape.Hkv, "D": shape.D,
            "N": shape.N, "G": shape.G, "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (q,k,v,dO,o = %d MiB), no flush" % ((3 * q_bytes + 2 * kv_bytes) >> 20)}


def run_reference(args, shape, world, rank):
    """The fp64 oracle timed on the host cores.  One step is one bounded sample
    of the workload (whole (head, group) units for about --ref-step-seconds);
    ms_per_step is the measured wall time of such a step, and the rate is the
    effective FLOPs the sample did divided by that time.  The time a whole
    workload step would take at that rate is reported under its own key."""
    if rank != 0:
        return
    fwd, bwd = effective_flops(shape)
    for _ in range(args.warmup):
        oracle_sample(shape, 0.0)
    total_s, total_units, total_flops, threads = 0.0, 0, 0.0, 1
    for _ in range(args.steps):
        el, u, fl, threads = oracle_sample(shape, args.ref_step_seconds)
        total_s += el
        total_units += u
        total_flops += fl
    tflops = total_flops / total_s / 1e12
    tokens_per_s = total_units * shape.G / total_s
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "tokens_per_s": tokens_per_s,
        "step": f"one bounded sample of the workload: whole (head, group) units of G={shape.G} rows, "
                f"fwd+bwd, for about {args.ref_step_seconds:g} s",
        "full_workload_step_ms_extrapolated": 1e3 * (fwd + bwd) / (tflops * 1e12),
        "config": workload_config(shape, world),
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{total_units} whole (head, group) units of G={shape.G} rows, "
                                   f"fwd+bwd, over {args.steps} steps ({total_s:.1f} s)"},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_ours(args, shape, world, rank, local):
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    q, k, v, do = I.make_inputs(shape, seed_offset=10 * rank)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((shape.B, shape.H, shape.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(s2.bwd_workspace_bytes(shape.B, shape.H, shape.Hkv, shape.N, shape.D, shape.G),
                     dtype=torch.uint8, device=dev)
    launches = [0]

    def step():
        s2.s2attn_forward(qd, kd, vd, shape.G, out=o, lse=lse)
        launches[0] += _lib.s2attn_last_launch_count()
        s2.s2attn_backward(qd, kd, vd, o, lse, dod, shape.G, dq=dq, dk=dk, dv=dv, workspace=ws)
        launches[0] += _lib.s2attn_last_launch_count()

    for _ in range(max(args.warmup, 3)):
        step()
    device_sync()
    if s2.device_status() != 0 or s2.device_status(ws) != 0:
        raise RuntimeError("device status reports a timeout during warm-up")

    # ---- device-timed region (inputs resident in HBM) ----
    # The headline loop runs with no per-kernel events between the launches.
    clocks = ClockSampler(local, args.clocks_csv_dir)
    clocks.start()
    time.sleep(0.3)
    launches[0] = 0
    barrier(world)
    device_sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    device_sync()
    barrier(world)
    ms_total = e0.elapsed_time(e1)
    gpu_launches = launches[0]
    # Per-kernel times: a second loop of the same steps with one CUDA-event pair
    # around each launch (on the launching stream).
    cap = 64 * args.steps + 8  # the split-dS backward runs several launches per step where it works in ranges
    assert _lib.s2attn_profile_start(cap) == 0
    for _ in range(args.steps):
        step()
    ms_arr = (ctypes.c_float * cap)()
    id_arr = (ctypes.c_int * cap)()
    n_rec = _lib.s2attn_profile_stop(ctypes.addressof(ms_arr), ctypes.addressof(id_arr), cap)
    device_sync()
    clk = clocks.stop()
    per_kernel = {}
    for i in range(max(n_rec, 0)):
        per_kernel.setdefault(id_arr[i], []).append(ms_arr[i])
    ms_step = max_over_ranks(ms_total / args.steps, world, dev)
    if s2.device_status() != 0 or s2.device_status(ws) != 0:
        raise RuntimeError("device status reports a timeout in the timed region")

    # ---- end-to-end through the public API with pinned host buffers ----
    # Every step copies its four inputs in from pinned host memory and its three
    # gradients out to pinned host memory.  The pipelined loop is how a training
    # input pipeline feeds the call: step i+1's inputs arrive (copy stream in) and
    # step i-1's gradients leave (copy stream out) while step i computes, on two
    # device sets of inputs and gradients.  The serial loop (copies and compute one
    # after another on one stream) is reported beside it.
    hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
    hdq, hdk, hdv = (torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv))
    host_in, host_out = (hq, hk, hv, hdo), (hdq, hdk, hdv)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    dev_in = [(qd, kd, vd, dod), tuple(torch.empty_like(t) for t in (qd, kd, vd, dod))]
    dev_out = [(dq, dk, dv), tuple(torch.empty_like(t) for t in (dq, dk, dv))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def compute(i):
        qi, ki, vi, doi = dev_in[i % 2]
        dqi, dki, dvi = dev_out[i % 2]
        s2.s2attn_forward(qi, ki, vi, shape.G, out=o, lse=lse)
        s2.s2attn_backward(qi, ki, vi, o, lse, doi, shape.G, dq=dqi, dk=dki, dv=dvi, workspace=ws)

    def e2e_serial(n):
        for _ in range(n):
            for d_, h_ in zip(dev_in[0], host_in):
                d_.copy_(h_, non_blocking=True)
            compute(0)
            for h_, d_ in zip(host_out, dev_out[0]):
                h_.copy_(d_, non_blocking=True)

    def e2e_pipelined(n):
        ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(n)] for _ in range(3))
        for i in range(n):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])  # the last reader of this input set
                for d_, h_ in zip(dev_in[i % 2], host_in):
                    d_.copy_(h_, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])  # this gradient set has left the device
            compute(i)
            ev_comp[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                for h_, d_ in zip(host_out, dev_out[i % 2]):
                    h_.copy_(d_, non_blocking=True)
                ev_out[i].record(s_out)

    def timed_e2e(loop, n, first, last):
        loop(2)
        device_sync()
        barrier(world)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(first)
        loop(n)
        f1.record(last)
        device_sync()
        barrier(world)
        return max_over_ranks(f0.elapsed_time(f1) / n, world, dev)

    e2e_steps = max(3, min(args.steps, 20))
    ms_e2e_serial = timed_e2e(e2e_serial, e2e_steps, stream, stream)
    ms_e2e = timed_e2e(e2e_pipelined, e2e_steps, s_in, s_out)
    if s2.device_status() != 0 or s2.device_status(ws) != 0:
        raise RuntimeError("device status reports a timeout in the end-to-end loop")
    # every step has the same inputs: the gradients that reached the host are
    # the device's -- bit for bit, except dq on the fused backward path, whose
    # fp32 reductions at L2 arrive in no fixed order (same values up to rounding)
    for name, h_, d_ in zip(("dq", "dk", "dv"), host_out, dev_out[1]):
        d_ = d_.cpu()
        if torch.equal(h_, d_):
            continue
        rel = float((h_.float() - d_.float()).norm() / d_.float().norm().clamp_min(1e-30))
        if not (name == "dq" and 4 in per_kernel and rel <= 1e-3):
            raise RuntimeError(f"end-to-end loop: {name} on the host differs from the device's (rel {rel:.2e})")

    # ---- report ----
    fwd, bwd = effective_flops(shape)
    total_flops = (fwd + bwd) * world
    tflops = total_flops / (ms_step * 1e-3) / 1e12
    tokens = shape.B * shape.N * world / (ms_step * 1e-3)
    peaks, peak_src = load_peaks()
    alg = kernel_algorithmic(shape, fused=4 in per_kernel)
    kern = {}
    for kid, times in per_kernel.items():
        # a kernel's work per step over its time per step (one launch per step
        # on every path but the split-dS backward in ranges, where dK/dV and
        # dQ-from-dS launch once per range)
        avg = sum(times) / len(times)
        step_ms = sum(times) / args.steps
        bound, work = alg[kid]
        if bound == "tensor":
            ach = work / (step_ms * 1e-3) / 1e12
            kern[KERNEL_NAMES[kid]] = {"avg_ms": avg, "launches": len(times), "ms_per_step": step_ms,
                                       "achieved": ach, "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"]}
        else:
            ach = work / (step_ms * 1e-3) / 1e9
            kern[KERNEL_NAMES[kid]] = {"avg_ms": avg, "launches": len(times), "ms_per_step": step_ms,
                                       "achieved": ach, "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}
    dom_id = max(per_kernel, key=lambda kid: sum(per_kernel[kid])) if per_kernel else 2
    dom = kern.get(KERNEL_NAMES[dom_id], {})
    bound = alg[dom_id][0]
    roofline = {
        "kernel": KERNEL_NAMES[dom_id], "bound": bound, "achieved": dom.get("achieved"),
        "peak": peaks["bf16_tflops"] if bound == "tensor" else peaks["hbm_gbs"],
        "unit": "TFLOP/s" if bound == "tensor" else "GB/s", "frac": dom.get("frac"),
        "traffic": recorded_traffic(KERNEL_NAMES[dom_id], shape.name), "peak_source": f"{peak_src} ({'bf16_tflops burst' if bound == 'tensor' else 'hbm_gbs'})",
        "share": (sum(per_kernel[dom_id]) / sum(sum(v) for v in per_kernel.values())) if per_kernel else None,
    }
    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "tokens_per_s": tokens,
        "frac_of_bf16_peak": tflops / (peaks["bf16_tflops"] * world),
        "config": workload_config(shape, world),
        "e2e": {"value": total_flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                "loop": "pipelined: copies in / out on two side streams overlap the neighbouring steps' compute",
                "serial_ms_per_step": ms_e2e_serial,
                "serial_value": total_flops / (ms_e2e_serial * 1e-3) / 1e12},
        "gpu_launches": gpu_launches,
        "roofline": roofline,
        "kernels": kern,
        "clocks": clk,
    }
    if not args.no_dense_ratio and rank == 0 and shape.G < shape.N:
        line["dense_comparison"] = dense_ratio(shape, dev, args)
    if not args.no_rope and rank == 0 and world == 1:
        line["rope"] = rope_step(shape, dev, peaks, ms_step)
    if not args.no_nf4 and rank == 0 and world == 1:
        line["nf4_qkv"] = nf4_projection(dev, peaks)
    if not args.no_hga and rank == 0 and world == 1:
        line["hga"] = hga_step(shape, dev, peaks)
    if not args.no_extra_workloads and world == 1:
        line["other_workloads"] = {s.name: other_workload(s, dev, peaks)
                                   for s in I.WORKLOADS if s.name in args.extra_workloads.split(",")}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        el, units, fl, threads = oracle_sample(shape, args.cpu_seconds)
        line["cpu_baseline"] = {"value": fl / el / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": f"{units} whole (head, group) units of G={shape.G} rows, fwd+bwd, "
                                          f"{el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def dense_ratio(shape: I.Shape, dev, args):
    """Same inputs through the same kernels with G = N (dense causal): time ratio."""
    import sparse_attention_attn_b200 as s2
    dense = shape.dense()
    q, k, v, do = (t.to(dev) for t in I.make_inputs(dense))
    # one workspace for both calls: the larger of the two plans' needs
    ws = torch.empty(max(s2.bwd_workspace_bytes(dense.B, dense.H, dense.Hkv, dense.N, dense.D, G)
                         for G in (shape.G, dense.G)), dtype=torch.uint8, device=dev)

    def timed(G, steps):
        for _ in range(3):
            o, lse = s2.s2attn_forward(q, k, v, G)
            s2.s2attn_backward(q, k, v, o, lse, do, G, workspace=ws)
        device_sync()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            o, lse = s2.s2attn_forward(q, k, v, G)
            s2.s2attn_backward(q, k, v, o, lse, do, G, workspace=ws)
        b.record()
        device_sync()
        return a.elapsed_time(b) / steps

    n = max(5, min(args.steps, 20))
    t_s2 = timed(shape.G, n)
    t_dense = timed(shape.N, n)
    return {"s2_ms": t_s2, "dense_ms": t_dense, "speedup": t_dense / t_s2}


def rope_step(shape: I.Shape, dev, peaks, ms_plain: float, steps: int = 10, warmup: int = 3):
    """The same step with RoPE + Position Interpolation (from 4096 tokens)
    before S2 attention: s2attn_fwd_rope (rotation passes for q and k, then the
    forward) and s2attn_bwd_rope (back-rotation fused into the dq conversion
    and the dK epilogue on the fused path).  Reports its time beside the plain
    step's and the rotation pass against the HBM bandwidth (bytes: read and
    write q and k; the table is L2-resident)."""
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib
    q, k, v, do = (t.to(dev) for t in I.make_inputs(shape))
    tab = s2.rope_table(shape.N, shape.D, min(1.0, 4096 / shape.N))
    o = torch.empty_like(q)
    lse = torch.empty((shape.B, shape.H, shape.N), dtype=torch.float32, device=dev)
    qr, kr = torch.empty_like(q), torch.empty_like(k)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(s2.bwd_workspace_bytes(shape.B, shape.H, shape.Hkv, shape.N, shape.D, shape.G),
                     dtype=torch.uint8, device=dev)

    def step():
        s2.s2attn_forward_rope(q, k, v, shape.G, tab, out=o, lse=lse, q_rot=qr, k_rot=kr)
        s2.s2attn_backward_rope(qr, kr, v, o, lse, do, shape.G, tab, dq=dq, dk=dk, dv=dv, workspace=ws)

    for _ in range(warmup):
        step()
    device_sync()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    device_sync()
    ms = a.elapsed_time(b) / steps
    cap = 8 * steps + 8
    assert _lib.s2attn_profile_start(cap) == 0
    for _ in range(steps):
        step()
    ms_arr, id_arr = (ctypes.c_float * cap)(), (ctypes.c_int * cap)()
    n = _lib.s2attn_profile_stop(ctypes.addressof(ms_arr), ctypes.addressof(id_arr), cap)
    if s2.device_status() != 0 or s2.device_status(ws) != 0:
        raise RuntimeError("device status reports a timeout in the RoPE step")
    rot = [ms_arr[i] for i in range(max(n, 0)) if id_arr[i] == 6]
    rot_bytes = 2.0 * (q.numel() + k.numel()) * 2 / 2  # per launch on average: q (H heads) or k (Hkv heads), read + write
    avg = sum(rot) / len(rot) if rot else None
    fwd, bwd = effective_flops(shape)
    out = {"ms_per_step": ms, "plain_ms_per_step": ms_plain, "overhead_ms": ms - ms_plain,
           "value": (fwd + bwd) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
           "pos_scale": min(1.0, 4096 / shape.N), "rope_base": 10000.0}
    if avg:
        out["rotation_pass"] = {"launches_per_step": len(rot) / steps, "avg_ms": avg,
                                "achieved": rot_bytes / (avg * 1e-3) / 1e9, "unit": "GB/s",
                                "frac": rot_bytes / (avg * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "bytes_per_launch": rot_bytes}
    return out


def hga_step(shape: I.Shape, dev, peaks, S: int = 8, steps: int = 10, warmup: int = 3):
    """HGA-style block-sparse attention on the workload's inputs: segments of
    G rows attended causally (no shift) plus S listed historical 128-row tiles
    per 256-row query block (random earlier tiles), forward + backward.
    Effective FLOPs: the local part counts as S2's (forward 2 GEMMs, backward
    2.5x), the historical part forward 2 GEMMs and backward 2 (dP and dQ; no
    dK/dV for detached keys)."""
    import sparse_attention_attn_b200 as s2
    q, k, v, do = (t.to(dev) for t in I.make_inputs(shape))
    hist = I.make_hga_selection(shape.B, shape.N, shape.G, S, seed=5).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((shape.B, shape.H, shape.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def step():
        s2.hga_forward(q, k, v, shape.G, hist, out=o, lse=lse)
        s2.hga_backward(q, k, v, o, lse, do, shape.G, hist, dq=dq, dk=dk, dv=dv)

    for _ in range(warmup):
        step()
    device_sync()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    device_sync()
    ms = a.elapsed_time(b) / steps
    if s2.device_status() != 0:
        raise RuntimeError("device status reports a timeout in the HGA step")
    n_hist = int((hist >= 0).sum().item())  # listed tiles over all blocks (each 256 rows x 128 keys)
    fwd_local, _ = effective_flops(shape)
    fwd_hist = 4.0 * shape.H * shape.D * n_hist * 256 * 128
    total = 3.5 * fwd_local + 2.0 * fwd_hist
    tf = total / (ms * 1e-3) / 1e12
    return {"ms_per_step": ms, "value": tf, "unit": "TFLOP/s", "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
            "tiles_per_block": S, "history_tiles_listed": n_hist, "steps": steps, "warmup": warmup}


def nf4_projection(dev, peaks, steps: int = 20, warmup: int = 3):
    """The QKV projection that feeds the attention, from NF4 weights with
    double quantization (LLaMA2-7B layer at 8192 tokens: x [8192, 4096],
    W [12288, 4096]): the fused kernel (dequantization inside the tensor-core
    GEMM) against the library's dequantization kernel followed by a cuBLAS
    GEMM (torch.matmul) on the dequantized weight.  Inputs and outputs (x
    64 MiB, codes 24 MiB, q/k/v 192 MiB) exceed the L2 together."""
    import sparse_attention_attn_b200 as s2
    c = I.NF4_LLAMA2_7B_8K
    M, K, H, Hkv, D = c["M"], c["K"], c["H"], c["Hkv"], c["D"]
    rows = (H + 2 * Hkv) * D
    codes, sq, c2 = (t.to(dev) for t in I.make_nf4_weights(rows, K, seed=3))
    x = I.randn_bf16((1, M, K), 90).to(dev)
    q = torch.empty((1, M, H, D), dtype=torch.bfloat16, device=dev)
    k = torch.empty((1, M, Hkv, D), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    w = torch.empty((rows, K), dtype=torch.bfloat16, device=dev)
    y = torch.empty((M, rows), dtype=torch.bfloat16, device=dev)

    def fused():
        s2.nf4_qkv(x, codes, sq, c2, H, Hkv, D, q=q, k=k, v=v)

    def unfused():
        s2.nf4_dequantize(codes, sq, c2, out=w)
        torch.matmul(x.view(M, K), w.t(), out=y)

    def dequant_only():
        s2.nf4_dequantize(codes, sq, c2, out=w)

    def timed(fn):
        for _ in range(warmup):
            fn()
        device_sync()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        device_sync()
        return a.elapsed_time(b) / steps

    ms_f, ms_u, ms_d = timed(fused), timed(unfused), timed(dequant_only)
    if s2.device_status() != 0:
        raise RuntimeError("device status reports a timeout in the NF4 projection")
    flops = 2.0 * M * rows * K
    dq_bytes = rows * K / 2 + rows * K / 64 + rows * K * 2  # codes + scale codes read, bf16 W' written
    tf = flops / (ms_f * 1e-3) / 1e12
    return {"workload": c["name"], "M": M, "K": K, "N_out": rows, "ms": ms_f, "achieved": tf, "unit": "TFLOP/s",
            "frac": tf / peaks["bf16_tflops"], "peak_source": "measured (bf16_tflops burst)",
            "unfused_ms": ms_u, "unfused": "nf4 dequantization kernel + cuBLAS bf16 GEMM (torch.matmul)",
            "speedup_vs_unfused": ms_u / ms_f,
            "dequant_kernel": {"ms": ms_d, "achieved": dq_bytes / (ms_d * 1e-3) / 1e9, "unit": "GB/s",
                               "frac": dq_bytes / (ms_d * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "steps": steps, "warmup": warmup}


def other_workload(shape: I.Shape, dev, peaks, steps: int = 5, warmup: int = 3):
    """ms per fwd+bwd step and fraction of the bf16 peak on another workload
    shape (a few steps; CUDA events on the launching stream)."""
    import sparse_attention_attn_b200 as s2
    q, k, v, do = (t.to(dev) for t in I.make_inputs(shape))
    o = torch.empty_like(q)
    lse = torch.empty((shape.B, shape.H, shape.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(s2.bwd_workspace_bytes(shape.B, shape.H, shape.Hkv, shape.N, shape.D, shape.G),
                     dtype=torch.uint8, device=dev)

    def step():
        s2.s2attn_forward(q, k, v, shape.G, out=o, lse=lse)
        s2.s2attn_backward(q, k, v, o, lse, do, shape.G, dq=dq, dk=dk, dv=dv, workspace=ws)

    for _ in range(warmup):
        step()
    device_sync()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    device_sync()
    if s2.device_status() != 0 or s2.device_status(ws) != 0:
        raise RuntimeError(f"device status reports a timeout on {shape.name}")
    ms = a.elapsed_time(b) / steps
    fwd, bwd = effective_flops(shape)
    tflops = (fwd + bwd) / (ms * 1e-3) / 1e12
    return {"ms_per_step": ms, "value": tflops, "unit": "TFLOP/s", "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
            "tokens_per_s": shape.B * shape.N / (ms * 1e-3), "steps": steps, "warmup": warmup}


def sweep_variants(shape: I.Shape):
    """Every variant the per-shape plan can select for a workload shape, as
    override strings: forward (work order x key tile x K/V ring depth) and
    backward (path x stages, and the dK/dV kernel's 128-query tiles).  The
    split-dS path keeps the plan's dS slots (every unit within the 4 GiB
    budget, else ranges)."""
    D = shape.D
    slots = (4,) if D == 128 else (4, 6, 8)
    fwd = [f"fwd_order={o},fwd_kv={s}" for o in ("snake", "pairs") for s in slots] + \
        [f"fwd_bn=64,fwd_order={o},fwd_kv={s}" for o in ("snake", "pairs") for s in ((8,) if D == 128 else (8, 12))]
    stages = (2, 3) if D == 128 else (3, 4)
    paths = ("split_ds", "split")
    bwd = (["bwd=fused"] if D == 128 else []) + [f"bwd={p},bwd_stages={s}" for p in paths for s in stages] + \
        ["bwd=split_ds,bwd_stages=3,bwd_qtile=128"]
    return fwd, bwd


def run_sweep(args, dev):
    """Times each selectable variant of the forward and of the backward on
    every workload shape (CUDA events on the launching stream, a few steps
    after warm-up) and prints one JSON line per (workload, variant) plus the
    plan the library selects for each shape."""
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    rows = []
    for shape in I.WORKLOADS:
        q, k, v, do = (t.to(dev) for t in I.make_inputs(shape))
        o = torch.empty_like(q)
        lse = torch.empty((shape.B, shape.H, shape.N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        steps = 10 if shape.N <= 16384 else 4
        fwd_specs, bwd_specs = sweep_variants(shape)
        _lib.s2attn_set_tile_override(None)
        chosen = _lib.s2attn_plan(shape.B, shape.H, shape.Hkv, shape.N, shape.D, shape.G, props.multi_processor_count)

        def timed(fn):
            for _ in range(3):
                fn()
            device_sync()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(steps):
                fn()
            b.record()
            device_sync()
            return a.elapsed_time(b) / steps

        for kind, specs in (("fwd", fwd_specs), ("bwd", bwd_specs)):
            for spec in specs:
                _lib.s2attn_set_tile_override(spec)
                try:
                    if kind == "fwd":
                        ms = timed(lambda: s2.s2attn_forward(q, k, v, shape.G, out=o, lse=lse))
                    else:
                        s2.s2attn_forward(q, k, v, shape.G, out=o, lse=lse)
                        ws = torch.empty(s2.bwd_workspace_bytes(shape.B, shape.H, shape.Hkv, shape.N, shape.D,
                                                                shape.G), dtype=torch.uint8, device=dev)
                        ms = timed(lambda: s2.s2attn_backward(q, k, v, o, lse, do, shape.G, dq=dq, dk=dk, dv=dv,
                                                              workspace=ws))
                        del ws
                    if s2.device_status() != 0:
                        raise RuntimeError(f"device status reports a timeout ({shape.name}, {spec})")
                finally:
                    _lib.s2attn_set_tile_override(None)
                fwd_f, bwd_f = effective_flops(shape)
                row = {"workload": shape.name, "kernel": kind, "variant": spec, "ms": ms,
                       "tflops": (fwd_f if kind == "fwd" else bwd_f) / (ms * 1e-3) / 1e12, "steps": steps}
                rows.append(row)
                print(json.dumps(row), flush=True)
        print(json.dumps({"workload": shape.name, "selected_plan": chosen}), flush=True)
        del q, k, v, do, o, lse, dq, dk, dv
        torch.cuda.empty_cache()
    return rows


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=I.LLAMA2_7B_8K.name,
                    choices=[s.name for s in I.WORKLOADS])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=None,
                    help="oracle seconds per reference step (default: ~2 minutes in total)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-csv-dir", default=None,
                    help="keep the raw nvidia-smi clock samples of the timed region in this directory")
    ap.add_argument("--no-dense-ratio", action="store_true",
                    help="skip timing G=N (dense causal) on the same inputs")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the few-step timing of the other workload shapes")
    ap.add_argument("--no-rope", action="store_true", help="skip the step with RoPE + Position Interpolation")
    ap.add_argument("--no-nf4", action="store_true", help="skip the NF4 QKV projection timing")
    ap.add_argument("--no-hga", action="store_true", help="skip the HGA block-sparse step timing")
    ap.add_argument("--nf4-only", action="store_true",
                    help="time only the NF4 QKV projection (--steps / --warmup launches) and print its JSON")
    ap.add_argument("--sweep", action="store_true",
                    help="time every selectable kernel variant on every workload shape and exit")
    ap.add_argument("--extra-workloads", default=f"{I.QWEN3_8B_16K.name},{I.LLAMA2_70B_32K.name}",
                    help="comma-separated workload names timed for a few steps beside the headline")
    args = ap.parse_args()
    shape = {s.name: s for s in I.WORKLOADS}[args.workload]
    if args.ref_step_seconds is None:
        args.ref_step_seconds = min(5.0, 120.0 / max(args.steps, 1))
    if args.sweep:
        run_sweep(args, torch.device("cuda", 0))
        return
    if args.nf4_only:
        print(json.dumps(nf4_projection(torch.device("cuda", 0), load_peaks()[0], steps=args.steps,
                                        warmup=args.warmup)), flush=True)
        return
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, shape, world, rank)
        else:
            run_ours(args, shape, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
