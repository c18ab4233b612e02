"""Benchmark of the Switch layer forward pass (tokens/s) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one switch_layer_fwd over one batch of synthetic tokens (router,
capacity scan, slot assignment with dispatch, both expert GEMMs with the gated
combine in the second one's epilogue; the scan runs inside the assignment
kernel when the per-tile histogram is small), inputs already resident in HBM.  Each step is timed with CUDA events
on the launching stream; an L2 flush (a 512 MiB write) runs between steps,
outside the events.  With --gpus N (under torchrun) every rank runs its own
batch (independent token groups, replicated experts: weak scaling, no
collective on the data path); time = max over ranks.

The JSON line also carries:
  roofline      the dominant kernel's achieved rate from per-launch CUDA
                events (the library's tracer) against the measured peak
  e2e           the same metric through the public API with pinned host
                buffers: x copied in and y/aux/counts copied out every step
  cpu_baseline  the fp64 oracle on the host cores over a bounded sample
  clocks        nvidia-smi samples taken during the timed region
--impl reference times the oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from sparse_mixture_experts_fp32_b200 import synth  # noqa: E402

METRIC = "Switch-layer fwd tokens/s on 1 B200; expert GEMM % bf16 peak; route/scatter GB/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "base8"
L2_FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank: int) -> int:
    """Every rank draws its own token batch; rank 0 keeps the workload's seed."""
    return wl.seed + 1000 * rank


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 50):
        self.lines: list[tuple[float, str]] = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", f"-lms", str(period_ms)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float) -> dict:
        rows = [l for (t, l) in self.lines if t0 - 0.06 <= t <= t1 + 0.06]
        if not rows:
            rows = [l for (_, l) in self.lines]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                mx.append(float(f[3]))
            except ValueError:
                continue
            for name, v in zip(names, f[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# algorithmic work per kernel launch
# ---------------------------------------------------------------------------
def kernel_work(wl, C, counts):
    """Algorithmic bytes (HBM) or flops per launch of each kernel of one step."""
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.num_experts
    s = 2 if wl.dtype == synth.BF16 else 4
    kept = np.minimum(counts, C)
    K = int(kept.sum())
    E_nz = int((kept > 0).sum())
    tiles = -(-T // 64)
    router_bytes = T * d * s + N * d * 4 + 8 * T + 8 * N * tiles
    return {
        "router_warp": ("hbm", router_bytes),
        "router_tiled": ("hbm", router_bytes),
        "router_staged": ("hbm", router_bytes),
        "router_tc": ("hbm", T * d * s + 3 * N * d * 2 + 8 * T + 8 * N * tiles),
        "router_weight_split": ("hbm", N * d * 4 + 3 * N * d * 2),
        "capacity_scan": ("hbm", 8 * N * tiles + 4 * N * tiles + 12 * N),
        "slot_assign_scatter": ("hbm", 4 * T + 4 * T + 4 * N * tiles + 4 * N * C + 2 * K * d * s + (T - K) * d * 4),
        "ffn_tc_gemm1_relu": ("tensor", 2.0 * K * d * F),
        "ffn_tc_gemm2_gated_scatter": ("tensor", 2.0 * K * F * d),
        "ffn_tc_fused": ("tensor", 4.0 * K * d * F),
        "ffn_simt_gemm1_relu": ("alu", 2.0 * K * d * F),
        "ffn_simt_gemm2": ("alu", 2.0 * K * F * d),
        "combine": ("hbm", T * d * 4 + K * d * 4 + 12 * T),
        "_meta": ("", dict(K=K, E_nz=E_nz, gemm_weight_bytes=2 * E_nz * d * F * s)),
    }


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def to_dev(a, device):
    import torch
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def run_gpu(args):
    import torch

    import sparse_mixture_experts_fp32_b200 as sm

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    wl = synth.WORKLOADS[args.workload]
    if args.capacity_factor is not None:
        wl = wl.with_capacity_factor(args.capacity_factor)
    # experts and router are shared by all ranks; every rank routes its own tokens
    w_in_np, w_out_np = synth.all_expert_weights(wl)
    inp = dict(x=synth.activations(wl, seed=rank_seed(wl, rank)), w_r=synth.router_weight(wl),
               bias=synth.router_bias(wl), w_in=w_in_np, w_out=w_out_np)
    C = sm.switch_capacity(wl.T, wl.num_experts, wl.capacity_factor)

    x = to_dev(inp["x"], device)
    w_r = to_dev(inp["w_r"], device)
    bias = to_dev(inp["bias"], device)
    w_in = to_dev(inp["w_in"], device)
    w_out = to_dev(inp["w_out"], device)
    dims = sm.layer_dims(x, w_in, capacity=C)
    ws = sm.workspace(dims, device)
    T, d, N = wl.T, wl.d_model, wl.num_experts
    out = dict(y=torch.empty(T, d, dtype=torch.float32, device=device),
               expert=torch.empty(T, dtype=torch.int32, device=device),
               gate=torch.empty(T, dtype=torch.float32, device=device),
               slot=torch.empty(T, dtype=torch.int32, device=device),
               counts=torch.empty(N, dtype=torch.int32, device=device),
               aux=torch.empty(1, dtype=torch.float32, device=device))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    L = sm.lib()
    import ctypes
    dref = ctypes.byref(dims)
    ptr = lambda t: None if t is None else t.data_ptr()
    call_args = (dref, ptr(x), ptr(w_r), ptr(bias), ptr(w_in), ptr(w_out), ptr(out["y"]), ptr(out["expert"]),
                 ptr(out["gate"]), ptr(out["slot"]), ptr(out["counts"]), ptr(out["aux"]), ptr(ws),
                 ws.numel(), stream.cuda_stream)

    def step():
        st = L.switch_layer_fwd(*call_args)
        if st != 0:
            raise sm.SwitchError(st, "switch_layer_fwd")

    # warm-up
    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize(device)
    status = sm.switch_check(ws)
    if status != 0:
        raise sm.SwitchError(status, "device status after warm-up")
    counts = out["counts"].cpu().numpy()

    # timed region: per-step events, L2 flush between steps (outside the events)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        time.sleep(0.3)
    launches0 = sm.launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    t_wall0 = time.time()
    for i in range(K):
        flush.fill_(float(i))
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(device)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    launches = sm.launch_count() - launches0
    clocks = sampler.summary(t_wall0, t_wall1) if sampler else None
    if sampler:
        sampler.stop()
    status = sm.switch_check(ws)
    if status != 0:
        raise sm.SwitchError(status, "device status after the timed steps")
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), world, device)
    ms_per_step = total_ms / K

    # the same K steps again with the library's per-launch tracer on: per-kernel
    # durations for the roofline (events between kernels serialise them, so
    # these steps are timed separately from the headline ones)
    sm.trace_start(K * 8)
    traced_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush.fill_(float(i))
        traced_ev[i][0].record(stream)
        step()
        traced_ev[i][1].record(stream)
    torch.cuda.synchronize(device)
    trace = sm.trace_read(K * 8)
    sm.trace_stop()
    traced_ms_per_step = sum(a.elapsed_time(b) for a, b in traced_ev) / K

    # per-kernel averages from the library's tracer (same steps)
    per_kernel: dict[str, list[float]] = {}
    for name, ms in trace:
        per_kernel.setdefault(name, []).append(ms)
    work = kernel_work(wl, C, counts)
    meta = work.pop("_meta")[1]
    peaks, peak_src = load_peaks()
    kernels = {}
    for name, times in per_kernel.items():
        avg = statistics.mean(times)
        kind, amount = work.get(name, ("?", 0))
        entry = {"launches": len(times), "avg_ms": round(avg, 5), "share": None}
        if kind == "hbm":
            entry.update(bound="hbm", achieved=amount / (avg * 1e-3) / 1e9, peak=peaks["hbm_gbs"], unit="GB/s")
        elif kind == "tensor":
            entry.update(bound="tensor", achieved=amount / (avg * 1e-3) / 1e12, peak=peaks["bf16_tflops"],
                         unit="TFLOP/s")
        elif kind == "alu":
            entry.update(bound="alu", achieved=amount / (avg * 1e-3) / 1e12, peak=74.4, unit="TFLOP/s")
        if "achieved" in entry:
            entry["achieved"] = round(entry["achieved"], 2)
            entry["frac"] = round(entry["achieved"] / entry["peak"], 4)
        kernels[name] = entry
    tot = sum(k["avg_ms"] * k["launches"] for k in kernels.values())
    for k in kernels.values():
        k["share"] = round(k["avg_ms"] * k["launches"] / tot, 4) if tot else None
    dominant = max(kernels, key=lambda n: kernels[n]["avg_ms"] * kernels[n]["launches"]) if kernels else None
    roofline = None
    if dominant and "achieved" in kernels[dominant]:
        k = kernels[dominant]
        roofline = {"kernel": dominant, "bound": k["bound"], "achieved": k["achieved"], "peak": k["peak"],
                    "unit": k["unit"], "frac": k["frac"], "traffic": traffic_from_profiles(dominant, wl.name),
                    "peak_source": (f"{peak_src} (burst bf16 matmul)" if k["bound"] == "tensor" else
                                    f"{peak_src} (copy bandwidth)" if k["bound"] == "hbm" else
                                    "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz (FFMA issue rate)")}

    # e2e through the public API with pinned host buffers
    e2e = run_e2e(args, sm, wl, inp, C, device, world)

    # capacity-factor sweep on the same tokens and weights (--sweep)
    sweep = []
    if args.sweep and wl.sweep:
        for c in wl.sweep:
            Cc = sm.switch_capacity(T, N, c)
            dc = sm.layer_dims(x, w_in, capacity=Cc)
            wsc = sm.workspace(dc, device)
            outc = sm.layer_fwd(x, w_r, w_in, w_out, capacity=Cc, logit_bias=bias, ws=wsc)
            for _ in range(args.warmup):
                flush.fill_(1.0)
                sm.layer_fwd(x, w_r, w_in, w_out, capacity=Cc, logit_bias=bias, ws=wsc, out=outc)
            torch.cuda.synchronize(device)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
            for i in range(K):
                flush.fill_(float(i))
                evs[i][0].record(stream)
                sm.layer_fwd(x, w_r, w_in, w_out, capacity=Cc, logit_bias=bias, ws=wsc, out=outc)
                evs[i][1].record(stream)
            torch.cuda.synchronize(device)
            if sm.switch_check(wsc) != 0:
                raise RuntimeError("device status after the sweep steps")
            msc = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, device) / K
            kept = int(np.minimum(outc["counts"].cpu().numpy(), Cc).sum())
            sweep.append({"capacity_factor": c, "capacity": Cc, "ms_per_step": round(msc, 5),
                          "value": round(world * T / (msc * 1e-3), 1), "kept_tokens": kept,
                          "drop_fraction": round(1 - kept / T, 6),
                          "expert_flops_per_step": 4.0 * kept * d * wl.d_ff})
            del wsc, outc
            torch.cuda.empty_cache()

    result = None
    if rank == 0:
        value = world * T / (ms_per_step * 1e-3)
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == synth.BF16 else "f32",
            "data": "synthetic (seeded numpy PCG64; per-rank token batches; experts replicated)",
            "config": {"workload": wl.name, "T": T, "d_model": d, "d_ff": wl.d_ff, "num_experts": N,
                       "capacity_factor": wl.capacity_factor, "capacity": C, "router": "fp32",
                       "experts": wl.dtype, "kept_tokens": meta["K"], "nonempty_experts": meta["E_nz"],
                       "drop_fraction": round(1 - meta["K"] / T, 6),
                       "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, outside the events)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": roofline,
            "kernels": kernels,
            "gpu_launches": int(launches),
            "traced_ms_per_step": round(traced_ms_per_step, 5),
            "e2e": e2e,
            "clocks": clocks,
            "wall_s_timed_region": round(t_wall1 - t_wall0, 4),
        }
        if sweep:
            result["sweep"] = sweep
        if not args.no_cpu_baseline and world == 1:
            result["cpu_baseline"] = cpu_baseline(wl, inp, C, budget_s=args.cpu_budget)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_e2e(args, sm, wl, inp, C, device, world):
    """Same metric through sm.layer_fwd with host-resident inputs and outputs.

    Every step copies its x from pinned host memory to the device, runs the
    layer and copies y, aux and counts back to pinned host memory.  The three
    parts run on their own streams with two sets of device buffers, so step
    i's output copy, step i+1's layer and step i+2's input copy overlap, as a
    caller streaming batches would run them; the time is from the first input
    copy to the last output copy."""
    import torch
    T, d, N = wl.T, wl.d_model, wl.num_experts
    tdt = torch.bfloat16 if wl.dtype == synth.BF16 else torch.float32
    x_host = to_dev(inp["x"], "cpu").pin_memory()
    w = {k: to_dev(inp[k], device) for k in ("w_r", "bias", "w_in", "w_out")}
    x_dev = [torch.empty(T, d, dtype=tdt, device=device) for _ in range(2)]
    y_host = [torch.empty(T, d, dtype=torch.float32).pin_memory() for _ in range(2)]
    aux_host = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(2)]
    counts_host = [torch.empty(N, dtype=torch.int32).pin_memory() for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    in_done = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    outs = [None, None]
    ws = None
    steps = max(3, min(args.steps, args.e2e_steps))

    def one(i):
        nonlocal ws
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(cmp_done[b])  # the layer of step i-2 has read x_dev[b]
            x_dev[b].copy_(x_host, non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_done[b])
            if i >= 2:
                s_cmp.wait_event(out_done[b])  # y of step i-2 has left outs[b]
            outs[b] = sm.layer_fwd(x_dev[b], w["w_r"], w["w_in"], w["w_out"], capacity=C, logit_bias=w["bias"],
                                   ws=ws, out=outs[b], stream=s_cmp)
            ws = outs[b]["workspace"]
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            y_host[b].copy_(outs[b]["y"], non_blocking=True)
            aux_host[b].copy_(outs[b]["aux"], non_blocking=True)
            counts_host[b].copy_(outs[b]["counts"], non_blocking=True)
            out_done[b].record(s_out)

    for i in range(4):
        one(i)
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        one(i + 4)
    end.record(s_out)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(start.elapsed_time(end) / steps, world, device)
    status = sm.switch_check(ws)
    if status != 0:
        raise sm.SwitchError(status, "device status after the e2e steps")
    return {"value": round(world * T / (ms * 1e-3), 1), "unit": UNIT, "ms_per_step": round(ms, 5),
            "steps": steps, "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
            "d2h_bytes_per_step": int(y_host[0].numel() * 4 + 4 + N * 4),
            "overlap": "input copy, layer and output copy on three streams, two buffer sets"}


def traffic_from_profiles(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    sources are unchanged since the counters were taken."""
    want = source_sha(kernel)
    for p in sorted((ROOT / "profiles").glob("*.md")):
        text = p.read_text()
        m = re.search(rf"^\s*traffic\[{re.escape(kernel)}@{re.escape(workload)}\]:\s*([0-9.eE+]+)\s+bytes"
                      rf"\s+source_sha=(\w+)", text, flags=re.M)
        if m and m.group(2) == want:
            return float(m.group(1))
    return None


# The source file of each traced kernel; its hash, with the shared headers,
# identifies the kernel as built.
KERNEL_SOURCE = {
    "router_warp": "route.cu", "router_tiled": "route.cu", "router_staged": "route.cu",
    "capacity_scan": "route.cu", "slot_assign": "route.cu", "slot_assign_scatter": "route.cu",
    "router_weight_split": "router_tc.cu", "router_tc": "router_tc.cu",
    "dispatch": "move.cu", "combine": "move.cu",
}


def source_sha(kernel: str) -> str:
    import hashlib
    csrc = ROOT / "sparse_mixture_experts_fp32_b200" / "csrc"
    src = KERNEL_SOURCE.get(kernel)
    if src is None and kernel.startswith(("ffn_tc", "ffn_simt")):
        src = "ffn_tc.cu" if kernel.startswith("ffn_tc") else "ffn_simt.cu"
    files = ["common.cuh", "internal.h"] + ([src] if src else sorted(p.name for p in csrc.glob("*.cu")))
    h = hashlib.sha1()
    for f in files:
        h.update((csrc / f).read_bytes())
    return h.hexdigest()[:12]


# ---------------------------------------------------------------------------
# the oracle: CPU baseline leg and reference arm
# ---------------------------------------------------------------------------
def cpu_baseline(wl, inp, C, budget_s=15.0):
    """Time the fp64 oracle on the host: routing + assignment for every token,
    expert FFN for a growing prefix of the kept tokens until about budget_s,
    extrapolated to all kept tokens."""
    import oracle
    orc = oracle.Oracle()
    t0 = time.perf_counter()
    r = orc.route(inp["x"], inp["w_r"], inp["bias"], capacity=C)
    t_route = time.perf_counter() - t0
    kept = np.flatnonzero(r["slot"] >= 0)
    n, t_ffn, done = 64, 0.0, 0
    while done < kept.size and t_ffn < budget_s:
        rows = kept[done:done + n]
        t1 = time.perf_counter()
        orc.output_rows(rows, inp["x"], inp["w_in"], inp["w_out"], r["expert"], r["slot"], r["gate"])
        t_ffn += time.perf_counter() - t1
        done += rows.size
        n = min(n * 2, kept.size)
    per_row = t_ffn / max(done, 1)
    est = t_route + per_row * kept.size
    return {"value": round(wl.T / est, 2), "unit": UNIT, "cores": orc.threads(), "kind": "oracle",
            "sample": (f"router/softmax/assignment/aux on all {wl.T} tokens ({t_route:.2f} s) + expert FFN on "
                       f"{done} of {kept.size} kept tokens ({t_ffn:.2f} s), extrapolated to all kept tokens"),
            "seconds_measured": round(t_route + t_ffn, 2)}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    wl = synth.WORKLOADS[args.workload]
    if args.capacity_factor is not None:
        wl = wl.with_capacity_factor(args.capacity_factor)
    inp = synth.inputs(wl)
    import oracle
    orc = oracle.Oracle()
    C = orc.capacity(wl.T, wl.num_experts, wl.capacity_factor)
    budget = max(1.0, args.cpu_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(wl, inp, C, budget_s=budget)
    vals = [cpu_baseline(wl, inp, C, budget_s=budget) for _ in range(args.steps)]
    value = statistics.mean(v["value"] for v in vals)
    ms = wl.T / value * 1e3
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
            "config": {"workload": wl.name, "T": wl.T, "d_model": wl.d_model, "d_ff": wl.d_ff,
                       "num_experts": wl.num_experts, "capacity_factor": wl.capacity_factor, "capacity": C},
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--capacity-factor", type=float, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle FFN time for cpu_baseline")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="also time every capacity factor of the workload's sweep")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, _ = dist_env()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    res = run_reference(args) if args.impl == "reference" else run_gpu(args)
    if res is not None and rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
