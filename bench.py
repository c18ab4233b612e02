"""Benchmark of the Switch layer forward pass (tokens/s) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one switch_layer_fwd over one batch of synthetic tokens (router,
capacity scan, slot assignment with dispatch, both expert GEMMs with the gated
combine in the second one's epilogue; the scan runs inside the assignment
kernel when the per-tile histogram is small), inputs already resident in HBM.
The default workload is the largest one, the Switch-Large-shaped layer
(T = 131072, d_model = 1024, d_ff = 4096, 128 experts, c = 1.25).  Each step is
timed with CUDA events on the launching stream; an L2 flush (a 512 MiB write)
runs between steps, outside the events.  With --gpus N (under torchrun) every
rank runs its own batch (independent token groups, replicated experts: weak
scaling, no collective on the data path); time = max over ranks.

The JSON line also carries:
  roofline      the dominant kernel's achieved rate from per-launch CUDA
                events (the library's tracer) against the measured peak
                (burst, and sustained for tensor-core kernels)
  kernels       every kernel's time, share and fraction of its roofline; for
                the kernels that write the float32 output, also the fraction
                with those rows counted at the activation dtype
  e2e           the same metric through the public API with pinned host
                buffers: x copied in and y/aux/counts copied out every step
  top2          the top-2 variant (switch_layer_fwd_top2) on the same tensors
  backward      a training step (training forward + switch_layer_bwd) on the same tensors
  entry_points  switch_dispatch and switch_combine called on their own
  sweep         the large-expert layer at every capacity factor of its sweep
                (drop fraction and tokens/s per c)
  cpu_baseline  the fp64 oracle on all host cores and on one core, over a
                bounded sample
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

import sparse_mixture_experts_fp32_b200 as swm  # noqa: E402  (flag constants; the library loads lazily)
from sparse_mixture_experts_fp32_b200 import synth  # noqa: E402

METRIC = "Switch-layer fwd tokens/s on 1 B200; expert GEMM % bf16 peak; route/scatter GB/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "large128"
SWEEP_WORKLOAD = "bigexpert64"
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


def workload_of(args):
    """The named workload, with the optional capacity factor and token count
    overrides (a reduced token count serves small profiler captures)."""
    wl = synth.WORKLOADS[args.workload]
    if args.capacity_factor is not None:
        wl = wl.with_capacity_factor(args.capacity_factor)
    if args.tokens is not None:
        wl = wl.with_tokens(args.tokens)
    return wl


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
WIDE_WAVES = 12  # the library's GEMM2 tile waves from which GEMM1 runs as its own launch


def ffn_two_launches(wl, C, counts, pairs=74):
    """Whether a layer call runs GEMM1 as its own launch and the fused kernel does GEMM2 only (else
    the fused kernel does both and GEMM1's launch, if any, exits without work): the library's own
    rule, from the same counts (256-row blocks x 256-wide GEMM2 column tiles)."""
    mt = int(np.sum((np.minimum(counts, C) + 255) // 256))
    return mt * (-(-wl.d_model // 256)) >= WIDE_WAVES * pairs


def kernel_work(wl, C, counts, pairs=74, flags=0):
    """Algorithmic work per launch of each kernel of one step: (bound, amount,
    amount with every activation-sized tensor counted at the activation dtype).

    The layer writes y (and zero rows of dropped tokens) in float32; the third
    figure counts those bytes at the activation dtype instead (T*d*s for the
    output), which is the algorithmic byte count of the combine and the
    dispatch as the layer's step table states them.  Of the fused FFN kernel
    and the two-launch GEMMs, the ones that exit without work in a layer call
    (the library decides on the device from the counts) get no work here."""
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.num_experts
    s = 2 if wl.dtype == synth.BF16 else 4
    kept = np.minimum(counts, C)
    K = int(kept.sum())
    E_nz = int((kept > 0).sum())
    tiles = -(-T // 64)
    router_bytes = T * d * s + N * d * 4 + 8 * T + 8 * N * tiles
    assign_common = 4 * T + 4 * T + 4 * N * tiles + 4 * N * C + 2 * K * d * s
    return {
        "router_warp": ("hbm", router_bytes, None),
        "router_tiled": ("hbm", router_bytes, None),
        "router_staged": ("hbm", router_bytes, None),
        "router_tc": ("hbm", T * d * s + 3 * N * d * 2 + 8 * T + 8 * N * tiles, None),
        # the same kernel against its tensor-core work: three exact bf16 terms of W_r per token, the
        # experts padded to the tile width (64 or 128)
        "router_tc/tensor": ("tensor", 6.0 * T * d * (64 if N <= 64 else 128), None),
        "router_weight_split": ("hbm", N * d * 4 + 3 * N * d * 2, None),
        "capacity_scan": ("hbm", 8 * N * tiles + 4 * N * tiles + 12 * N, None),
        "slot_assign_scatter": ("hbm", assign_common + (T - K) * d * 4, assign_common + (T - K) * d * s),
        "ffn_tc_gemm1_relu": ("tensor", 2.0 * K * d * F, None),
        "ffn_tc_gemm2_gated_scatter": ("tensor", 2.0 * K * F * d, None),
        "ffn_tc_fused": ("tensor", 4.0 * K * d * F, None),
        "ffn_simt_gemm1_relu": ("alu", 2.0 * K * d * F, None),
        "ffn_simt_gemm2": ("alu", 2.0 * K * F * d, None),
        "combine": ("hbm", T * d * 4 + K * d * 4 + 12 * T, T * d * s + K * d * s + 12 * T),
        "dispatch": ("hbm", 2 * K * d * s + 4 * N * C + 4 * N, None),
        "_meta": ("", dict(K=K, E_nz=E_nz, gemm_weight_bytes=2 * E_nz * d * F * s), None),
    } | ({} if flags & (swm.SWITCH_FLAG_GEMM_1CTA | swm.SWITCH_FLAG_FFN_TWO_LAUNCHES) else  # no fused kernel
          {"ffn_tc_fused": ("tensor", 2.0 * K * F * d, None)} if ffn_two_launches(wl, C, counts, pairs) else
          {"ffn_tc_gemm1_relu": ("?", 0, None)})


def kernel_entry(kind, amount, amount_act, avg_ms, launches, peaks):
    """One kernel's achieved rate against the measured peaks."""
    entry = {"launches": launches, "avg_ms": round(avg_ms, 5), "share": None}
    sec = avg_ms * 1e-3
    if kind == "hbm":
        entry.update(bound="hbm", achieved=amount / sec / 1e9, peak=peaks["hbm_gbs"], unit="GB/s")
    elif kind == "tensor":
        entry.update(bound="tensor", achieved=amount / sec / 1e12, peak=peaks["bf16_tflops"], unit="TFLOP/s")
    elif kind == "alu":
        entry.update(bound="alu", achieved=amount / sec / 1e12, peak=74.4, unit="TFLOP/s")
    if "achieved" in entry:
        entry["frac"] = round(entry["achieved"] / entry["peak"], 4)
        entry["achieved"] = round(entry["achieved"], 2)
        if kind == "tensor" and "bf16_tflops_sustained" in peaks:
            entry["frac_sustained"] = round(entry["achieved"] / peaks["bf16_tflops_sustained"], 4)
        if amount_act is not None:
            # the same kernel with the float32 output rows counted at the activation dtype
            entry["achieved_act_dtype"] = round(amount_act / sec / 1e9, 2)
            entry["frac_act_dtype"] = round(amount_act / sec / 1e9 / entry["peak"], 4)
    return entry


DOMINANT_WORK_TEXT = {
    "ffn_tc_fused": "4*K*d_model*d_ff (K = kept tokens; both expert GEMMs), or 2*K*d_ff*d_model when GEMM1 "
                    "ran as its own launch (GEMM2 only)",
    "ffn_tc_gemm1_relu": "2*K*d_model*d_ff (K = kept tokens; the first expert GEMM)",
    "ffn_tc_gemm2_gated_scatter": "2*K*d_ff*d_model (K = kept tokens; the second expert GEMM)",
    "router_tc": "T*d*s + 6*N*d + 8*T + 8*N*ceil(T/64)",
    "router_staged": "T*d*s + 4*N*d + 8*T + 8*N*ceil(T/64)",
    "slot_assign_scatter": "8*T + 4*N*ceil(T/64) + 4*N*C + 2*K*d*s + 4*(T-K)*d",
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
    wl = workload_of(args)
    # experts and router are shared by all ranks; every rank routes its own tokens
    inp = dict(x=synth.activations(wl, seed=rank_seed(wl, rank)), w_r=synth.router_weight(wl),
               bias=synth.router_bias(wl))
    C = sm.switch_capacity(wl.T, wl.num_experts, wl.capacity_factor)
    experts = None
    if wl.zipf_s is not None:
        # Skewed routing sends every token to a few experts: draw the weights of the experts
        # that receive tokens (found by routing on the GPU) and leave the others zero.  The
        # layer never reads an expert without kept tokens, so the timed work is the same.
        r = sm.route(to_dev(inp["x"], device), to_dev(inp["w_r"], device), capacity=C,
                     logit_bias=to_dev(inp["bias"], device), d_ff=wl.d_ff)
        experts = np.flatnonzero(r["counts"].cpu().numpy() > 0)
        if world > 1:  # every rank holds the same experts: the union over ranks
            import torch.distributed as tdist
            mask = torch.zeros(wl.num_experts, dtype=torch.int32, device=device)
            mask[torch.from_numpy(experts).to(device)] = 1
            tdist.all_reduce(mask, op=tdist.ReduceOp.MAX)
            experts = np.flatnonzero(mask.cpu().numpy() > 0)
        del r
    inp["w_in"], inp["w_out"] = synth.all_expert_weights(wl, experts=experts)

    x = to_dev(inp["x"], device)
    w_r = to_dev(inp["w_r"], device)
    bias = to_dev(inp["bias"], device)
    w_in = to_dev(inp["w_in"], device)
    w_out = to_dev(inp["w_out"], device)
    dims = sm.layer_dims(x, w_in, capacity=C, flags=args.flags)
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
    work = kernel_work(wl, C, counts, torch.cuda.get_device_properties(device).multi_processor_count // 2,
                       args.flags)
    meta = work.pop("_meta")[1]
    peaks, peak_src = load_peaks()
    kernels = {}
    for name, times in per_kernel.items():
        kind, amount, amount_act = work.get(name, ("?", 0, None))
        kernels[name] = kernel_entry(kind, amount, amount_act, statistics.mean(times), len(times), peaks)
        if name + "/tensor" in work:  # a second roofline for the same kernel
            t_kind, t_amount, _ = work[name + "/tensor"]
            t = kernel_entry(t_kind, t_amount, None, statistics.mean(times), len(times), peaks)
            kernels[name]["tensor_achieved_tflops"] = t["achieved"]
            kernels[name]["frac_tensor"] = t["frac"]
    tot = sum(k["avg_ms"] * k["launches"] for k in kernels.values())
    for k in kernels.values():
        k["share"] = round(k["avg_ms"] * k["launches"] / tot, 4) if tot else None
    dominant = max(kernels, key=lambda n: kernels[n]["avg_ms"] * kernels[n]["launches"]) if kernels else None
    roofline = None
    if dominant and "achieved" in kernels[dominant]:
        k = kernels[dominant]
        roofline = {"kernel": dominant, "bound": k["bound"], "achieved": k["achieved"], "peak": k["peak"],
                    "unit": k["unit"], "frac": k["frac"], "traffic": traffic_from_profiles(dominant, wl.name),
                    "units_per_launch": ("flops" if k["bound"] in ("tensor", "alu") else "bytes") + " = " +
                                        DOMINANT_WORK_TEXT.get(dominant, "see kernel_work"),
                    "peak_source": (f"{peak_src} (burst bf16 matmul)" if k["bound"] == "tensor" else
                                    f"{peak_src} (copy bandwidth)" if k["bound"] == "hbm" else
                                    "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz (FFMA issue rate)")}
        if "frac_sustained" in k:
            roofline["frac_sustained"] = k["frac_sustained"]
            roofline["peak_sustained"] = peaks.get("bf16_tflops_sustained")
        if clocks and clocks.get("sm_mhz"):
            roofline["sm_mhz_median"] = clocks["sm_mhz"]

    # e2e through the public API with pinned host buffers
    e2e = run_e2e(args, sm, wl, inp, C, device, world)

    # the top-2 variant of the layer on the same tokens and weights
    top2 = time_top2(args, sm, wl, x, w_r, bias, w_in, w_out, C, flush, stream, device) \
        if (world == 1 and not args.no_top2 and wl.num_experts >= 2) else None

    # the backward pass (training forward + switch_layer_bwd) on the same tokens and weights
    backward = time_backward(args, sm, wl, x, w_r, bias, w_in, w_out, C, flush, stream, device) \
        if (world == 1 and not args.no_backward and wl.dtype == synth.BF16) else None

    # standalone dispatch and combine entry points on the same workload
    entry_points = time_entry_points(sm, wl, x, w_r, bias, C, flush, stream, device) if world == 1 else None

    # capacity-factor sweep of the large-expert layer (its own inputs)
    sweep = run_sweep(args, sm, device, flush, stream) if (world == 1 and not args.no_sweep) else None

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
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       **({"flags": args.flags} if args.flags else {})},
            "roofline": roofline,
            "kernels": kernels,
            "gpu_launches": int(launches),
            "traced_ms_per_step": round(traced_ms_per_step, 5),
            "e2e": e2e,
            "clocks": clocks,
            "wall_s_timed_region": round(t_wall1 - t_wall0, 4),
        }
        if top2:
            result["top2"] = top2
        if backward:
            result["backward"] = backward
        if entry_points:
            result["entry_points"] = entry_points
        if sweep:
            result["sweep"] = sweep
        if not args.no_cpu_baseline and world == 1:
            result["cpu_baseline"] = cpu_baseline(wl, inp, C, budget_s=args.cpu_budget)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def _time_events(fn, flush, stream, reps):
    """Average CUDA-event time of fn() over reps calls, L2 flushed before each (outside the events)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i in range(reps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / reps


def time_top2(args, sm, wl, x, w_r, bias, w_in, w_out, C, flush, stream, device):
    """The top-2 layer (switch_layer_fwd_top2) on the workload's tensors: ms per
    step, tokens/s and each kernel's fraction of its roofline."""
    import torch
    T = wl.T
    out = sm.layer_fwd_top2(x, w_r, w_in, w_out, capacity=C, logit_bias=bias)
    ws = out["workspace"]
    fn = lambda: sm.layer_fwd_top2(x, w_r, w_in, w_out, capacity=C, logit_bias=bias, ws=ws, out=out)
    for _ in range(args.warmup):
        flush.fill_(1.0)
        fn()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 20))
    ms = _time_events(fn, flush, stream, steps)
    sm.trace_start(steps * 8)
    _time_events(fn, flush, stream, steps)
    trace = sm.trace_read(steps * 8)
    sm.trace_stop()
    if sm.switch_check(ws) != 0:
        raise RuntimeError("device status after the top-2 steps")
    counts = out["counts"].cpu().numpy()
    kept = np.minimum(counts, C)
    K = int(kept.sum())
    s = x.element_size()
    d, F, N = wl.d_model, wl.d_ff, wl.num_experts
    tiles = -(-T // 64)
    work = {
        "router_tc": ("hbm", T * d * s + 3 * N * d * 2 + 16 * T + 12 * N * tiles, None),
        "router_staged": ("hbm", T * d * s + 4 * N * d + 16 * T + 12 * N * tiles, None),
        "router_tiled": ("hbm", T * d * s + 4 * N * d + 16 * T + 12 * N * tiles, None),
        "router_weight_split": ("hbm", N * d * 4 + 3 * N * d * 2, None),
        "capacity_scan": ("hbm", 20 * N * tiles + 12 * N, None),
        "slot_assign_scatter": ("hbm", 16 * T + 8 * N * tiles + 4 * N * C + 2 * K * d * s, None),
        "ffn_tc_gemm1_relu": ("tensor", 2.0 * K * d * F, None),
        "ffn_tc_gemm2": ("tensor", 2.0 * K * F * d, None),
        "combine_top2": ("hbm", T * d * 4 + K * d * 4 + 24 * T, T * d * s + K * d * s + 24 * T),
    }
    peaks, _ = load_peaks()
    per_kernel: dict[str, list[float]] = {}
    for name, kms in trace:
        per_kernel.setdefault(name, []).append(kms)
    kernels = {}
    for name, times in per_kernel.items():
        kind, amount, amount_act = work.get(name, ("?", 0, None))
        kernels[name] = kernel_entry(kind, amount, amount_act, statistics.mean(times), len(times) // steps, peaks)
    result = {"ms_per_step": round(ms, 5), "value": round(T / (ms * 1e-3), 1), "unit": UNIT, "steps": steps,
              "capacity": C, "kept_assignments": K, "dropped_assignments": int(2 * T - K),
              "expert_flops_per_step": 4.0 * K * d * F, "kernels": kernels}
    del out, ws
    torch.cuda.empty_cache()
    return result


def time_backward(args, sm, wl, x, w_r, bias, w_in, w_out, C, flush, stream, device):
    """A training step of the layer: the training forward (SWITCH_FLAG_TRAINING) and
    switch_layer_bwd with a fixed upstream gradient, timed together and per kernel."""
    import torch
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.num_experts
    dy = torch.randn(T, d, device=device, generator=torch.Generator(device).manual_seed(7))
    fwd = sm.layer_fwd(x, w_r, w_in, w_out, capacity=C, logit_bias=bias, flags=sm.SWITCH_FLAG_TRAINING)
    grads = sm.layer_bwd(fwd, x, w_r, w_in, w_out, dy, 0.01, logit_bias=bias)

    def step():
        sm.layer_fwd(x, w_r, w_in, w_out, capacity=C, logit_bias=bias, flags=sm.SWITCH_FLAG_TRAINING,
                     ws=fwd["workspace"], out=fwd)
        d_ = sm.layer_dims(x, w_in, capacity=C, flags=sm.SWITCH_FLAG_TRAINING)
        sm.switch_layer_bwd(d_, x, w_r, w_in, w_out, fwd["expert"], fwd["gate"], fwd["slot"], fwd["counts"], dy,
                            0.01, grads["dx"], grads["dw_r"], grads["dbias"], grads["dw_in"], grads["dw_out"],
                            fwd["workspace"])
    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    ms = _time_events(step, flush, stream, steps)
    sm.trace_start(steps * 32)
    _time_events(step, flush, stream, steps)
    trace = sm.trace_read(steps * 32)
    sm.trace_stop()
    if sm.switch_check(fwd["workspace"]) != 0:
        raise RuntimeError("device status after the backward steps")
    K = int(np.minimum(fwd["counts"].cpu().numpy(), C).sum())
    s = x.element_size()
    per_kernel: dict[str, list[float]] = {}
    for name, kms in trace:
        per_kernel.setdefault(name, []).append(kms)
    Np = -(-N // 64) * 64
    Tc = max(256, -(-(-(-T // 64)) // 128) * 128)                       # tokens per dW_r chunk
    chunks = -(-T // Tc)
    kept_e = np.minimum(fwd["counts"].cpu().numpy().astype(np.int64), C)
    tails = np.where(kept_e > 0, np.minimum(C, -(-kept_e // 64) * 64) - kept_e, 0)
    zero_tails = int(tails.sum()) * (2 * d + 2 * F) * s  # rows zeroed in dE, xbuf, H and dZ
    # the router operand splits: dh -> [T][6 Np] and W_r -> [d][6 Np] (dx), dh -> [3N][chunk tokens] (dW_r)
    splits = (4 * T * N + 2 * T * 6 * Np) + (4 * N * d + 2 * d * 6 * Np) + (4 * T * N + 2 * 3 * N * chunks * Tc)
    work = {
        "bwd_gate_softmax": ("hbm", 4 * T * d + 4 * K * d + 2 * K * d + 8 * T * N, None),
        "bwd_tc_gemm_dz": ("tensor", 2.0 * K * d * F, None),
        "bwd_tc_gemm_dx": ("tensor", 2.0 * K * F * d, None),
        "bwd_tc_gemm_dw": ("tensor", 2.0 * K * d * F, None),
        "bwd_router_dx": ("alu", 2.0 * T * N * d, None),
        "bwd_router_dw": ("alu", 2.0 * T * N * d, None),
        # bf16 MMA flops executed on the exact splits: six term pairs (dx), three dh terms (dW_r)
        "bwd_router_tc_dx": ("tensor", 2.0 * T * d * 6 * N, None),
        "bwd_router_tc_dw": ("tensor", 2.0 * T * d * 3 * N, None),
        "ffn_tc_gemm1_relu": ("tensor", 2.0 * K * d * F, None),
        "ffn_tc_gemm2": ("tensor", 2.0 * K * F * d, None),
    }
    peaks, _ = load_peaks()
    kernels = {}
    for name, times in per_kernel.items():
        n_per_step = len(times) // steps
        if name in ("bwd_router_split", "bwd_zero_tails"):
            total = splits if name == "bwd_router_split" else zero_tails
            kernels[name] = kernel_entry("hbm", total / max(n_per_step, 1), None, statistics.mean(times),
                                         n_per_step, peaks)
            continue
        kind, amount, amount_act = work.get(name, ("?", 0, None))
        kernels[name] = kernel_entry(kind, amount, amount_act, statistics.mean(times), n_per_step, peaks)
    tot = sum(k["avg_ms"] * k["launches"] for k in kernels.values())
    for k in kernels.values():
        k["share"] = round(k["avg_ms"] * k["launches"] / tot, 4) if tot else None
    result = {"ms_per_step": round(ms, 5), "value": round(T / (ms * 1e-3), 1), "unit": UNIT,
              "what": "training forward (SWITCH_FLAG_TRAINING) + switch_layer_bwd per step", "steps": steps,
              "kept_tokens": K, "expert_flops_per_step": 12.0 * K * d * F, "kernels": kernels}
    del fwd, grads, dy
    torch.cuda.empty_cache()
    return result


def time_entry_points(sm, wl, x, w_r, bias, C, flush, stream, device, reps=10):
    """switch_dispatch and switch_combine called on their own (the layer path
    fuses both into its neighbours), timed with CUDA events, with their
    achieved HBM bandwidth over the algorithmic bytes."""
    import torch
    T, d, N = wl.T, wl.d_model, wl.num_experts
    r = sm.route(x, w_r, capacity=C, logit_bias=bias, d_ff=wl.d_ff)
    if sm.switch_check(r["workspace"]) != 0:
        raise RuntimeError("device status after route")
    dims = sm.dims(T, d, wl.d_ff, N, C, x.dtype)
    xbuf = torch.empty(N * C * d, dtype=x.dtype, device=device)
    ybuf = torch.randn(N * C * d, dtype=torch.float32, device=device)
    y = torch.empty(T, d, dtype=torch.float32, device=device)
    counts = r["counts"]
    for _ in range(3):
        sm.switch_dispatch(dims, x, r["slot_token"], counts, xbuf)
        sm.switch_combine(dims, ybuf, r["expert"], r["slot"], r["gate"], y)
    torch.cuda.synchronize()
    ms_d = _time_events(lambda: sm.switch_dispatch(dims, x, r["slot_token"], counts, xbuf), flush, stream, reps)
    ms_c = _time_events(lambda: sm.switch_combine(dims, ybuf, r["expert"], r["slot"], r["gate"], y), flush,
                        stream, reps)
    K = int(torch.clamp(counts, max=C).sum().item())
    s = x.element_size()
    peaks, _ = load_peaks()
    bytes_d = 2 * K * d * s + 4 * N * C + 4 * N
    bytes_c = T * d * 4 + K * d * 4 + 12 * T
    bytes_c_act = T * d * s + K * d * s + 12 * T
    out = {}
    for name, ms, b, b_act in (("dispatch", ms_d, bytes_d, None), ("combine", ms_c, bytes_c, bytes_c_act)):
        e = kernel_entry("hbm", b, b_act, ms, reps, peaks)
        e.pop("share", None)
        e["bytes"] = b
        out[name] = e
    del xbuf, ybuf, y, r
    torch.cuda.empty_cache()
    return out


def run_sweep(args, sm, device, flush, stream):
    """The large-expert layer at every capacity factor of its sweep, on one
    seeded input: ms per step, tokens/s, kept tokens and drop fraction per c.

    With the Zipf(0.8) logit bias only a few experts receive tokens; the
    weights of the others are left as zeros on the device (the layer never
    reads an expert without kept tokens), which spares drawing ~10 GB of
    random weights on the host."""
    import torch
    wl = synth.WORKLOADS[SWEEP_WORKLOAD]
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.num_experts
    x = to_dev(synth.activations(wl), device)
    w_r = to_dev(synth.router_weight(wl), device)
    bias = to_dev(synth.router_bias(wl), device)
    r = sm.route(x, w_r, capacity=1, logit_bias=bias, d_ff=F)
    if sm.switch_check(r["workspace"]) != 0:
        raise RuntimeError("device status after route")
    used = np.flatnonzero(r["counts"].cpu().numpy() > 0)
    del r
    w_in = torch.zeros(N, F, d, dtype=x.dtype, device=device)
    w_out = torch.zeros(N, d, F, dtype=x.dtype, device=device)
    for e in used:
        wi, wo = synth.expert_weights(wl, int(e))
        w_in[int(e)].copy_(to_dev(wi, device))
        w_out[int(e)].copy_(to_dev(wo, device))
    steps = max(3, min(args.steps, 20))
    out = {"workload": wl.name, "T": T, "d_model": d, "d_ff": F, "num_experts": N,
           "nonzero_weight_experts": int(used.size), "steps": steps, "points": []}
    for c in wl.sweep:
        Cc = sm.switch_capacity(T, N, c)
        dc = sm.layer_dims(x, w_in, capacity=Cc)
        wsc = sm.workspace(dc, device)
        outc = sm.layer_fwd(x, w_r, w_in, w_out, capacity=Cc, logit_bias=bias, ws=wsc)
        fn = lambda: sm.layer_fwd(x, w_r, w_in, w_out, capacity=Cc, logit_bias=bias, ws=wsc, out=outc)
        for _ in range(args.warmup):
            flush.fill_(1.0)
            fn()
        torch.cuda.synchronize()
        ms = _time_events(fn, flush, stream, steps)
        if sm.switch_check(wsc) != 0:
            raise RuntimeError("device status after the sweep steps")
        kept = int(np.minimum(outc["counts"].cpu().numpy(), Cc).sum())
        out["points"].append({"capacity_factor": c, "capacity": Cc, "ms_per_step": round(ms, 5),
                              "value": round(T / (ms * 1e-3), 1), "unit": UNIT, "kept_tokens": kept,
                              "drop_fraction": round(1 - kept / T, 6),
                              "expert_flops_per_step": 4.0 * kept * d * F})
        del wsc, outc
        torch.cuda.empty_cache()
    del x, w_r, bias, w_in, w_out
    torch.cuda.empty_cache()
    return out


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
def _oracle_sample(orc, wl, inp, C, budget_s, route_tokens=None):
    """Oracle time per token: routing (logits, softmax, top-1) on the first
    `route_tokens` tokens (all when None) plus the capacity assignment and
    aux on all ids, and the expert FFN on a growing prefix of the kept tokens
    until about budget_s; returns (seconds extrapolated to the whole
    workload, description)."""
    T = wl.T
    n_route = T if route_tokens is None else min(T, route_tokens)
    x = inp["x"]
    t0 = time.perf_counter()
    h = orc.router_logits(x[:n_route], inp["w_r"], inp["bias"])
    r = orc.softmax_top1(h)
    t_route = time.perf_counter() - t0
    if n_route == T:
        ids = r["expert"]
    else:  # ids of the tokens not routed here come from a full routing done outside the timing
        ids = inp["_oracle_expert"]
    t1 = time.perf_counter()
    a = orc.assign(ids, wl.num_experts, C)
    orc.aux(T, a["counts"], np.zeros(wl.num_experts))
    t_assign = time.perf_counter() - t1
    kept = np.flatnonzero(a["slot"] >= 0)
    gate = np.ones(T)
    n, t_ffn, done = 16, 0.0, 0
    while done < kept.size and t_ffn < budget_s:
        rows = kept[done:done + n]
        t2 = time.perf_counter()
        orc.output_rows(rows, x, inp["w_in"], inp["w_out"], ids, a["slot"], gate)
        t_ffn += time.perf_counter() - t2
        done += rows.size
        n = min(n * 2, kept.size)
    est = t_route * T / n_route + t_assign + (t_ffn / max(done, 1)) * kept.size
    desc = (f"routing on {n_route} of {T} tokens ({t_route:.2f} s), assignment + aux on all ({t_assign:.2f} s), "
            f"expert FFN on {done} of {kept.size} kept tokens ({t_ffn:.2f} s); extrapolated to the whole workload")
    return est, desc, t_route + t_assign + t_ffn


def cpu_baseline(wl, inp, C, budget_s=15.0, one_core=True):
    """Time the fp64 oracle on the host cores over a bounded sample of the
    workload, extrapolated to tokens/s of the whole workload: once with all
    host threads and once on a single core."""
    import oracle
    orc = oracle.Oracle()
    all_threads = orc.threads()
    est, desc, measured = _oracle_sample(orc, wl, inp, C, budget_s)
    out = {"value": round(wl.T / est, 2), "unit": UNIT, "cores": all_threads, "kind": "oracle",
           "sample": desc, "seconds_measured": round(measured, 2)}
    if one_core:
        if "_oracle_expert" not in inp:
            inp["_oracle_expert"] = orc.softmax_top1(orc.router_logits(inp["x"], inp["w_r"], inp["bias"]))["expert"]
        orc.set_threads(1)
        try:
            est1, desc1, measured1 = _oracle_sample(orc, wl, inp, C, budget_s / 3, route_tokens=2048)
        finally:
            orc.set_threads(all_threads)
        out["one_core"] = {"value": round(wl.T / est1, 2), "unit": UNIT, "cores": 1, "sample": desc1,
                           "seconds_measured": round(measured1, 2)}
    return out


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    wl = workload_of(args)
    inp = synth.inputs(wl)
    import oracle
    orc = oracle.Oracle()
    C = orc.capacity(wl.T, wl.num_experts, wl.capacity_factor)
    budget = max(1.0, args.cpu_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(wl, inp, C, budget_s=budget, one_core=False)
    vals = [cpu_baseline(wl, inp, C, budget_s=budget, one_core=False) for _ in range(args.steps)]
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--capacity-factor", type=float, default=None)
    ap.add_argument("--tokens", type=int, default=None, help="token count override (small profiler captures)")
    ap.add_argument("--flags", type=int, default=0, help="SWITCH_FLAG_* bits for the timed layer (diagnostic paths)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle FFN time for cpu_baseline")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-top2", action="store_true", help="skip timing the top-2 variant of the layer")
    ap.add_argument("--no-backward", action="store_true", help="skip timing the backward pass")
    ap.add_argument("--no-sweep", action="store_true",
                    help=f"skip the capacity-factor sweep of the {SWEEP_WORKLOAD} workload")
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
