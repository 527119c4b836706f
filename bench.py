#!/usr/bin/env python
"""Benchmark of the gated bidirectional TTT-MLP layer on B200.

One step = one full layer (fused Q/K/V projections, forward scan with gate,
reverse projections, reverse scan with gate) over one synthetic 313,344-token
sequence of width 3072 (48 heads, d = 64, hidden 256, b = 64), inputs already
resident in HBM.  Multi-GPU (torchrun): each rank runs its own sequence
(independent replicas, weak scaling, no collective on the data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--model mlp|linear]

Prints one JSON line on rank 0.  --model linear measures the TTT-Linear layer
(f(u; W) = W u) on the same sequence instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "TTT-MLP tokens/s (48 heads, bidirectional) at T≈313k; % of roofline"
METRIC_LINEAR = "TTT-Linear tokens/s (48 heads, bidirectional) at T≈313k; % of roofline"
UNIT = "tokens/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "traffic.json")
# Fallback peaks of the profiling recipe (used only if MEASURED_PEAKS.json is absent).
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
TF32_PER_BF16 = 1.1 / 2.25          # nominal dense tf32 / bf16 ratio
N_SM, FP32_LANES = 148, 128         # FP32 FMA lanes per SM


# ------------------------------------------------------------------ helpers
def _peaks():
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        p["_source"] = "measured"
        return p
    p = dict(FALLBACK)
    p["_source"] = "fallback"
    return p


def _src_hash(*files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "test_rnn_layer_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# kernel name -> source files whose content the ncu traffic figure belongs to
KERNEL_SRC = {
    "scan_chunk_simt": ("scan_chunk_simt.cu",),
    "scan_chunk_tc": ("scan_chunk_tc.cu",),
    "scan_chunk_tc2": ("scan_chunk_tc2.cu",),
    "scan_token": ("scan_token.cu",),
    "proj_full_simt": ("proj_simt.cu",),
    "proj_full_tc": ("proj_tc.cu",),
    "proj_per_head": ("proj_simt.cu",),
    "gate": ("gate.cu",),
    "scan_linear": ("scan_linear.cu",),
    "scan_linear_tc": ("scan_linear_tc.cu",),
}


def _traffic(name: str, units_scale: float):
    """DRAM bytes per launch of `name` from the committed ncu summary, or None
    if absent or taken on a different version of the kernel's source."""
    try:
        with open(TRAFFIC_PATH) as f:
            rec = json.load(f).get(name)
        if not rec or rec.get("src_hash") != _src_hash(*KERNEL_SRC[name]):
            return None
        return rec["bytes_per_launch_per_unit"] * units_scale
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks/throttle reasons every 200 ms for one GPU (by UUID)."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons, power = [], None, set(), []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8 or (self.uuid and parts[0] != self.uuid):
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------ workload
def _workload(args):
    from test_rnn_layer_b200 import synth as S
    w = S.FULL63S
    if args.T:
        w = w.with_T(args.T)
    return w


def _config(w, extra=None):
    cfg = {"workload": w.name, "T": w.T, "D": w.model_dim, "H": w.H, "d": w.d, "hidden": w.m, "b": w.b,
           "dirs": w.dirs, "x_dtype": w.dtype, "state": "fp32", "eta": f"{w.eta}/d", "alpha": w.alpha,
           "inputs": "seeded Gaussian stand-ins for video tokens (X~N(0,1), theta~N(0,1/D), W1_0~N(0,1/d), "
                     "W2_0~N(0,1/4d))",
           "l2": "no flush: every input is larger than the 126 MB L2 (X 1.9 GB, Q/K/V 11.5 GB)",
           "parallelism": "replicas (one sequence per GPU)"}
    if extra:
        cfg.update(extra)
    return cfg


def _algorithmic(w):
    """Algorithmic work of each kernel kind over one direction of the layer
    (all of that direction's launches together)."""
    T, D, H, d, m, b = w.T, w.model_dim, w.H, w.d, w.m, w.b
    scan_flops = H * T * (7 * 2 * d * m + 2 * b * (d + m))
    proj_flops = 2.0 * T * D * 3 * D
    return {
        "scan_chunk_tc": ("tensor_tf32", scan_flops),
        "scan_chunk_tc2": ("tensor_tf32", scan_flops),
        "scan_chunk_simt": ("alu", scan_flops),
        "scan_token": ("alu", H * T * 7 * 2 * d * m),
        "proj_full_tc": ("tensor_bf16", proj_flops),
        "proj_full_simt": ("alu", proj_flops),
        "proj_per_head": ("hbm", T * D * (2 + 12)),
        # forward: x bf16 + z fp32 read, X' fp32 + bf16 increment written (12 B);
        # reverse: X' fp32 + z fp32 read, Y bf16 written (10 B); 11 B on average
        "gate": ("hbm", T * D * 11),
        # TTT-Linear per head-token: e = W_c k (2 d^2), update (2 d^2), z = W q (2 d^2)
        "scan_linear": ("alu", H * T * 6 * d * d),
        # chunk form on the tensor cores: W K^T, W Q^T, update (3 x 2 d^2) + Q K^T and the masked
        # correction (2 x 2 b d over the causal half)
        "scan_linear_tc": ("tensor_tf32", H * T * (6 * d * d + 2 * b * d)),
    }


def _roofline(name, ms_per_launch, launches_per_step, w, peaks, clocks):
    """Roofline of one launch of `name`: the step's algorithmic work for that
    kernel (both directions for a bidirectional layer) divided evenly over its
    launches, against the average launch duration."""
    bound, work_dir = _algorithmic(w)[name]
    ndir = 2 if w.dirs == "bidir" else 1
    work = work_dir * ndir / launches_per_step
    sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    src = "of " + peaks["_source"]
    if bound == "tensor_bf16":
        peak, unit, kind, note = sus, "TFLOP/s", "tensor", f"bf16 dense sustained {src}"
        achieved = work / (ms_per_launch * 1e-3) / 1e12
    elif bound == "tensor_tf32":
        peak, unit, kind = sus * TF32_PER_BF16, "TFLOP/s", "tensor"
        note = f"tf32 dense = bf16 sustained {src} x 1.1/2.25 (nominal ratio)"
        achieved = work / (ms_per_launch * 1e-3) / 1e12
    elif bound == "alu":
        mhz = peaks.get("sm_max_mhz", 1965.0)
        peak = N_SM * FP32_LANES * 2 * mhz * 1e6 / 1e12
        unit, kind, note = "TFLOP/s", "alu", f"FP32 FMA: 148 SM x 128 lanes x 2 x {mhz:.0f} MHz"
        achieved = work / (ms_per_launch * 1e-3) / 1e12
    else:
        peak, unit, kind, note = peaks["hbm_gbs"], "GB/s", "hbm", f"HBM copy {src}"
        achieved = work / (ms_per_launch * 1e-3) / 1e9
    units = w.T * ndir / launches_per_step / 1024.0   # traffic records are stored per 1024 tokens
    return {"kernel": name, "bound": kind, "achieved": round(achieved, 3), "peak": round(peak, 2), "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": _traffic(name, units), "peak_note": note,
            "ms_per_launch": round(ms_per_launch, 4), "work_per_launch": work}


# ------------------------------------------------------------------ multi-rank bookkeeping
def rank_seed(rank: int) -> int:
    """Each replica draws its own sequence."""
    return rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (all ranks call this in the same order)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Tokens of all replicas per second, timed by the slowest rank."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


# ------------------------------------------------------------------ CPU side (oracle)
def _cpu_sample(w, tokens: int, seed: int = 0):
    """A bounded sample of the workload for the fp64 oracle: the first `tokens`
    tokens of the sequence, forward direction, `heads` heads (one OpenMP thread
    each), with their share of the projections."""
    import numpy as np
    import torch

    from oracle import ttt_oracle as O
    from test_rnn_layer_b200 import synth as S

    threads = O.num_threads()
    heads = list(range(min(w.H, threads)))
    inp = S.make_inputs(w.with_T(tokens), seed=seed, device="cpu")
    X = inp["X"].float().numpy()
    th = [inp[k].float().numpy() for k in ("theta_q", "theta_k", "theta_v")]
    W1, W2 = inp["W1_0"].double().numpy(), inp["W2_0"].double().numpy()

    def run():
        t0 = time.perf_counter()
        O.full_mode_heads(X, *th, W1, W2, w.eta_eff, w.b, heads)
        return time.perf_counter() - t0

    # metric units: tokens through all H heads in both directions
    scale = len(heads) / (w.H * 2.0)
    sample = (f"first {tokens} tokens, {len(heads)} of {w.H} heads, forward direction only (fp64 oracle incl. "
              f"those heads' Q/K/V projections); tokens/s scaled by {len(heads)}/({w.H}*2)")
    return run, scale, threads, sample


def _cpu_sample_linear(w, tokens: int, seed: int = 0):
    """As _cpu_sample, for the TTT-Linear layer."""
    import numpy as np

    from oracle import ttt_oracle as O
    from test_rnn_layer_b200 import synth as S

    threads = O.num_threads()
    heads = list(range(min(w.H, threads)))
    inp = S.make_linear_inputs(w.with_T(tokens), seed=seed, device="cpu")
    X = inp["X"].float().numpy()
    rows = np.concatenate([np.arange(h * w.d, (h + 1) * w.d) for h in heads])
    th = [inp[k].float().numpy()[rows] for k in ("theta_q", "theta_k", "theta_v")]
    W0 = inp["W_0"].double().numpy()[heads]

    def run():
        t0 = time.perf_counter()
        Q, K, V = [O.project_full(X, t).reshape(tokens, len(heads), w.d).transpose(1, 0, 2) for t in th]
        O.linear_scan_heads(Q, K, V, W0, w.eta_eff, w.b)
        return time.perf_counter() - t0

    scale = len(heads) / (w.H * 2.0)
    sample = (f"first {tokens} tokens, {len(heads)} of {w.H} heads, forward direction only (fp64 TTT-Linear "
              f"oracle incl. those heads' Q/K/V projections); tokens/s scaled by {len(heads)}/({w.H}*2)")
    return run, scale, threads, sample


# ------------------------------------------------------------------ arms
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = _workload(args)
    tokens = args.ref_tokens
    run, scale, threads, sample = (_cpu_sample_linear if args.model == "linear" else _cpu_sample)(w, tokens)
    for _ in range(args.warmup):
        run()
    times = [run() for _ in range(args.steps)]
    step_s = sum(times) / len(times)
    value = tokens * scale / step_s
    line = {"impl": "reference", "metric": METRIC_LINEAR if args.model == "linear" else METRIC, "value": value,
            "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, {"sample": sample}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from test_rnn_layer_b200 import synth as S
    from test_rnn_layer_b200 import tttmlp as L

    L.lib()   # loud failure if the CUDA library is missing
    if args.kernels == "simt":
        L.check(L.ttt_mlp_select_kernels(1, 1), "ttt_mlp_select_kernels")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = _workload(args)
    inp = S.make_inputs(w, seed=rank_seed(rank), device=dev)
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    direction = L.DIRS[w.dirs]
    ws = L.alloc_workspace(desc, w.b, direction, dev, host_io=True)
    ws_dev_bytes = L.ttt_mlp_workspace_size(desc, w.b, direction)
    Y = torch.empty_like(inp["X"])
    stream = torch.cuda.current_stream()

    def step():
        st = L.ttt_mlp_forward(desc, inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"],
                               inp["W2_0"], w.eta_eff, w.b, direction, inp["alpha_f"], inp["alpha_r"], Y, None, None,
                               None, ws, ws_dev_bytes, stream)
        if st != L.TTT_OK:
            raise L.TTTError(st, "ttt_mlp_forward")

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    L.check(L.ttt_mlp_status(ws, stream), "warm-up status")

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    n_launch0 = L.ttt_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = L.ttt_launch_count() - n_launch0
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    L.check(L.ttt_mlp_status(ws, stream), "timed-run status")
    ms_per_step = ms / args.steps
    value = whole_job_tokens_per_s(world, w.T, ms_per_step)

    # per-kernel device times over a second timed pass (events on the launch stream)
    L.ttt_kernel_timing(True)
    kpass = max(1, min(args.steps, 3))
    for _ in range(kpass):
        step()
    torch.cuda.synchronize()
    ktimes = L.ttt_kernel_times()
    L.ttt_kernel_timing(False)
    total = sum(v[0] for v in ktimes.values()) or 1.0
    top = max(ktimes, key=lambda k: ktimes[k][0])
    peaks = _peaks()
    roof = _roofline(top, ktimes[top][0] / ktimes[top][1], ktimes[top][1] / kpass, w, peaks, clocks)
    roof["share"] = round(ktimes[top][0] / total, 4)   # of the summed kernel time (streams overlap)
    roof["ms_per_step"] = round(ktimes[top][0] / kpass, 3)
    kernels = {k: {"ms_per_step": round(v[0] / kpass, 3), "launches_per_step": v[1] // kpass,
                   "share": round(v[0] / total, 4)} for k, v in ktimes.items()}

    # end to end through the public host-buffer entry point: H2D of X, layer, D2H of Y
    e2e = None
    if not args.no_e2e:
        Xh = inp["X"].cpu().pin_memory()
        Yh = torch.empty_like(Xh).pin_memory()
        ns = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            st = L.ttt_mlp_forward_host(desc, Xh, inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"],
                                        inp["W2_0"], w.eta_eff, w.b, direction, inp["alpha_f"], inp["alpha_r"], Yh, ws,
                                        ws.numel(), stream)
            L.check(st, "ttt_mlp_forward_host")

        e2e_step()
        barrier()
        t0 = time.perf_counter()
        for _ in range(ns):
            e2e_step()
        barrier()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev) / ns
        nbytes = Xh.numel() * Xh.element_size()
        e2e = {"value": whole_job_tokens_per_s(world, w.T, e2e_s * 1e3), "unit": UNIT, "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "ms_per_step": e2e_s * 1e3, "steps": ns}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        run, scale, threads, sample = _cpu_sample(w, args.cpu_tokens)
        t = run()
        cpu = {"value": args.cpu_tokens * scale / t, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": sample, "seconds": round(t, 2)}

    if rank == 0:
        scan_impl = "tensor-core" if any(k.endswith("_tc") for k in ktimes) else "simt"
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": "bf16-in/tf32-mma/fp32-state" if scan_impl == "tensor-core" else "fp32",
                "data": "synthetic",
                "config": _config(w, {"kernels": scan_impl}), "gpu_launches": launches,
                "clocks": clocks, "roofline": roof, "kernels": kernels, "e2e": e2e, "cpu_baseline": cpu,
                "impl": "ours"}
        print(json.dumps(line), flush=True)
    return 0


def run_ours_linear(args, rank, world, local_rank):
    """The TTT-Linear layer on the same sequence (fp32 scan), same JSON line."""
    import torch

    from test_rnn_layer_b200 import synth as S
    from test_rnn_layer_b200 import tttmlp as L

    L.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = _workload(args)
    inp = S.make_linear_inputs(w, seed=rank_seed(rank), device=dev)
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    direction = L.DIRS[w.dirs]
    n_ws = L.ttt_linear_workspace_size(desc, w.b, direction)
    ws = torch.empty(n_ws, dtype=torch.uint8, device=dev)
    Y = torch.empty_like(inp["X"])
    stream = torch.cuda.current_stream()

    def step(X=None, Yo=None):
        st = L.ttt_linear_forward(desc, inp["X"] if X is None else X, inp["theta_q"], inp["theta_k"],
                                  inp["theta_v"], inp["W_0"], w.eta_eff, w.b, direction, inp["alpha_f"],
                                  inp["alpha_r"], Y if Yo is None else Yo, None, None, ws, n_ws, stream)
        L.check(st, "ttt_linear_forward")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    L.check(L.ttt_mlp_status(ws, stream), "warm-up status")
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    n_launch0 = L.ttt_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = L.ttt_launch_count() - n_launch0
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    L.check(L.ttt_mlp_status(ws, stream), "timed-run status")
    ms_per_step = ms / args.steps
    value = whole_job_tokens_per_s(world, w.T, ms_per_step)

    L.ttt_kernel_timing(True)
    kpass = max(1, min(args.steps, 3))
    for _ in range(kpass):
        step()
    torch.cuda.synchronize()
    ktimes = L.ttt_kernel_times()
    L.ttt_kernel_timing(False)
    total = sum(v[0] for v in ktimes.values()) or 1.0
    peaks = _peaks()
    scan = "scan_linear_tc" if "scan_linear_tc" in ktimes else "scan_linear"
    roof = _roofline(scan, ktimes[scan][0] / ktimes[scan][1], ktimes[scan][1] / kpass, w, peaks, clocks)
    roof["share"] = round(ktimes[scan][0] / total, 4)
    kernels = {k: {"ms_per_step": round(v[0] / kpass, 3), "launches_per_step": v[1] // kpass,
                   "share": round(v[0] / total, 4)} for k, v in ktimes.items()}

    e2e = None
    if not args.no_e2e:   # pinned host X in, host Y out, through the device entry point
        Xh = inp["X"].cpu().pin_memory()
        Yh = torch.empty_like(Xh).pin_memory()
        Xd = torch.empty_like(inp["X"])
        ns = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            Xd.copy_(Xh, non_blocking=True)
            step(Xd, Y)
            Yh.copy_(Y, non_blocking=True)
            L.check(L.ttt_mlp_status(ws, stream), "status")

        e2e_step()
        t0 = time.perf_counter()
        for _ in range(ns):
            e2e_step()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev) / ns
        nbytes = Xh.numel() * Xh.element_size()
        e2e = {"value": whole_job_tokens_per_s(world, w.T, e2e_s * 1e3), "unit": UNIT,
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes, "ms_per_step": e2e_s * 1e3,
               "steps": ns}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        run, scale, threads, sample = _cpu_sample_linear(w, args.cpu_tokens)
        t = run()
        cpu = {"value": args.cpu_tokens * scale / t, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": sample, "seconds": round(t, 2)}
    if rank == 0:
        line = {"metric": METRIC_LINEAR, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": "bf16-in/tf32-mma/fp32-state" if scan == "scan_linear_tc" else "bf16-in/fp32-scan",
                "data": "synthetic",
                "config": _config(w, {"model": "ttt-linear", "state": "W [64 x 64] fp32 per head"}),
                "gpu_launches": launches, "clocks": clocks, "roofline": roof, "kernels": kernels, "e2e": e2e,
                "cpu_baseline": cpu, "impl": "ours"}
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--model", choices=["mlp", "linear"], default="mlp")
    ap.add_argument("--kernels", choices=["auto", "simt"], default="auto",
                    help="simt: the fp32 SIMT scan and projection kernels (reference kernels)")
    ap.add_argument("--T", type=int, default=0, help="override the sequence length (quick checks only)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-tokens", type=int, default=65536)
    ap.add_argument("--ref-tokens", type=int, default=8192)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.model == "linear":
            return run_ours_linear(args, rank, world, local_rank)
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
