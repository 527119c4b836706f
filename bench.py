#!/usr/bin/env python
"""Benchmark of the gated bidirectional TTT-MLP layer on B200.

One step = one full layer (fused Q/K/V projections, forward scan with gate,
reverse projections, reverse scan with gate) over one synthetic 313,344-token
sequence of width 3072 (48 heads, d = 64, hidden 256, b = 64), inputs already
resident in HBM.  Multi-GPU (torchrun): each rank runs its own sequence
(independent replicas, weak scaling, no collective on the data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--model mlp|linear]
                    [--workload full63s|scale18s|minibatch|causal|tiny]

Prints one JSON line on rank 0.  With --gpus N > 1 and no torchrun
environment, bench.py starts N ranks itself (torch.distributed.run, one
process per GPU).  --model linear measures the TTT-Linear layer
(f(u; W) = W u) on the same sequence instead.  --workload picks one of the
other workloads of the description (default: the 313,344-token layer); the
b = 1 per-token workloads also report the time per token.
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
    "scan_chunk_tc3": ("scan_chunk_tc3.cu",),
    "scan_token": ("scan_token.cu",),
    "scan_token_cluster": ("scan_token_cluster.cu",),
    "proj_full_simt": ("proj_simt.cu",),
    "proj_full_tc": ("proj_tc.cu",),
    "proj_per_head": ("proj_simt.cu",),
    "gate": ("gate.cu",),
    "scan_linear": ("scan_linear.cu",),
    "scan_linear_tc": ("scan_linear_tc.cu",),
    "attn_seg_tc": ("attn_seg_tc.cu",),
}


def _layout_key(w) -> str:
    return f"{'head' if w.per_head else 'full'}-H{w.H}-d{w.d}"


def _traffic(name: str, units_scale: float, w=None):
    """DRAM bytes per launch of `name` from the committed ncu summary, or None
    if absent, taken on a different version of the kernel's source, or taken
    on another layout (head count, per-head vs full width) than `w`'s."""
    try:
        with open(TRAFFIC_PATH) as f:
            rec = json.load(f).get(name)
        if not rec or rec.get("src_hash") != _src_hash(*KERNEL_SRC[name]):
            return None
        if w is not None and rec.get("layout", "full-H48-d64") != _layout_key(w):
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
WORKLOAD_NAMES = ("full63s", "scale18s", "minibatch", "causal", "tiny")


def _workload(args):
    from test_rnn_layer_b200 import synth as S
    w = {"full63s": S.FULL63S, "scale18s": S.SCALE18S, "minibatch": S.MINIBATCH, "causal": S.CAUSAL,
         "tiny": S.TINY}[args.workload]
    if args.T:
        w = w.with_T(args.T)
    return w


def _metric(w, model: str) -> str:
    from test_rnn_layer_b200 import synth as S
    if w.name == S.FULL63S.name:
        return METRIC_LINEAR if model == "linear" else METRIC
    kind = "TTT-Linear" if model == "linear" else "TTT-MLP"
    return f"{kind} tokens/s ({w.H} heads, {w.dirs}, b={w.b}, {w.dtype}) at T={w.T}; % of roofline"


def _input_bytes(w) -> int:
    return w.H * w.T * w.d * (2 if w.dtype == "bf16" else 4) if w.per_head else w.T * w.model_dim * 2


def _config(w, extra=None):
    """The workload description; identical in both arms for the same workload."""
    th = f"theta~N(0,1/{'d' if w.per_head else 'D'})"
    xb = _input_bytes(w)
    l2 = ("no flush: every input is larger than the 126 MB L2" if xb > 126e6 else
          "no flush: the inputs fit in L2 (a small workload; reported for its per-token latency)")
    cfg = {"workload": w.name, "T": w.T, "D": w.model_dim, "H": w.H, "d": w.d, "hidden": w.m, "b": w.b,
           "dirs": w.dirs, "x_dtype": w.dtype, "state": "fp32", "eta": f"{w.eta}/d", "alpha": w.alpha,
           "layout": "per-head X [H,T,d]" if w.per_head else "full width X [T,D]",
           "inputs": f"seeded Gaussian stand-ins for video tokens (X~N(0,1), {th}, W1_0~N(0,1/d), "
                     "W2_0~N(0,1/4d))",
           "l2": l2, "parallelism": "replicas (one sequence per GPU)"}
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
        # tf32 for the two d-by-m products that read the fp32 state (A, Aq0), fp16 for the rest
        "scan_chunk_tc3": ("tensor_mixed", scan_flops),
        "scan_chunk_simt": ("alu", scan_flops),
        "scan_token": ("alu", H * T * 7 * 2 * d * m),
        "scan_token_cluster": ("alu", H * T * 7 * 2 * d * m),
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
        # backward of the scan: the forward chunk recomputed plus its reverse-mode derivative, counted
        # as three forward passes (the kernel does more: the state walk that keeps the chunk-start
        # states); its products run on tf32 tensor cores, in the split form (three products each) for
        # fp32 layers
        "scan_backward": ("tensor_tf32" if w.dtype == "bf16" else "tensor_3xtf32",
                          3 * H * T * (7 * 2 * d * m + 2 * b * (d + m))),
        # projections' gradients: dX += dU theta and dtheta += dU^T X for the three projections
        "grad_gemm": ("alu", 2 * 3 * 2.0 * T * D * (d if w.per_head else D)),
        "gate_backward": ("hbm", T * D * 16),
    }


def _tf32_share(w) -> float:
    """Share of the scan's algorithmic flops that the split-group kernel runs
    with tf32 operands: A^T = W1 K^T and Aq0 = W1 Q^T (they read the fp32
    state in tensor memory); every other product takes fp16 operands."""
    return 2 * 2 * w.d * w.m / (7 * 2 * w.d * w.m + 2 * w.b * (w.d + w.m))


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
    elif bound == "tensor_mixed":
        f = _tf32_share(w)
        peak = 1.0 / (f / (sus * TF32_PER_BF16) + (1.0 - f) / sus)
        unit, kind = "TFLOP/s", "tensor"
        note = (f"{f:.3f} of the flops at tf32 (bf16 sustained {src} x 1.1/2.25), the rest at fp16 (= bf16 "
                f"sustained {src}): the time-weighted peak")
        achieved = work / (ms_per_launch * 1e-3) / 1e12
    elif bound == "tensor_tf32":
        peak, unit, kind = sus * TF32_PER_BF16, "TFLOP/s", "tensor"
        note = f"tf32 dense = bf16 sustained {src} x 1.1/2.25 (nominal ratio)"
        achieved = work / (ms_per_launch * 1e-3) / 1e12
    elif bound == "tensor_3xtf32":   # every product taken as three tf32 products
        peak, unit, kind = sus * TF32_PER_BF16 / 3, "TFLOP/s", "tensor"
        note = f"tf32 dense = bf16 sustained {src} x 1.1/2.25 (nominal ratio), / 3 for the split products"
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
            "frac": round(achieved / peak, 4), "traffic": _traffic(name, units, w), "peak_note": note,
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
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _cpu_sample(w, tokens: int, model: str = "mlp", seed: int = 0):
    """A bounded sample of the workload for the fp64 oracle: the first `tokens`
    tokens of the sequence, the first direction only, as many heads as the
    oracle has threads (one OpenMP thread per head), with those heads' share of
    the projections.  Both the reference arm and the CPU baseline time exactly
    this sample.  Returns (run, scale, threads, description): run() times one
    pass in seconds; tokens x scale / seconds is in the metric's units (tokens
    through all heads and directions)."""
    import numpy as np

    from oracle import ttt_oracle as O
    from test_rnn_layer_b200 import synth as S

    threads = O.num_threads()
    heads = list(range(min(w.H, threads)))
    tokens = min(tokens, w.T)
    ws = w.with_T(tokens)
    inp = (S.make_linear_inputs if model == "linear" else S.make_inputs)(ws, seed=seed, device="cpu")
    reverse = w.dirs == "rev"
    ndir = 2 if w.dirs == "bidir" else 1
    if w.per_head:
        X = inp["X"].double().numpy()[heads]
        th = [inp[k].double().numpy()[heads] for k in ("theta_q", "theta_k", "theta_v")]
    else:
        X = inp["X"].float().numpy()
        rows = np.concatenate([np.arange(h * w.d, (h + 1) * w.d) for h in heads])
        th = [inp[k].float().numpy()[rows] for k in ("theta_q", "theta_k", "theta_v")]

    if model == "linear":
        W0 = inp["W_0"].double().numpy()[heads]

        def work():
            if w.per_head:
                O.linear_direction(X, *th, W0, w.eta_eff, w.b, reverse, per_head=True)
            else:
                Q, K, V = [O.project_full(X, t).reshape(tokens, len(heads), w.d).transpose(1, 0, 2) for t in th]
                O.linear_scan_heads(Q, K, V, W0, w.eta_eff, w.b, reverse)
    else:
        W1, W2 = inp["W1_0"].double().numpy()[heads], inp["W2_0"].double().numpy()[heads]

        def work():
            if w.per_head:
                O.direction(X, *th, W1, W2, w.eta_eff, w.b, reverse, per_head=True)
            else:
                O.full_mode_heads(X, *th, W1, W2, w.eta_eff, w.b, list(range(len(heads))), reverse=reverse)

    def run():
        t0 = time.perf_counter()
        work()
        return time.perf_counter() - t0

    scale = len(heads) / (w.H * float(ndir))
    kind = "TTT-Linear" if model == "linear" else "TTT-MLP"
    sample = (f"first {tokens} tokens, {len(heads)} of {w.H} heads, {'reverse' if reverse else 'forward'} direction "
              f"only (fp64 {kind} oracle incl. those heads' Q/K/V projections); tokens/s scaled by "
              f"{len(heads)}/({w.H}*{ndir})")
    return run, scale, threads, sample


def cpu_baseline(w, args) -> dict:
    """The oracle on this host's cores, on the reference arm's sample, repeated
    args.cpu_reps times (about 10-30 s of CPU work at the full layer)."""
    run, scale, threads, sample = _cpu_sample(w, args.sample_tokens, args.model)
    times = [run() for _ in range(args.cpu_reps)]
    t = sum(times) / len(times)
    tokens = min(args.sample_tokens, w.T)
    return {"value": tokens * scale / t, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
            "seconds": round(sum(times), 2), "reps": len(times), "cpu_model": cpu_model()}


# ------------------------------------------------------------------ arms
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = _workload(args)
    run, scale, threads, sample = _cpu_sample(w, args.sample_tokens, args.model)
    tokens = min(args.sample_tokens, w.T)
    for _ in range(args.warmup):
        run()
    times = [run() for _ in range(args.steps)]
    step_s = sum(times) / len(times)
    value = tokens * scale / step_s
    line = {"impl": "reference", "metric": _metric(w, args.model), "value": value, "unit": UNIT,
            "n_gpus": max(world, args.gpus), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": _config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def _timed_steps(step, args, world, local_rank, stream, flush_l2):
    """W untimed warm-up steps, then K timed steps between barriers and
    synchronisations, timed by CUDA events on `stream`; the maximum over
    ranks.  With flush_l2 a buffer larger than L2 is written before each
    step and every step is timed alone (the flush outside the timed spans)."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    scrub = torch.empty(64 << 22, dtype=torch.float32, device=stream.device) if flush_l2 else None   # 1 GiB
    barrier()
    torch.cuda.synchronize()
    if flush_l2:
        ms = 0.0
        for _ in range(args.steps):
            scrub.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            e1.synchronize()
            ms += e0.elapsed_time(e1)
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(ms, world, torch.device("cuda", local_rank))


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from test_rnn_layer_b200 import synth as S
    from test_rnn_layer_b200 import tttmlp as L

    L.lib()   # loud failure if the CUDA library is missing
    sel = {"auto": None, "simt": (1, 1), "cluster": (2, 0), "split": (4, 0)}[args.kernels]
    if sel:
        L.check(L.ttt_mlp_select_kernels(*sel), "ttt_mlp_select_kernels")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = _workload(args)
    linear = args.model == "linear"
    inp = (S.make_linear_inputs if linear else S.make_inputs)(w, seed=rank_seed(rank), device=dev)
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    direction = L.DIRS[w.dirs]
    if linear:
        ws_dev_bytes = L.ttt_linear_workspace_size(desc, w.b, direction)
        ws = torch.empty(L.ttt_linear_host_io_workspace_size(desc, w.b, direction), dtype=torch.uint8, device=dev)
    else:
        ws = L.alloc_workspace(desc, w.b, direction, dev, host_io=True)
        ws_dev_bytes = L.ttt_mlp_workspace_size(desc, w.b, direction)
    Y = torch.empty_like(inp["X"])
    stream = torch.cuda.current_stream()

    def step(X=None, Yo=None):
        X = inp["X"] if X is None else X
        Yo = Y if Yo is None else Yo
        if linear:
            st = L.ttt_linear_forward(desc, X, inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W_0"],
                                      w.eta_eff, w.b, direction, inp["alpha_f"], inp["alpha_r"], Yo, None, None, ws,
                                      ws_dev_bytes, stream)
        else:
            st = L.ttt_mlp_forward(desc, X, inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"],
                                   inp["W2_0"], w.eta_eff, w.b, direction, inp["alpha_f"], inp["alpha_r"], Yo, None,
                                   None, None, ws, ws_dev_bytes, stream)
        if st != L.TTT_OK:
            raise L.TTTError(st, "ttt_linear_forward" if linear else "ttt_mlp_forward")

    flush_l2 = _input_bytes(w) <= 126e6
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    L.check(L.ttt_mlp_status(ws, stream), "warm-up status")

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    time.sleep(0.3)
    n_launch0 = L.ttt_launch_count()
    ms = _timed_steps(step, argparse.Namespace(warmup=0, steps=args.steps), world, local_rank, stream, flush_l2)
    launches = L.ttt_launch_count() - n_launch0
    clocks = sampler.stop()
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
    scans = [k for k in ktimes if k.startswith("scan")]
    top = max(scans or ktimes, key=lambda k: ktimes[k][0]) if linear else max(ktimes, key=lambda k: ktimes[k][0])
    peaks = _peaks()
    roof = _roofline(top, ktimes[top][0] / ktimes[top][1], ktimes[top][1] / kpass, w, peaks, clocks)
    roof["share"] = round(ktimes[top][0] / total, 4)   # of the summed kernel time (streams overlap)
    roof["ms_per_step"] = round(ktimes[top][0] / kpass, 3)
    kernels = {k: {"ms_per_step": round(v[0] / kpass, 3), "launches_per_step": v[1] // kpass,
                   "share": round(v[0] / total, 4)} for k, v in ktimes.items()}

    # end to end through the public API with pinned host buffers: H2D of X, layer, D2H of Y
    e2e = None
    if not args.no_e2e:
        Xh = inp["X"].cpu().pin_memory()
        Yh = torch.empty_like(Xh).pin_memory()
        ns = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            if linear:
                st = L.ttt_linear_forward_host(desc, Xh, inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W_0"],
                                               w.eta_eff, w.b, direction, inp["alpha_f"], inp["alpha_r"], Yh, ws,
                                               ws.numel(), stream)
                L.check(st, "ttt_linear_forward_host")
            else:
                st = L.ttt_mlp_forward_host(desc, Xh, inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"],
                                            inp["W2_0"], w.eta_eff, w.b, direction, inp["alpha_f"], inp["alpha_r"],
                                            Yh, ws, ws.numel(), stream)
                L.check(st, "ttt_mlp_forward_host")

        e2e_step()
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        t0 = time.perf_counter()
        for _ in range(ns):
            e2e_step()
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev) / ns
        nbytes = Xh.numel() * Xh.element_size()
        e2e = {"value": whole_job_tokens_per_s(world, w.T, e2e_s * 1e3), "unit": UNIT, "h2d_bytes_per_step": nbytes,
               "d2h_bytes_per_step": nbytes, "ms_per_step": e2e_s * 1e3, "steps": ns}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(w, args)

    if rank == 0:
        tc = any("_tc" in k for k in ktimes)
        scan_name = next((k for k in ktimes if k.startswith("scan")), "")
        if linear:
            dtype = "bf16-in/tf32-mma/fp32-state" if tc else f"{w.dtype}-in/fp32-scan"
        elif "scan_chunk_tc3" in ktimes:
            dtype = "bf16-in/tf32+fp16-mma/fp32-state"
        else:
            dtype = "bf16-in/tf32-mma/fp32-state" if tc else "fp32"
        line = {"metric": _metric(w, args.model), "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic", "config": _config(w),
                "kernels_impl": "tensor-core" if tc else "simt", "gpu_launches": launches, "clocks": clocks,
                "roofline": roof, "kernels": kernels, "e2e": e2e, "cpu_baseline": cpu, "impl": "ours"}
        if w.b == 1:   # the per-token rule: the sequential chain per token
            line["ns_per_token"] = ms_per_step * 1e6 / w.T
            line["scan_ns_per_token"] = ktimes[scan_name][0] / kpass * 1e6 / (w.T * (2 if w.dirs == "bidir" else 1))
        print(json.dumps(line), flush=True)
    return 0


METRIC_BLOCK = ("block tokens/s (segment-local attention in 21 segments + bidirectional TTT-MLP layer, 48 heads) "
                "at T≈313k; % of roofline")


def _attention_flops(T: int, D: int, L: int) -> float:
    """Q K^T and P V over every segment and head: 2 x 2 L_s^2 D flops per segment."""
    return sum(4.0 * (min(s0 + L, T) - s0) ** 2 * D for s0 in range(0, T, L))


def cpu_baseline_block(w, L_seg, args) -> dict:
    """The oracles on a bounded sample: the attention of the first 256 query
    rows of a segment for every head (each against the segment's keys), and
    the layer's own sample (cpu_baseline); block tokens/s = 1 / (attention
    seconds per token + layer seconds per token)."""
    from oracle import seg_attention as A
    from test_rnn_layer_b200 import synth as S

    rows = 256
    a = S.make_attention_inputs(w.with_T(L_seg), seed=0, device="cpu")
    Q, K, V = (a[k].double().numpy() for k in ("Q_a", "K_a", "V_a"))

    def att():
        t0 = time.perf_counter()
        for h in range(w.H):
            c = slice(h * w.d, (h + 1) * w.d)
            A.attention_segment(Q[:rows, c], K[:, c], V[:, c])
        return time.perf_counter() - t0

    t_att = min(att() for _ in range(2)) / rows
    layer = cpu_baseline(w, args)
    value = 1.0 / (t_att + 1.0 / layer["value"])
    return {"value": value, "unit": UNIT, "cores": max(layer["cores"], os.cpu_count() or 1), "kind": "oracle",
            "sample": (f"attention: {rows} query rows of a {L_seg}-token segment, all {w.H} heads (fp64, numpy); "
                       f"layer: {layer['sample']}; combined as seconds per token"),
            "attention_s_per_token": t_att, "layer_tokens_per_s": layer["value"], "cpu_model": cpu_model()}


def run_block(args, rank, world, local_rank):
    """One step = the block: segment-local attention (21 segments) feeding the
    bidirectional layer, through ttt_block_forward; besides it, the attention
    and the layer timed alone, the two calls one after the other, and the
    interleaved schedule (each segment's attention beside the scan)."""
    import torch
    import torch.distributed as dist

    from test_rnn_layer_b200 import synth as S
    from test_rnn_layer_b200 import tttmlp as L

    L.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = _workload(args)
    if w.per_head or w.dirs != "bidir" or w.dtype != "bf16":
        raise SystemExit("--block needs the full-width bidirectional bf16 layer (--workload full63s)")
    L_seg = S.segment_length(S.FULL63S.T)   # the tokens of one 3-s segment of the 63-s video, whatever --T is
    inp = S.make_inputs(w, seed=rank_seed(rank), device=dev)
    inp.update(S.make_attention_inputs(w, seed=rank_seed(rank), device=dev))
    desc = L.make_desc(w.T, w.H, w.d, False, True)
    nws = L.ttt_block_workspace_size(desc, w.b)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    aws = torch.empty(L.ttt_seg_attention_workspace_size(), dtype=torch.uint8, device=dev)
    X = torch.empty_like(inp["X"])
    Y = torch.empty_like(inp["X"])
    stream = torch.cuda.current_stream()
    th = (inp["theta_q"], inp["theta_k"], inp["theta_v"])

    def block(Qa=None, Ka=None, Va=None, Xr=None):
        L.check(L.ttt_block_forward(desc, L_seg, inp["Q_a"] if Qa is None else Qa, inp["K_a"] if Ka is None else Ka,
                                    inp["V_a"] if Va is None else Va, w.D, inp["X"] if Xr is None else Xr, X, *th,
                                    inp["W1_0"], inp["W2_0"], w.eta_eff, w.b, inp["alpha_f"], inp["alpha_r"], Y, ws,
                                    nws, stream), "ttt_block_forward")

    def attention():
        L.check(L.ttt_seg_attention(w.T, w.H, w.d, L_seg, inp["Q_a"], inp["K_a"], inp["V_a"], w.D, inp["X"], X, w.D,
                                    0, w.T, aws, aws.numel(), stream), "ttt_seg_attention")

    def layer():
        L.check(L.ttt_mlp_forward(desc, X, *th, inp["W1_0"], inp["W2_0"], w.eta_eff, w.b, L.TTT_BIDIR,
                                  inp["alpha_f"], inp["alpha_r"], Y, None, None, None, ws, nws, stream),
                "ttt_mlp_forward")

    for _ in range(args.warmup):
        block()
    torch.cuda.synchronize()
    L.check(L.ttt_mlp_status(ws, stream), "warm-up status")
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    time.sleep(0.3)
    n_launch0 = L.ttt_launch_count()
    ms = _timed_steps(block, argparse.Namespace(warmup=0, steps=args.steps), world, local_rank, stream, False)
    launches = L.ttt_launch_count() - n_launch0
    clocks = sampler.stop()
    L.check(L.ttt_mlp_status(ws, stream), "timed-run status")
    ms_per_step = ms / args.steps
    value = whole_job_tokens_per_s(world, w.T, ms_per_step)

    def alone(fn, n=3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    # per-kernel device times of the block (events on each launch's stream)
    L.ttt_kernel_timing(True)
    kpass = 2
    for _ in range(kpass):
        block()
    torch.cuda.synchronize()
    ktimes = L.ttt_kernel_times()
    L.ttt_kernel_timing(False)
    total = sum(v[0] for v in ktimes.values()) or 1.0
    kernels = {k: {"ms_per_step": round(v[0] / kpass, 3), "launches_per_step": v[1] // kpass,
                   "share": round(v[0] / total, 4)} for k, v in ktimes.items()}
    att_ms = alone(attention)
    layer_ms = alone(layer)
    two_calls_ms = alone(lambda: (attention(), layer()))
    L.check(L.ttt_debug_set_block_front(95), "ttt_debug_set_block_front")
    interleaved_ms = alone(block)
    L.check(L.ttt_debug_set_block_front(-1), "ttt_debug_set_block_front")
    L.check(L.ttt_mlp_status(ws, stream), "comparison status")

    peaks = _peaks()
    src = "of " + peaks["_source"]
    flops = _attention_flops(w.T, w.D, L_seg)
    k_att = ktimes["attn_seg_tc"]
    att_launch_ms = k_att[0] / k_att[1]
    achieved = flops * kpass / k_att[1] / (att_launch_ms * 1e-3) / 1e12
    roof = {"kernel": "attn_seg_tc", "bound": "tensor", "achieved": round(achieved, 2),
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
            "traffic": _traffic("attn_seg_tc", w.T / 1024.0), "peak_note": f"bf16 dense burst {src} (kernel timed "
            "alone, one launch of the whole sequence)", "ms_per_launch": round(att_launch_ms, 3),
            "work_per_launch": flops, "work": "4 L_s^2 D flops per segment (Q K^T and P V, all heads)",
            "share": round(k_att[0] / total, 4)}

    e2e = None
    if not args.no_e2e:
        host = {k: inp[k].cpu().pin_memory() for k in ("Q_a", "K_a", "V_a", "X")}
        dev_in = {k: torch.empty_like(inp[k]) for k in host}
        Yh = torch.empty_like(host["X"]).pin_memory()
        ns = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            for k in host:
                dev_in[k].copy_(host[k], non_blocking=True)
            block(dev_in["Q_a"], dev_in["K_a"], dev_in["V_a"], dev_in["X"])
            Yh.copy_(Y, non_blocking=True)
            L.check(L.ttt_mlp_status(ws, stream), "status")

        e2e_step()
        t0 = time.perf_counter()
        for _ in range(ns):
            e2e_step()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev) / ns
        nb = host["X"].numel() * 2
        e2e = {"value": whole_job_tokens_per_s(world, w.T, e2e_s * 1e3), "unit": UNIT, "h2d_bytes_per_step": 4 * nb,
               "d2h_bytes_per_step": nb, "ms_per_step": e2e_s * 1e3, "steps": ns}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_block(w, L_seg, args)
    if rank == 0:
        nseg = -(-w.T // L_seg)
        cfg = _config(w, {"workload": "block-" + w.name, "attention": f"segment-local, {nseg} segments of {L_seg} "
                          f"tokens (the last {w.T - (nseg - 1) * L_seg}), full inside a segment, Q/K/V ~N(0,1) bf16, "
                          "residual X", "schedule": "attention of every row, then the layer"})
        line = {"metric": METRIC_BLOCK, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16-in/bf16-mma-attention/tf32+fp16-mma-scan/fp32-state",
                "data": "synthetic", "config": cfg, "gpu_launches": launches, "clocks": clocks, "roofline": roof,
                "kernels": kernels, "schedules_ms": {"block": round(ms_per_step, 2), "attention_alone":
                round(att_ms, 2), "layer_alone": round(layer_ms, 2), "attention_then_layer_two_calls":
                round(two_calls_ms, 2), "interleaved_front95": round(interleaved_ms, 2)},
                "e2e": e2e, "cpu_baseline": cpu, "impl": "ours"}
        print(json.dumps(line), flush=True)
    return 0


def run_backward(args, rank, world, local_rank):
    """One training step of the layer: ttt_mlp_backward (the forward pass
    recomputed inside, then the gradients of every input) for a seeded
    upstream gradient dY; tokens/s of that step."""
    import torch

    from test_rnn_layer_b200 import synth as S
    from test_rnn_layer_b200 import tttmlp as L

    L.lib()
    sel = {"auto": None, "simt": (1, 1), "cluster": (2, 0), "split": (4, 0)}[args.kernels]
    if sel:
        L.check(L.ttt_mlp_select_kernels(*sel), "ttt_mlp_select_kernels")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = _workload(args)
    inp = S.make_inputs(w, seed=rank_seed(rank), device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    dY = torch.randn(inp["X"].shape, generator=gen, device=dev, dtype=torch.float32)
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    direction = L.DIRS[w.dirs]
    nbytes = L.ttt_mlp_backward_workspace_size(desc, w.b, direction)
    if nbytes == 0:
        raise L.TTTError(L.TTT_ERR_INVALID_ARG, "ttt_mlp_backward_workspace_size: " + L.ttt_last_error())
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    outs = [torch.empty(inp["X"].shape, **f32)] + [torch.empty(inp[k].shape, **f32) for k in
                                                   ("theta_q", "theta_k", "theta_v", "W1_0", "W2_0")]
    da_f, da_r = torch.empty(w.model_dim, **f32), torch.empty(w.model_dim, **f32)
    stream = torch.cuda.current_stream()

    def step(X=None, dy=None, dX=None):
        st = L.ttt_mlp_backward(desc, inp["X"] if X is None else X, inp["theta_q"], inp["theta_k"], inp["theta_v"],
                                inp["W1_0"], inp["W2_0"], w.eta_eff, w.b, direction, inp["alpha_f"], inp["alpha_r"],
                                dY if dy is None else dy, outs[0] if dX is None else dX, *outs[1:], da_f, da_r, ws,
                                nbytes, stream)
        if st != L.TTT_OK:
            raise L.TTTError(st, "ttt_mlp_backward")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    L.check(L.ttt_mlp_status(ws, stream), "warm-up status")
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    time.sleep(0.3)
    n_launch0 = L.ttt_launch_count()
    ms = _timed_steps(step, argparse.Namespace(warmup=0, steps=args.steps), world, local_rank, stream,
                      _input_bytes(w) <= 126e6)
    launches = L.ttt_launch_count() - n_launch0
    clocks = sampler.stop()
    L.check(L.ttt_mlp_status(ws, stream), "timed-run status")
    ms_per_step = ms / args.steps
    L.ttt_kernel_timing(True)
    step()
    torch.cuda.synchronize()
    ktimes = L.ttt_kernel_times()
    L.ttt_kernel_timing(False)
    total = sum(v[0] for v in ktimes.values()) or 1.0
    top = max(ktimes, key=lambda k: ktimes[k][0])
    roof = None
    if top in _algorithmic(w):
        roof = _roofline(top, ktimes[top][0] / ktimes[top][1], ktimes[top][1], w, _peaks(), clocks)
        roof["share"] = round(ktimes[top][0] / total, 4)
    kernels = {k: {"ms_per_step": round(v[0], 3), "launches_per_step": v[1], "share": round(v[0] / total, 4)}
               for k, v in ktimes.items()}
    e2e = None
    if not args.no_e2e:   # X and dY from pinned host memory, dX back to it
        Xh, dYh = inp["X"].cpu().pin_memory(), dY.cpu().pin_memory()
        dXh = torch.empty(dYh.shape, dtype=torch.float32).pin_memory()
        Xd, dYd = torch.empty_like(inp["X"]), torch.empty_like(dY)
        ns = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            Xd.copy_(Xh, non_blocking=True)
            dYd.copy_(dYh, non_blocking=True)
            step(Xd, dYd)
            dXh.copy_(outs[0], non_blocking=True)
            L.check(L.ttt_mlp_status(ws, stream), "status")

        e2e_step()
        t0 = time.perf_counter()
        for _ in range(ns):
            e2e_step()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev) / ns
        e2e = {"value": whole_job_tokens_per_s(world, w.T, e2e_s * 1e3), "unit": UNIT,
               "h2d_bytes_per_step": Xh.numel() * Xh.element_size() + dYh.numel() * 4,
               "d2h_bytes_per_step": dXh.numel() * 4, "ms_per_step": e2e_s * 1e3, "steps": ns}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_backward(w, args)
    if rank == 0:
        line = {"metric": "TTT-MLP training step (forward + backward) " + _metric(w, "mlp"),
                "value": whole_job_tokens_per_s(world, w.T, ms_per_step), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None,
                "dtype": ("bf16-in/tf32-mma/fp32-state-backward" if w.dtype == "bf16"
                          else "fp32-in/3xtf32-mma/fp32-state-backward"),
                "data": "synthetic",
                "config": _config(w, {"step": "forward recomputed + backward of every input"}),
                "gpu_launches": launches, "clocks": clocks, "roofline": roof, "kernels": kernels, "e2e": e2e,
                "cpu_baseline": cpu, "impl": "ours"}
        print(json.dumps(line), flush=True)
    return 0


def cpu_baseline_backward(w, args) -> dict:
    """The backward oracle (fp64 autograd) on a bounded sample: the first
    1.5 x sample_tokens tokens (at most 24,576: about 12 s on 16 host cores)
    of two heads."""
    import numpy as np
    import torch

    from oracle import ttt_backward as B
    from test_rnn_layer_b200 import synth as S

    tokens = min(w.T, max(16, min(24576, args.sample_tokens * 3 // 2)))
    heads = min(w.H, 2)
    ws = w.with_(T=tokens, H=heads, D=heads * w.d if not w.per_head else 0)
    inp = S.make_inputs(ws, seed=0)
    dY = np.random.default_rng(0).normal(size=tuple(inp["X"].shape))
    t0 = time.perf_counter()
    B.layer_backward({k: inp[k].double().numpy() for k in B.NAMES}, dY, w.eta_eff, w.b, w.dirs, w.per_head)
    t = time.perf_counter() - t0
    scale = heads / w.H
    return {"value": tokens * scale / t, "unit": UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"first {tokens} tokens, {heads} of {w.H} heads (fp64 autograd of the oracle's forward, "
                      f"{'the full width reduced to those heads' if not w.per_head else 'per-head inputs'}); "
                      f"tokens/s scaled by {heads}/{w.H}", "seconds": round(t, 2), "cpu_model": cpu_model()}


def run_dry_host(args, rank, world):
    """Host plumbing only (no GPU, no library): the rank layout, the process
    group (gloo), the barrier-bracketed timing of `steps` steps that sleep
    (10 ms x (rank + 1)), the maximum over ranks and rank 0's JSON line.
    Used by the CPU tests of the launcher."""
    import torch
    import torch.distributed as dist
    w = _workload(args)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(0.010 * (rank + 1))
    if world > 1:
        dist.barrier()
    ms = max_over_ranks((time.perf_counter() - t0) * 1e3, world, torch.device("cpu"))
    if rank == 0:
        ms_per_step = ms / args.steps
        print(json.dumps({"metric": _metric(w, args.model), "value": whole_job_tokens_per_s(world, w.T, ms_per_step),
                          "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": ms_per_step, "dry_run": True, "config": _config(w)}), flush=True)
    return 0


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_command(argv, n: int, port: int) -> list:
    """torch.distributed.run command that runs this script as n ranks on one node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]


def run_sharded(args, rank, world, local_rank):
    """One sequence of the full-width bidirectional layer with its heads split over
    the ranks (test_rnn_layer_b200/shard.py): per rank the forward phase of its
    heads, an all-reduce of the gate increment, the reverse phase, an
    all-reduce of Y.  Strong scaling: `value` is the sequence's tokens per
    second of the slowest rank."""
    import torch
    import torch.distributed as dist

    from test_rnn_layer_b200 import shard
    from test_rnn_layer_b200 import synth as S
    from test_rnn_layer_b200 import tttmlp as L

    L.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = _workload(args)
    if w.per_head or w.dirs != "bidir" or w.dtype != "bf16":
        raise SystemExit("--shard-heads needs the full-width bidirectional bf16 layer (--workload full63s)")
    inp = S.make_inputs(w, seed=0, device=dev)   # the same sequence on every rank
    th = [inp["theta_q"], inp["theta_k"], inp["theta_v"]]
    desc = L.make_desc(w.T, w.H, w.d, False, True)
    h0, hn = shard.head_range(w.H, rank, world)
    ws = shard.heads_workspace(desc, hn, w.b, dev)
    stream = torch.cuda.current_stream()
    all_reduce = (lambda t: dist.all_reduce(t)) if world > 1 else (lambda t: None)

    def fwd(X, theta, W1_0, W2_0, eta, b, alpha_f, r, n):
        return shard.shard_forward(X, theta, W1_0, W2_0, eta, b, alpha_f, r, n, workspace=ws, stream=stream)

    def rev(X, theta, W1_0, W2_0, eta, b, alpha_r, inc, Xp, r, n):
        return shard.shard_reverse(X, theta, W1_0, W2_0, eta, b, alpha_r, inc, Xp, r, n, workspace=ws,
                                   stream=stream)

    def step():
        shard.sharded_layer_forward(inp["X"], th, inp["W1_0"], inp["W2_0"], w.eta_eff, w.b, inp["alpha_f"],
                                    inp["alpha_r"], rank, world, all_reduce, forward_step=fwd, reverse_step=rev)

    n_launch0 = L.ttt_launch_count()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    time.sleep(0.3)
    ms = _timed_steps(step, args, world, local_rank, stream, _input_bytes(w) <= 126e6)
    clocks = sampler.stop()
    launches = (L.ttt_launch_count() - n_launch0) * args.steps // (args.steps + args.warmup)
    L.check(L.ttt_mlp_status(ws, stream), "timed-run status")
    ms_per_step = ms / args.steps
    if rank == 0:
        line = {"metric": _metric(w, "mlp"), "value": w.T / (ms_per_step * 1e-3), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": "bf16-in/tf32+fp16-mma/fp32-state", "data": "synthetic",
                "config": _config(w, {"parallelism": f"heads split over {world} rank(s), one sequence",
                                      "heads_per_rank": hn}),
                "clocks": clocks, "gpu_launches": launches}
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--model", choices=["mlp", "linear"], default="mlp")
    ap.add_argument("--workload", choices=WORKLOAD_NAMES, default="full63s")
    ap.add_argument("--kernels", choices=["auto", "simt", "cluster", "split"], default="auto",
                    help="simt: the fp32 SIMT scan and projection kernels (reference kernels); cluster / split: "
                         "the two-CTA tensor-core scan with all warps on every stage / with state and output warp "
                         "groups a chunk apart")
    ap.add_argument("--T", type=int, default=0, help="override the sequence length (quick checks only)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--sample-tokens", type=int, default=16384,
                    help="tokens of the oracle's sample (reference arm and CPU baseline alike)")
    ap.add_argument("--cpu-reps", type=int, default=4, help="passes of the oracle's sample for the CPU baseline")
    ap.add_argument("--backward", action="store_true",
                    help="time one training step (forward recomputed + backward) instead of the forward layer")
    ap.add_argument("--shard-heads", action="store_true",
                    help="one sequence of the full-width layer split by heads over the ranks (strong scaling; "
                         "an all-reduce of the gate increment between the directions) instead of replicas")
    ap.add_argument("--block", action="store_true",
                    help="time the block (segment-local attention feeding the layer, ttt_block_forward) instead "
                         "of the layer alone")
    ap.add_argument("--dry-run-host", action="store_true", help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")

    if "WORLD_SIZE" not in os.environ and args.gpus > 1 and args.impl == "ours":
        # one process per GPU: start the ranks and wait for them (rank 0 prints the line)
        return subprocess.call(spawn_command(sys.argv[1:], args.gpus, _free_port()))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        if args.dry_run_host:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        else:
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local_rank))
    try:
        if args.dry_run_host:
            return run_dry_host(args, rank, world)
        if args.backward:
            return run_backward(args, rank, world, local_rank)
        if args.shard_heads:
            return run_sharded(args, rank, world, local_rank)
        if args.block:
            return run_block(args, rank, world, local_rank)
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
