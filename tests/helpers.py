"""Shared helpers for the parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them."""
from __future__ import annotations

import numpy as np
import torch

from oracle import ttt_oracle as O
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

# Tolerances on the max-normalised error max|g - o| / max|o|: 1e-3 when the
# whole path is fp32, 2e-2 when X and theta are bf16 (fp32 state/accumulate).
TOL_F32 = 1e-3
TOL_BF16 = 2e-2


def tol(w: S.Workload) -> float:
    return TOL_BF16 if w.dtype == "bf16" else TOL_F32


def maxrel(g, o) -> float:
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    scale = np.abs(o).max()
    if scale == 0:
        return float(np.abs(g).max())
    return float(np.abs(g - o).max() / scale)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_args(inp: dict):
    return [to_np(inp[k]) for k in ("X", "theta_q", "theta_k", "theta_v", "W1_0", "W2_0")]


def run_gpu(w: S.Workload, inp: dict, dirs: str | None = None, eta: float | None = None, **kw) -> dict:
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    return L.layer_forward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W1_0"], g["W2_0"],
                           w.eta_eff if eta is None else eta, w.b, dirs or w.dirs, alpha_f=g["alpha_f"],
                           alpha_r=g["alpha_r"], per_head=w.per_head, **kw)


def run_oracle(w: S.Workload, inp: dict, dirs: str | None = None, eta: float | None = None) -> dict:
    return O.layer_forward(*oracle_args(inp), w.eta_eff if eta is None else eta, w.b, dirs or w.dirs,
                           alpha_f=to_np(inp["alpha_f"]), alpha_r=to_np(inp["alpha_r"]), per_head=w.per_head)


def head_slice(inp: dict, heads) -> dict:
    """Per-head mode: the inputs of a subset of heads (X, theta, W_0 and alpha rows)."""
    out = dict(inp)
    idx = torch.tensor(list(heads))
    for k in ("X", "theta_q", "theta_k", "theta_v", "W1_0", "W2_0"):
        out[k] = inp[k].index_select(0, idx)
    d = inp["X"].shape[2]
    cols = torch.cat([torch.arange(h * d, (h + 1) * d) for h in heads])
    out["alpha_f"] = inp["alpha_f"][cols]
    out["alpha_r"] = inp["alpha_r"][cols]
    return out
