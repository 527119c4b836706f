"""Head-sharded bidirectional TTT-MLP layer over R ranks (host logic).

Every head's chain is independent (paper notes page, "关键设计 / TTT-MLP 层":
each head keeps its own hidden state), so the heads split over ranks; the one
coupling is the reverse direction's projection, which reads every channel of
the forward direction's output ("关键设计 / 门控 + 双向机制": the reverse pass
runs on X' = X + tanh(alpha_f) z_f, and theta_Q/K/V mix all channels).  Rank r
of R owns heads [r H/R, (r+1) H/R) and holds the replicated inputs (X, theta,
W_0, alpha).  A layer is:

  1. forward phase (ttt_mlp_forward_heads, TTT_PHASE_FWD): X' and the gate
     increment bf16(tanh(alpha_f) z_f) in this rank's columns, zero elsewhere;
  2. a sum over ranks of the increment arrays (all-reduce: each column has one
     non-zero contributor, so the sum is exact);
  3. reverse phase (TTT_PHASE_REV): Y in this rank's columns, zero elsewhere;
  4. a sum over ranks of Y, so that every rank holds the layer's output.

Steps 1 and 3 are per-rank functions of their own so that a caller can run
the ranks one after another (one device) or concurrently (one process per
device, the sums as collectives).
"""
from __future__ import annotations

from typing import Callable

import torch

from . import tttmlp as L


def head_range(H: int, rank: int, world: int) -> tuple[int, int]:
    """(first head, head count) of `rank`: equal shards of the H heads."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    hn = H // world
    return rank * hn, hn


def heads_workspace(desc: L.ttt_mlp_desc, hn: int, b: int, device) -> torch.Tensor:
    n = L.ttt_mlp_heads_workspace_size(desc, hn, b)
    if n == 0:
        raise L.TTTError(L.TTT_ERR_INVALID_ARG, "ttt_mlp_heads_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _desc(X, W1_0) -> L.ttt_mlp_desc:
    T, _ = X.shape
    H, _, d = W1_0.shape
    return L.make_desc(T, H, d, False, True)


def shard_forward(X, theta, W1_0, W2_0, eta: float, b: int, alpha_f, rank: int, world: int,
                  workspace: torch.Tensor | None = None, stream=None):
    """Step 1 for one rank: returns (X' fp32 [T, D], increment bf16 [T, D]), both
    holding only this rank's columns (the increment is zero elsewhere)."""
    desc = _desc(X, W1_0)
    h0, hn = head_range(desc.H, rank, world)
    T, D = X.shape
    Xp = torch.empty((T, D), dtype=torch.float32, device=X.device)
    inc = torch.zeros((T, D), dtype=torch.bfloat16, device=X.device)
    ws = workspace if workspace is not None else heads_workspace(desc, hn, b, X.device)
    st = L.ttt_mlp_forward_heads(desc, h0, hn, L.TTT_PHASE_FWD, X, theta[0], theta[1], theta[2], W1_0, W2_0, eta, b,
                                 alpha_f, None, Xp, inc, ws, ws.numel(), stream)
    L.check(st, "ttt_mlp_forward_heads (forward phase)")
    return Xp, inc


def shard_reverse(X, theta, W1_0, W2_0, eta: float, b: int, alpha_r, inc_all, Xp, rank: int, world: int,
                  workspace: torch.Tensor | None = None, stream=None):
    """Step 3 for one rank: Y bf16 [T, D] in this rank's columns, zero elsewhere.
    inc_all: every rank's increment summed; Xp: this rank's step-1 X'."""
    desc = _desc(X, W1_0)
    h0, hn = head_range(desc.H, rank, world)
    Y = torch.zeros(X.shape, dtype=torch.bfloat16, device=X.device)
    ws = workspace if workspace is not None else heads_workspace(desc, hn, b, X.device)
    st = L.ttt_mlp_forward_heads(desc, h0, hn, L.TTT_PHASE_REV, X, theta[0], theta[1], theta[2], W1_0, W2_0, eta, b,
                                 alpha_r, inc_all, Xp, Y, ws, ws.numel(), stream)
    L.check(st, "ttt_mlp_forward_heads (reverse phase)")
    return Y


def sharded_layer_forward(X, theta, W1_0, W2_0, eta: float, b: int, alpha_f, alpha_r, rank: int, world: int,
                          all_reduce: Callable[[torch.Tensor], None], forward_step=shard_forward,
                          reverse_step=shard_reverse):
    """The bidirectional layer with this rank's heads; `all_reduce(t)` sums t
    over the ranks in place (e.g. torch.distributed.all_reduce).  Returns Y
    (bf16 [T, D]), the same on every rank.  forward_step / reverse_step compute
    steps 1 and 3 (the defaults run them through the CUDA library)."""
    Xp, inc = forward_step(X, theta, W1_0, W2_0, eta, b, alpha_f, rank, world)
    all_reduce(inc)
    Y = reverse_step(X, theta, W1_0, W2_0, eta, b, alpha_r, inc, Xp, rank, world)
    all_reduce(Y)
    return Y
