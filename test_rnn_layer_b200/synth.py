"""Seeded synthetic inputs for the TTT-MLP layer (shared by tests, smoke and bench).

This module holds no arithmetic of the method: it only draws the inputs the
pages' workloads would feed the layer (Gaussian stand-ins for CogVideo-X
tokens, fan-in initialised projections and hidden states) at the pages'
sequence lengths.  Both the CUDA path and the oracle receive exactly these
tensors.

Draw order with one torch.Generator seeded by ``seed`` on ``device``:
X, theta_Q, theta_K, theta_V, W1_0, W2_0, each drawn as fp32 N(0, 1) and
scaled by the stated standard deviation, then rounded to bf16 where the
workload is bf16 (X and theta only; W_0 and alpha stay fp32).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int            # heads
    d: int            # head dim; the hidden width is m = 4 d
    T: int            # tokens
    b: int            # chunk (mini-batch) size; 1 = per-token rule
    dirs: str         # "fwd" | "rev" | "bidir"
    dtype: str        # "f32" | "bf16" (X, theta, Y)
    per_head: bool    # True: X [H,T,d], theta [H,d,d]; False: X [T,D], theta [H*d, D]
    eta: float        # learning rate as the workload states it
    alpha: float = 0.1
    D: int = 0        # model dim (full mode); H*d in per-head mode

    @property
    def m(self) -> int:
        return 4 * self.d

    @property
    def model_dim(self) -> int:
        return self.D if self.D else self.H * self.d

    @property
    def eta_eff(self) -> float:
        """The step size passed to the layer: eta / d.

        With the literal squared-norm loss the stated eta diverges within a
        few tokens even in fp64; eta / d is the same rule written for the
        mean-squared loss (1/d)||.||^2, and stays finite over 313k tokens.
        """
        return self.eta / self.d

    def with_T(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the benchmark description, in order.
TINY = Workload("tiny-h1-d16-T256-b1-fwd-f32", H=1, d=16, T=256, b=1, dirs="fwd", dtype="f32",
                per_head=True, eta=0.1)
CAUSAL = Workload("causal-h4-d64-T4096-b1-fwd-f32", H=4, d=64, T=4096, b=1, dirs="fwd", dtype="f32",
                  per_head=True, eta=0.05)
MINIBATCH = Workload("bidir-h48-d64-T32768-b16-bf16", H=48, d=64, T=32768, b=16, dirs="bidir",
                     dtype="bf16", per_head=True, eta=0.05)
SCALE18S = Workload("bidir-h48-d64-T102400-b64-bf16", H=48, d=64, T=102400, b=64, dirs="bidir",
                    dtype="bf16", per_head=True, eta=0.05)
FULL63S = Workload("layer-D3072-h48-d64-T313344-b64-bidir-bf16", H=48, d=64, T=313344, b=64,
                   dirs="bidir", dtype="bf16", per_head=False, eta=0.05, D=3072)

WORKLOADS = [TINY, CAUSAL, MINIBATCH, SCALE18S, FULL63S]


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def make_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu") -> dict:
    """Draw X, theta_Q/K/V, W1_0, W2_0, alpha_f, alpha_r for workload ``w``."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    dt = torch_dtype(w)

    def draw(shape, std):
        t = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t

    H, d, m, T = w.H, w.d, w.m, w.T
    if w.per_head:
        X = draw((H, T, d), 1.0).to(dt)
        th_std = math.sqrt(1.0 / d)
        thetas = [draw((H, d, d), th_std).to(dt) for _ in range(3)]
    else:
        D = w.model_dim
        X = draw((T, D), 1.0).to(dt)
        th_std = math.sqrt(1.0 / D)
        thetas = [draw((H * d, D), th_std).to(dt) for _ in range(3)]
    W1_0 = draw((H, m, d), math.sqrt(1.0 / d))
    W2_0 = draw((H, d, m), math.sqrt(1.0 / m))
    D = w.model_dim
    alpha_f = torch.full((D,), w.alpha, dtype=torch.float32, device=dev)
    alpha_r = torch.full((D,), w.alpha, dtype=torch.float32, device=dev)
    return dict(X=X, theta_q=thetas[0], theta_k=thetas[1], theta_v=thetas[2], W1_0=W1_0, W2_0=W2_0,
                alpha_f=alpha_f, alpha_r=alpha_r)


def make_linear_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu") -> dict:
    """The inputs of make_inputs plus the TTT-Linear initial state W_0 [H, d, d]
    ~ N(0, 1/d) (fan-in), drawn afterwards from the same generator sequence."""
    inp = make_inputs(w, seed, device)
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 1_000_003)
    inp["W_0"] = torch.randn((w.H, w.d, w.d), generator=g, device=dev, dtype=torch.float32).mul_(
        math.sqrt(1.0 / w.d))
    return inp


# The segment-local attention before the layer: 63 s of video in 3-s segments.
SEGMENTS_63S = 21


def segment_length(T: int, n_segments: int = SEGMENTS_63S) -> int:
    """Tokens per segment when T tokens cover ``n_segments`` equal segments
    (ceil(T / n); the last one is shorter when n does not divide T)."""
    return -(-T // n_segments)


def make_attention_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu",
                          qk_std: float = 1.0) -> dict:
    """Q_a, K_a, V_a [T, D] bf16 for the attention sublayer: Q_a and K_a
    N(0, qk_std^2), V_a N(0, 1), drawn in that order from a generator seeded
    ``seed + 2_000_003`` (independent of make_inputs' draws, whose X is the
    sublayer's residual)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 2_000_003)
    T, D = w.T, w.model_dim
    out = {}
    for k, std in (("Q_a", qk_std), ("K_a", qk_std), ("V_a", 1.0)):
        t = torch.randn((T, D), generator=g, device=dev, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out[k] = t.to(torch.bfloat16)
    return out
