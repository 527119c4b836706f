"""fp64 CPU oracle of the TTT-MLP layer's backward pass (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the CUDA library never uses it.

Training the layer adjusts the projections theta_Q/K/V, the initial hidden
state W_0 and the gate vectors (paper notes page, "损失函数 / 训练策略": the TTT
layers and gates are fine-tuned; "关键设计 / 门控 + 双向机制": the gate vectors
are learned).  For a scalar training loss with upstream gradient dY = dLoss/dY
this module returns the gradients with respect to X, theta_Q/K/V, W1_0, W2_0,
alpha_f and alpha_r.  It writes the layer's forward computation once more in
plain PyTorch fp64 -- the same definition as ttt_oracle.c, step for step:

  per chunk of b tokens in walking order, state (W1, W2) at the chunk start:
    a_s = W1 k_s, g_s = GELU(a_s), e_s = W2 g_s - v_s                 (every s of the chunk)
    dl/dW2 (s) = 2 e_s g_s^T,  dl/dW1 (s) = [2 (W2^T e_s) * GELU'(a_s)] k_s^T
    W_t = W_chunk_start - eta * sum_{s <= t} dl/dW (s)                 (a running sum)
    z_t = W2_t GELU(W1_t q_t)
  out = x + tanh(alpha) * z;  bidirectional: forward on X, reverse on X'

-- and lets torch.autograd form the vector-Jacobian product (a library
primitive as one step).  The forward restatement is pinned to the C oracle's
forward and the gradients to central finite differences of the C oracle.
"""
from __future__ import annotations

import math

import numpy as np
import torch

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def gelu(a: torch.Tensor) -> torch.Tensor:
    """erf-GELU: a * Phi(a)."""
    return 0.5 * a * (1.0 + torch.erf(a / _SQRT2))


def gelu_prime(a: torch.Tensor) -> torch.Tensor:
    """d GELU / da = Phi(a) + a phi(a)."""
    return 0.5 * (1.0 + torch.erf(a / _SQRT2)) + a * torch.exp(-0.5 * a * a) * _INV_SQRT_2PI


def scan(Q, K, V, W1, W2, eta: float, b: int, reverse: bool):
    """One direction for H heads at once.  Q, K, V [H, T, d]; W1 [H, m, d];
    W2 [H, d, m] (torch fp64).  Returns (Z [H, T, d], W1_T, W2_T)."""
    T = Q.shape[1]
    order = torch.arange(T - 1, -1, -1) if reverse else torch.arange(T)
    zs = []
    for s0 in range(0, T, b):
        idx = order[s0:s0 + b]
        q, k, v = Q[:, idx], K[:, idx], V[:, idx]                    # [H, n, d]
        a = torch.einsum("hij,hnj->hni", W1, k)                       # [H, n, m]
        g = gelu(a)
        e = torch.einsum("hji,hni->hnj", W2, g) - v                   # [H, n, d]
        G2 = 2.0 * e[..., :, None] * g[..., None, :]                  # [H, n, d, m]
        delta = 2.0 * torch.einsum("hnj,hji->hni", e, W2) * gelu_prime(a)
        G1 = delta[..., :, None] * k[..., None, :]                    # [H, n, m, d]
        W1t = W1[:, None] - eta * torch.cumsum(G1, dim=1)             # prefix states, token by token
        W2t = W2[:, None] - eta * torch.cumsum(G2, dim=1)
        aq = torch.einsum("hnij,hnj->hni", W1t, q)
        zs.append(torch.einsum("hnji,hni->hnj", W2t, gelu(aq)))
        W1, W2 = W1t[:, -1], W2t[:, -1]
    Z = torch.cat(zs, dim=1)                                          # walking order
    if reverse:
        Z = Z.flip(1)
    return Z, W1, W2


def _project(X, theta, per_head: bool, H: int, d: int):
    if per_head:
        return torch.einsum("hed,htd->hte", theta, X)                 # [H, T, d]
    T = X.shape[0]
    return (X @ theta.T).reshape(T, H, d).permute(1, 0, 2)            # [T, H d] -> [H, T, d]


def _to_layout(Zh, per_head: bool):
    if per_head:
        return Zh
    H, T, d = Zh.shape
    return Zh.permute(1, 0, 2).reshape(T, H * d)


def _alpha(alpha, per_head: bool, H: int, d: int):
    return alpha.reshape(H, 1, d) if per_head else alpha


def layer_forward(X, theta_q, theta_k, theta_v, W1_0, W2_0, alpha_f, alpha_r, eta: float, b: int, dirs: str,
                  per_head: bool) -> dict:
    """The gated layer in torch fp64 (differentiable); the same composition as
    ttt_oracle.layer_forward.  Returns Y and the pre-gate Z of each direction."""
    H, m, d = W1_0.shape
    out = {}

    def direction(src, reverse):
        U = [_project(src, th, per_head, H, d) for th in (theta_q, theta_k, theta_v)]
        Zh, _, _ = scan(U[0], U[1], U[2], W1_0, W2_0, eta, b, reverse)
        return _to_layout(Zh, per_head)

    src = X
    if dirs in ("fwd", "bidir"):
        Zf = direction(X, False)
        out["Z_f"] = Zf
        src = X + torch.tanh(_alpha(alpha_f, per_head, H, d)) * Zf
        if dirs == "fwd":
            out["Y"] = src
            return out
    Zr = direction(src, True)
    out["Z_r"] = Zr
    out["Y"] = src + torch.tanh(_alpha(alpha_r, per_head, H, d)) * Zr
    return out


NAMES = ("X", "theta_q", "theta_k", "theta_v", "W1_0", "W2_0", "alpha_f", "alpha_r")


def layer_backward(inputs: dict, dY, eta: float, b: int, dirs: str, per_head: bool) -> dict:
    """Gradients of sum(dY * Y) with respect to every input (fp64 numpy out).

    inputs: X, theta_q, theta_k, theta_v, W1_0, W2_0, alpha_f, alpha_r as
    arrays or tensors (any float dtype; converted to fp64).  The gradient of a
    gate vector that the direction does not use is zero."""
    t = {k: torch.tensor(np.asarray(inputs[k], dtype=np.float64), requires_grad=True) for k in NAMES}
    out = layer_forward(t["X"], t["theta_q"], t["theta_k"], t["theta_v"], t["W1_0"], t["W2_0"], t["alpha_f"],
                        t["alpha_r"], eta, b, dirs, per_head)
    dy = torch.tensor(np.asarray(dY, dtype=np.float64))
    grads = torch.autograd.grad(out["Y"], [t[k] for k in NAMES], grad_outputs=dy, allow_unused=True)
    res = {}
    for k, g in zip(NAMES, grads):
        res["d" + k] = np.zeros(t[k].shape) if g is None else g.detach().numpy()
    res["Y"] = out["Y"].detach().numpy()
    return res
