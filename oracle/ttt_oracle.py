"""fp64 CPU oracle of the TTT-MLP layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA path:
the recurrence itself lives in ``ttt_oracle.c`` (plain C, fp64), the dense
steps around it are numpy fp64 matrix products written out below.

Sources (One-Minute Video Generation with Test-Time Training):
  * paper notes page, "关键设计 / TTT-MLP 层": f(u;W) = W2 GELU(W1 u) with hidden
    width 4d, the loss ||f(theta_K x; W) - theta_V x||^2, one gradient step per
    token, output z_t = f(theta_Q x_t; W_t);
  * paper notes page, "关键设计 / 门控 + 双向": gate(TTT, X; alpha) =
    tanh(alpha) * TTT(X) + X with alpha a learned vector; a forward TTT pass,
    then a reverse one, sharing theta but each with its own gate.

Readings taken where the pages are silent:
  * the reverse pass runs on the gated forward output X' (sequential
    composition: the forward pass first, the reverse pass after it);
  * both directions start from the same W_0 and use the same theta;
  * per-head mode: X is [H, T, d] and theta is [H, d, d] (one projection per
    head); full mode: X is [T, D] and theta is [H*d, D] (nn.Linear layout),
    the heads' outputs concatenated back to D = H*d channels, no output
    projection;
  * chunks (b > 1) take every gradient at the chunk-start state and read token
    t with the prefix state (see ttt_oracle.c).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ttt_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libttt_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile ttt_oracle.c into libttt_oracle.so next to it (gcc, fp64, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-D_GNU_SOURCE", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def configure(lib):
    """Declare the argument and result types of the C functions on a loaded
    ctypes library (the oracle's own, or a copy built from another source)."""
    lib.ttt_ref_gelu.restype = ctypes.c_double
    lib.ttt_ref_gelu.argtypes = [ctypes.c_double]
    lib.ttt_ref_gelu_prime.restype = ctypes.c_double
    lib.ttt_ref_gelu_prime.argtypes = [ctypes.c_double]
    lib.ttt_ref_inner_loss_grad.restype = ctypes.c_double
    lib.ttt_ref_inner_loss_grad.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp]
    lib.ttt_ref_mlp_apply.restype = None
    lib.ttt_ref_mlp_apply.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp]
    lib.ttt_ref_scan_per_token.restype = None
    lib.ttt_ref_scan_per_token.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] + [_dp] * 6
    lib.ttt_ref_scan_chunked.restype = None
    lib.ttt_ref_scan_chunked.argtypes = [ctypes.c_int] * 6 + [ctypes.c_double] + [_dp] * 6
    lib.ttt_ref_scan_heads.restype = None
    lib.ttt_ref_scan_heads.argtypes = [ctypes.c_int] * 6 + [ctypes.c_double] + [_dp] * 6
    lib.ttt_ref_num_threads.restype = ctypes.c_int
    lib.ttt_ref_num_threads.argtypes = []
    lib.ttt_ref_linear_grad.restype = ctypes.c_double
    lib.ttt_ref_linear_grad.argtypes = [ctypes.c_int, _dp, _dp, _dp, _dp]
    lib.ttt_ref_linear_apply.restype = None
    lib.ttt_ref_linear_apply.argtypes = [ctypes.c_int, _dp, _dp, _dp]
    lib.ttt_ref_linear_scan_per_token.restype = None
    lib.ttt_ref_linear_scan_per_token.argtypes = [ctypes.c_int] * 3 + [ctypes.c_double] + [_dp] * 5
    lib.ttt_ref_linear_scan_chunked.restype = None
    lib.ttt_ref_linear_scan_chunked.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] + [_dp] * 5
    lib.ttt_ref_linear_scan_heads.restype = None
    lib.ttt_ref_linear_scan_heads.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double] + [_dp] * 5
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_dp)


def num_threads() -> int:
    """OpenMP threads the C scan uses."""
    return int(_load().ttt_ref_num_threads())


# ---------------------------------------------------------------- inner model
def gelu(a: float) -> float:
    """erf-GELU of one value (fp64)."""
    return float(_load().ttt_ref_gelu(float(a)))


def gelu_prime(a: float) -> float:
    """Derivative of erf-GELU at one value (fp64)."""
    return float(_load().ttt_ref_gelu_prime(float(a)))


def inner_loss_grad(W1, W2, k, v):
    """Loss ||W2 GELU(W1 k) - v||^2 and its gradients (G1 [m,d], G2 [d,m])."""
    W1, W2, k, v = _f64(W1), _f64(W2), _f64(k), _f64(v)
    m, d = W1.shape
    G1 = np.empty((m, d)); G2 = np.empty((d, m))
    loss = _load().ttt_ref_inner_loss_grad(d, m, _ptr(W1), _ptr(W2), _ptr(k), _ptr(v), _ptr(G1), _ptr(G2))
    return float(loss), G1, G2


def mlp_apply(W1, W2, u) -> np.ndarray:
    """f(u; W) = W2 GELU(W1 u)."""
    W1, W2, u = _f64(W1), _f64(W2), _f64(u)
    m, d = W1.shape
    z = np.empty(d)
    _load().ttt_ref_mlp_apply(d, m, _ptr(W1), _ptr(W2), _ptr(u), _ptr(z))
    return z


# ---------------------------------------------------------------- the scan
def scan(Q, K, V, W1_0, W2_0, eta: float, b: int, reverse: bool = False, zmode: int = 0,
         per_token: bool = False):
    """One head, one direction.  Q, K, V: [T, d].  Returns (Z [T,d], W1_T, W2_T).

    per_token=True runs the literal per-token rule (no chunk code at all);
    otherwise the chunked primal form with chunk size b (zmode 1 = chunk-end
    reading, used only to show it differs from the graded prefix reading).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    W1 = _f64(W1_0).copy(); W2 = _f64(W2_0).copy()
    T, d = Q.shape
    m = W1.shape[0]
    Z = np.zeros((T, d))
    lib = _load()
    if per_token:
        lib.ttt_ref_scan_per_token(T, d, m, int(reverse), float(eta), _ptr(Q), _ptr(K), _ptr(V),
                                   _ptr(W1), _ptr(W2), _ptr(Z))
    else:
        lib.ttt_ref_scan_chunked(T, d, m, int(b), int(reverse), int(zmode), float(eta), _ptr(Q), _ptr(K),
                                 _ptr(V), _ptr(W1), _ptr(W2), _ptr(Z))
    return Z, W1, W2


def scan_heads(Q, K, V, W1_0, W2_0, eta: float, b: int, reverse: bool = False):
    """H heads in parallel (OpenMP).  Q, K, V: [H, T, d]; W1_0 [H, m, d]; W2_0 [H, d, m]."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    W1 = _f64(W1_0).copy(); W2 = _f64(W2_0).copy()
    H, T, d = Q.shape
    m = W1.shape[1]
    Z = np.zeros((H, T, d))
    _load().ttt_ref_scan_heads(H, T, d, m, int(b), int(reverse), float(eta), _ptr(Q), _ptr(K), _ptr(V),
                               _ptr(W1), _ptr(W2), _ptr(Z))
    return Z, W1, W2


# ---------------------------------------------------------------- projections
def project_per_head(X, theta) -> np.ndarray:
    """Per-head mode: u[h, t] = theta[h] @ x[h, t].  X [H,T,d], theta [H,d,d] -> [H,T,d]."""
    X, theta = _f64(X), _f64(theta)
    return np.einsum("hed,htd->hte", theta, X)


def project_full(X, theta, row_block: int = 1 << 15) -> np.ndarray:
    """Full mode: U = X @ theta^T.  X [T,D], theta [N,D] -> [T,N] (fp64, by row blocks)."""
    theta = _f64(theta)
    T = X.shape[0]
    out = np.empty((T, theta.shape[0]))
    for r0 in range(0, T, row_block):
        out[r0:r0 + row_block] = _f64(X[r0:r0 + row_block]) @ theta.T
    return out


def gate(X, Z, alpha) -> np.ndarray:
    """tanh(alpha) * Z + X, alpha broadcast over the channel (last) axis."""
    return _f64(X) + np.tanh(_f64(alpha)) * _f64(Z)


# ---------------------------------------------------------------- the layer
def _heads_from_full(U, H: int, d: int) -> np.ndarray:
    T = U.shape[0]
    return np.ascontiguousarray(U.reshape(T, H, d).transpose(1, 0, 2))


def _full_from_heads(Zh) -> np.ndarray:
    H, T, d = Zh.shape
    return np.ascontiguousarray(Zh.transpose(1, 0, 2).reshape(T, H * d))


def direction(X, theta_q, theta_k, theta_v, W1_0, W2_0, eta: float, b: int, reverse: bool,
              per_head: bool, H: int | None = None):
    """One TTT direction on input X; returns (Z in X's layout, W1_T, W2_T)."""
    if per_head:
        Q = project_per_head(X, theta_q); K = project_per_head(X, theta_k); V = project_per_head(X, theta_v)
        Z, W1, W2 = scan_heads(Q, K, V, W1_0, W2_0, eta, b, reverse)
        return Z, W1, W2
    d = W1_0.shape[2]
    H = H if H is not None else W1_0.shape[0]
    Q = _heads_from_full(project_full(X, theta_q), H, d)
    K = _heads_from_full(project_full(X, theta_k), H, d)
    V = _heads_from_full(project_full(X, theta_v), H, d)
    Zh, W1, W2 = scan_heads(Q, K, V, W1_0, W2_0, eta, b, reverse)
    return _full_from_heads(Zh), W1, W2


def _alpha_layout(alpha, X, per_head: bool):
    """alpha has D = H*d entries; in per-head mode channel (h, j) is alpha[h*d + j]."""
    a = _f64(alpha)
    if per_head:
        H, _, d = X.shape
        return a.reshape(H, 1, d)
    return a


def layer_forward(X, theta_q, theta_k, theta_v, W1_0, W2_0, eta: float, b: int, dirs: str,
                  alpha_f=None, alpha_r=None, per_head: bool = True) -> dict:
    """The gated TTT layer.

    dirs: "fwd" -> Y = gate_f(X, fwd(X));  "rev" -> Y = gate_r(X, rev(X));
          "bidir" -> X' = gate_f(X, fwd(X)), Y = gate_r(X', rev(X')).
    Returns dict with Y, Z_f / Z_r (pre-gate), X' (bidir) and final states.
    """
    out = {}
    if dirs in ("fwd", "bidir"):
        Zf, W1f, W2f = direction(X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, False, per_head)
        Xp = gate(X, Zf, _alpha_layout(alpha_f, X, per_head))
        out.update(Z_f=Zf, W1_f=W1f, W2_f=W2f)
        if dirs == "fwd":
            out["Y"] = Xp
            return out
        out["Xp"] = Xp
        src = Xp
    else:
        src = _f64(X)
    Zr, W1r, W2r = direction(src, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, True, per_head)
    out.update(Z_r=Zr, W1_r=W1r, W2_r=W2r, Y=gate(src, Zr, _alpha_layout(alpha_r, X, per_head)))
    return out


def full_mode_heads(X, theta_q, theta_k, theta_v, W1_0, W2_0, eta: float, b: int, heads,
                    reverse: bool = False):
    """Full mode, a subset of heads only: the pre-gate Z of the listed heads for one
    direction run directly on X ([T, len(heads)*d]; head order as listed).

    Used for sampled checks at full size: the forward pass of a head needs only
    that head's rows of theta; the reverse pass equals this when the forward
    gate is zero (alpha_f = 0 makes X' = X exactly).
    """
    d = W1_0.shape[2]
    rows = np.concatenate([np.arange(h * d, (h + 1) * d) for h in heads])
    sel = lambda th: np.asarray(th)[rows]
    nh = len(heads)
    Q = _heads_from_full(project_full(X, sel(theta_q)), nh, d)
    K = _heads_from_full(project_full(X, sel(theta_k)), nh, d)
    V = _heads_from_full(project_full(X, sel(theta_v)), nh, d)
    W1 = _f64(W1_0)[list(heads)]; W2 = _f64(W2_0)[list(heads)]
    Zh, W1T, W2T = scan_heads(Q, K, V, W1, W2, eta, b, reverse)
    return _full_from_heads(Zh), W1T, W2T


# ---------------------------------------------------------------- TTT-Linear
# The linear variant (paper notes page, "实验关键数据 / 消融实验": TTT-Linear):
# f(u; W) = W u with W [d, d]; loss, update rule, prefix reading, gate and
# directions as for the MLP state.
def linear_grad(W, k, v):
    """Loss ||W k - v||^2 and its gradient 2 (W k - v) k^T."""
    W, k, v = _f64(W), _f64(k), _f64(v)
    d = W.shape[0]
    G = np.empty((d, d))
    loss = _load().ttt_ref_linear_grad(d, _ptr(W), _ptr(k), _ptr(v), _ptr(G))
    return float(loss), G


def linear_apply(W, u) -> np.ndarray:
    """f(u; W) = W u."""
    W, u = _f64(W), _f64(u)
    z = np.empty(W.shape[0])
    _load().ttt_ref_linear_apply(W.shape[0], _ptr(W), _ptr(u), _ptr(z))
    return z


def linear_scan(Q, K, V, W_0, eta: float, b: int, reverse: bool = False, per_token: bool = False):
    """One head, one direction.  Q, K, V: [T, d].  Returns (Z [T, d], W_T)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    W = _f64(W_0).copy()
    T, d = Q.shape
    Z = np.zeros((T, d))
    lib = _load()
    if per_token:
        lib.ttt_ref_linear_scan_per_token(T, d, int(reverse), float(eta), _ptr(Q), _ptr(K), _ptr(V), _ptr(W),
                                          _ptr(Z))
    else:
        lib.ttt_ref_linear_scan_chunked(T, d, int(b), int(reverse), float(eta), _ptr(Q), _ptr(K), _ptr(V),
                                        _ptr(W), _ptr(Z))
    return Z, W


def linear_scan_heads(Q, K, V, W_0, eta: float, b: int, reverse: bool = False):
    """H heads (OpenMP).  Q, K, V: [H, T, d]; W_0 [H, d, d]."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    W = _f64(W_0).copy()
    H, T, d = Q.shape
    Z = np.zeros((H, T, d))
    _load().ttt_ref_linear_scan_heads(H, T, d, int(b), int(reverse), float(eta), _ptr(Q), _ptr(K), _ptr(V),
                                      _ptr(W), _ptr(Z))
    return Z, W


def linear_direction(X, theta_q, theta_k, theta_v, W_0, eta: float, b: int, reverse: bool, per_head: bool):
    """One TTT-Linear direction on input X; returns (Z in X's layout, W_T)."""
    if per_head:
        Q = project_per_head(X, theta_q); K = project_per_head(X, theta_k); V = project_per_head(X, theta_v)
        return linear_scan_heads(Q, K, V, W_0, eta, b, reverse)
    H, d = W_0.shape[0], W_0.shape[2]
    Q = _heads_from_full(project_full(X, theta_q), H, d)
    K = _heads_from_full(project_full(X, theta_k), H, d)
    V = _heads_from_full(project_full(X, theta_v), H, d)
    Zh, W = linear_scan_heads(Q, K, V, W_0, eta, b, reverse)
    return _full_from_heads(Zh), W


def linear_layer_forward(X, theta_q, theta_k, theta_v, W_0, eta: float, b: int, dirs: str, alpha_f=None,
                         alpha_r=None, per_head: bool = True) -> dict:
    """The gated TTT-Linear layer, composed as layer_forward composes the MLP one."""
    out = {}
    if dirs in ("fwd", "bidir"):
        Zf, Wf = linear_direction(X, theta_q, theta_k, theta_v, W_0, eta, b, False, per_head)
        Xp = gate(X, Zf, _alpha_layout(alpha_f, X, per_head))
        out.update(Z_f=Zf, W_f=Wf)
        if dirs == "fwd":
            out["Y"] = Xp
            return out
        out["Xp"] = Xp
        src = Xp
    else:
        src = _f64(X)
    Zr, Wr = linear_direction(src, theta_q, theta_k, theta_v, W_0, eta, b, True, per_head)
    out.update(Z_r=Zr, W_r=Wr, Y=gate(src, Zr, _alpha_layout(alpha_r, X, per_head)))
    return out
