"""Pins of the fp64 TTT-Linear oracle against things other than itself.

The linear variant (One-Minute Video Generation with Test-Time Training, paper
notes page, "实验关键数据 / 消融实验": TTT-Linear, a linear hidden state) is the
same layer with f(u; W) = W u.  Independent means: central finite differences,
torch autograd, exact rational arithmetic on a scalar hand case, a separately
written matrix (dual) form of the chunk, closed forms and invariants.  A dropped
factor 2, a wrong sign, a transposed gradient, gradients at the running state
or z read before the update fails at least one of them.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as O


def _rand(shape, rng, scale=1.0):
    return rng.normal(size=shape) * scale


@pytest.mark.parametrize("d", [1, 2, 3, 5])
def test_linear_gradient_central_differences(d):
    rng = np.random.default_rng(d)
    W, k, v = _rand((d, d), rng), _rand(d, rng), _rand(d, rng)
    loss, G = O.linear_grad(W, k, v)
    assert loss == pytest.approx(float(np.sum((W @ k - v) ** 2)), rel=1e-13)
    h = 1e-6
    for i in range(d):
        for j in range(d):
            Wp, Wm = W.copy(), W.copy()
            Wp[i, j] += h
            Wm[i, j] -= h
            fd = (O.linear_grad(Wp, k, v)[0] - O.linear_grad(Wm, k, v)[0]) / (2 * h)
            assert G[i, j] == pytest.approx(fd, rel=1e-6, abs=1e-8)


def test_linear_gradient_matches_autograd():
    rng = np.random.default_rng(7)
    d = 6
    W, k, v = _rand((d, d), rng), _rand(d, rng), _rand(d, rng)
    Wt = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    loss = ((Wt @ torch.tensor(k) - torch.tensor(v)) ** 2).sum()
    loss.backward()
    np.testing.assert_allclose(O.linear_grad(W, k, v)[1], Wt.grad.numpy(), rtol=1e-13, atol=1e-13)


def _hand_scalar(q, k, v, w0, eta, b):
    """d = 1 in exact rational arithmetic, written from the rule: the gradient
    of (w k - v)^2 is 2 (w k - v) k, taken at the chunk-start w; token t is
    read with the running w after its own update."""
    w = Fraction(w0)
    z = []
    for s0 in range(0, len(q), b):
        wc = w
        for t in range(s0, min(s0 + b, len(q))):
            w = w - Fraction(eta) * 2 * (wc * Fraction(k[t]) - Fraction(v[t])) * Fraction(k[t])
            z.append(w * Fraction(q[t]))
    return [float(x) for x in z], float(w)


@pytest.mark.parametrize("b", [1, 2, 3])
def test_linear_scalar_hand_case_exact(b):
    q = [0.5, -1.25, 2.0, 0.75, -0.5]
    k = [1.0, 0.5, -1.5, 2.0, 0.25]
    v = [0.25, -1.0, 0.5, 1.0, -2.0]
    w0, eta = 0.75, 0.125
    z_ref, w_ref = _hand_scalar(q, k, v, w0, eta, b)
    arr = lambda x: np.array(x, dtype=np.float64).reshape(-1, 1)
    Z, W = O.linear_scan(arr(q), arr(k), arr(v), np.array([[w0]]), eta, b)
    np.testing.assert_allclose(Z[:, 0], z_ref, rtol=1e-15, atol=1e-15)
    assert W[0, 0] == pytest.approx(w_ref, rel=1e-15)


def _dual_chunked(Q, K, V, W0, eta, b):
    """The chunk as matrix products, written independently of the oracle:
    E = K Wc^T - V, Z = Q Wc^T - 2 eta tril(Q K^T) E, W = Wc - 2 eta E^T K."""
    W = W0.copy()
    Z = np.zeros_like(Q)
    for s0 in range(0, Q.shape[0], b):
        sl = slice(s0, min(s0 + b, Q.shape[0]))
        q, k, v = Q[sl], K[sl], V[sl]
        E = k @ W.T - v
        Z[sl] = q @ W.T - 2 * eta * np.tril(q @ k.T) @ E
        W = W - 2 * eta * E.T @ k
    return Z, W


@pytest.mark.parametrize("b,T", [(1, 9), (4, 17), (16, 40), (64, 130)])
def test_linear_primal_matches_dual_form(b, T):
    rng = np.random.default_rng(b * 100 + T)
    d = 8
    Q, K, V = _rand((T, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    W0 = _rand((d, d), rng, 1 / np.sqrt(d))
    eta = 0.01
    Z, W = O.linear_scan(Q, K, V, W0, eta, b)
    Zd, Wd = _dual_chunked(Q, K, V, W0, eta, b)
    np.testing.assert_allclose(Z, Zd, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(W, Wd, rtol=1e-11, atol=1e-11)


def test_linear_chunk_of_one_is_the_per_token_rule():
    rng = np.random.default_rng(3)
    T, d = 50, 5
    Q, K, V = _rand((T, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    W0 = _rand((d, d), rng, 0.3)
    Z1, W1 = O.linear_scan(Q, K, V, W0, 0.02, 1)
    Zp, Wp = O.linear_scan(Q, K, V, W0, 0.02, 1, per_token=True)
    np.testing.assert_array_equal(Z1, Zp)
    np.testing.assert_array_equal(W1, Wp)


def test_linear_eta_zero_closed_form():
    rng = np.random.default_rng(5)
    T, d = 20, 4
    Q, K, V = _rand((T, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    W0 = _rand((d, d), rng)
    Z, W = O.linear_scan(Q, K, V, W0, 0.0, 4)
    np.testing.assert_allclose(Z, Q @ W0.T, rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(W, W0)


def test_linear_descent_property_small_eta():
    rng = np.random.default_rng(11)
    T, d = 30, 6
    Q, K, V = _rand((T, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    W = _rand((d, d), rng, 0.3)
    for t in range(T):
        before = O.linear_grad(W, K[t], V[t])[0]
        _, W = O.linear_scan(Q[t:t + 1], K[t:t + 1], V[t:t + 1], W, 1e-3, 1)
        assert O.linear_grad(W, K[t], V[t])[0] < before


def test_linear_reverse_is_flip_forward_flip():
    rng = np.random.default_rng(13)
    T, d, b = 37, 4, 8
    Q, K, V = _rand((T, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    W0 = _rand((d, d), rng, 0.5)
    Zr, Wr = O.linear_scan(Q, K, V, W0, 0.01, b, reverse=True)
    Zf, Wf = O.linear_scan(Q[::-1], K[::-1], V[::-1], W0, 0.01, b)
    np.testing.assert_array_equal(Zr, Zf[::-1])
    np.testing.assert_array_equal(Wr, Wf)


def test_linear_heads_equal_single_head_runs():
    rng = np.random.default_rng(17)
    H, T, d, b = 3, 21, 4, 5
    Q, K, V = _rand((H, T, d), rng), _rand((H, T, d), rng), _rand((H, T, d), rng)
    W0 = _rand((H, d, d), rng, 0.5)
    Z, W = O.linear_scan_heads(Q, K, V, W0, 0.01, b)
    for h in range(H):
        Zh, Wh = O.linear_scan(Q[h], K[h], V[h], W0[h], 0.01, b)
        np.testing.assert_array_equal(Z[h], Zh)
        np.testing.assert_array_equal(W[h], Wh)


def test_linear_layer_alpha_zero_is_identity_and_bidir_composes():
    rng = np.random.default_rng(19)
    H, T, d = 2, 12, 4
    X = _rand((H, T, d), rng)
    th = [_rand((H, d, d), rng, 0.5) for _ in range(3)]
    W0 = _rand((H, d, d), rng, 0.5)
    zero = np.zeros(H * d)
    out = O.linear_layer_forward(X, *th, W0, 0.01, 4, "bidir", alpha_f=zero, alpha_r=zero, per_head=True)
    np.testing.assert_array_equal(out["Y"], X)
    a = np.full(H * d, 0.1)
    out = O.linear_layer_forward(X, *th, W0, 0.01, 4, "bidir", alpha_f=a, alpha_r=a, per_head=True)
    Zf, _ = O.linear_direction(X, *th, W0, 0.01, 4, False, True)
    Xp = X + np.tanh(0.1) * Zf
    Zr, _ = O.linear_direction(Xp, *th, W0, 0.01, 4, True, True)
    np.testing.assert_allclose(out["Y"], Xp + np.tanh(0.1) * Zr, rtol=1e-14, atol=1e-14)


def test_linear_full_mode_with_block_diagonal_theta_equals_per_head_mode():
    rng = np.random.default_rng(23)
    H, T, d = 3, 10, 4
    D = H * d
    Xh = _rand((H, T, d), rng)
    th_h = [_rand((H, d, d), rng, 0.5) for _ in range(3)]
    W0 = _rand((H, d, d), rng, 0.5)
    Xf = Xh.transpose(1, 0, 2).reshape(T, D)
    th_f = []
    for th in th_h:
        full = np.zeros((D, D))
        for h in range(H):
            full[h * d:(h + 1) * d, h * d:(h + 1) * d] = th[h]
        th_f.append(full)
    a = np.full(D, 0.1)
    ph = O.linear_layer_forward(Xh, *th_h, W0, 0.01, 3, "bidir", alpha_f=a, alpha_r=a, per_head=True)
    fm = O.linear_layer_forward(Xf, *th_f, W0, 0.01, 3, "bidir", alpha_f=a, alpha_r=a, per_head=False)
    np.testing.assert_allclose(fm["Y"], ph["Y"].transpose(1, 0, 2).reshape(T, D), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("b", [1, 8])
def test_linear_scan_is_causal_token_by_token(b):
    rng = np.random.default_rng(31 + b)
    T, d, t0 = 21, 4, 11
    Q, K, V = _rand((T, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    W0 = _rand((d, d), rng, 0.5)
    K2, V2 = K.copy(), V.copy()
    K2[t0] += 0.5
    V2[t0] -= 0.5
    for reverse in (False, True):
        Z, _ = O.linear_scan(Q, K, V, W0, 0.02, b, reverse=reverse)
        Zp, _ = O.linear_scan(Q, K2, V2, W0, 0.02, b, reverse=reverse)
        same = slice(t0 + 1, T) if reverse else slice(0, t0)
        np.testing.assert_array_equal(Z[same], Zp[same])
        assert np.abs(Z[t0] - Zp[t0]).max() > 1e-6
