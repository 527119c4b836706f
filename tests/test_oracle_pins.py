"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against mathematics the pages fix (One-Minute
Video Generation with Test-Time Training, paper notes page, "关键设计":
TTT-MLP layer definition; gate + bidirectional section), using independent
means: finite differences, torch autograd, mpmath at 40 digits, a separately
written dual (matrix) form of the chunk, closed forms and invariants.  A
dropped term, a wrong sign or index, a transposed operand or reading z with
the pre-update state fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import erf as sp_erf, ndtr

from oracle import ttt_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return np.array(rows)


def _np_gelu(a):
    return 0.5 * a * (1.0 + sp_erf(a / math.sqrt(2.0)))


def _np_gelu_prime(a):
    return ndtr(a) + a * np.exp(-0.5 * a * a) / math.sqrt(2 * math.pi)


def _rand_head(rng, T, d, scale_w=1.0):
    m = 4 * d
    Q = rng.normal(size=(T, d)); K = rng.normal(size=(T, d)); V = rng.normal(size=(T, d))
    W1 = rng.normal(size=(m, d)) * math.sqrt(1.0 / d) * scale_w
    W2 = rng.normal(size=(d, m)) * math.sqrt(1.0 / m) * scale_w
    return Q, K, V, W1, W2


# ------------------------------------------------------------------ GELU
def test_gelu_matches_normal_cdf_table():
    tab = _table("normal_cdf.txt")
    for x, phi in tab:
        assert O.gelu(x) == pytest.approx(x * phi, rel=1e-15, abs=1e-300)


def test_gelu_and_derivative_against_library_and_fd():
    xs = np.linspace(-6, 6, 97)
    for x in xs:
        assert O.gelu(x) == pytest.approx(x * ndtr(x), rel=1e-14, abs=1e-15)
        h = 1e-5
        fd = (O.gelu(x + h) - O.gelu(x - h)) / (2 * h)
        assert O.gelu_prime(x) == pytest.approx(fd, rel=1e-8, abs=1e-9)
    assert O.gelu_prime(0.0) == 0.5
    assert O.gelu(0.0) == 0.0


# ------------------------------------------------------------------ inner gradient
@pytest.mark.parametrize("d", [1, 2, 4])
def test_inner_gradient_central_differences(d):
    rng = np.random.default_rng(10 + d)
    m = 4 * d
    W1 = rng.normal(size=(m, d)); W2 = rng.normal(size=(d, m)) * 0.5
    k = rng.normal(size=d); v = rng.normal(size=d)
    _, G1, G2 = O.inner_loss_grad(W1, W2, k, v)
    h = 1e-6
    fd1 = np.zeros_like(W1); fd2 = np.zeros_like(W2)
    for idx in np.ndindex(*W1.shape):
        Wp = W1.copy(); Wp[idx] += h; Wm = W1.copy(); Wm[idx] -= h
        fd1[idx] = (O.inner_loss_grad(Wp, W2, k, v)[0] - O.inner_loss_grad(Wm, W2, k, v)[0]) / (2 * h)
    for idx in np.ndindex(*W2.shape):
        Wp = W2.copy(); Wp[idx] += h; Wm = W2.copy(); Wm[idx] -= h
        fd2[idx] = (O.inner_loss_grad(W1, Wp, k, v)[0] - O.inner_loss_grad(W1, Wm, k, v)[0]) / (2 * h)
    assert np.abs(fd1 - G1).max() <= 1e-6 * np.abs(G1).max()
    assert np.abs(fd2 - G2).max() <= 1e-6 * np.abs(G2).max()


def test_inner_gradient_matches_autograd():
    rng = np.random.default_rng(3)
    d, m = 8, 32
    W1 = rng.normal(size=(m, d)) / math.sqrt(d); W2 = rng.normal(size=(d, m)) / math.sqrt(m)
    k = rng.normal(size=d); v = rng.normal(size=d)
    loss, G1, G2 = O.inner_loss_grad(W1, W2, k, v)
    w1 = torch.tensor(W1, requires_grad=True); w2 = torch.tensor(W2, requires_grad=True)
    L = ((w2 @ torch.nn.functional.gelu(w1 @ torch.tensor(k)) - torch.tensor(v)) ** 2).sum()
    g1, g2 = torch.autograd.grad(L, [w1, w2])
    assert loss == pytest.approx(L.item(), rel=1e-14)
    np.testing.assert_allclose(G1, g1.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(G2, g2.numpy(), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ scan: independent forms
def _autograd_scan(Q, K, V, W1, W2, eta, b, reverse=False):
    """Brute force with torch autograd: gradient at the chunk-start state for every
    token, prefix state for the output (b = 1 is the per-token rule)."""
    gelu = torch.nn.functional.gelu
    W1 = torch.tensor(W1); W2 = torch.tensor(W2)
    T = Q.shape[0]
    order = list(range(T))[::-1] if reverse else list(range(T))
    Z = np.zeros_like(Q)
    for c0 in range(0, T, b):
        chunk = order[c0:c0 + b]
        W1c, W2c = W1.clone(), W2.clone()
        for t in chunk:
            w1 = W1c.clone().requires_grad_(True); w2 = W2c.clone().requires_grad_(True)
            L = ((w2 @ gelu(w1 @ torch.tensor(K[t])) - torch.tensor(V[t])) ** 2).sum()
            g1, g2 = torch.autograd.grad(L, [w1, w2])
            W1 = W1 - eta * g1; W2 = W2 - eta * g2
            Z[t] = (W2 @ gelu(W1 @ torch.tensor(Q[t]))).numpy()
    return Z, W1.numpy(), W2.numpy()


def _dual_scan(Q, K, V, W1, W2, eta, b):
    """The chunk written as matrix products (what a tensor-core kernel computes):
    A = K W1^T, G = GELU(A), E = G W2^T - V, Delta = (2E W2) * GELU'(A),
    Aq = Q W1^T - eta tril(Q K^T) Delta, Gq = GELU(Aq),
    Z = Gq W2^T - eta tril(Gq G^T) 2E; then W1 -= eta Delta^T K, W2 -= eta (2E)^T G."""
    W1 = W1.copy(); W2 = W2.copy()
    T = Q.shape[0]
    Z = np.zeros_like(Q)
    for s0 in range(0, T, b):
        k = K[s0:s0 + b]; q = Q[s0:s0 + b]; v = V[s0:s0 + b]
        n = k.shape[0]
        A = k @ W1.T
        G = _np_gelu(A)
        E2 = 2.0 * (G @ W2.T - v)
        Delta = (E2 @ W2) * _np_gelu_prime(A)
        tril = np.tril(np.ones((n, n)))
        Aq = q @ W1.T - eta * (tril * (q @ k.T)) @ Delta
        Gq = _np_gelu(Aq)
        Z[s0:s0 + b] = Gq @ W2.T - eta * (tril * (Gq @ G.T)) @ E2
        W1 -= eta * Delta.T @ k
        W2 -= eta * E2.T @ G
    return Z, W1, W2


@pytest.mark.parametrize("b,T", [(1, 7), (2, 7), (3, 7), (4, 8)])
def test_scan_matches_autograd_brute_force(b, T):
    rng = np.random.default_rng(100 + b)
    Q, K, V, W1, W2 = _rand_head(rng, T, 2)
    eta = 0.05
    for reverse in (False, True):
        Zo, W1o, W2o = O.scan(Q, K, V, W1, W2, eta, b, reverse=reverse)
        Zb, W1b, W2b = _autograd_scan(Q, K, V, W1, W2, eta, b, reverse=reverse)
        np.testing.assert_allclose(Zo, Zb, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(W1o, W1b, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(W2o, W2b, rtol=1e-12, atol=1e-13)


def test_scan_mpmath_hand_case():
    """d = 1, m = 4, T = 2 at 40 digits, gradients by mpmath numerical differentiation
    (no chain rule written anywhere): b = 1 and b = 2 (prefix reading)."""
    mp = pytest.importorskip("mpmath")
    mp.mp.dps = 40
    W1_0 = [0.7, -0.4, 1.1, 0.2]          # W1 [4 x 1]
    W2_0 = [0.3, 0.9, -0.5, 0.6]          # W2 [1 x 4]
    ks, vs, qs = [0.8, -1.3], [0.5, 0.2], [-0.6, 1.4]
    eta = 0.1

    def f(w1, w2, u):
        return mp.fsum(w2[i] * (u * w1[i]) * (1 + mp.erf(u * w1[i] / mp.sqrt(2))) / 2 for i in range(4))

    def grad(w1, w2, k, v):
        x0 = list(w1) + list(w2)
        loss = lambda *w: (f(w[:4], w[4:], k) - v) ** 2
        return [mp.diff(loss, x0, tuple(1 if j == i else 0 for j in range(8))) for i in range(8)]

    for b in (1, 2):
        w = [mp.mpf(x) for x in W1_0 + W2_0]
        zs = []
        for c0 in range(0, 2, b):
            wc = list(w)
            for t in range(c0, min(c0 + b, 2)):
                g = grad(wc[:4], wc[4:], mp.mpf(ks[t]), mp.mpf(vs[t]))
                w = [w[i] - eta * g[i] for i in range(8)]
                zs.append(f(w[:4], w[4:], mp.mpf(qs[t])))
        Z, W1T, W2T = O.scan(np.array(qs)[:, None], np.array(ks)[:, None], np.array(vs)[:, None],
                             np.array(W1_0)[:, None], np.array(W2_0)[None, :], eta, b)
        for t in range(2):
            assert Z[t, 0] == pytest.approx(float(zs[t]), rel=1e-13, abs=1e-15)
        np.testing.assert_allclose(W1T[:, 0], [float(x) for x in w[:4]], rtol=1e-13)
        np.testing.assert_allclose(W2T[0], [float(x) for x in w[4:]], rtol=1e-13)


@pytest.mark.parametrize("b,T", [(4, 37), (8, 64), (16, 50), (64, 128)])
def test_primal_matches_dual_form(b, T):
    rng = np.random.default_rng(200 + b)
    Q, K, V, W1, W2 = _rand_head(rng, T, 8)
    eta = 0.05 / 8
    Zo, W1o, W2o = O.scan(Q, K, V, W1, W2, eta, b)
    Zd, W1d, W2d = _dual_scan(Q, K, V, W1, W2, eta, b)
    scale = np.abs(Zo).max()
    assert np.abs(Zo - Zd).max() <= 1e-12 * scale
    np.testing.assert_allclose(W1o, W1d, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(W2o, W2d, rtol=1e-11, atol=1e-13)


def test_chunk_of_one_is_the_per_token_rule():
    rng = np.random.default_rng(5)
    Q, K, V, W1, W2 = _rand_head(rng, 40, 4)
    for reverse in (False, True):
        Zc, W1c, W2c = O.scan(Q, K, V, W1, W2, 0.01, 1, reverse=reverse)
        Zp, W1p, W2p = O.scan(Q, K, V, W1, W2, 0.01, 1, reverse=reverse, per_token=True)
        assert np.array_equal(Zc, Zp) and np.array_equal(W1c, W1p) and np.array_equal(W2c, W2p)


def test_eta_zero_closed_form():
    """eta = 0: the state never moves, z_t = W2_0 GELU(W1_0 theta_Q x_t)."""
    rng = np.random.default_rng(6)
    H, T, d = 2, 9, 4
    m = 4 * d
    X = rng.normal(size=(H, T, d))
    th = [rng.normal(size=(H, d, d)) / 2 for _ in range(3)]
    W1 = rng.normal(size=(H, m, d)) / 2; W2 = rng.normal(size=(H, d, m)) / 4
    for b in (1, 3):
        out = O.layer_forward(X, *th, W1, W2, 0.0, b, "fwd", alpha_f=np.full(H * d, 0.3), per_head=True)
        for h in range(H):
            for t in range(T):
                q = th[0][h] @ X[h, t]
                z = W2[h] @ (0.5 * (W1[h] @ q) * (1 + sp_erf((W1[h] @ q) / math.sqrt(2))))
                np.testing.assert_allclose(out["Z_f"][h, t], z, rtol=1e-13, atol=1e-14)
        np.testing.assert_array_equal(out["W1_f"], W1)


def test_descent_property_small_eta():
    """A small step lowers each token's own loss: l(W_t; x_t) < l(W_{t-1}; x_t)."""
    rng = np.random.default_rng(7)
    Q, K, V, W1, W2 = _rand_head(rng, 30, 4)
    eta = 1e-4 / 4
    for t in range(30):
        before = O.inner_loss_grad(W1, W2, K[t], V[t])[0]
        _, W1, W2 = O.scan(Q[t:t + 1], K[t:t + 1], V[t:t + 1], W1, W2, eta, 1)
        after = O.inner_loss_grad(W1, W2, K[t], V[t])[0]
        assert after < before


def test_reverse_is_flip_forward_flip():
    rng = np.random.default_rng(8)
    Q, K, V, W1, W2 = _rand_head(rng, 23, 4)
    for b in (1, 5, 8):
        Zr, W1r, W2r = O.scan(Q, K, V, W1, W2, 0.02, b, reverse=True)
        Zf, W1f, W2f = O.scan(Q[::-1], K[::-1], V[::-1], W1, W2, 0.02, b)
        np.testing.assert_array_equal(Zr, Zf[::-1])
        np.testing.assert_array_equal(W1r, W1f)


def test_segmented_scan_equals_one_shot():
    rng = np.random.default_rng(9)
    Q, K, V, W1, W2 = _rand_head(rng, 48, 4)
    Z, W1T, W2T = O.scan(Q, K, V, W1, W2, 0.02, 8)
    Za, W1a, W2a = O.scan(Q[:24], K[:24], V[:24], W1, W2, 0.02, 8)
    Zb, W1b, W2b = O.scan(Q[24:], K[24:], V[24:], W1a, W2a, 0.02, 8)
    np.testing.assert_array_equal(Z, np.concatenate([Za, Zb]))
    np.testing.assert_array_equal(W1T, W1b)


def test_prefix_and_chunk_end_readings_differ():
    """The two readings of which state produces z_t inside a chunk agree at b = 1
    and differ clearly at b = 16, so the choice (prefix) is fixed by a test."""
    rng = np.random.default_rng(11)
    Q, K, V, W1, W2 = _rand_head(rng, 64, 8)
    eta = 0.05 / 8
    Zp = O.scan(Q, K, V, W1, W2, eta, 1, zmode=0)[0]
    Ze = O.scan(Q, K, V, W1, W2, eta, 1, zmode=1)[0]
    np.testing.assert_array_equal(Zp, Ze)
    Zp = O.scan(Q, K, V, W1, W2, eta, 16, zmode=0)[0]
    Ze = O.scan(Q, K, V, W1, W2, eta, 16, zmode=1)[0]
    assert np.abs(Zp - Ze).max() > 1e-3 * np.abs(Zp).max()


# ------------------------------------------------------------------ gate and directions
def test_gate_identity_at_alpha_zero_and_init_value():
    tab = _table("gate_init.txt")
    assert np.tanh(tab[0, 0]) == pytest.approx(tab[0, 1], rel=1e-15)
    rng = np.random.default_rng(12)
    H, T, d = 2, 11, 4
    m = 4 * d
    X = rng.normal(size=(H, T, d))
    th = [rng.normal(size=(H, d, d)) / 2 for _ in range(3)]
    W1 = rng.normal(size=(H, m, d)) / 2; W2 = rng.normal(size=(H, d, m)) / 4
    zero = np.zeros(H * d)
    for dirs in ("fwd", "rev", "bidir"):
        out = O.layer_forward(X, *th, W1, W2, 0.01, 4, dirs, alpha_f=zero, alpha_r=zero, per_head=True)
        np.testing.assert_array_equal(out["Y"], X)
    a = np.full(H * d, tab[0, 0])
    out = O.layer_forward(X, *th, W1, W2, 0.01, 4, "fwd", alpha_f=a, per_head=True)
    np.testing.assert_allclose(out["Y"] - X, tab[0, 1] * out["Z_f"], rtol=1e-13, atol=1e-15)


def test_bidirectional_is_forward_then_reverse_on_gated_output():
    rng = np.random.default_rng(13)
    H, T, d = 2, 13, 4
    m = 4 * d
    X = rng.normal(size=(H, T, d))
    th = [rng.normal(size=(H, d, d)) / 2 for _ in range(3)]
    W1 = rng.normal(size=(H, m, d)) / 2; W2 = rng.normal(size=(H, d, m)) / 4
    af = rng.normal(size=H * d) * 0.1; ar = rng.normal(size=H * d) * 0.1
    out = O.layer_forward(X, *th, W1, W2, 0.01, 3, "bidir", alpha_f=af, alpha_r=ar, per_head=True)
    f = O.layer_forward(X, *th, W1, W2, 0.01, 3, "fwd", alpha_f=af, per_head=True)
    r = O.layer_forward(f["Y"], *th, W1, W2, 0.01, 3, "rev", alpha_r=ar, per_head=True)
    np.testing.assert_array_equal(out["Y"], r["Y"])
    # the reverse direction is the forward one on the flipped sequence
    rf = O.layer_forward(f["Y"][:, ::-1], *th, W1, W2, 0.01, 3, "fwd", alpha_f=ar, per_head=True)
    np.testing.assert_allclose(out["Y"], rf["Y"][:, ::-1], rtol=1e-14, atol=1e-15)


def test_full_mode_with_block_diagonal_theta_equals_per_head_mode():
    """Full mode (X [T, D], theta [H*d, D]) with block-diagonal theta is the per-head
    mode: fixes the projection layout and the head/channel bookkeeping."""
    rng = np.random.default_rng(14)
    H, T, d = 3, 10, 4
    m, D = 4 * d, 3 * 4
    Xh = rng.normal(size=(H, T, d))
    th = [rng.normal(size=(H, d, d)) / 2 for _ in range(3)]
    W1 = rng.normal(size=(H, m, d)) / 2; W2 = rng.normal(size=(H, d, m)) / 4
    af = rng.normal(size=D) * 0.2; ar = rng.normal(size=D) * 0.2
    Xf = Xh.transpose(1, 0, 2).reshape(T, D)
    thf = []
    for t in th:
        big = np.zeros((H * d, D))
        for h in range(H):
            big[h * d:(h + 1) * d, h * d:(h + 1) * d] = t[h]
        thf.append(big)
    ph = O.layer_forward(Xh, *th, W1, W2, 0.02, 4, "bidir", alpha_f=af, alpha_r=ar, per_head=True)
    fm = O.layer_forward(Xf, *thf, W1, W2, 0.02, 4, "bidir", alpha_f=af, alpha_r=ar, per_head=False)
    np.testing.assert_allclose(fm["Y"], ph["Y"].transpose(1, 0, 2).reshape(T, D), rtol=1e-13, atol=1e-14)
    # sampled-head helper agrees with the whole layer's forward pre-gate output
    Zs, _, _ = O.full_mode_heads(Xf, *thf, W1, W2, 0.02, 4, heads=[2, 0])
    Zfull = fm["Z_f"]
    np.testing.assert_allclose(Zs[:, :d], Zfull[:, 2 * d:3 * d], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(Zs[:, d:], Zfull[:, 0:d], rtol=1e-14, atol=1e-15)


def test_literal_eta_diverges_and_eta_over_d_does_not():
    """With the squared-norm loss and the stated eta = 0.1 (d = 16) the state blows up
    within a few tokens even in fp64; eta / d (mean-squared loss) stays finite."""
    import test_rnn_layer_b200.synth as S
    w = S.TINY
    inp = S.make_inputs(w, seed=0)
    args = [inp[k].double().numpy() for k in ("X", "theta_q", "theta_k", "theta_v", "W1_0", "W2_0")]
    with np.errstate(all="ignore"):
        bad = O.layer_forward(*args, w.eta, 1, "fwd", alpha_f=inp["alpha_f"].numpy(), per_head=True)
    assert not np.isfinite(bad["Y"]).all()
    good = O.layer_forward(*args, w.eta_eff, 1, "fwd", alpha_f=inp["alpha_f"].numpy(), per_head=True)
    assert np.isfinite(good["Y"]).all() and np.isfinite(good["W1_f"]).all()


@pytest.mark.parametrize("b", [1, 8])
def test_scan_is_causal_token_by_token(b):
    """Forward: z_t depends on tokens 0..t only, also inside a chunk (the prefix
    reading); reverse: on tokens t..T-1 only.  Perturbing token t0 must leave the
    earlier (forward) or later (reverse) outputs exactly unchanged and change z_t0."""
    rng = np.random.default_rng(29 + b)
    T, d, m, t0 = 21, 3, 12, 11
    Q, K, V = rng.normal(size=(T, d)), rng.normal(size=(T, d)), rng.normal(size=(T, d))
    W1, W2 = rng.normal(size=(m, d)) / np.sqrt(d), rng.normal(size=(d, m)) / np.sqrt(m)
    Q2, K2, V2 = Q.copy(), K.copy(), V.copy()
    K2[t0] += 0.5
    V2[t0] -= 0.5
    for reverse in (False, True):
        Z, _, _ = O.scan(Q, K, V, W1, W2, 0.02, b, reverse=reverse)
        Zp, _, _ = O.scan(Q2, K2, V2, W1, W2, 0.02, b, reverse=reverse)
        same = slice(t0 + 1, T) if reverse else slice(0, t0)
        np.testing.assert_array_equal(Z[same], Zp[same])
        assert np.abs(Z[t0] - Zp[t0]).max() > 1e-6


def test_heads_equal_single_head_runs():
    """The multi-head driver (OpenMP over heads, [H, T, d] streams) equals H
    separate single-head scans with eta > 0: fixes its head strides for Q, K, V,
    W1, W2 and Z, for the per-token rule (b = 1) and the chunk form, both ways."""
    rng = np.random.default_rng(21)
    H, T, d = 3, 29, 4
    m = 4 * d
    Q, K, V = (rng.normal(size=(H, T, d)) for _ in range(3))
    W1 = rng.normal(size=(H, m, d)) / math.sqrt(d)
    W2 = rng.normal(size=(H, d, m)) / math.sqrt(m)
    for b in (1, 6):
        for reverse in (False, True):
            Z, W1T, W2T = O.scan_heads(Q, K, V, W1, W2, 0.05 / d, b, reverse)
            for h in range(H):
                z, w1, w2 = O.scan(Q[h], K[h], V[h], W1[h], W2[h], 0.05 / d, b, reverse=reverse, per_token=b == 1)
                assert np.array_equal(Z[h], z) and np.array_equal(W1T[h], w1) and np.array_equal(W2T[h], w2)
            assert np.abs(W1T - W1).max() > 1e-6   # the state moved
