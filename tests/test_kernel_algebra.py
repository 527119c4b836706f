"""The chunk algebra the tensor-core scan kernels implement, restated in numpy
fp64 exactly as the kernels arrange it, against the oracle (CPU only).

The parity tests compare the kernels with the oracle on the GPU; these tests
pin, on the CPU, the derivations the kernels are built on, so that a reader can
check them without a GPU:
  * the cluster MLP scan: hidden units split over two CTAs, transposed forms,
    z read as W2_old Gq plus the prefix-masked correction, and z completed
    from per-CTA partials (the masked correction is linear in N, so each CTA
    may mask its own partial N);
  * the TTT-Linear tensor-core scan: E'^T = -2 eta (W K^T - V^T),
    Z^T = W Q^T + E'^T M^T, W += E'^T K.
"""
import numpy as np
import pytest
from scipy.special import erf

from oracle import ttt_oracle as O


def gelu(a):
    return 0.5 * a * (1.0 + erf(a / np.sqrt(2.0)))


def gelu_prime(a):
    return 0.5 * (1.0 + erf(a / np.sqrt(2.0))) + a * np.exp(-0.5 * a * a) / np.sqrt(2 * np.pi)


def _chunks(T, b, reverse):
    """Row ranges of the walk's chunks in natural row order (the kernels keep rows in natural order)."""
    out = []
    for c in range((T + b - 1) // b):
        bc = min(b, T - c * b)
        y0 = T - c * b - bc if reverse else c * b
        out.append((y0, bc))
    return out


def _prefix_mask(n, reverse):
    """keep[t, s]: s is not after t in the walk (rows in natural order)."""
    t = np.arange(n)[:, None]
    s = np.arange(n)[None, :]
    return (s >= t) if reverse else (s <= t)


def cluster_mlp_scan(Q, K, V, W1, W2, eta, b, reverse):
    """The cluster kernel's per-chunk arrangement, CTA r owning hidden units [r m/2, (r+1) m/2)."""
    T, d = Q.shape
    m = W1.shape[0]
    halves = [slice(0, m // 2), slice(m // 2, m)]
    W1 = W1.copy(); W2 = W2.copy()
    Z = np.zeros((T, d))
    for y0, bc in _chunks(T, b, reverse):
        q, k, v = Q[y0:y0 + bc], K[y0:y0 + bc], V[y0:y0 + bc]
        keep = _prefix_mask(bc, reverse)
        # A^T = W1 K^T per CTA; G = GELU(A); Y^T = sum over CTAs of W2[:, mine] G[:, mine]^T (exchange)
        AT = [W1[h] @ k.T for h in halves]
        G = [gelu(a.T) for a in AT]
        Y = sum(G[r] @ W2[:, halves[r]].T for r in range(2))
        D2 = -2.0 * eta * (Y - v)                                       # D2' [t][j]
        Dl = [(D2 @ W2[:, halves[r]]) * gelu_prime(AT[r].T) for r in range(2)]   # P * G'
        M = np.where(keep, q @ k.T, 0.0)                                # M[t, s]
        Aq = [(W1[halves[r]] @ q.T).T + M @ Dl[r] for r in range(2)]    # W1_old Q^T + Dl^T M^T
        W2_old = W2.copy()
        for r, h in enumerate(halves):                                  # the chunk's state update
            W1[h] += Dl[r].T @ k
            W2[:, h] += D2.T @ G[r]
        Gq = [gelu(a) for a in Aq]
        # per CTA: Z1_r = W2_old[:, mine] Gq_r, N_r = G_r Gq_r^T, Np_r[t, s] = N_r[s, t] (s not after t)
        z = np.zeros((bc, d))
        for r, h in enumerate(halves):
            Z1 = Gq[r] @ W2_old[:, h].T
            N = G[r] @ Gq[r].T
            Np = np.where(keep, N.T, 0.0)
            z += Z1 + Np @ D2                                           # the CTA's partial z
        Z[y0:y0 + bc] = z
    return Z, W1, W2


def linear_tc_scan(Q, K, V, W, eta, b, reverse):
    """The TTT-Linear tensor-core kernel's per-chunk arrangement."""
    T, d = Q.shape
    W = W.copy()
    Z = np.zeros((T, d))
    for y0, bc in _chunks(T, b, reverse):
        q, k, v = Q[y0:y0 + bc], K[y0:y0 + bc], V[y0:y0 + bc]
        ET = -2.0 * eta * (W @ k.T - v.T)                               # E'^T [i][t]
        M = np.where(_prefix_mask(bc, reverse), q @ k.T, 0.0)
        Z[y0:y0 + bc] = (W @ q.T + ET @ M.T).T
        W = W + ET @ k
    return Z, W


def _inputs(T, d, m, seed):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.normal(size=(T, d)) for _ in range(3))
    W1 = rng.normal(size=(m, d)) / np.sqrt(d)
    W2 = rng.normal(size=(d, m)) / np.sqrt(m)
    return Q, K, V, W1, W2


@pytest.mark.parametrize("b,T", [(1, 7), (4, 13), (8, 32), (6, 37)])
@pytest.mark.parametrize("reverse", [False, True])
def test_cluster_mlp_chunk_algebra_matches_the_oracle(b, T, reverse):
    d, m = 4, 16
    Q, K, V, W1, W2 = _inputs(T, d, m, b * 100 + T)
    eta = 0.05 / d
    Zk, W1k, W2k = cluster_mlp_scan(Q, K, V, W1, W2, eta, b, reverse)
    Zo, W1o, W2o = O.scan(Q, K, V, W1, W2, eta, b, reverse=reverse)
    np.testing.assert_allclose(Zk, Zo, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(W1k, W1o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(W2k, W2o, rtol=1e-11, atol=1e-12)


def test_masking_the_sum_of_partials_equals_summing_masked_partials():
    """The reason each CTA may finish its own z partial: the prefix mask and the
    correction product are linear in N."""
    rng = np.random.default_rng(1)
    n, d = 9, 5
    N0, N1 = rng.normal(size=(n, n)), rng.normal(size=(n, n))
    D2 = rng.normal(size=(n, d))
    keep = _prefix_mask(n, False)
    lhs = np.where(keep, (N0 + N1).T, 0.0) @ D2
    rhs = np.where(keep, N0.T, 0.0) @ D2 + np.where(keep, N1.T, 0.0) @ D2
    np.testing.assert_allclose(lhs, rhs, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("b,T", [(2, 9), (16, 40), (64, 130)])
@pytest.mark.parametrize("reverse", [False, True])
def test_linear_tc_chunk_algebra_matches_the_oracle(b, T, reverse):
    rng = np.random.default_rng(b * 10 + T)
    d = 8
    Q, K, V = (rng.normal(size=(T, d)) for _ in range(3))
    W0 = rng.normal(size=(d, d)) / np.sqrt(d)
    eta = 0.05 / d
    Zk, Wk = linear_tc_scan(Q, K, V, W0, eta, b, reverse)
    Zo, Wo = O.linear_scan(Q, K, V, W0, eta, b, reverse=reverse)
    np.testing.assert_allclose(Zk, Zo, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Wk, Wo, rtol=1e-11, atol=1e-12)
