"""Pins of the fp64 segment-local attention oracle against things other than
itself: torch's own scaled-dot-product attention with a block-diagonal mask
(a library routine, fp64 on the CPU), closed forms (zero queries give the
segment mean of V; one dominant key gives a two-value softmax whose weights
are known exactly; length-1 segments give V), and invariants (tokens of other
segments change nothing; permuting a segment's keys with their values changes
nothing).  Planted mistakes -- a d instead of sqrt(d) scale, a causal mask,
segments one token off, the softmax taken over the queries, K and V swapped --
each fail at least one pin (last test).

Source: One-Minute Video Generation with Test-Time Training, paper notes page,
"方法详解 / 整体框架" (self-attention only inside each 3-second segment).
"""
import numpy as np
import pytest
import torch

from oracle import seg_attention as A


def _qkv(T, H, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return [rng.normal(size=(T, H * d)) * scale for _ in range(3)]


def _library(Q, K, V, H, L):
    """torch's scaled_dot_product_attention, fp64, mask = same segment."""
    T, D = Q.shape
    d = D // H
    seg = torch.arange(T) // L
    mask = seg[:, None] == seg[None, :]
    to = lambda M: torch.tensor(M, dtype=torch.float64).view(T, H, d).permute(1, 0, 2)
    out = torch.nn.functional.scaled_dot_product_attention(to(Q), to(K), to(V), attn_mask=mask)
    return out.permute(1, 0, 2).reshape(T, D).numpy()


# Each pin takes an attention function att(Q, K, V, H, L) -> [T, H d] and
# raises AssertionError when it does not hold.
def pin_library(att):
    for (T, H, d, L, seed) in [(37, 3, 8, 10, 1), (64, 2, 16, 64, 2), (50, 1, 4, 7, 3)]:
        Q, K, V = _qkv(T, H, d, seed)
        np.testing.assert_allclose(att(Q, K, V, H, L), _library(Q, K, V, H, L), rtol=1e-11, atol=1e-12)


def pin_zero_queries(att):
    T, H, d, L = 29, 2, 4, 8
    _, K, V = _qkv(T, H, d, 4)
    out = att(np.zeros((T, H * d)), K, V, H, L)
    for s0 in range(0, T, L):
        s1 = min(s0 + L, T)
        np.testing.assert_allclose(out[s0:s1], np.broadcast_to(V[s0:s1].mean(axis=0), (s1 - s0, H * d)),
                                   rtol=1e-12, atol=1e-13)


def pin_dominant_key(att):
    """One segment of n keys: k_u = e_u (unit vectors, d >= n), q_t = c e_{u*(t)}.
    Scores are c / sqrt(d) for u*(t) and 0 for the rest, so
    A[t] = (e^a v_{u*} + sum_{u != u*} v_u) / (e^a + n - 1),  a = c / sqrt(d)."""
    n, d, c = 6, 8, 3.0
    rng = np.random.default_rng(5)
    K = np.zeros((n, d))
    K[np.arange(n), np.arange(n)] = 1.0
    V = rng.normal(size=(n, d))
    star = rng.permutation(n)
    Q = c * K[star]
    a = c / np.sqrt(d)
    want = np.empty((n, d))
    for t in range(n):
        want[t] = (np.exp(a) * V[star[t]] + V.sum(axis=0) - V[star[t]]) / (np.exp(a) + n - 1)
    np.testing.assert_allclose(att(Q, K, V, 1, n), want, rtol=1e-13, atol=1e-14)


def pin_unit_segments(att):
    Q, K, V = _qkv(11, 2, 4, 6)
    np.testing.assert_allclose(att(Q, K, V, 2, 1), V, rtol=1e-14, atol=1e-15)


def pin_locality(att):
    T, H, d, L = 40, 2, 4, 9
    Q, K, V = _qkv(T, H, d, 7)
    base = att(Q, K, V, H, L)
    for s0 in range(0, T, L):
        s1 = min(s0 + L, T)
        Q2, K2, V2 = _qkv(T, H, d, 100 + s0)
        for M, M2 in ((Q2, Q), (K2, K), (V2, V)):
            M[s0:s1] = M2[s0:s1]
        np.testing.assert_allclose(att(Q2, K2, V2, H, L)[s0:s1], base[s0:s1], rtol=1e-13, atol=1e-14)


def pin_key_permutation(att):
    T, H, d, L = 30, 2, 4, 10
    Q, K, V = _qkv(T, H, d, 8)
    base = att(Q, K, V, H, L)
    perm = np.concatenate([s0 + np.random.default_rng(s0).permutation(min(L, T - s0)) for s0 in range(0, T, L)])
    np.testing.assert_allclose(att(Q, K[perm], V[perm], H, L), base, rtol=1e-12, atol=1e-13)


PINS = [pin_library, pin_zero_queries, pin_dominant_key, pin_unit_segments, pin_locality, pin_key_permutation]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_holds_pin(pin):
    pin(A.seg_attention)


def test_segments_cover_the_sequence_once():
    for T, L in [(1, 1), (10, 3), (313344, 14922), (64, 64), (65, 64)]:
        seg = A.segments(T, L)
        assert seg[0][0] == 0 and seg[-1][1] == T
        assert all(a1 == b0 for (_, a1), (b0, _) in zip(seg, seg[1:]))
        assert all(0 < s1 - s0 <= L for s0, s1 in seg)


def test_rows_subset_equals_whole():
    T, H, d, L = 45, 3, 4, 16
    Q, K, V = _qkv(T, H, d, 9)
    rows = np.array([0, 5, 15, 16, 31, 44])
    # the same arithmetic on fewer rows (a matrix product may block rows differently: last-bit differences)
    np.testing.assert_allclose(A.seg_attention(Q, K, V, H, L, rows), A.seg_attention(Q, K, V, H, L)[rows],
                               rtol=1e-14, atol=1e-15)


def test_block_input_is_residual_plus_attention():
    T, H, d, L = 20, 2, 4, 7
    Q, K, V = _qkv(T, H, d, 10)
    X = np.random.default_rng(11).normal(size=(T, H * d))
    np.testing.assert_array_equal(A.block_input(X, Q, K, V, H, L), X + A.seg_attention(Q, K, V, H, L))
    rows = np.array([3, 19])
    np.testing.assert_allclose(A.block_input(X, Q, K, V, H, L, rows), (X + A.seg_attention(Q, K, V, H, L))[rows],
                               rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------- planted mistakes
def _causal(Q, K, V, H, L):
    T, D = Q.shape
    d = D // H
    out = np.empty((T, D))
    for s0, s1 in A.segments(T, L):
        for t in range(s0, s1):
            for h in range(H):
                c = slice(h * d, (h + 1) * d)
                out[t, c] = A.attention_segment(Q[t:t + 1, c], K[s0:t + 1, c], V[s0:t + 1, c])[0]
    return out


def _softmax_over_queries(Q, K, V, H, L):
    T, D = Q.shape
    d = D // H
    out = np.empty((T, D))
    for s0, s1 in A.segments(T, L):
        for h in range(H):
            c = slice(h * d, (h + 1) * d)
            s = Q[s0:s1, c] @ K[s0:s1, c].T / np.sqrt(d)
            p = np.exp(s - s.max(axis=0, keepdims=True))
            out[s0:s1, c] = (p / p.sum(axis=0, keepdims=True)) @ V[s0:s1, c]
    return out


MUTANTS = {
    "scale 1/d": lambda Q, K, V, H, L: A.seg_attention(Q / np.sqrt(Q.shape[1] // H), K, V, H, L),
    "causal": _causal,
    "segments one longer": lambda Q, K, V, H, L: A.seg_attention(Q, K, V, H, L + 1),
    "softmax over queries": _softmax_over_queries,
    "K and V swapped": lambda Q, K, V, H, L: A.seg_attention(Q, V, K, H, L),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    failed = []
    for pin in PINS:
        try:
            pin(MUTANTS[name])
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake '{name}'"
