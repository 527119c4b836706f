"""fp64 CPU oracle of the segment-local attention sublayer that feeds the TTT
layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA path.

Source (One-Minute Video Generation with Test-Time Training, paper notes
page, "方法详解 / 整体框架" and "亮点与洞察"): the pretrained diffusion
transformer keeps its self-attention, but only over the tokens of each
3-second segment; the gated TTT layer inserted after that attention layer
runs over the whole sequence.

Readings taken where the pages are silent:
  * segment s holds the tokens [s L, min((s + 1) L, T)) for a segment length
    L (63 s of video in 3-s segments: 21 segments, L = ceil(T / 21));
  * inside a segment the attention is full, not causal (a diffusion model
    denoises every frame of a clip at once), with the usual 1/sqrt(d) scale:
        A[t, h] = sum_{u in seg(t)} softmax_u(q_t . k_u / sqrt(d)) v_u
    for head h with q, k, v its d columns of Q, K, V ([T, H d], heads
    side by side, the TTT layer's channel layout);
  * the TTT layer's input is the sublayer's residual sum X = Xres + A; the
    backbone's Q/K/V and output projections and its norms need trained
    weights and are outside this path (Q, K, V are inputs).
"""
from __future__ import annotations

import numpy as np


def segments(T: int, L: int) -> list[tuple[int, int]]:
    """The token ranges [s L, min((s + 1) L, T)) of the segments."""
    if L <= 0:
        raise ValueError("segment length must be positive")
    return [(s0, min(s0 + L, T)) for s0 in range(0, T, L)]


def attention_segment(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v for one head on one segment, fp64.

    q: [n, d] queries, k, v: [n, d] keys and values of the same segment.  The
    row maximum is subtracted before the exponential (the quotient is the
    same; it only keeps exp from overflowing).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = (q @ k.T) / np.sqrt(q.shape[1])
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p / p.sum(axis=1, keepdims=True)) @ v


def seg_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, H: int, L: int, rows=None) -> np.ndarray:
    """Segment-local attention A [T, H d] (or the listed rows of it), fp64.

    Q, K, V: [T, H d] (head h in columns [h d, (h + 1) d)).  ``rows``: an
    optional sorted array of token indices; only those rows of A are formed
    (each still attends over its whole segment).
    """
    T, D = Q.shape
    d = D // H
    if d * H != D or K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K, V must be [T, H d] alike")
    want = np.arange(T) if rows is None else np.asarray(rows)
    out = np.empty((len(want), D))
    for s0, s1 in segments(T, L):
        sel = np.nonzero((want >= s0) & (want < s1))[0]
        if len(sel) == 0:
            continue
        for h in range(H):
            c = slice(h * d, (h + 1) * d)
            out[sel, c] = attention_segment(Q[want[sel], c], K[s0:s1, c], V[s0:s1, c])
    return out


def block_input(Xres: np.ndarray, Q: np.ndarray, K: np.ndarray, V: np.ndarray, H: int, L: int,
                rows=None) -> np.ndarray:
    """The TTT layer's input X = Xres + A (fp64), whole or the listed rows."""
    A = seg_attention(Q, K, V, H, L, rows)
    base = np.asarray(Xres, dtype=np.float64)
    return (base if rows is None else base[np.asarray(rows)]) + A
