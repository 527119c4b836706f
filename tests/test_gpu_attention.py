"""Parity of the tensor-core segment-local attention and of the block
(attention, then the bidirectional layer, in one schedule) against the fp64
oracles, on seeded inputs.

Tolerance of the attention, on max|g - o| / max|o| of the attention part:
1e-2.  The result is rounded to bf16 (relative 2^-9 = 2.0e-3 per element) and
the softmax weights enter P V as bf16 (each weight relative 2^-9; with weights
that sum to one the error of an output is at most 2^-9 max|v| and in practice
far less, as the rounding errors of thousands of weights do not line up); Q K^T
of bf16 inputs accumulates in fp32 exactly enough (2^-24 relative).  The mean
error is held to 3e-3 of the mean magnitude as well.
"""
import numpy as np
import pytest
import torch

from oracle import seg_attention as A
from oracle import ttt_oracle as O
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

from helpers import maxrel, to_np, TOL_BF16

pytestmark = pytest.mark.gpu

TOL_ATTN = 1e-2
TOL_ATTN_MEAN = 3e-3


def _run(T, H, Lseg, Q, K, V, ld_qkv, Xres=None, rows=None, ld_out=None, out=None):
    D = H * 64
    ld_out = ld_out or D
    if out is None:
        out = torch.full((T, ld_out), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.ttt_seg_attention_workspace_size(), dtype=torch.uint8, device="cuda")
    r0, r1 = rows or (0, T)
    L.check(L.ttt_seg_attention(T, H, 64, Lseg, Q, K, V, ld_qkv, Xres, out, ld_out, r0, r1, ws, ws.numel()),
            "ttt_seg_attention")
    assert L.ttt_mlp_status(ws, None) == L.TTT_OK
    return out


def _compare(g, ref_att, base=None):
    """g: the GPU rows (fp64), ref_att: the oracle's attention rows, base: the residual rows (or None).

    Without a residual the attention itself is held to TOL_ATTN (max-normalised)
    and TOL_ATTN_MEAN (mean).  With one, g = bf16(base + A): the bf16 rounding of
    the sum (at most one bf16 step, 2^-8 relative, of |base + A|) hides A's own
    last bits, so each element is held to that step plus TOL_ATTN max|A|."""
    if base is None:
        e = maxrel(g, ref_att)
        mean = float(np.abs(g - ref_att).mean() / np.abs(ref_att).mean())
        print(f"attention: max-normalised error {e:.2e}, mean relative {mean:.2e}")
        assert e < TOL_ATTN and mean < TOL_ATTN_MEAN
        return e
    want = base + ref_att
    excess = np.abs(g - want) - 2.0 ** -8 * np.abs(want)
    e = float(max(excess.max(), 0.0) / np.abs(ref_att).max())
    print(f"attention + residual: error beyond one bf16 step of the sum {e:.2e} of max|A|")
    assert e < TOL_ATTN
    return e


CASES = [   # T, H, segment length, residual, rows
    (1000, 3, 300, False, None),          # three whole segments and a short one; ragged key and query tiles
    (1000, 3, 300, True, (137, 811)),     # a row range cutting segments, with the residual
    (777, 2, 777, True, None),            # one segment
    (515, 1, 128, False, None),           # segments of exactly one key tile
    (260, 2, 64, False, (5, 250)),        # segments shorter than a tile
    (2048, 4, 2048, False, (1000, 1300)), # sixteen key tiles, a middle slice of the queries
]


@pytest.mark.parametrize("T,H,Lseg,res,rows", CASES)
def test_attention_matches_oracle(T, H, Lseg, res, rows):
    w = S.FULL63S.with_(T=T, H=H, D=H * 64)
    a = S.make_attention_inputs(w, seed=T + H, device="cuda")
    Xres = S.make_inputs(w, seed=T, device="cuda")["X"] if res else None
    out = _run(T, H, Lseg, a["Q_a"], a["K_a"], a["V_a"], H * 64, Xres, rows)
    r0, r1 = rows or (0, T)
    idx = np.arange(r0, r1)
    ref = A.seg_attention(to_np(a["Q_a"]), to_np(a["K_a"]), to_np(a["V_a"]), H, Lseg, idx)
    _compare(to_np(out)[r0:r1], ref, to_np(Xres)[r0:r1] if res else None)
    # rows outside the range are untouched
    o = out.float().cpu()
    assert torch.all(o[:r0] == 7.0) and torch.all(o[r1:] == 7.0)


def test_unit_segments_return_v_exactly():
    T, H = 300, 2
    a = S.make_attention_inputs(S.FULL63S.with_(T=T, H=H, D=H * 64), seed=3, device="cuda")
    out = _run(T, H, 1, a["Q_a"], a["K_a"], a["V_a"], H * 64)
    assert torch.equal(out, a["V_a"])


@pytest.mark.parametrize("qk_std", [2.0, 3.0])
def test_peaked_attention(qk_std):
    """Scores of standard deviation qk_std^2: tile maxima that pass the running
    maximum by more than 2^8 occur, so the rescaling of O and the row sum runs."""
    T, H, Lseg = 3000, 2, 1400
    w = S.FULL63S.with_(T=T, H=H, D=H * 64)
    a = S.make_attention_inputs(w, seed=11, device="cuda", qk_std=qk_std)
    out = _run(T, H, Lseg, a["Q_a"], a["K_a"], a["V_a"], H * 64)
    ref = A.seg_attention(to_np(a["Q_a"]), to_np(a["K_a"]), to_np(a["V_a"]), H, Lseg)
    _compare(to_np(out), ref)


def test_rising_scores_rescale_every_tile():
    """q_t . k_u grows with u: every key tile raises the row maximum by more
    than 8 (log2 units), so O and the row sum are rescaled at every tile."""
    T, H, Lseg = 1024, 1, 1024
    u = torch.arange(T, dtype=torch.float32)
    Q = torch.zeros(T, 64)
    Q[:, 0] = 1.0
    K = torch.zeros(T, 64)
    K[:, 0] = u * (8.0 * 9.0 / 128.0 / 1.4426950408889634)   # +9 log2 units per 128 keys
    V = torch.randn(T, 64, generator=torch.Generator().manual_seed(5))
    Qd, Kd, Vd = (t.to(torch.bfloat16).cuda() for t in (Q, K, V))
    out = _run(T, H, Lseg, Qd, Kd, Vd, 64)
    ref = A.seg_attention(to_np(Qd), to_np(Kd), to_np(Vd), H, Lseg)
    _compare(to_np(out), ref)


def test_fused_qkv_layout_and_wide_output():
    """Q, K, V as column blocks of one [T, 3D] array; Out with a row stride
    wider than D (the extra columns stay untouched)."""
    T, H = 900, 3
    D = H * 64
    w = S.FULL63S.with_(T=T, H=H, D=D)
    a = S.make_attention_inputs(w, seed=21, device="cuda")
    qkv = torch.cat([a["Q_a"], a["K_a"], a["V_a"]], dim=1).contiguous()
    out = torch.full((T, D + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    base = qkv.data_ptr()
    _run(T, H, 400, base, base + D * 2, base + 2 * D * 2, 3 * D, None, None, D + 64, out)
    ref = A.seg_attention(to_np(a["Q_a"]), to_np(a["K_a"]), to_np(a["V_a"]), H, 400)
    _compare(to_np(out[:, :D]), ref)
    assert torch.all(out[:, D:].float() == 7.0)


def test_residual_in_place():
    T, H = 640, 2
    w = S.FULL63S.with_(T=T, H=H, D=H * 64)
    a = S.make_attention_inputs(w, seed=31, device="cuda")
    X = S.make_inputs(w, seed=31, device="cuda")["X"]
    X0 = to_np(X)
    _run(T, H, 200, a["Q_a"], a["K_a"], a["V_a"], H * 64, X, None, None, X)
    ref = A.seg_attention(to_np(a["Q_a"]), to_np(a["K_a"]), to_np(a["V_a"]), H, 200)
    _compare(to_np(X), ref, X0)


def test_nonfinite_input_is_reported():
    T, H = 500, 1
    a = S.make_attention_inputs(S.FULL63S.with_(T=T, H=H, D=64), seed=41, device="cuda")
    a["V_a"][123, 7] = float("nan")
    out = torch.empty(T, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.ttt_seg_attention_workspace_size(), dtype=torch.uint8, device="cuda")
    L.check(L.ttt_seg_attention(T, H, 64, 250, a["Q_a"], a["K_a"], a["V_a"], 64, None, out, 64, 0, T, ws,
                                ws.numel()), "ttt_seg_attention")
    assert L.ttt_mlp_status(ws, None) == L.TTT_ERR_NONFINITE


def test_full_size_sampled_rows():
    """T = 313,344 tokens, 48 heads, 21 segments of 14,922 (the last 14,904):
    the whole launch, 96 sampled rows (segment edges, the ragged last segment,
    random rows) checked for every head."""
    w = S.FULL63S
    T, H = w.T, w.H
    Lseg = S.segment_length(T)
    a = S.make_attention_inputs(w, seed=0, device="cuda")
    Xres = S.make_inputs(w, seed=0, device="cuda")["X"]
    out = _run(T, H, Lseg, a["Q_a"], a["K_a"], a["V_a"], w.D, Xres)
    rng = np.random.default_rng(0)
    last = (T - 1) // Lseg * Lseg
    picks = [0, 1, 127, 128, Lseg - 1, Lseg, 10 * Lseg + 5000, last, last + 129, T - 2, T - 1]
    rows = np.unique(np.concatenate([picks, rng.integers(0, T, 96 - len(picks))]))
    segs = sorted({int(r) // Lseg for r in rows})
    g = to_np(out[torch.as_tensor(rows, device="cuda")])
    base = to_np(Xres[torch.as_tensor(rows, device="cuda")])
    ref = np.empty_like(g)
    for s in segs:   # each sampled row against its own segment's keys and values
        s0, s1 = s * Lseg, min((s + 1) * Lseg, T)
        sel = np.nonzero((rows >= s0) & (rows < s1))[0]
        Qs = to_np(a["Q_a"][torch.as_tensor(rows[sel], device="cuda")])
        Ks, Vs = to_np(a["K_a"][s0:s1]), to_np(a["V_a"][s0:s1])
        for h in range(H):
            c = slice(h * 64, (h + 1) * 64)
            ref[sel, c] = A.attention_segment(Qs[:, c], Ks[:, c], Vs[:, c])
    _compare(g, ref, base)


# ---------------------------------------------------------------- the block
def _block_inputs(w, seed):
    inp = S.make_inputs(w, seed=seed, device="cuda")
    inp.update(S.make_attention_inputs(w, seed=seed, device="cuda"))
    return inp


def _block(w, inp, Lseg, front=None):
    desc = L.make_desc(w.T, w.H, w.d, False, True)
    ws = torch.empty(L.ttt_block_workspace_size(desc, w.b), dtype=torch.uint8, device="cuda")
    X = torch.empty_like(inp["X"])
    Y = torch.empty_like(inp["X"])
    if front is not None:
        L.check(L.ttt_debug_set_block_front(front), "ttt_debug_set_block_front")
    try:
        L.check(L.ttt_block_forward(desc, Lseg, inp["Q_a"], inp["K_a"], inp["V_a"], w.D, inp["X"], X,
                                    inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"],
                                    w.eta_eff, w.b, inp["alpha_f"], inp["alpha_r"], Y, ws, ws.numel()),
                "ttt_block_forward")
        assert L.ttt_mlp_status(ws, None) == L.TTT_OK
    finally:
        L.ttt_debug_set_block_front(-1)
    return X, Y


def _two_calls(w, inp, Lseg):
    X = _run(w.T, w.H, Lseg, inp["Q_a"], inp["K_a"], inp["V_a"], w.D, inp["X"])
    Y = L.layer_forward(X, inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"], w.eta_eff,
                        w.b, "bidir", alpha_f=inp["alpha_f"], alpha_r=inp["alpha_r"], per_head=False)["Y"]
    return X, Y


@pytest.mark.parametrize("front", [None, 0, 50, 100])
def test_block_equals_attention_then_layer(front):
    """Same kernels, same per-row arithmetic: the block's X and Y equal the two
    calls' bit for bit, whatever the head start."""
    w = S.FULL63S.with_T(8192)
    inp = _block_inputs(w, 3)
    Lseg = S.segment_length(w.T)
    Xb, Yb = _block(w, inp, Lseg, front)
    Xs, Ys = _two_calls(w, inp, Lseg)
    assert torch.equal(Xb, Xs)
    assert torch.equal(Yb, Ys)


@pytest.mark.parametrize("T", [1500, 3000])
def test_block_matches_oracle(T):
    """The block on 4 heads against the oracles: attention in fp64, the layer's
    input rounded to bf16 (the block's X is bf16), the layer in fp64."""
    w = S.FULL63S.with_(T=T, H=4, D=256)
    inp = _block_inputs(w, 7)
    Lseg = S.segment_length(T)
    Xg, Yg = _block(w, inp, Lseg)
    att = A.seg_attention(to_np(inp["Q_a"]), to_np(inp["K_a"]), to_np(inp["V_a"]), w.H, Lseg)
    base = to_np(inp["X"])
    _compare(to_np(Xg), att, base)
    X_ref = torch.tensor(base + att).to(torch.bfloat16).double().numpy()
    ref = O.layer_forward(X_ref, *(to_np(inp[k]) for k in ("theta_q", "theta_k", "theta_v", "W1_0", "W2_0")),
                          w.eta_eff, w.b, "bidir", alpha_f=to_np(inp["alpha_f"]), alpha_r=to_np(inp["alpha_r"]),
                          per_head=False)
    e = maxrel(to_np(Yg), ref["Y"])
    print(f"block Y: max-normalised error {e:.2e}")
    assert e < TOL_BF16
