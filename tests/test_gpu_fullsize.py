"""Parity at the workloads' full sequence lengths, in the launch configuration
bench.py times (automatic kernel choice, whole layer in one call).

The oracle cannot redo whole 48-head layers at these lengths in test time, so
each test checks outputs it can compute one by one:
  * per-head inputs: every head is independent in both directions (X' of a
    head depends only on that head), so sampled heads are checked completely,
    forward and reverse, over the full length;
  * the 3072-wide layer: the forward pass of a head needs only that head's
    rows of theta, so sampled heads' forward outputs are checked over the full
    length; the reverse pass mixes all heads through theta X', except when the
    forward gate is zero (X' = X exactly), which a second run uses to check
    sampled heads' reverse outputs.
Tolerance: max-normalised error 2e-2 (bf16 inputs, fp32 state).
"""
import numpy as np
import pytest
import torch

from helpers import TOL_BF16, maxrel, to_np
from oracle import ttt_oracle as O
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu


def _gpu_layer(w, inp, dev):
    g = {k: v.to(dev) for k, v in inp.items()}
    out = L.layer_forward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W1_0"], g["W2_0"], w.eta_eff, w.b,
                          w.dirs, alpha_f=g["alpha_f"], alpha_r=g["alpha_r"], per_head=w.per_head, want_z=True)
    return out


@pytest.mark.parametrize("w,heads", [(S.MINIBATCH, [5, 42]), (S.SCALE18S, [11])],
                         ids=["b16-T32768", "b64-T102400"])
def test_per_head_workloads_full_length_sampled_heads(w, heads):
    dev = torch.device("cuda")
    inp = S.make_inputs(w, seed=0, device=dev)
    out = _gpu_layer(w, inp, dev)
    idx = torch.tensor(heads, device=dev)
    sub = {k: v.index_select(0, idx).cpu() for k, v in inp.items() if k in ("X", "theta_q", "theta_k", "theta_v",
                                                                         "W1_0", "W2_0")}
    cols = torch.cat([torch.arange(h * w.d, (h + 1) * w.d) for h in heads])
    af, ar = inp["alpha_f"].cpu()[cols], inp["alpha_r"].cpu()[cols]
    ref = O.layer_forward(*[to_np(sub[k]) for k in ("X", "theta_q", "theta_k", "theta_v", "W1_0", "W2_0")],
                          w.eta_eff, w.b, "bidir", alpha_f=to_np(af), alpha_r=to_np(ar), per_head=True)
    Zf = to_np(out["Z"][0].index_select(0, idx))
    Zr = to_np(out["Z"][1].index_select(0, idx))
    Y = to_np(out["Y"].index_select(0, idx))
    errs = {"Z_f": maxrel(Zf, ref["Z_f"]), "Z_r": maxrel(Zr, ref["Z_r"]), "Y": maxrel(Y, ref["Y"])}
    assert all(v <= TOL_BF16 for v in errs.values()), errs


def _full_layer_sampled(alpha_f_value, heads):
    w = S.FULL63S
    dev = torch.device("cuda")
    inp = S.make_inputs(w, seed=0, device=dev)
    inp["alpha_f"].fill_(alpha_f_value)
    out = _gpu_layer(w, inp, dev)
    d = w.d
    cols = torch.cat([torch.arange(h * d, (h + 1) * d) for h in heads]).to(dev)
    Zf = to_np(out["Z"][0].index_select(1, cols))
    Zr = to_np(out["Z"][1].index_select(1, cols))
    del out
    torch.cuda.empty_cache()
    X = inp["X"].cpu().float().numpy()
    th = [inp[k].cpu().float().numpy() for k in ("theta_q", "theta_k", "theta_v")]
    W1, W2 = to_np(inp["W1_0"].cpu()), to_np(inp["W2_0"].cpu())
    return w, X, th, W1, W2, Zf, Zr


def test_full_layer_full_length_forward_sampled_head():
    heads = [17]
    w, X, th, W1, W2, Zf, _ = _full_layer_sampled(S.FULL63S.alpha, heads)
    ref, _, _ = O.full_mode_heads(X, *th, W1, W2, w.eta_eff, w.b, heads)
    assert maxrel(Zf, ref) <= TOL_BF16


def test_full_layer_full_length_reverse_sampled_head_with_zero_forward_gate():
    heads = [30]
    w, X, th, W1, W2, Zf, Zr = _full_layer_sampled(0.0, heads)
    ref_r, _, _ = O.full_mode_heads(X, *th, W1, W2, w.eta_eff, w.b, heads, reverse=True)
    assert maxrel(Zr, ref_r) <= TOL_BF16
