"""Parity at the workloads' full sequence lengths, in the launch configuration
bench.py times (automatic kernel choice, whole layer in one call).

  * per-head inputs: every head is independent in both directions (X' of a
    head depends only on that head), so sampled heads are checked completely,
    forward and reverse, over the full length, against the oracle run here;
  * the 3072-wide layer with both gates at 0.1: the reverse pass mixes every
    head through theta X', so the oracle's expected outputs come from a full
    48-head forward pass and the sampled heads' reverse pass written once by
    tests/golden/make_full_layer_golden.py (oracle only); this test compares
    Z_f, Z_r, Y and both final states of those heads on six 128-token windows
    spread from the first token to the last.  The forward pass of one head
    (which needs only that head's rows of theta) is also checked over the
    whole length against the oracle run here;
  * the 3072-wide TTT-Linear layer the same way, from the expected values
    tests/golden/make_full_linear_golden.py wrote.
Tolerance: max-normalised error 2e-2 (bf16 inputs, fp32 state).  Every error
is printed (pytest -s) with the prefix PARITY.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

from helpers import TOL_BF16, maxrel, to_np
from oracle import ttt_oracle as O
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
GOLDEN_FULL = os.path.join(GOLDEN_DIR, "full_layer_T313344_seed0.npz")


def _report(name, errs):
    print(f"PARITY {name} " + " ".join(f"{k}={v:.3e}" for k, v in errs.items()), flush=True)


def _gpu_layer(w, inp, dev, want_state=False):
    g = {k: v.to(dev) for k, v in inp.items()}
    return L.layer_forward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W1_0"], g["W2_0"], w.eta_eff, w.b,
                           w.dirs, alpha_f=g["alpha_f"], alpha_r=g["alpha_r"], per_head=w.per_head, want_z=True,
                           want_state=want_state)


@pytest.mark.parametrize("w,heads", [(S.MINIBATCH, [0, 5, 29, 42]), (S.SCALE18S, [11, 23, 36, 47])],
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
    _report(f"{w.name} heads={heads}", errs)
    assert all(v <= TOL_BF16 for v in errs.values()), errs


def _golden_digest():
    spec = importlib.util.spec_from_file_location("make_full_layer_golden",
                                                  os.path.join(GOLDEN_DIR, "make_full_layer_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.input_digest


def test_full_layer_full_length_both_directions_with_the_gates():
    g = np.load(GOLDEN_FULL)
    w = S.FULL63S
    inp = S.make_inputs(w, seed=0, device="cpu")   # the generator the expected values were written from
    assert _golden_digest()(inp) == str(g["digest"]), "inputs differ from those of the stored expected values"
    assert int(g["T"]) == w.T and int(g["b"]) == w.b and float(g["eta"]) == w.eta_eff
    dev = torch.device("cuda")
    out = _gpu_layer(w, inp, dev, want_state=True)
    heads = [int(h) for h in g["heads"]]
    win = int(g["window"])
    rows = torch.cat([torch.arange(int(s), int(s) + win) for s in g["starts"]]).to(dev)
    cols = torch.cat([torch.arange(h * w.d, (h + 1) * w.d) for h in heads]).to(dev)
    pick = lambda t: to_np(t.index_select(0, rows).index_select(1, cols))
    Zf, Zr, Y = pick(out["Z"][0]), pick(out["Z"][1]), pick(out["Y"])
    hidx = torch.tensor(heads, device=dev)
    st = {k: to_np(out[k][di].index_select(0, hidx)) for k, di in (("W1_T", 0), ("W2_T", 0))}
    st_r = {k: to_np(out[k][1].index_select(0, hidx)) for k in ("W1_T", "W2_T")}
    del out
    torch.cuda.empty_cache()
    # the oracle's Y on the sampled elements from its own z: Y = gate_r(gate_f(X, z_f), z_r)
    Xs = inp["X"].double()[rows.cpu()][:, cols.cpu()].numpy()
    af, ar = to_np(inp["alpha_f"][cols.cpu()]), to_np(inp["alpha_r"][cols.cpu()])
    Zf_o, Zr_o = g["Z_f"].astype(np.float64), g["Z_r"].astype(np.float64)
    Y_o = O.gate(O.gate(Xs, Zf_o, af), Zr_o, ar)
    errs = {"Z_f": maxrel(Zf, Zf_o), "Z_r": maxrel(Zr, Zr_o), "Y": maxrel(Y, Y_o),
            "W1_f": maxrel(st["W1_T"], g["W1_f"]), "W2_f": maxrel(st["W2_T"], g["W2_f"]),
            "W1_r": maxrel(st_r["W1_T"], g["W1_r"]), "W2_r": maxrel(st_r["W2_T"], g["W2_r"])}
    _report(f"{w.name} heads={heads} windows={list(map(int, g['starts']))}x{win}", errs)
    assert all(v <= TOL_BF16 for v in errs.values()), errs


def test_full_layer_full_length_forward_sampled_head():
    heads = [17]
    w = S.FULL63S
    dev = torch.device("cuda")
    inp = S.make_inputs(w, seed=0, device=dev)
    out = _gpu_layer(w, inp, dev)
    cols = torch.cat([torch.arange(h * w.d, (h + 1) * w.d) for h in heads]).to(dev)
    Zf = to_np(out["Z"][0].index_select(1, cols))
    del out
    torch.cuda.empty_cache()
    X = inp["X"].cpu().float().numpy()
    th = [inp[k].cpu().float().numpy() for k in ("theta_q", "theta_k", "theta_v")]
    W1, W2 = to_np(inp["W1_0"].cpu()), to_np(inp["W2_0"].cpu())
    ref, _, _ = O.full_mode_heads(X, *th, W1, W2, w.eta_eff, w.b, heads)
    err = maxrel(Zf, ref)
    _report(f"{w.name} forward head={heads} all tokens", {"Z_f": err})
    assert err <= TOL_BF16


GOLDEN_LINEAR = os.path.join(GOLDEN_DIR, "full_linear_T313344_seed0.npz")


def test_linear_full_layer_full_length_both_directions_with_the_gates():
    """The 3072-wide TTT-Linear layer at 313,344 tokens, both gates at 0.1, against
    the expected values tests/golden/make_full_linear_golden.py wrote from the
    oracle: Z_f, Z_r, Y and both final states of three heads on six windows."""
    g = np.load(GOLDEN_LINEAR)
    w = S.FULL63S
    inp = S.make_linear_inputs(w, seed=0, device="cpu")
    spec = importlib.util.spec_from_file_location("make_full_linear_golden",
                                                  os.path.join(GOLDEN_DIR, "make_full_linear_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert mod.input_digest(inp) == str(g["digest"]), "inputs differ from those of the stored expected values"
    assert int(g["T"]) == w.T and int(g["b"]) == w.b and float(g["eta"]) == w.eta_eff
    dev = torch.device("cuda")
    d_in = {k: v.to(dev) for k, v in inp.items()}
    out = L.linear_layer_forward(d_in["X"], d_in["theta_q"], d_in["theta_k"], d_in["theta_v"], d_in["W_0"],
                                 w.eta_eff, w.b, w.dirs, alpha_f=d_in["alpha_f"], alpha_r=d_in["alpha_r"],
                                 per_head=False, want_z=True, want_state=True)
    heads = [int(h) for h in g["heads"]]
    win = int(g["window"])
    rows = torch.cat([torch.arange(int(s), int(s) + win) for s in g["starts"]]).to(dev)
    cols = torch.cat([torch.arange(h * w.d, (h + 1) * w.d) for h in heads]).to(dev)
    pick = lambda t: to_np(t.index_select(0, rows).index_select(1, cols))
    Zf, Zr, Y = pick(out["Z"][0]), pick(out["Z"][1]), pick(out["Y"])
    hidx = torch.tensor(heads, device=dev)
    Wf, Wr = to_np(out["W_T"][0].index_select(0, hidx)), to_np(out["W_T"][1].index_select(0, hidx))
    del out, d_in
    torch.cuda.empty_cache()
    Xs = inp["X"].double()[rows.cpu()][:, cols.cpu()].numpy()
    af, ar = to_np(inp["alpha_f"][cols.cpu()]), to_np(inp["alpha_r"][cols.cpu()])
    Zf_o, Zr_o = g["Z_f"].astype(np.float64), g["Z_r"].astype(np.float64)
    Y_o = O.gate(O.gate(Xs, Zf_o, af), Zr_o, ar)
    errs = {"Z_f": maxrel(Zf, Zf_o), "Z_r": maxrel(Zr, Zr_o), "Y": maxrel(Y, Y_o),
            "W_f": maxrel(Wf, g["W_f"]), "W_r": maxrel(Wr, g["W_r"])}
    _report(f"linear {w.name} heads={heads} windows={list(map(int, g['starts']))}x{win}", errs)
    assert all(v <= TOL_BF16 for v in errs.values()), errs
