"""TTT-Linear on the GPU (through the C ABI) against the fp64 oracle, element
by element: pre-gate z of each direction, the layer output Y and the final
state, at sizes the oracle finishes in seconds, with ragged chunks, tiles
spanning chunks (b > 64), T = 1, head dims 16/32/64 and both input layouts."""
import numpy as np
import pytest
import torch

from helpers import maxrel, to_np, tol
from oracle import ttt_oracle as O
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu

CASES = [
    S.TINY,                                                        # fp32, d = 16, b = 1, fwd
    S.CAUSAL.with_(T=1000),                                        # fp32, d = 64, b = 1, fwd
    S.MINIBATCH.with_(T=1003, H=4),                                # bf16, b = 16, bidir, ragged
    S.SCALE18S.with_(T=1000, H=4),                                 # bf16, b = 64, bidir, ragged
    S.FULL63S.with_(T=777, H=4, D=256),                            # bf16 full width, b = 64, bidir
    S.CAUSAL.with_(T=300, H=3, d=32, b=5, dirs="rev"),             # fp32, d = 32, reverse only
    S.CAUSAL.with_(T=350, H=2, b=100, dirs="bidir"),               # fp32, chunks spanning two tiles
    S.MINIBATCH.with_(T=1, H=2),                                   # a single token
    S.FULL63S.with_(T=3000, H=4, D=256),                           # full width, three chunk segments
    S.FULL63S.with_(T=3000, H=4, D=256, dirs="rev"),               # ... reverse only
]
IDS = ["tiny-d16-b1", "causal-d64-b1", "b16-bidir-bf16", "b64-bidir-bf16", "full-width-bf16", "d32-b5-rev",
       "b100-bidir", "T1", "full-width-segmented", "full-width-segmented-rev"]


def _oracle(w, inp):
    f = lambda k: inp[k].double().numpy()
    return O.linear_layer_forward(f("X"), f("theta_q"), f("theta_k"), f("theta_v"), f("W_0"), w.eta_eff, w.b,
                                  w.dirs, alpha_f=f("alpha_f"), alpha_r=f("alpha_r"), per_head=w.per_head)


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_linear_layer_matches_oracle(w):
    inp = S.make_linear_inputs(w, seed=0)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = L.linear_layer_forward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W_0"], w.eta_eff, w.b,
                                 w.dirs, alpha_f=g["alpha_f"], alpha_r=g["alpha_r"], per_head=w.per_head,
                                 want_z=True, want_state=True)
    o = _oracle(w, inp)
    errs = {"Y": maxrel(to_np(out["Y"]), o["Y"])}
    if w.dirs == "bidir":
        errs["Z_f"] = maxrel(to_np(out["Z"][0]), o["Z_f"])
        errs["Z_r"] = maxrel(to_np(out["Z"][1]), o["Z_r"])
        errs["W_f"] = maxrel(to_np(out["W_T"][0]), o["W_f"])
        errs["W_r"] = maxrel(to_np(out["W_T"][1]), o["W_r"])
    else:
        key = "f" if w.dirs == "fwd" else "r"
        errs["Z_" + key] = maxrel(to_np(out["Z"][0]), o["Z_" + key])
        errs["W_" + key] = maxrel(to_np(out["W_T"][0]), o["W_" + key])
    bad = {k: v for k, v in errs.items() if not v <= tol(w)}
    assert not bad, errs


def test_linear_eta_zero_gives_the_initial_map():
    """eta = 0 keeps W = W_0, so z = W_0 q exactly up to fp32 rounding."""
    w = S.CAUSAL.with_(T=200, H=2)
    inp = S.make_linear_inputs(w)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = L.linear_layer_forward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W_0"], 0.0, 16, "fwd",
                                 alpha_f=g["alpha_f"], per_head=True, want_z=True, want_state=True)
    Q = np.einsum("hed,htd->hte", inp["theta_q"].double().numpy(), inp["X"].double().numpy())
    ref = np.einsum("hij,htj->hti", inp["W_0"].double().numpy(), Q)
    assert maxrel(to_np(out["Z"][0]), ref) < 1e-5
    assert torch.equal(out["W_T"][0].cpu(), inp["W_0"])


def test_linear_nonfinite_state_is_reported():
    w = S.MINIBATCH.with_(T=100, H=2)
    inp = S.make_linear_inputs(w)
    inp["W_0"][1, 3, 5] = float("nan")
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = L.linear_layer_forward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W_0"], w.eta_eff, w.b,
                                 w.dirs, alpha_f=g["alpha_f"], alpha_r=g["alpha_r"], per_head=True,
                                 check_status=False)
    assert L.ttt_mlp_status(out["workspace"]) == L.TTT_ERR_NONFINITE


@pytest.mark.parametrize("w", [S.FULL63S.with_(T=3000, H=4, D=256), S.MINIBATCH.with_(T=500, H=3),
                               S.FULL63S.with_(T=3000, H=4, D=256, dirs="rev")],
                         ids=["full-bidir-segmented", "per-head-bidir", "full-rev"])
def test_linear_host_buffers_equal_device_call(w):
    """ttt_linear_forward_host (X in from pinned host memory, Y back to it; on the segmented path the copies
    go segment by segment) runs the same kernels on the same values as ttt_linear_forward: the same bits."""
    inp = S.make_linear_inputs(w, seed=2)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = L.linear_layer_forward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W_0"], w.eta_eff, w.b, w.dirs,
                                 alpha_f=g["alpha_f"], alpha_r=g["alpha_r"], per_head=w.per_head)
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    direction = L.DIRS[w.dirs]
    n = L.ttt_linear_host_io_workspace_size(desc, w.b, direction)
    assert n > L.ttt_linear_workspace_size(desc, w.b, direction)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    Xh = inp["X"].contiguous().pin_memory()
    Yh = torch.empty_like(Xh).pin_memory()
    L.check(L.ttt_linear_forward_host(desc, Xh, g["theta_q"], g["theta_k"], g["theta_v"], g["W_0"], w.eta_eff, w.b,
                                      direction, g["alpha_f"], g["alpha_r"], Yh, ws, n), "ttt_linear_forward_host")
    assert torch.equal(Yh, out["Y"].cpu())
