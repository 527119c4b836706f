"""Pins of the backward-pass oracle (oracle/ttt_backward.py) against things
other than itself:
  * its torch forward restatement equals the C oracle's forward (per-head and
    full-width layers, per-token and chunked, every direction);
  * its gradients equal central finite differences of the C oracle's forward
    for every input (X, theta_Q/K/V, W1_0, W2_0, alpha_f, alpha_r);
  * eta = 0: the keys and values never reach the output, so dtheta_K and
    dtheta_V are exactly zero;
  * alpha_f = alpha_r = 0: Y = X, so dX = dY, every weight gradient is zero and
    dalpha is the closed form sum_t dY * z (tanh'(0) = 1), z from the C oracle.
"""
import numpy as np
import pytest

from oracle import ttt_backward as B
from oracle import ttt_oracle as O


def _inputs(rng, H=2, T=11, d=4, per_head=True):
    m, D = 4 * d, H * d   # the heads' outputs concatenate back to the model width
    if per_head:
        X = rng.normal(size=(H, T, d))
        th = [rng.normal(size=(H, d, d)) / np.sqrt(d) for _ in range(3)]
    else:
        X = rng.normal(size=(T, D))
        th = [rng.normal(size=(H * d, D)) / np.sqrt(D) for _ in range(3)]
    return {"X": X, "theta_q": th[0], "theta_k": th[1], "theta_v": th[2],
            "W1_0": rng.normal(size=(H, m, d)) / np.sqrt(d), "W2_0": rng.normal(size=(H, d, m)) / np.sqrt(m),
            "alpha_f": rng.normal(size=H * d) * 0.3, "alpha_r": rng.normal(size=H * d) * 0.3}


def _c_forward(inp, eta, b, dirs, per_head):
    return O.layer_forward(inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"], eta, b,
                           dirs, alpha_f=inp["alpha_f"], alpha_r=inp["alpha_r"], per_head=per_head)


@pytest.mark.parametrize("per_head", [True, False])
@pytest.mark.parametrize("b", [1, 3])
@pytest.mark.parametrize("dirs", ["fwd", "rev", "bidir"])
def test_torch_forward_equals_c_oracle(per_head, b, dirs):
    import torch
    rng = np.random.default_rng(40 + b)
    inp = _inputs(rng, per_head=per_head)
    t = {k: torch.tensor(v) for k, v in inp.items()}
    out = B.layer_forward(t["X"], t["theta_q"], t["theta_k"], t["theta_v"], t["W1_0"], t["W2_0"], t["alpha_f"],
                          t["alpha_r"], 0.05, b, dirs, per_head)
    ref = _c_forward(inp, 0.05, b, dirs, per_head)
    scale = np.abs(ref["Y"]).max()
    assert np.abs(out["Y"].numpy() - ref["Y"]).max() <= 1e-12 * scale
    for k in ("Z_f", "Z_r"):
        if k in ref:
            assert np.abs(out[k].numpy() - ref[k]).max() <= 1e-12 * np.abs(ref[k]).max()


@pytest.mark.parametrize("per_head,b,dirs", [(True, 1, "fwd"), (True, 3, "bidir"), (True, 2, "rev"),
                                             (False, 2, "bidir")])
def test_gradients_match_central_differences_of_the_c_oracle(per_head, b, dirs):
    rng = np.random.default_rng(70 + b)
    inp = _inputs(rng, H=2, T=7, d=2, per_head=per_head)
    dY = rng.normal(size=inp["X"].shape)
    eta = 0.1
    g = B.layer_backward(inp, dY, eta, b, dirs, per_head)
    loss = lambda q: float((dY * _c_forward(q, eta, b, dirs, per_head)["Y"]).sum())
    h = 1e-6
    for name in B.NAMES:
        fd = np.zeros_like(inp[name])
        for idx in np.ndindex(*inp[name].shape):
            qp = {k: v.copy() for k, v in inp.items()}
            qm = {k: v.copy() for k, v in inp.items()}
            qp[name][idx] += h
            qm[name][idx] -= h
            fd[idx] = (loss(qp) - loss(qm)) / (2 * h)
        scale = max(np.abs(fd).max(), 1e-12)
        if (name == "alpha_f" and dirs == "rev") or (name == "alpha_r" and dirs == "fwd"):
            assert np.abs(g["d" + name]).max() == 0.0 and np.abs(fd).max() == 0.0
            continue
        assert np.abs(g["d" + name] - fd).max() <= 2e-7 * scale, name


def test_eta_zero_keys_and_values_do_not_reach_the_output():
    rng = np.random.default_rng(5)
    inp = _inputs(rng, H=2, T=9, d=4)
    dY = rng.normal(size=inp["X"].shape)
    g = B.layer_backward(inp, dY, 0.0, 4, "bidir", True)
    assert np.abs(g["dtheta_k"]).max() == 0.0 and np.abs(g["dtheta_v"]).max() == 0.0
    assert np.abs(g["dtheta_q"]).max() > 1e-3 and np.abs(g["dW1_0"]).max() > 1e-3


def test_zero_gates_closed_form():
    rng = np.random.default_rng(6)
    inp = _inputs(rng, H=2, T=10, d=4)
    inp["alpha_f"] = np.zeros(8)
    inp["alpha_r"] = np.zeros(8)
    dY = rng.normal(size=inp["X"].shape)
    g = B.layer_backward(inp, dY, 0.05, 3, "bidir", True)
    assert np.array_equal(g["dX"], dY)
    for k in ("theta_q", "theta_k", "theta_v", "W1_0", "W2_0"):
        assert np.abs(g["d" + k]).max() == 0.0, k
    ref = _c_forward(inp, 0.05, 3, "bidir", True)     # z_r here runs on X' = X
    da_f = (dY * ref["Z_f"]).sum(axis=1).reshape(-1)   # per-head layout [H, T, d] -> channel h*d + e
    da_r = (dY * ref["Z_r"]).sum(axis=1).reshape(-1)
    np.testing.assert_allclose(g["dalpha_f"], da_f, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g["dalpha_r"], da_r, rtol=1e-12, atol=1e-13)
