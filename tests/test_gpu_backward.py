"""Backward pass of the layer (ttt_mlp_backward through the C ABI) against the
fp64 backward oracle (oracle/ttt_backward.py: autograd of the primal chunk
form, pinned to the C oracle and to finite differences), gradient by gradient:
dX, dtheta_Q/K/V, dW1_0, dW2_0, dalpha_f, dalpha_r for a seeded upstream
gradient dY.  Tolerances: 1e-3 max-normalised for fp32 inputs (the scan
backward's products in the split, fp32-accurate tf32 form), 2e-2 for bf16
inputs (the forward pass recomputed inside and the scan backward's products
run on single tf32 / fp16 / bf16 tensor-core products there)."""
import numpy as np
import pytest
import torch

from helpers import maxrel, to_np
from oracle import ttt_backward as B
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu

CASES = [
    S.Workload("bwd-head-bf16-b16", H=2, d=64, T=150, b=16, dirs="bidir", dtype="bf16", per_head=True, eta=0.05),
    S.Workload("bwd-head-f32-b1", H=2, d=16, T=40, b=1, dirs="fwd", dtype="f32", per_head=True, eta=0.1),
    S.Workload("bwd-head-f32-b5-rev", H=3, d=32, T=77, b=5, dirs="rev", dtype="f32", per_head=True, eta=0.05),
    S.Workload("bwd-full-bf16-b64", H=2, d=64, T=200, b=64, dirs="bidir", dtype="bf16", per_head=False, eta=0.05,
               D=128),
    S.Workload("bwd-full-f32-b8", H=2, d=16, T=45, b=8, dirs="bidir", dtype="f32", per_head=False, eta=0.1, D=32),
    S.Workload("bwd-head-T1", H=2, d=64, T=1, b=16, dirs="bidir", dtype="bf16", per_head=True, eta=0.05),
    # long runs: 128 chunks of 16, and 65 chunks of 64 with a ragged last one (several segments when the
    # backward is built with sparser checkpoints)
    S.Workload("bwd-head-bf16-b16-128chunks", H=2, d=64, T=2048, b=16, dirs="bidir", dtype="bf16", per_head=True,
               eta=0.05),
    S.Workload("bwd-full-bf16-b64-65chunks", H=4, d=64, T=4131, b=64, dirs="bidir", dtype="bf16", per_head=False,
               eta=0.05, D=256),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_the_oracle(w):
    inp = S.make_inputs(w, seed=0)
    gen = torch.Generator().manual_seed(77)
    dY = torch.randn(inp["X"].shape, generator=gen, dtype=torch.float32)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = L.layer_backward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W1_0"], g["W2_0"], w.eta_eff, w.b,
                           w.dirs, g["alpha_f"], g["alpha_r"], dY.to(dev), per_head=w.per_head)
    torch.cuda.synchronize()
    ref = B.layer_backward({k: to_np(inp[k]) for k in B.NAMES}, dY.double().numpy(), w.eta_eff, w.b, w.dirs,
                           w.per_head)
    tol = 2e-2 if w.dtype == "bf16" else 1e-3
    errs = {k: maxrel(to_np(out["d" + k]), ref["d" + k]) for k in B.NAMES}
    print(f"PARITY backward {w.name} " + " ".join(f"d{k}={v:.3e}" for k, v in errs.items()), flush=True)
    assert all(v <= tol for v in errs.values()), errs


@pytest.mark.parametrize("w", [CASES[2], CASES[7]], ids=lambda w: w.name)
def test_backward_cluster_of_two_ctas_equals_one_cta(w):
    # a head's backward scan on one CTA or on a cluster of two: the same operations for every value
    inp = S.make_inputs(w, seed=3)
    gen = torch.Generator().manual_seed(5)
    dY = torch.randn(inp["X"].shape, generator=gen, dtype=torch.float32).cuda()
    g = {k: v.cuda() for k, v in inp.items()}
    outs = []
    try:
        for ctas in (1, 2):
            L.check(L.ttt_debug_set_backward_ctas(ctas), "ttt_debug_set_backward_ctas")
            outs.append(L.layer_backward(g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W1_0"], g["W2_0"],
                                         w.eta_eff, w.b, w.dirs, g["alpha_f"], g["alpha_r"], dY,
                                         per_head=w.per_head))
            torch.cuda.synchronize()
    finally:
        L.ttt_debug_set_backward_ctas(0)
    for k in ("dX", "dtheta_q", "dtheta_k", "dtheta_v", "dW1_0", "dW2_0"):
        assert torch.equal(outs[0][k], outs[1][k]), k
    # dalpha sums over tokens with atomic adds, in an order that varies from run to run
    for k in ("dalpha_f", "dalpha_r"):
        assert torch.allclose(outs[0][k], outs[1][k], rtol=1e-5, atol=1e-5 * float(outs[0][k].abs().max())), k


def test_backward_rejects_chunks_above_64():
    w = S.SCALE18S.with_(T=300, b=100, H=2)
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, True)
    assert L.ttt_mlp_backward_workspace_size(desc, 100, L.TTT_BIDIR) == 0
    assert "64" in L.ttt_last_error()

