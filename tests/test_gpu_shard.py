"""Head-sharded layer on one GPU: R ranks emulated one after another through
ttt_mlp_forward_heads (test_rnn_layer_b200/shard.py's per-rank steps; the
sums over ranks are plain additions, since each column has one non-zero
contributor).  No kernel waits on another: the ranks' launches are ordinary
stream-ordered launches.

The assembled Y must equal ttt_mlp_forward's bidirectional full-width layer
bit for bit (the same kernels, the same per-element arithmetic), and X' and
the gate increment must too; one case is also compared with the fp64 oracle.
The 48-head, 8-rank case gives each rank 6 heads, so the projection's last
column tile is partial."""
import numpy as np
import pytest
import torch

from helpers import maxrel, to_np
from oracle import ttt_oracle as O
from test_rnn_layer_b200 import shard
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu

CASES = [("h8-T1000", 8, 1000, [1, 2, 4, 8]), ("h48-T700", 48, 700, [8, 5])]


def _inputs(H, T, seed=0):
    w = S.FULL63S.with_(T=T, H=H, D=H * 64)
    inp = S.make_inputs(w, seed=seed, device=torch.device("cuda"))
    return w, inp


def _emulated(w, inp, world):
    th = [inp["theta_q"], inp["theta_k"], inp["theta_v"]]
    steps = [shard.shard_forward(inp["X"], th, inp["W1_0"], inp["W2_0"], w.eta_eff, w.b, inp["alpha_f"], r, world)
             for r in range(world)]
    inc_all = sum(inc for _, inc in steps)
    Y = sum(shard.shard_reverse(inp["X"], th, inp["W1_0"], inp["W2_0"], w.eta_eff, w.b, inp["alpha_r"], inc_all,
                                steps[r][0], r, world) for r in range(world))
    torch.cuda.synchronize()
    return Y, inc_all


@pytest.mark.parametrize("name,H,T,worlds", CASES, ids=[c[0] for c in CASES])
def test_emulated_ranks_equal_the_single_gpu_layer(name, H, T, worlds):
    w, inp = _inputs(H, T)
    full = L.layer_forward(inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"],
                           w.eta_eff, w.b, "bidir", alpha_f=inp["alpha_f"], alpha_r=inp["alpha_r"], per_head=False)
    for world in worlds:
        if H % world:
            with pytest.raises(ValueError):
                _emulated(w, inp, world)
            continue
        Y, inc_all = _emulated(w, inp, world)
        assert torch.isfinite(Y.float()).all()
        assert torch.equal(Y, full["Y"]), (world, (Y.float() - full["Y"].float()).abs().max().item())


def test_sharded_layer_matches_the_oracle():
    w, inp = _inputs(8, 600, seed=5)
    Y, _ = _emulated(w, inp, 4)
    c = {k: to_np(v) for k, v in inp.items()}
    ref = O.layer_forward(c["X"], c["theta_q"], c["theta_k"], c["theta_v"], c["W1_0"], c["W2_0"], w.eta_eff, w.b,
                          "bidir", alpha_f=c["alpha_f"], alpha_r=c["alpha_r"], per_head=False)["Y"]
    err = maxrel(to_np(Y), ref)
    print(f"PARITY shard-h8-T600-4ranks Y={err:.3e}", flush=True)
    assert err <= 2e-2


def test_bad_head_ranges_and_layouts_are_refused():
    w, inp = _inputs(8, 128)
    desc = L.make_desc(w.T, w.H, w.d, False, True)
    n = L.ttt_mlp_heads_workspace_size(desc, 2, w.b)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    Xp = torch.empty(w.T, w.H * w.d, dtype=torch.float32, device="cuda")
    out = torch.zeros(w.T, w.H * w.d, dtype=torch.bfloat16, device="cuda")
    args = (inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"], w.eta_eff, w.b,
            inp["alpha_f"], None, Xp, out, ws, n)
    assert L.ttt_mlp_forward_heads(desc, 7, 2, L.TTT_PHASE_FWD, *args) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_mlp_forward_heads(desc, 0, 2, 5, *args) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_mlp_forward_heads(desc, 0, 2, L.TTT_PHASE_REV, *args) == L.TTT_ERR_INVALID_ARG   # no delta_all
    small = L.ttt_mlp_forward_heads(desc, 0, 2, L.TTT_PHASE_FWD, *args[:-1], n - 256)
    assert small == L.TTT_ERR_INVALID_ARG
    head_desc = L.make_desc(w.T, w.H, w.d, True, True)
    assert L.ttt_mlp_forward_heads(head_desc, 0, 2, L.TTT_PHASE_FWD, *args) == L.TTT_ERR_UNSUPPORTED
