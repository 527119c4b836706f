"""ttt_mlp_forward_noalloc: the entry point for callers that cannot allocate
device memory (an embedding framework owns the allocator, a plug-in may not
call cudaMalloc, a service may not allocate after start-up).  It must give the
same results as ttt_mlp_forward with a caller workspace, call after call,
even though every call reuses the library's one fixed scratch array.

Collected last on purpose (file name), so a failure here does not hide the
other GPU tests in a run that stops at the first failure.
"""
import pytest
import torch

from helpers import maxrel, tol, to_np
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu

CASES = [
    S.MINIBATCH.with_(T=1000, H=8),          # bf16, b = 16, bidirectional, ragged tail
    S.CAUSAL,                                # fp32, b = 1, forward (4 heads x 4096 tokens)
]


def _both(w, seed):
    dev = torch.device("cuda")
    inp = {k: v.to(dev) for k, v in S.make_inputs(w, seed=seed).items()}
    ref = L.layer_forward(inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"],
                          w.eta_eff, w.b, w.dirs, alpha_f=inp["alpha_f"], alpha_r=inp["alpha_r"],
                          per_head=w.per_head, want_z=True)
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    nd = 2 if w.dirs == "bidir" else 1
    Y = torch.empty_like(inp["X"])
    Z = torch.empty((nd,) + tuple(inp["X"].shape), dtype=torch.float32, device=dev)
    st = L.ttt_mlp_forward_noalloc(desc, inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"],
                                   inp["W2_0"], w.eta_eff, w.b, L.DIRS[w.dirs], inp["alpha_f"], inp["alpha_r"], Y, Z,
                                   None, None)
    L.check(st, "ttt_mlp_forward_noalloc")
    torch.cuda.synchronize()
    return ref, Y, Z


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"H{w.H}-T{w.T}-b{w.b}-{w.dirs}-{w.dtype}")
def test_noalloc_matches_workspace_entry_point_twice_in_a_row(w):
    for seed in (0, 1):       # two calls in a row on the shared scratch, different inputs
        ref, Y, Z = _both(w, seed)
        assert maxrel(to_np(Y), to_np(ref["Y"])) <= tol(w)
        assert maxrel(to_np(Z), to_np(ref["Z"])) <= tol(w)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = S.FULL63S.with_T(20000)              # needs about 1.4 GB of scratch
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, True)
    dev = torch.device("cuda")
    x = torch.zeros(16, device=dev)
    st = L.ttt_mlp_forward_noalloc(desc, x, x, x, x, x, x, w.eta_eff, w.b, L.TTT_BIDIR, x, x, x, None, None, None)
    assert st == L.TTT_ERR_UNSUPPORTED
    assert "32" in L.ttt_last_error() or "bytes" in L.ttt_last_error()
