"""ttt_mlp_forward_noalloc: the entry point for callers that cannot allocate
device memory (an embedding framework owns the allocator, a plug-in may not
call cudaMalloc, a service may not allocate after start-up).  It runs the same
kernels with the same arithmetic as ttt_mlp_forward, so its outputs must equal
that entry point's bit for bit, call after call, even though every call reuses
the library's one fixed scratch array; and a call must not change the
device's allocated memory.

Collected last on purpose (file name), so a failure here does not hide the
other GPU tests in a run that stops at the first failure.
"""
import pytest
import torch

from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu

CASES = [
    S.MINIBATCH.with_(T=1000, H=8),           # bf16, b = 16, bidirectional, ragged tail (cluster scan)
    S.CAUSAL,                                 # fp32, b = 1, forward (4 heads x 4096 tokens)
    S.FULL63S.with_(T=1500, H=4, D=256),      # full width, bf16, b = 64, bidirectional: ttt_mlp_forward runs
                                              # it in chunk segments on its own streams, this entry point on
                                              # the caller's stream alone
]


def _inputs(w, seed):
    dev = torch.device("cuda")
    return {k: v.to(dev) for k, v in S.make_inputs(w, seed=seed).items()}


def _reference(w, inp):
    return L.layer_forward(inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"],
                           w.eta_eff, w.b, w.dirs, alpha_f=inp["alpha_f"], alpha_r=inp["alpha_r"],
                           per_head=w.per_head, want_z=True, want_state=True)


def _outputs(w, inp):
    nd = 2 if w.dirs == "bidir" else 1
    dev = inp["X"].device
    return {"Y": torch.empty_like(inp["X"]),
            "Z": torch.empty((nd,) + tuple(inp["X"].shape), dtype=torch.float32, device=dev),
            "W1_T": torch.empty((nd,) + tuple(inp["W1_0"].shape), dtype=torch.float32, device=dev),
            "W2_T": torch.empty((nd,) + tuple(inp["W2_0"].shape), dtype=torch.float32, device=dev)}


def _noalloc(w, inp, out):
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    return L.ttt_mlp_forward_noalloc(desc, inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"],
                                     inp["W2_0"], w.eta_eff, w.b, L.DIRS[w.dirs], inp["alpha_f"], inp["alpha_r"],
                                     out["Y"], out["Z"], out["W1_T"], out["W2_T"])


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"{'head' if w.per_head else 'full'}-H{w.H}-T{w.T}-b{w.b}-"
                                                   f"{w.dirs}-{w.dtype}")
def test_noalloc_equals_workspace_entry_point_twice_in_a_row_and_allocates_nothing(w):
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, w.dtype == "bf16")
    assert L.ttt_mlp_workspace_size(desc, w.b, L.DIRS[w.dirs]) <= 32 << 20
    # everything the test needs is allocated up front; only the no-alloc calls run in between
    inps = [_inputs(w, seed) for seed in (0, 1)]   # two calls in a row on the shared scratch, different inputs
    refs = [_reference(w, inp) for inp in inps]
    outs = [_outputs(w, inp) for inp in inps]
    torch.cuda.synchronize()
    for k in range(2):
        if k == 1:
            before = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
        L.check(_noalloc(w, inps[k], outs[k]), "ttt_mlp_forward_noalloc")
        L.check(L.ttt_mlp_noalloc_status(), "ttt_mlp_noalloc_status")
        torch.cuda.synchronize()
        if k == 1:
            after = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
            assert after == before, (before, after)
        for name in ("Y", "Z", "W1_T", "W2_T"):
            assert torch.equal(outs[k][name], refs[k][name]), (k, name)


def test_noalloc_status_reports_an_expired_wait_and_the_next_call_is_clean():
    w = CASES[0]
    inp = _inputs(w, 0)
    ref = _reference(w, inp)
    out = _outputs(w, inp)
    L.ttt_debug_inject_wait_timeout(True)
    try:
        L.check(_noalloc(w, inp, out), "ttt_mlp_forward_noalloc")
        assert L.ttt_mlp_noalloc_status() == L.TTT_ERR_TIMEOUT
    finally:
        L.ttt_debug_inject_wait_timeout(False)
    L.check(_noalloc(w, inp, out), "ttt_mlp_forward_noalloc")
    assert L.ttt_mlp_noalloc_status() == L.TTT_OK
    assert torch.equal(out["Y"], ref["Y"]) and torch.equal(out["Z"], ref["Z"])


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = S.FULL63S.with_T(20000)              # needs about 1.4 GB of scratch
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, True)
    dev = torch.device("cuda")
    x = torch.zeros(16, device=dev)
    st = L.ttt_mlp_forward_noalloc(desc, x, x, x, x, x, x, w.eta_eff, w.b, L.TTT_BIDIR, x, x, x, None, None, None)
    assert st == L.TTT_ERR_UNSUPPORTED
    assert "32" in L.ttt_last_error() or "bytes" in L.ttt_last_error()
