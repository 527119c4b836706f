"""Failure detection on the GPU without faulting it: a bounded wait made to
expire (test hook) must come back as TTT_ERR_TIMEOUT with the CUDA context
still usable, and non-finite inputs must come back as TTT_ERR_NONFINITE."""
import pytest
import torch

from helpers import maxrel, run_gpu, run_oracle, to_np, tol
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives():
    w = S.MINIBATCH.with_(T=300, H=2)   # bf16 inputs: the cluster tensor-core scan
    inp = S.make_inputs(w)
    L.ttt_debug_inject_wait_timeout(True)
    try:
        g = run_gpu(w, inp, check_status=False)
        st = L.ttt_mlp_status(g["workspace"])
    finally:
        L.ttt_debug_inject_wait_timeout(False)
    assert st == L.TTT_ERR_TIMEOUT
    # the next call on the same context runs normally and is correct
    g = run_gpu(w, inp, want_z=True)
    o = run_oracle(w, inp)
    assert maxrel(to_np(g["Z"][0]), o["Z_f"]) <= tol(w)
    assert maxrel(to_np(g["Y"]), o["Y"]) <= tol(w)


def _poison(inp, key, value):
    t = inp[key]
    flat = t.view(-1)
    flat[flat.numel() // 3] = value


@pytest.mark.parametrize("w,key,value", [
    (S.MINIBATCH.with_(T=200, H=2), "X", float("nan")),
    (S.TINY, "X", float("nan")),
    (S.FULL63S.with_(T=700, H=4, D=256), "X", float("nan")),
    (S.FULL63S.with_(T=700, H=4, D=256), "theta_k", float("inf")),
    (S.MINIBATCH.with_(T=200, H=2), "theta_v", float("nan")),
    (S.MINIBATCH.with_(T=200, H=2), "W1_0", float("nan")),
    (S.FULL63S.with_(T=700, H=4, D=256), "W2_0", float("-inf")),
], ids=["per-head-X", "per-token-X", "full-layer-X", "full-layer-theta_k", "per-head-theta_v", "per-head-W1_0",
        "full-layer-W2_0"])
def test_nonfinite_input_reports_nonfinite(w, key, value):
    """A NaN or Inf anywhere in the inputs comes back as TTT_ERR_NONFINITE,
    whichever kernel it meets first (projection, scan state load, gate)."""
    inp = S.make_inputs(w)
    _poison(inp, key, value)
    g = run_gpu(w, inp, check_status=False)
    assert L.ttt_mlp_status(g["workspace"]) == L.TTT_ERR_NONFINITE
