"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Workloads are the five of the benchmark description (tiny per-token scan,
4-head causal scan, 48-head bidirectional mini-batch scans, full 3072-wide
layer) at sizes the oracle finishes in seconds with ragged last chunks, plus
edge cases.  Full-length runs are in test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

from helpers import TOL_BF16, TOL_F32, maxrel, oracle_args, run_gpu, run_oracle, tol, to_np
from oracle import ttt_oracle as O
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu

IMPLS = [0, 1]   # 0 = automatic kernel choice, 1 = SIMT reference kernels


@pytest.fixture(params=IMPLS, ids=["auto", "simt"])
def impl(request):
    L.check(L.ttt_mlp_select_kernels(request.param, request.param), "select")
    yield request.param
    L.ttt_mlp_select_kernels(0, 0)


def _compare(w, g, o, dirs=None):
    dirs = dirs or w.dirs
    errs = {"Y": maxrel(to_np(g["Y"]), o["Y"])}
    if g["Z"] is not None:
        if dirs == "bidir":
            errs["Z_f"] = maxrel(to_np(g["Z"][0]), o["Z_f"])
            errs["Z_r"] = maxrel(to_np(g["Z"][1]), o["Z_r"])
        else:
            key = "Z_f" if dirs == "fwd" else "Z_r"
            errs[key] = maxrel(to_np(g["Z"][0]), o[key])
    if g["W1_T"] is not None:
        first = "f" if dirs in ("fwd", "bidir") else "r"
        errs["W1_T"] = maxrel(to_np(g["W1_T"][0]), o["W1_" + first])
        errs["W2_T"] = maxrel(to_np(g["W2_T"][0]), o["W2_" + first])
    return errs


def _check(w, dirs=None, eta=None, impl=None, **inp_kw):
    inp = S.make_inputs(w, seed=0)
    g = run_gpu(w, inp, dirs=dirs, eta=eta, want_z=True, want_state=True)
    o = run_oracle(w, inp, dirs=dirs, eta=eta)
    errs = _compare(w, g, o, dirs)
    print(f"PARITY {w.name} T={w.T} b={w.b} {dirs or w.dirs} " + " ".join(f"{k}={v:.3e}" for k, v in errs.items()),
          flush=True)
    bad = {k: v for k, v in errs.items() if not v <= tol(w)}
    assert not bad, f"{w.name}: {errs}"
    return errs


def test_tiny_workload(impl):
    _check(S.TINY)


def test_causal_workload(impl):
    _check(S.CAUSAL)


@pytest.mark.parametrize("T", [1000, 1003])
def test_minibatch_b16_bidir_ragged(impl, T):
    _check(S.MINIBATCH.with_T(T))


@pytest.mark.parametrize("T", [1000, 64 * 9])
def test_b64_bidir_ragged(impl, T):
    _check(S.SCALE18S.with_T(T))


def test_full_layer_short(impl):
    _check(S.FULL63S.with_T(777))


@pytest.mark.parametrize("T", [3000, 64 * 50])
@pytest.mark.parametrize("dirs", ["bidir", "rev"])
def test_full_layer_segmented_pipeline(T, dirs):
    """On the tensor-core path the full layer runs each direction as several
    chunk segments (state carried between launches, projection and gate on a
    second stream): lengths that give three segments, with and without a
    ragged last chunk, checked with the final state."""
    _check(S.FULL63S.with_(T=T, H=4, D=256, dirs=dirs))


@pytest.mark.parametrize("dirs", ["fwd", "rev", "bidir"])
@pytest.mark.parametrize("b", [1, 5, 64])
def test_directions_and_chunks_f32(impl, dirs, b):
    w = S.Workload("edge", H=3, d=32, T=150, b=b, dirs=dirs, dtype="f32", per_head=True, eta=0.05)
    _check(w)


@pytest.mark.parametrize("T,b", [(1, 1), (1, 16), (7, 16), (64, 64), (65, 64)])
def test_short_sequences(impl, T, b):
    _check(S.SCALE18S.with_(T=T, b=b, H=4))


def test_full_mode_f32(impl):
    w = S.Workload("full-f32", H=4, d=64, T=300, b=16, dirs="bidir", dtype="f32", per_head=False, eta=0.05,
                   D=256)
    _check(w)


def test_d16_chunked_bidir(impl):
    _check(S.TINY.with_(b=8, dirs="bidir", H=2))


def test_eta_zero_state_unchanged():
    w = S.SCALE18S.with_(T=200, H=2)
    inp = S.make_inputs(w)
    g = run_gpu(w, inp, eta=0.0, want_z=True, want_state=True)
    np.testing.assert_array_equal(g["W1_T"][0].cpu().numpy(), inp["W1_0"].numpy())
    np.testing.assert_array_equal(g["W2_T"][1].cpu().numpy(), inp["W2_0"].numpy())
    o = run_oracle(w, inp, eta=0.0)
    assert maxrel(to_np(g["Z"][0]), o["Z_f"]) < 1e-3


def test_alpha_zero_is_identity():
    for w in (S.TINY, S.MINIBATCH.with_(T=300, H=3), S.FULL63S.with_(T=100)):
        inp = S.make_inputs(w)
        inp["alpha_f"].zero_(); inp["alpha_r"].zero_()
        g = run_gpu(w, inp)
        assert torch.equal(g["Y"].cpu(), inp["X"])


def test_literal_eta_reports_nonfinite():
    w = S.TINY
    inp = S.make_inputs(w)
    g = run_gpu(w, inp, eta=w.eta, check_status=False)
    assert L.ttt_mlp_status(g["workspace"]) == L.TTT_ERR_NONFINITE
    # the status word is cleared by the read
    assert L.ttt_mlp_status(g["workspace"]) == L.TTT_OK


def test_reverse_equals_flipped_forward_on_gpu():
    w = S.MINIBATCH.with_(T=2000, H=4, dirs="rev")
    inp = S.make_inputs(w)
    g_rev = run_gpu(w, inp, dirs="rev", want_z=True)
    flipped = dict(inp)
    flipped["X"] = inp["X"].flip(1).contiguous()
    flipped["alpha_f"] = inp["alpha_r"]
    g_fwd = run_gpu(w, flipped, dirs="fwd", want_z=True)
    # Same arithmetic up to the order of the token sums inside the tf32 MMAs
    # (the reverse pass holds its tokens in natural order): a few tf32 ulps.
    assert maxrel(to_np(g_rev["Z"][0]), to_np(g_fwd["Z"][0].flip(1))) < 1e-3


@pytest.mark.parametrize("w", [S.MINIBATCH.with_(T=500, H=4), S.FULL63S.with_(T=3000, H=4, D=256),
                               S.FULL63S.with_(T=3000, H=4, D=256, dirs="rev")],
                         ids=["per-head", "full-layer-segmented", "full-layer-segmented-rev"])
def test_host_io_entry_point_matches_device_entry_point(w):
    """Host buffers in and out (copied segment by segment, overlapped with the
    computation, on the segmented full-layer path) give the device entry
    point's result bit for bit."""
    inp = S.make_inputs(w)
    dev = torch.device("cuda")
    gd = {k: v.to(dev) for k, v in inp.items()}
    ref = run_gpu(w, inp)["Y"].cpu()
    desc = L.make_desc(w.T, w.H, w.d, w.per_head, True)
    direction = L.DIRS[w.dirs]
    ws = L.alloc_workspace(desc, w.b, direction, dev, host_io=True)
    Xh = inp["X"].pin_memory()
    Yh = torch.empty_like(Xh).pin_memory()
    st = L.ttt_mlp_forward_host(desc, Xh, gd["theta_q"], gd["theta_k"], gd["theta_v"], gd["W1_0"], gd["W2_0"],
                                w.eta_eff, w.b, direction, gd["alpha_f"], gd["alpha_r"], Yh, ws, ws.numel())
    L.check(st, "ttt_mlp_forward_host")
    assert torch.equal(Yh, ref)


def test_launches_are_counted():
    w = S.TINY
    inp = S.make_inputs(w)
    n0 = L.ttt_launch_count()
    run_gpu(w, inp)
    assert L.ttt_launch_count() - n0 >= 2


@pytest.mark.parametrize("T", [1000, 128])
def test_full_layer_eta_zero_isolates_projection(impl, T):
    """eta = 0 freezes the state, so z = W2_0 GELU(W1_0 q) depends only on the
    projections: a tight check of the full-layer projection kernels (forward
    pass, and the reverse pass's accumulation onto the forward projections).
    The scan is pinned to the fp32 kernel so only the projection kernel varies."""
    L.check(L.ttt_mlp_select_kernels(1, impl), "select")
    w = S.FULL63S.with_T(T)
    inp = S.make_inputs(w)
    g = run_gpu(w, inp, eta=0.0, want_z=True)
    o = run_oracle(w, inp, eta=0.0)
    assert maxrel(to_np(g["Z"][0]), o["Z_f"]) < 1e-5
    assert maxrel(to_np(g["Z"][1]), o["Z_r"]) < 2e-4


@pytest.mark.parametrize("w", [S.MINIBATCH.with_T(1000), S.SCALE18S.with_T(1000), S.FULL63S.with_T(777)],
                         ids=["b16-per-head", "b64-per-head", "full-layer"])
def test_one_cta_tensor_core_scan(w):
    """The tensor-core scan with one CTA per head (the default runs each head on
    a two-CTA cluster) against the oracle."""
    L.check(L.ttt_mlp_select_kernels(3, 0), "select")
    try:
        _check(w)
    finally:
        L.ttt_mlp_select_kernels(0, 0)


@pytest.mark.parametrize("dirs", ["fwd", "rev", "bidir"])
@pytest.mark.parametrize("sel", [0, 3], ids=["four-cta-cluster", "one-cta"])
@pytest.mark.parametrize("per_head", [True, False], ids=["per-head", "full-width"])
def test_per_token_kernels_d64(sel, dirs, per_head):
    """b = 1 at d = 64: the per-token scan with each head's state over a cluster of
    four CTAs (automatic) and with one CTA per head (selector 3), every direction,
    a token count that is not a multiple of the 32-token staging block."""
    w = S.Workload("tok-d64", H=3, d=64, T=150, b=1, dirs=dirs, dtype="f32", per_head=per_head, eta=0.05,
                   D=0 if per_head else 192)
    L.check(L.ttt_mlp_select_kernels(sel, 0), "select")
    try:
        _check(w)
    finally:
        L.ttt_mlp_select_kernels(0, 0)
