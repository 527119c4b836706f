"""The two-CTA tensor-core scans, each selected explicitly, against the fp64
oracle: the kernel whose every warp walks every stage of a chunk (scan
selector 2) and the one whose state and output warp groups run a chunk apart
(selector 4).  Workloads: the bidirectional mini-batch scans at b = 16 and 64
with ragged last chunks, both directions alone, short sequences (a single
ragged chunk, exact multiples of 64), the 3072-wide layer in one launch and
in chunk segments, fp32 inputs, and the final states.  Tolerance 2e-2 (tf32
and fp16 operands, fp32 accumulation and state)."""
import pytest

from helpers import TOL_BF16, maxrel, run_gpu, run_oracle, to_np
from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[2, 4], ids=["cluster", "cluster-split-groups"])
def scan_impl(request):
    L.check(L.ttt_mlp_select_kernels(request.param, 0), "select")
    yield request.param
    L.ttt_mlp_select_kernels(0, 0)


def _check(w, dirs=None):
    inp = S.make_inputs(w, seed=0)
    g = run_gpu(w, inp, dirs=dirs, want_z=True, want_state=True)
    o = run_oracle(w, inp, dirs=dirs)
    dirs = dirs or w.dirs
    errs = {"Y": maxrel(to_np(g["Y"]), o["Y"])}
    keys = {"fwd": ["Z_f"], "rev": ["Z_r"], "bidir": ["Z_f", "Z_r"]}[dirs]
    for i, k in enumerate(keys):
        errs[k] = maxrel(to_np(g["Z"][i]), o[k])
    first = "f" if dirs in ("fwd", "bidir") else "r"
    errs["W1_T"] = maxrel(to_np(g["W1_T"][0]), o["W1_" + first])
    errs["W2_T"] = maxrel(to_np(g["W2_T"][0]), o["W2_" + first])
    print(f"PARITY {w.name} T={w.T} b={w.b} {dirs} " + " ".join(f"{k}={v:.3e}" for k, v in errs.items()), flush=True)
    assert all(v <= TOL_BF16 for v in errs.values()), errs


@pytest.mark.parametrize("T", [1000, 2048])
def test_bidir_b16(scan_impl, T):
    _check(S.MINIBATCH.with_(T=T, H=6))


@pytest.mark.parametrize("T", [1500, 4096])
def test_bidir_b64(scan_impl, T):
    _check(S.SCALE18S.with_(T=T, H=6))


@pytest.mark.parametrize("dirs", ["fwd", "rev"])
def test_one_direction(scan_impl, dirs):
    _check(S.SCALE18S.with_(T=777, H=3), dirs=dirs)


@pytest.mark.parametrize("T,b", [(1, 16), (7, 16), (64, 64), (65, 64), (128, 64), (200, 2), (300, 33)])
def test_short_sequences_and_odd_chunks(scan_impl, T, b):
    _check(S.SCALE18S.with_(T=T, b=b, H=2))


def test_full_layer_one_launch(scan_impl):
    _check(S.FULL63S.with_(T=777, H=4, D=256))


@pytest.mark.parametrize("T", [3000, 64 * 50])
def test_full_layer_segments(scan_impl, T):
    _check(S.FULL63S.with_(T=T, H=4, D=256))


def test_fp32_inputs(scan_impl):
    _check(S.Workload("f32-tc", H=3, d=64, T=500, b=32, dirs="bidir", dtype="f32", per_head=True, eta=0.05))
