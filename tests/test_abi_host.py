"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/tttmlp.h declares, sizes workspaces, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from test_rnn_layer_b200 import build as B
from test_rnn_layer_b200 import tttmlp as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def _declared():
    src = open(os.path.join(ROOT, "include", "tttmlp.h")).read()
    return sorted(set(re.findall(r"TTT_API\s+[\w\s\*]+?\b(ttt_\w+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = _declared()
    assert "ttt_mlp_forward" in names and len(names) >= 8
    out = subprocess.run(["nm", "-D", "--defined-only", L.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (ttt_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    lib = L.lib()
    for n in names:
        assert getattr(lib, n) is not None
    assert set(L.EXPORTED) == set(names)


def test_library_needs_no_driver_at_load_time():
    out = subprocess.run(["ldd", L.library_path()], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "not found" not in out


def _desc(**kw):
    base = dict(T=1024, H=4, d=64, per_head=True, bf16=False)
    base.update(kw)
    return L.make_desc(base["T"], base["H"], base["d"], base["per_head"], base["bf16"])


def test_workspace_sizes():
    d = _desc()
    n1 = L.ttt_mlp_workspace_size(d, 1, L.TTT_FWD)
    nb = L.ttt_mlp_workspace_size(d, 1, L.TTT_BIDIR)
    assert n1 >= 3 * 1024 * 256 * 4 and nb >= n1 + 1024 * 256 * 4
    assert L.ttt_mlp_host_io_workspace_size(d, 1, L.TTT_FWD) >= n1 + 2 * 1024 * 256 * 4
    full = _desc(T=313344, H=48, per_head=False, bf16=True)
    n = L.ttt_mlp_workspace_size(full, 64, L.TTT_BIDIR)
    # Q, K, V and X' in fp32 plus the bf16 gate increment: at least 9.0 bytes per element
    assert n >= 313344 * 3072 * 18
    assert n % 256 == 0


@pytest.mark.parametrize("bad", [dict(T=0), dict(H=0), dict(d=48), dict(d=0)])
def test_bad_desc_rejected(bad):
    d = _desc(**bad)
    assert L.ttt_mlp_workspace_size(d, 1, L.TTT_FWD) == 0
    assert L.ttt_last_error()


def test_bad_m_and_D_rejected():
    d = _desc()
    d.m = 200
    assert L.ttt_mlp_workspace_size(d, 1, L.TTT_FWD) == 0 and "m=" in L.ttt_last_error()
    d = _desc()
    d.D = 100
    assert L.ttt_mlp_workspace_size(d, 1, L.TTT_FWD) == 0 and "D=" in L.ttt_last_error()


@pytest.mark.parametrize("b", [0, -1, 257])
def test_bad_chunk_rejected(b):
    assert L.ttt_mlp_workspace_size(_desc(), b, L.TTT_FWD) == 0


def _fwd(desc, **over):
    args = dict(X=0x1000, tq=0x2000, tk=0x3000, tv=0x4000, W1=0x5000, W2=0x6000, eta=0.01, b=16,
                dir=L.TTT_BIDIR, af=0x7000, ar=0x8000, Y=0x90000000, Z=None, W1T=None, W2T=None,
                ws=0x100000000, wsb=1 << 40)
    args.update(over)
    return L.ttt_mlp_forward(desc, args["X"], args["tq"], args["tk"], args["tv"], args["W1"], args["W2"],
                             args["eta"], args["b"], args["dir"], args["af"], args["ar"], args["Y"], args["Z"],
                             args["W1T"], args["W2T"], args["ws"], args["wsb"], 0)


def test_forward_argument_errors_before_any_cuda_call():
    """Every call below is rejected by argument checks, so the fake addresses
    never reach the device.  Still skipped where a GPU exists."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake device addresses are only used where no GPU exists")
    d = _desc()
    assert _fwd(d, X=None) == L.TTT_ERR_INVALID_ARG
    assert _fwd(d, ar=None) == L.TTT_ERR_INVALID_ARG and "alpha_r" in L.ttt_last_error()
    assert _fwd(d, eta=float("nan")) == L.TTT_ERR_INVALID_ARG
    assert _fwd(d, eta=-1.0) == L.TTT_ERR_INVALID_ARG
    assert _fwd(d, X=0x1004) == L.TTT_ERR_INVALID_ARG and "aligned" in L.ttt_last_error()
    assert _fwd(d, ws=0x100000010) == L.TTT_ERR_INVALID_ARG and "256" in L.ttt_last_error()
    assert _fwd(d, wsb=1024) == L.TTT_ERR_INVALID_ARG and "too small" in L.ttt_last_error()
    assert _fwd(d, Y=0x1000) == L.TTT_ERR_INVALID_ARG and "alias" in L.ttt_last_error()
    assert _fwd(d, b=0) == L.TTT_ERR_INVALID_ARG
    assert _fwd(_desc(d=48)) == L.TTT_ERR_UNSUPPORTED


def test_kernel_selector_validation():
    assert L.ttt_mlp_select_kernels(5, 0) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_mlp_select_kernels(-1, 0) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_mlp_select_kernels(0, 3) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_mlp_select_kernels(0, 0) == L.TTT_OK


def test_status_null_workspace():
    assert L.lib().ttt_mlp_status(None, None) == L.TTT_ERR_INVALID_ARG


def test_linear_workspace_sizes_and_desc_checks():
    d = _desc()
    d.m = 12345   # not used by the linear layer
    n1 = L.ttt_linear_workspace_size(d, 16, L.TTT_FWD)
    nb = L.ttt_linear_workspace_size(d, 16, L.TTT_BIDIR)
    # Q, K, V and z in fp32 (+ X' for both directions)
    assert n1 >= 4 * 1024 * 256 * 4 and nb >= n1 + 1024 * 256 * 4 and n1 % 256 == 0
    assert L.ttt_linear_workspace_size(_desc(d=48), 16, L.TTT_FWD) == 0
    assert L.ttt_linear_workspace_size(_desc(), 0, L.TTT_FWD) == 0


def test_linear_forward_argument_errors_before_any_cuda_call():
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake device addresses are only used where no GPU exists")
    d = _desc()

    def fwd(**over):
        a = dict(X=0x1000, tq=0x2000, tk=0x3000, tv=0x4000, W=0x5000, eta=0.01, b=16, dir=L.TTT_BIDIR,
                 af=0x7000, ar=0x8000, Y=0x90000000, Z=None, WT=None, ws=0x100000000, wsb=1 << 40)
        a.update(over)
        return L.ttt_linear_forward(d, a["X"], a["tq"], a["tk"], a["tv"], a["W"], a["eta"], a["b"], a["dir"],
                                    a["af"], a["ar"], a["Y"], a["Z"], a["WT"], a["ws"], a["wsb"], 0)

    assert fwd(W=None) == L.TTT_ERR_INVALID_ARG
    assert fwd(af=None) == L.TTT_ERR_INVALID_ARG and "alpha_f" in L.ttt_last_error()
    assert fwd(eta=float("inf")) == L.TTT_ERR_INVALID_ARG
    assert fwd(Y=0x1000) == L.TTT_ERR_INVALID_ARG and "alias" in L.ttt_last_error()
    assert fwd(wsb=4096) == L.TTT_ERR_INVALID_ARG and "too small" in L.ttt_last_error()
    assert fwd(WT=0x1008) == L.TTT_ERR_INVALID_ARG and "aligned" in L.ttt_last_error()


@pytest.mark.parametrize("nchunks", [1, 15, 16, 17, 47, 128, 1000, 1603, 4896])
def test_pipeline_segments_tile_the_walk(nchunks):
    """The pipelined full-width layer splits a direction's walk into chunk
    segments: contiguous, non-empty, covering [0, nchunks) exactly; the first
    and last segments are the shortest (their projection or gate is not
    overlapped), no segment exceeds max(16, ceil(nchunks / 16))."""
    seg = L.ttt_debug_pipe_segments(nchunks)
    assert seg[0][0] == 0 and seg[-1][1] == nchunks
    for (a0, a1), (b0, _) in zip(seg, seg[1:]):
        assert a1 == b0
    sizes = [e - b for b, e in seg]
    assert min(sizes) >= 1
    cap = max(16, -(-nchunks // 16))
    assert max(sizes) <= cap
    if len(seg) > 2:
        assert sizes[0] <= min(sizes[1:-1]) and sizes[-1] <= min(sizes[1:-1])
    assert L.lib().ttt_debug_pipe_segments(0, None, 0) == -1


def test_pipeline_segments_of_the_benchmark_layer():
    """313,344 tokens in 64-token chunks: 4,896 chunks; the ramp grows by 3/2
    from 16 at both ends and the middle is split into equal pieces."""
    sizes = [e - b for b, e in L.ttt_debug_pipe_segments(4896)]
    assert sizes[:4] == [16, 24, 36, 54] and sizes[-4:] == [54, 36, 24, 16]
    middle = sizes[8:-8]   # between the two ramps (8 segments each: 16 ... 271), at most 306 = 4896 / 16
    assert max(middle) - min(middle) <= 1 and max(middle) <= 306


def test_attention_argument_errors_before_any_cuda_call():
    """ttt_seg_attention and ttt_block_forward reject bad arguments before any
    CUDA call (fake device addresses; skipped where a GPU exists)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake device addresses are only used where no GPU exists")
    T, H = 1000, 2
    Q, K, V, O, W = 0x10000000, 0x20000000, 0x30000000, 0x40000000, 0x50000000

    def att(**kw):
        a = dict(T=T, H=H, d=64, L=300, Q=Q, K=K, V=V, ld=128, X=None, O=O, ldo=128, r0=0, r1=T, ws=W, wsb=256)
        a.update(kw)
        return L.ttt_seg_attention(a["T"], a["H"], a["d"], a["L"], a["Q"], a["K"], a["V"], a["ld"], a["X"], a["O"],
                                   a["ldo"], a["r0"], a["r1"], a["ws"], a["wsb"], 0)

    assert L.ttt_seg_attention_workspace_size() == 256
    assert att(d=32) == L.TTT_ERR_UNSUPPORTED
    assert att(L=0) == L.TTT_ERR_INVALID_ARG
    assert att(ld=120) == L.TTT_ERR_INVALID_ARG and "strides" in L.ttt_last_error()
    assert att(ldo=132) == L.TTT_ERR_INVALID_ARG
    assert att(V=None) == L.TTT_ERR_INVALID_ARG
    assert att(Q=Q + 8) == L.TTT_ERR_INVALID_ARG and "aligned" in L.ttt_last_error()
    assert att(O=K + 4096) == L.TTT_ERR_INVALID_ARG and "overlap" in L.ttt_last_error()
    assert att(r0=10, r1=5) == L.TTT_ERR_INVALID_ARG
    assert att(r1=T + 1) == L.TTT_ERR_INVALID_ARG
    assert att(ws=None) == L.TTT_ERR_INVALID_ARG
    assert att(wsb=16) == L.TTT_ERR_INVALID_ARG
    d = L.make_desc(T, H, 64, False, True)
    assert L.ttt_block_workspace_size(d, 64) == L.ttt_mlp_workspace_size(d, 64, L.TTT_BIDIR) > 0
    ph = L.make_desc(T, H, 64, True, True)
    blk = lambda desc, **kw: L.ttt_block_forward(desc, kw.get("L", 300), Q, K, V, 128, None, kw.get("X", O), 0x60000000,
                                                 0x61000000, 0x62000000, 0x63000000, 0x64000000, 0.01, 64,
                                                 0x65000000, 0x66000000, 0x67000000, W, 1 << 40, 0)
    assert blk(ph) == L.TTT_ERR_UNSUPPORTED
    assert blk(d, L=0) == L.TTT_ERR_INVALID_ARG
    assert blk(d, X=Q) == L.TTT_ERR_INVALID_ARG and "overlap" in L.ttt_last_error()
    assert L.ttt_debug_set_block_front(101) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_debug_set_block_front(-1) == L.TTT_OK
    assert L.ttt_debug_set_backward_ctas(3) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_debug_set_backward_ctas(-1) == L.TTT_ERR_INVALID_ARG
    assert L.ttt_debug_set_backward_ctas(0) == L.TTT_OK
