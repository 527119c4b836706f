"""The segmented full layer forks its work onto the library's own streams and
joins back with events; it must also work inside a CUDA graph capture (the
usual way to replay a fixed-shape layer without host launch overhead)."""
import pytest
import torch

from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dirs", ["bidir", "fwd"])
def test_full_layer_captured_in_cuda_graph_matches_eager(dirs):
    w = S.FULL63S.with_(T=3000, H=4, D=256, dirs=dirs)
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in S.make_inputs(w).items()}
    desc = L.make_desc(w.T, w.H, w.d, False, True)
    direction = L.DIRS[dirs]
    ws = L.alloc_workspace(desc, w.b, direction, dev)

    def call(Y, stream):
        return L.ttt_mlp_forward(desc, g["X"], g["theta_q"], g["theta_k"], g["theta_v"], g["W1_0"], g["W2_0"],
                                 w.eta_eff, w.b, direction, g["alpha_f"], g["alpha_r"], Y, None, None, None, ws,
                                 ws.numel(), stream)

    Y_eager = torch.empty_like(g["X"])
    L.check(call(Y_eager, torch.cuda.current_stream()), "eager")
    L.check(L.ttt_mlp_status(ws), "eager status")

    s = torch.cuda.Stream()
    Y = torch.empty_like(g["X"])
    with torch.cuda.stream(s):   # warm-up on the capture stream
        L.check(call(Y, s), "warm-up")
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        st = call(Y, s)
    assert st == L.TTT_OK, L.ttt_last_error()
    Y.zero_()
    torch.cuda.synchronize()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_eager)
    L.check(L.ttt_mlp_status(ws), "replay status")
    del graph
