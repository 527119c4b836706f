"""Two callers on two streams: the segmented full-width layer runs on a set of
library streams per caller stream, so two layers enqueued on different
streams (both enqueued before either is synchronised) must give the same
bits as the same layers run one after the other."""
import pytest
import torch

from test_rnn_layer_b200 import synth as S
from test_rnn_layer_b200 import tttmlp as L

pytestmark = pytest.mark.gpu


def _call(w, inp, Y, ws, stream):
    desc = L.make_desc(w.T, w.H, w.d, False, True)
    st = L.ttt_mlp_forward(desc, inp["X"], inp["theta_q"], inp["theta_k"], inp["theta_v"], inp["W1_0"], inp["W2_0"],
                           w.eta_eff, w.b, L.TTT_BIDIR, inp["alpha_f"], inp["alpha_r"], Y, None, None, None, ws,
                           ws.numel(), stream)
    L.check(st, "ttt_mlp_forward")


def test_two_caller_streams_equal_sequential_calls():
    w = S.FULL63S.with_T(3000)
    dev = torch.device("cuda")
    inps = [S.make_inputs(w, seed=s, device=dev) for s in (11, 12)]
    desc = L.make_desc(w.T, w.H, w.d, False, True)
    wss = [L.alloc_workspace(desc, w.b, L.TTT_BIDIR, dev) for _ in range(2)]
    seq = [torch.empty_like(inp["X"]) for inp in inps]
    cur = torch.cuda.current_stream()
    for k in range(2):
        _call(w, inps[k], seq[k], wss[k], cur)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    par = [torch.empty_like(inp["X"]) for inp in inps]
    for _ in range(2):   # the second round reuses each stream's library streams and events
        for k in range(2):
            streams[k].wait_stream(cur)
            with torch.cuda.stream(streams[k]):
                _call(w, inps[k], par[k], wss[k], streams[k])
        torch.cuda.synchronize()
        for k in range(2):
            assert L.ttt_mlp_status(wss[k], streams[k]) == L.TTT_OK
            assert torch.equal(par[k], seq[k])
