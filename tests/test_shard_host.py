"""Host logic of the head-sharded layer (test_rnn_layer_b200/shard.py) on CPU.

Two gloo ranks run sharded_layer_forward with steps computed by the fp64
oracle for their heads (the same quantities the CUDA phases write: X' and the
bf16 gate increment in the rank's columns; Y in the rank's columns after a
reverse pass on X + the summed increments).  Checks: the two-rank result
equals the one-rank result bit for bit (the sums have one non-zero
contributor per column), it matches the unsharded oracle layer within the
bf16 rounding of the increment and of Y, and the head ranges tile the heads.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from test_rnn_layer_b200 import shard

ETA, B, T, H, D_HEAD = 0.05 / 4, 4, 24, 4, 4   # eta = 0.05 / d, as the workloads use


def _inputs(seed=3):
    g = np.random.default_rng(seed)
    D, m = H * D_HEAD, 4 * D_HEAD
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)
    return {"X": bf(g.normal(size=(T, D))),
            "theta": [bf(g.normal(size=(D, D)) / np.sqrt(D)) for _ in range(3)],
            "W1_0": torch.tensor(g.normal(size=(H, m, D_HEAD)) / np.sqrt(D_HEAD), dtype=torch.float32),
            "W2_0": torch.tensor(g.normal(size=(H, D_HEAD, m)) / np.sqrt(m), dtype=torch.float32),
            "alpha_f": torch.tensor(g.normal(size=D) * 0.5, dtype=torch.float32),
            "alpha_r": torch.tensor(g.normal(size=D) * 0.5, dtype=torch.float32)}


def _cols(rank, world):
    h0, hn = shard.head_range(H, rank, world)
    return slice(h0 * D_HEAD, (h0 + hn) * D_HEAD), list(range(h0, h0 + hn))


def oracle_forward_step(X, theta, W1_0, W2_0, eta, b, alpha_f, rank, world):
    from oracle import ttt_oracle as O
    cols, heads = _cols(rank, world)
    Xf = X.double().numpy()
    z, _, _ = O.full_mode_heads(Xf, *[t.double().numpy() for t in theta], W1_0.numpy(), W2_0.numpy(), eta, b,
                                heads, reverse=False)
    incr = np.tanh(alpha_f.double().numpy()[cols]) * z
    Xp = torch.zeros(X.shape, dtype=torch.float32)
    inc = torch.zeros(X.shape, dtype=torch.bfloat16)
    Xp[:, cols] = torch.tensor(Xf[:, cols] + incr, dtype=torch.float32)
    inc[:, cols] = torch.tensor(incr, dtype=torch.float32).to(torch.bfloat16)
    return Xp, inc


def oracle_reverse_step(X, theta, W1_0, W2_0, eta, b, alpha_r, inc_all, Xp, rank, world):
    from oracle import ttt_oracle as O
    cols, heads = _cols(rank, world)
    Xr = X.double().numpy() + inc_all.double().numpy()   # X' as the reverse projection reads it
    z, _, _ = O.full_mode_heads(Xr, *[t.double().numpy() for t in theta], W1_0.numpy(), W2_0.numpy(), eta, b,
                                heads, reverse=True)
    Y = torch.zeros(X.shape, dtype=torch.bfloat16)
    Y[:, cols] = torch.tensor(Xp[:, cols].double().numpy() + np.tanh(alpha_r.double().numpy()[cols]) * z,
                              dtype=torch.float32).to(torch.bfloat16)
    return Y


def _sum_over_ranks(t):   # gloo sums fp32; every column has one non-zero contributor
    f = t.float()
    dist.all_reduce(f)
    t.copy_(f.to(t.dtype))


def _run(inp, rank, world, all_reduce):
    return shard.sharded_layer_forward(inp["X"], inp["theta"], inp["W1_0"], inp["W2_0"], ETA, B, inp["alpha_f"],
                                       inp["alpha_r"], rank, world, all_reduce, forward_step=oracle_forward_step,
                                       reverse_step=oracle_reverse_step)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Y = _run(_inputs(), rank, world, _sum_over_ranks)
        out[rank] = Y.float().numpy().tobytes()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_equal_one_rank_and_the_unsharded_oracle():
    from oracle import ttt_oracle as O
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]                                   # every rank holds the whole output
    inp = _inputs()
    one = _run(inp, 0, 1, lambda t: None)
    two = np.frombuffer(res[0], dtype=np.float32).reshape(T, H * D_HEAD)
    assert np.isfinite(two).all()
    assert np.array_equal(two, one.float().numpy())           # the split changes nothing
    ref = O.layer_forward(inp["X"].double().numpy(), *[t.double().numpy() for t in inp["theta"]],
                          inp["W1_0"].numpy(), inp["W2_0"].numpy(), ETA, B, "bidir",
                          alpha_f=inp["alpha_f"].numpy(), alpha_r=inp["alpha_r"].numpy(), per_head=False)["Y"]
    err = np.abs(two - ref).max() / np.abs(ref).max()
    assert err < 1e-2, err                                    # bf16 increment and bf16 Y


@pytest.mark.parametrize("world", [1, 2, 4])
def test_head_ranges_tile_the_heads(world):
    got = [shard.head_range(48, r, world) for r in range(world)]
    assert got[0][0] == 0 and all(hn == 48 // world for _, hn in got)
    assert all(got[r][0] + got[r][1] == got[r + 1][0] for r in range(world - 1))
    assert got[-1][0] + got[-1][1] == 48


def test_uneven_or_bad_ranks_are_refused():
    with pytest.raises(ValueError):
        shard.head_range(48, 0, 5)
    with pytest.raises(ValueError):
        shard.head_range(48, 2, 2)
