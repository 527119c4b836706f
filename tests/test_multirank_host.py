"""Host logic of the multi-GPU path on CPU: two gloo ranks run bench.py's
replica bookkeeping (per-rank seeds, max-over-ranks timing, whole-job
throughput).  The layer runs as independent replicas, so no collective
touches the data path; only the timing reduction crosses ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    from test_rnn_layer_b200 import synth as S
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = S.TINY.with_T(32)
        inp = S.make_inputs(w, seed=bench.rank_seed(rank))
        ms = 10.0 + 5.0 * rank                   # the second rank is the slower one
        worst = bench.max_over_ranks(ms, world, torch.device("cpu"))
        value = bench.whole_job_tokens_per_s(world, w.T, worst)
        dist.barrier()
        out[rank] = (worst, value, float(inp["X"].sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replica_bookkeeping():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0                      # max over ranks
    assert res[0][1] == res[1][1] == pytest.approx(2 * 32 / 0.015)
    assert res[0][2] != res[1][2]                              # each replica draws its own sequence


def test_single_rank_bookkeeping_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_tokens_per_s(1, 313344, 200.0) == pytest.approx(313344 / 0.2)


def test_bench_starts_its_own_ranks_and_reports_the_slowest():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself; rank 0
    alone prints the line, with n_gpus 2 and the slower rank's time (the host
    plumbing only: each step sleeps 10 ms x (rank + 1), gloo, no GPU)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--steps", "3", "--warmup", "3", "--dry-run-host",
                        "--workload", "tiny"], capture_output=True, text=True, timeout=240, cwd=root, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["dry_run"] is True
    assert line["ms_per_step"] >= 20.0                       # the second rank sleeps 20 ms per step
    assert line["value"] == pytest.approx(2 * 256 / (line["ms_per_step"] * 1e-3))
