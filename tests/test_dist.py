"""Multi-rank host logic of the benchmark (world size 2, gloo on CPU): per-rank independent
inputs, max-over-ranks timing and the whole-job throughput."""
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


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import synthetic
    local_ms = 100.0 + 25.0 * rank                      # rank 1 is the slower one
    worst = bench.max_over_ranks(local_ms, torch.device("cpu"))
    seed = bench.rank_seed(5, rank)
    cfg = synthetic.config("tiny", n_q=16, max_len=16)
    first = synthetic.gen_q_idx(cfg, seed)[0][0, 0, :8].tolist()
    q.put((rank, worst, seed, first))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_weak_scaling_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, s0, f0), (r1, w1, s1, f1) = res
    assert w0 == w1 == 125.0                          # every rank reports the slowest rank's time
    assert s0 != s1 and f0 != f1                      # independent sequences per rank
    import bench
    assert bench.aggregate_value(131072, 10, 2, 125.0) == pytest.approx(131072 * 10 * 2 / 0.125)
