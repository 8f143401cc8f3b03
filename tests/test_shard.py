"""Query-row sharding of one prefill sequence (host logic; the exchange runs as gloo ranks on CPU).

The kernels' side of it, that a chunk call computes exactly the chunk's rows of the whole
call, is `tests/test_parity_gpu.py::test_query_chunks_match_one_call`."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_long_indexer_b200 import shard


@pytest.mark.parametrize("L", [0, 1, 5, 4096, 131072])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_partition_covers_the_rows_in_order_and_balances_the_work(L, world):
    k = 2048
    parts = shard.row_partition(L, world, k)
    assert len(parts) == world and parts[0][0] == 0 and parts[-1][1] == L
    for (a0, a1), (b0, b1) in zip(parts, parts[1:]):
        assert a0 <= a1 == b0 <= b1
    total = shard.cost_prefix(L, k)
    # one row's work is at most the last row's; a part is within one row of its share
    row_max = shard.cost_prefix(L, k) - shard.cost_prefix(max(L - 1, 0), k)
    for r0, r1 in parts:
        work = shard.cost_prefix(r1, k) - shard.cost_prefix(r0, k)
        assert abs(work - total / world) <= row_max + 1e-9 * total


def test_cost_prefix_is_the_row_sum():
    k = 7
    for t in range(0, 40):
        direct = sum((u + 1) * 2.0 + 3.0 * min(u + 1, k) for u in range(t))
        assert shard.cost_prefix(t, k, pair_w=2.0, row_w=3.0) == pytest.approx(direct)


def test_indexer_only_weights_give_the_square_root_split():
    # with attention free, the causal indexer work of rows [0, t) grows as t^2 / 2, so two
    # ranks split at L / sqrt(2)
    L = 1 << 20
    (_, b), _ = shard.row_partition(L, 2, 2048, pair_w=1.0, row_w=0.0)
    assert abs(b - L / 2 ** 0.5) <= 2


def test_later_ranks_get_fewer_rows():
    parts = shard.row_partition(131072, 4, 2048)
    sizes = [r1 - r0 for r0, r1 in parts]
    assert sizes == sorted(sizes, reverse=True) and sizes[0] > sizes[-1]


def test_chunk_call_positions_follow_the_header():
    parts = shard.row_partition(10000, 3, 2048)
    for r, (r0, r1) in enumerate(parts):
        c = shard.chunk_call(parts, r)
        # query i of the chunk sits at position length - n_q + i = r0 + i
        assert (c.row0, c.n_q, c.length) == (r0, r1 - r0, r1)
        assert c.length - c.n_q == c.row0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from sparse_attention_long_indexer_b200 import shard as sh
    L = 1000
    parts = sh.row_partition(L, world, 64)
    full = torch.arange(L * 3, dtype=torch.int32).reshape(L, 3) * 7 + 1        # the reference rows
    kv = torch.randn(L, 5, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    r0, r1 = parts[rank]
    got_i = sh.all_gather_rows(full[r0:r1].clone(), parts)
    got_b = sh.all_gather_rows(kv[r0:r1].clone(), parts)
    q.put((rank, bool(torch.equal(got_i, full)), bool(torch.equal(got_b.view(torch.int16), kv.view(torch.int16))),
           [r1 - r0 for r0, r1 in parts]))
    dist.barrier()
    dist.destroy_process_group()


def test_all_gather_assembles_uneven_row_ranges():
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_i, ok_b, sizes in res:
        assert ok_i and ok_b, rank
        assert len(set(sizes)) > 1                         # the ranges really are uneven
