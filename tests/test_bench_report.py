"""Host logic of the benchmark's report (no GPU): algorithmic work and the JSON line's shape for
the prefill and decode workloads."""
import types

import pytest

import bench
import synthetic


def _args(**kw):
    d = dict(seed=0, steps=10, warmup=3, stage="all", no_cpu_baseline=True, cpu_budget=1.0)
    d.update(kw)
    return types.SimpleNamespace(**d)


def _res(launches):
    return dict(total_ms=20.0, idx_ms=[1.2] * 10, att_ms=[0.8] * 10, clocks=None, e2e=None,
                launches_per_step=launches)


def test_decode_work_follows_the_seeded_lengths():
    cfg = synthetic.config("decode")
    lens = [int(x) for x in synthetic.lengths(cfg, 0)]
    w = bench._work(cfg, 0)
    # the decode query sits at position len-1 and scores every cached key 0..len-1
    assert w["pairs"] == sum(lens)
    assert w["sel_rows"] == sum(min(cfg.topk, n) for n in lens)
    assert w["indexer_flop"] == sum(lens) * 2 * 64 * 128
    # keys are read once: 128 code bytes and a 4-byte scale each, plus the query side and idx
    assert w["indexer_bytes"] == sum(lens) * 132 + cfg.batch * (64 * 130 + 4 + cfg.topk * 4)
    assert w["attn_bytes"] == w["sel_rows"] * 1152 + cfg.batch * (128 * (1088 * 2 + 4) + cfg.topk * 4)


def test_prefill_work_is_the_causal_count():
    cfg = synthetic.config("prefill_4k")
    w = bench._work(cfg, 0)
    L, k = 4096, 2048
    assert w["pairs"] == L * (L + 1) // 2
    assert w["sel_rows"] == k * (k + 1) // 2 + (L - k) * k


def test_decode_line_is_hbm_bound_in_sequences_per_second():
    cfg = synthetic.config("decode")
    line = bench.report(_args(), cfg, _res(3), 1)
    assert line["unit"] == "sequences/s" and line["metric"].startswith("DSA decode")
    assert line["value"] == pytest.approx(64 * 10 / 0.020)
    assert line["gpu_launches"] == 30
    for st in line["stages"].values():
        assert st["bound"] == "hbm" and st["unit"] == "GB/s"
        assert st["frac"] == pytest.approx(st["achieved"] / st["peak"])
    assert line["roofline"]["kernel"] == "indexer_topk"


def test_other_prefill_workloads_name_their_own_sizes():
    cfg = synthetic.config("prefill_4k")
    line = bench.report(_args(), cfg, _res(2), 1)
    assert line["metric"] == "DSA prefill query-tokens/s (indexer+top-k+sparse MLA) at L=4096, k=2048"
    assert line["unit"] == "query-tokens/s"


def test_prefill_line_keeps_the_headline_metric():
    cfg = synthetic.config("prefill_128k")
    line = bench.report(_args(), cfg, _res(2), 1)
    assert line["metric"] == bench.METRIC and line["unit"] == "query-tokens/s"
    assert line["stages"]["indexer_topk"]["bound"] == "tensor"
    assert line["gpu_launches"] == 20


def test_rank_row_work_sums_to_the_sequence():
    from sparse_attention_long_indexer_b200 import shard
    cfg = synthetic.config("prefill_32k")
    parts = shard.row_partition(cfg.n_q, 3, cfg.topk)
    whole = bench._work(cfg, 0)
    per = [bench._work_rows(cfg, r0, r1) for r0, r1 in parts]
    for key in ("pairs", "sel_rows", "indexer_flop", "attn_flop"):
        assert sum(w[key] for w in per) == whole[key]


def test_row_sharded_line_is_strong_scaling_over_the_whole_sequence():
    from sparse_attention_long_indexer_b200 import shard
    cfg = synthetic.config("prefill_128k")
    parts = shard.row_partition(cfg.n_q, 4, cfg.topk)
    res = dict(_res(2), gather_ms=[0.4] * 10, shard={"parts": parts, "rank0_rows": parts[0]})
    line = bench.report(_args(), cfg, res, 4)
    assert line["scaling"] == "strong" and line["n_gpus"] == 4
    # one sequence per step over the slowest rank's time, not four
    assert line["value"] == pytest.approx(cfg.n_q * 10 / 0.020)
    assert line["stages"]["allgather"]["bytes"] == cfg.max_len * (128 + 4 + 576 * 2)
    w0 = bench._work_rows(cfg, *parts[0])
    assert line["stages"]["indexer_topk"]["achieved"] == pytest.approx(w0["indexer_flop"] / 1.2e-3 / 1e12)


def test_torchrun_command_runs_this_bench_as_n_local_ranks():
    cmd = bench.torchrun_command(4, ["--gpus", "4", "--steps", "3"], 29512)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd and "--master-port=29512" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"] and cmd[-5].endswith("bench.py")


def test_gpus_2_spawns_two_ranks_with_their_environment():
    # `bench.py --gpus 2` outside torchrun relaunches itself as two ranks; --print-ranks makes each
    # rank report its environment and exit before touching a GPU
    import json
    import os
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.abspath(bench.__file__), "--gpus", "2", "--print-ranks"],
                         capture_output=True, text=True, timeout=240, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    ranks = [json.loads(line) for line in out.stdout.splitlines() if line.startswith("{")]
    assert sorted(r["RANK"] for r in ranks) == ["0", "1"]
    assert all(r["WORLD_SIZE"] == "2" and r["MASTER_ADDR"] == "127.0.0.1" for r in ranks)
    assert sorted(r["LOCAL_RANK"] for r in ranks) == ["0", "1"]
