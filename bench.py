#!/usr/bin/env python
"""Benchmark of the DSA forward path (lightning indexer + top-k + sparse MLA attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill_128k] [--impl ours|reference]

One step = the whole hot path over one 128K-token causal prefill (B=1, L=131072, H_I=64,
d_I=128 FP8, H=128, d_qk=576, d_v=512, k=2048), inputs resident in HBM, timed with CUDA
events on the launching stream; metric = query-tokens/s. Under torchrun each rank runs its
own independent sequence (weak scaling, no collective on the data path); timing is the max
over ranks. Prints one JSON line on rank 0.

--impl reference times the fp64 CPU oracle on a bounded sample of the same workload (rank 0
only; other ranks exit 0 without work).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synthetic  # noqa: E402

METRIC = "DSA prefill query-tokens/s (indexer+top-k+sparse MLA) at 128K ctx, k=2048"
UNIT = "query-tokens/s"
DECODE_METRIC = "DSA decode sequences/s (indexer+top-k+sparse MLA), 64 sequences, len ~ U[4K,128K], k=2048"
DECODE_UNIT = "sequences/s"


def _workload_name(cfg):
    d = cfg.description
    return d if d.startswith(cfg.name + ":") else f"{cfg.name}: {d}"


def _metric(cfg):
    """The headline metric on the 128K prefill; the same quantity, named for its own sizes, on
    the other prefill workloads."""
    if cfg.is_decode:
        return DECODE_METRIC, DECODE_UNIT
    if cfg.name == "prefill_128k":
        return METRIC, UNIT
    return f"DSA prefill query-tokens/s (indexer+top-k+sparse MLA) at L={cfg.max_len}, k={cfg.topk}", UNIT


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def _work(cfg, seed=0):
    """Algorithmic work per launch of each stage.

    Prefill: B causal sequences of length L. Decode: one query per sequence at position
    len_b - 1 over its len_b cached keys (lengths from the seeded generator). The byte counts
    are the compulsory HBM traffic: every input read once, every output written once."""
    B, k = cfg.batch, cfg.topk
    if cfg.is_decode:
        lens = [int(x) for x in synthetic.lengths(cfg, seed)]
        pairs = sum(lens)
        sel_rows = sum(min(k, n) for n in lens)
    else:
        L = cfg.max_len
        pairs = B * L * (L + 1) // 2                              # causal (t, s) pairs, s <= t
        kk = min(k, L)
        sel_rows = B * (kk * (kk + 1) // 2 + (L - kk) * k)        # sum over t of min(k, t+1)
    n_tok = B * cfg.n_q
    keys = pairs if cfg.is_decode else B * cfg.max_len            # keys read once per launch
    return {
        "indexer_flop": pairs * 2 * cfg.n_idx_heads * cfg.idx_dim,                     # FP8 MACs x 2
        "attn_flop": sel_rows * 2 * cfg.n_heads * (cfg.d_qk + cfg.d_v),                 # QK^T + PV
        "attn_gather_bytes": sel_rows * cfg.d_qk * 2,
        "indexer_bytes": keys * (cfg.idx_dim + 4) + n_tok * (cfg.n_idx_heads * (cfg.idx_dim + 2) + 4 + k * 4),
        "attn_bytes": sel_rows * cfg.d_qk * 2 + n_tok * (cfg.n_heads * ((cfg.d_qk + cfg.d_v) * 2 + 4) + k * 4),
        "pairs": pairs, "sel_rows": sel_rows,
    }


def _traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    import hashlib
    src = os.path.join(ROOT, "sparse_attention_long_indexer_b200", "csrc",
                       "indexer_topk.cuh" if kernel == "indexer" else "sparse_mla.cuh")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:12]
    for line in open(path):
        m = re.match(r"\|\s*(\w+)\s*\|\s*(\w+)\s*\|\s*([0-9.eE+]+)\s*\|\s*([0-9a-f]{12})\s*\|", line)
        if m and m.group(1) == kernel and m.group(2) == workload and m.group(4) == sha:
            return float(m.group(3))
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms",
                 "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows)}


# ----------------------------------------------------------------------------- oracle timing (CPU)
def _oracle_rows(cfg, seed, rows, cache=None):
    """Runs the fp64 oracle (full path) on query rows of sequence 0.

    Returns (oracle seconds, BLAS threads, cache); ``cache`` keeps the regenerated keys and
    latent rows of the sequence so later calls only regenerate the per-query inputs."""
    import oracle
    from tests.dsa_cases import u16
    if cache is None:
        kc, ks = synthetic.gen_k_idx(cfg, seed, b=0)
        cache = {"k": (kc.numpy(), ks.numpy()),
                 "kv": u16(synthetic.gen_kv(cfg, seed, b=0, positions=range(0, cfg.max_len)))}
    qc, qs = synthetic.gen_q_idx(cfg, seed, tokens=rows)
    w = synthetic.gen_w(cfg, seed, tokens=rows)
    q = synthetic.gen_q(cfg, seed, tokens=rows)
    t0 = time.perf_counter()
    for j, t in enumerate(rows):
        oracle.dsa_row(qc[j].numpy(), float(qs[j]), u16(w[j]), cache["k"][0], cache["k"][1], u16(q[j]), cache["kv"],
                       t, cfg.topk, cfg.d_v, cfg.softmax_scale)
    dt = time.perf_counter() - t0
    threads = 1
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        pass
    return dt, threads, cache


def _shuffled_rows(cfg, n, seed):
    rows = synthetic.sample_rows(cfg.n_q, n, seed)
    return [rows[i] for i in np.random.default_rng(seed).permutation(len(rows))]


def _oracle_decode(cfg, seed, seqs):
    """Runs the fp64 oracle (full path) on the decode queries of the listed sequences.

    Each sequence's caches (its len_b keys and latent rows) are regenerated first; only the
    oracle itself is timed. Returns (oracle seconds, BLAS threads)."""
    import oracle
    from tests.dsa_cases import u16
    lens = synthetic.lengths(cfg, seed)
    spent, threads = 0.0, 1
    for b in seqs:
        n = int(lens[b])
        kc, ks = synthetic.gen_k_idx(cfg, seed, b=b, s_range=range(0, n))
        kv = u16(synthetic.gen_kv(cfg, seed, b=b, positions=range(0, n)))
        qc, qs = synthetic.gen_q_idx(cfg, seed, tokens=[b * cfg.n_q])
        w = synthetic.gen_w(cfg, seed, tokens=[b * cfg.n_q])
        q = synthetic.gen_q(cfg, seed, tokens=[b * cfg.n_q])
        t0 = time.perf_counter()
        oracle.dsa_row(qc[0].numpy(), float(qs[0]), u16(w[0]), kc.numpy(), ks.numpy(), u16(q[0]), kv, n - 1,
                       cfg.topk, cfg.d_v, cfg.softmax_scale)
        spent += time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        pass
    return spent, threads


def cpu_baseline_decode(cfg, seed, budget_s=20.0):
    order = [int(i) for i in np.random.default_rng(seed + 99).permutation(cfg.batch)]
    t_start = time.perf_counter()
    done, spent, threads = 0, 0.0, 1
    for b in order:
        # cache regeneration (about 3 s per sequence on the host) dominates the wall time, so the
        # sample also stops after twice the oracle budget of wall time
        if spent >= budget_s or (done > 0 and time.perf_counter() - t_start >= 2 * budget_s):
            break
        dt, threads = _oracle_decode(cfg, seed, [b])
        spent += dt
        done += 1
    return {"value": done / spent, "unit": DECODE_UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} seeded random sequences of the decode workload (full path per sequence: fp64 index "
                      f"scores over its len_b cached keys, stable sort, fp64 attention over the k selected rows); "
                      f"{spent:.1f} s of oracle time, {time.perf_counter() - t_start:.1f} s wall incl. cache "
                      f"regeneration"}


def cpu_baseline(cfg, seed, budget_s=20.0):
    rows_all = _shuffled_rows(cfg, 4096, seed + 99)
    t_start = time.perf_counter()
    done, spent, cache, threads = 0, 0.0, None, 1
    i = 0
    while spent < budget_s and i < len(rows_all):
        chunk = rows_all[i:i + 8]
        dt, threads, cache = _oracle_rows(cfg, seed, chunk, cache)
        spent += dt
        done += len(chunk)
        i += 8
    return {"value": done / spent, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} seeded uniformly-random query rows of the {cfg.name} workload (full path per row: "
                      f"fp64 index scores over keys 0..t, stable sort, fp64 attention over the k selected rows); "
                      f"{spent:.1f} s of oracle time, {time.perf_counter() - t_start:.1f} s wall incl. input "
                      f"regeneration"}


# ----------------------------------------------------------------------------- multi-rank helpers
def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own independent sequence (weak scaling)."""
    return seed + rank


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank scalar over the process group (the job's time is its slowest rank)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' query tokens over the slowest rank's time."""
    return tokens_per_rank_step * steps * world / (max_ms / 1e3)


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args, cfg, rank, world, local_rank):
    import sparse_attention_long_indexer_b200 as dsa
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    seed = rank_seed(args.seed, rank)
    do_idx = args.stage in ("all", "indexer")
    do_att = args.stage in ("all", "attention")
    do_loss = args.with_loss
    attn_fn = dsa.dsa_masked_mqa_attn if args.attn_mode == "masked" else dsa.dsa_sparse_mla_attn
    k_idx, k_scale = synthetic.gen_k_idx(cfg, seed, dev)
    if args.chunk_queries:
        # the call for the last C queries of one sequence (n_q = C over the whole key side), as the
        # chunked and row-sharded runs make it; for profiling a long context at a small footprint
        import dataclasses
        toks = range(cfg.max_len - args.chunk_queries, cfg.max_len)
        cfg = dataclasses.replace(cfg, n_q=args.chunk_queries)
        q_idx, q_scale = synthetic.gen_q_idx(cfg, seed, dev, tokens=toks)
        g = {"q_idx": q_idx.view(1, cfg.n_q, cfg.n_idx_heads, cfg.idx_dim), "k_idx": k_idx,
             "w": synthetic.gen_w(cfg, seed, dev, tokens=toks).view(1, cfg.n_q, -1),
             "lengths": synthetic.lengths(cfg, seed).to(dev)}
        if do_att:
            g["q"] = synthetic.gen_q(cfg, seed, dev, tokens=toks).view(1, cfg.n_q, cfg.n_heads, cfg.d_qk)
            g["kv"] = synthetic.gen_kv(cfg, seed, dev)
    else:
        q_idx, q_scale = synthetic.gen_q_idx(cfg, seed, dev)
        g = {"q_idx": q_idx, "k_idx": k_idx, "w": synthetic.gen_w(cfg, seed, dev),
             "lengths": synthetic.lengths(cfg, seed).to(dev)}
        if do_att:
            g["q"] = synthetic.gen_q(cfg, seed, dev)
            g["kv"] = synthetic.gen_kv(cfg, seed, dev)
    scales = torch.cat([q_scale.reshape(-1), k_scale.reshape(-1)]).contiguous()
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk, device=dev)
    idx = torch.empty((cfg.batch, cfg.n_q, cfg.topk), dtype=torch.int32, device=dev)
    if do_att:
        out = torch.empty((cfg.batch, cfg.n_q, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((cfg.batch, cfg.n_q, cfg.n_heads), dtype=torch.float32, device=dev)
    idx_scores = torch.empty((cfg.batch, cfg.n_q, cfg.topk), dtype=torch.float32, device=dev) if do_loss else None
    loss = torch.empty((cfg.batch, cfg.n_q), dtype=torch.float32, device=dev) if do_loss else None
    stream = torch.cuda.current_stream(dev)

    if not do_idx:   # the attention still needs real selections: compute them once, untimed
        dsa.dsa_indexer_topk(dims, g["q_idx"], g["w"], g["k_idx"], scales, g["lengths"], cfg.topk, idx, ws.buf,
                             stream)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if do_idx and do_loss:       # the selection with the index score of every selected entry
            dsa.dsa_indexer_topk_scores(dims, g["q_idx"], g["w"], g["k_idx"], scales, g["lengths"], cfg.topk, idx,
                                        idx_scores, ws.buf, stream)
        elif do_idx:
            dsa.dsa_indexer_topk(dims, g["q_idx"], g["w"], g["k_idx"], scales, g["lengths"], cfg.topk, idx, ws.buf,
                                 stream)
        if ev is not None:
            ev[1].record(stream)
        if do_att:
            attn_fn(dims, g["q"], g["kv"], idx, cfg.topk, out, lse, ws.buf, stream)
        if ev is not None:
            ev[2].record(stream)
        if do_loss:
            dsa.dsa_indexer_kl_loss(dims, g["q"], g["kv"], idx, idx_scores, lse, cfg.topk, loss, ws.buf, stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    ws.check()

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    end.record(stream)
    barrier()
    clocks = sampler.stop() if sampler else None
    ws.check()
    total_ms = start.elapsed_time(end)
    idx_ms = [e[0].elapsed_time(e[1]) for e in evs]
    att_ms = [e[1].elapsed_time(e[2]) for e in evs]
    loss_ms = [e[2].elapsed_time(e[3]) for e in evs] if do_loss else None
    total_ms = max_over_ranks(total_ms, dev)

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, cfg, dsa, dims, g, scales, ws, dev, stream, world)
    # kernels per step: the indexer is one launch (decode: scoring kernel + row select, or + merge), the
    # attention one;
    # dims other than the production ones add the copies into padded layouts (3 before the
    # indexer; 2 before and 2 after the attention)
    padded = (cfg.n_idx_heads, cfg.idx_dim, cfg.n_heads, cfg.d_latent, cfg.d_rope) != (64, 128, 128, 512, 64)
    # a prefill whose items reach the indexer's sampled threshold adds its exact pass (a second
    # launch of the same kernel over the items, if any, whose sampled threshold failed)
    sampled = (not cfg.is_decode) and cfg.topk >= 1024 and cfg.max_len >= 64 * 128
    idx_launches = 2 if cfg.is_decode else (2 if sampled else 1)
    att_launches = (2 if args.attn_mode == "masked" else 1) + (4 if padded else 0)     # masked: bitmap kernel
    launches = ((idx_launches + (3 if padded else 0)) * int(do_idx) + att_launches * int(do_att) +
                (1 + (2 if padded else 0)) * int(do_loss))
    return dict(total_ms=total_ms, idx_ms=idx_ms, att_ms=att_ms, loss_ms=loss_ms, clocks=clocks, e2e=e2e,
                launches_per_step=launches)




def _work_rows(cfg, r0, r1):
    """Algorithmic work of query rows [r0, r1) of one causal prefill sequence."""
    k = cfg.topk

    def sel(t):                                                  # sum over u < t of min(k, u + 1)
        return t * (t + 1) // 2 if t <= k else k * (k + 1) // 2 + (t - k) * k
    pairs = r1 * (r1 + 1) // 2 - r0 * (r0 + 1) // 2
    sel_rows = sel(r1) - sel(r0)
    return {"indexer_flop": pairs * 2 * cfg.n_idx_heads * cfg.idx_dim,
            "attn_flop": sel_rows * 2 * cfg.n_heads * (cfg.d_qk + cfg.d_v),
            "attn_gather_bytes": sel_rows * cfg.d_qk * 2, "pairs": pairs, "sel_rows": sel_rows}


def run_sharded(args, cfg, rank, world, local_rank):
    """One sequence's query rows split over the ranks (strong scaling).

    Every rank draws the same sequence. It generates only its own rows' query-side inputs and
    its own tokens' key-side cache rows. The timed step is the all-gather of the key side, then
    the rank's indexer and attention calls on its rows as one chunk (n_q = r1 - r0, lengths =
    r1)."""
    import sparse_attention_long_indexer_b200 as dsa
    from sparse_attention_long_indexer_b200 import shard
    import dataclasses
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    seed = args.seed
    L = cfg.max_len
    parts = shard.row_partition(L, world, cfg.topk)
    c = shard.chunk_call(parts, rank)
    r0, r1 = parts[rank]
    rows = range(r0, r1)
    step_q = 8192
    qc, qs = [], []
    for a in range(r0, r1, step_q):                      # the query codes in bounded pieces
        x, y = synthetic.gen_q_idx(cfg, seed, dev, tokens=range(a, min(r1, a + step_q)))
        qc.append(x)
        qs.append(y)
    q_idx = torch.cat(qc) if qc else torch.empty((0, cfg.n_idx_heads, cfg.idx_dim), dtype=torch.uint8, device=dev)
    q_scale = torch.cat(qs) if qs else torch.empty((0,), dtype=torch.float32, device=dev)
    w = synthetic.gen_w(cfg, seed, dev, tokens=rows)
    q = synthetic.gen_q(cfg, seed, dev, tokens=rows)
    k_loc, ks_loc = synthetic.gen_k_idx(cfg, seed, dev, b=0, s_range=rows)
    kv_loc = synthetic.gen_kv(cfg, seed, dev, b=0, positions=rows)
    ccfg = dataclasses.replace(cfg, n_q=c.n_q)
    dims = dsa.dims_for(ccfg)
    ws = dsa.Workspace.create(dims, cfg.topk, device=dev)
    lengths = torch.tensor([c.length], dtype=torch.int32, device=dev)
    idx = torch.empty((1, c.n_q, cfg.topk), dtype=torch.int32, device=dev)
    out = torch.empty((1, c.n_q, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, c.n_q, cfg.n_heads), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        k_full = shard.all_gather_rows(k_loc, parts).view(1, L, cfg.idx_dim)
        ks_full = shard.all_gather_rows(ks_loc, parts)
        kv_full = shard.all_gather_rows(kv_loc, parts).view(1, L, cfg.d_qk)
        scales = torch.cat([q_scale, ks_full])
        if ev is not None:
            ev[1].record(stream)
        dsa.dsa_indexer_topk(dims, q_idx, w, k_full, scales, lengths, cfg.topk, idx, ws.buf, stream)
        if ev is not None:
            ev[2].record(stream)
        dsa.dsa_sparse_mla_attn(dims, q, kv_full, idx, cfg.topk, out, lse, ws.buf, stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    ws.check()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    end.record(stream)
    torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    ws.check()
    total_ms = max_over_ranks(start.elapsed_time(end), dev)
    return dict(total_ms=total_ms, gather_ms=[e[0].elapsed_time(e[1]) for e in evs],
                idx_ms=[e[1].elapsed_time(e[2]) for e in evs], att_ms=[e[2].elapsed_time(e[3]) for e in evs],
                clocks=clocks, e2e=None, launches_per_step=2, shard={"parts": parts, "rank0_rows": parts[0]})


def run_e2e_whole(args, cfg, dsa, dims, g, scales, ws, dev, stream, world):
    """Same step, inputs copied from pinned host memory and results read back every step, as one call."""
    names = ["q_idx", "w", "k_idx", "q", "kv", "lengths"]
    try:
        host = {k: torch.empty(g[k].shape, dtype=g[k].dtype, pin_memory=True) for k in names}
        host_scales = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
        host_out = torch.empty((cfg.batch, cfg.n_q, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, pin_memory=True)
        host_lse = torch.empty((cfg.batch, cfg.n_q, cfg.n_heads), dtype=torch.float32, pin_memory=True)
        host_idx = torch.empty((cfg.batch, cfg.n_q, cfg.topk), dtype=torch.int32, pin_memory=True)
        pinned = True
    except RuntimeError:
        return {"value": None, "unit": UNIT, "note": "pinned host allocation failed"}
    for k in names:
        host[k].copy_(g[k])
    host_scales.copy_(scales)
    dev_in = {k: torch.empty_like(g[k]) for k in names}
    dev_scales = torch.empty_like(scales)
    out = torch.empty(host_out.shape, dtype=host_out.dtype, device=dev)
    lse = torch.empty(host_lse.shape, dtype=host_lse.dtype, device=dev)
    idx = torch.empty(host_idx.shape, dtype=host_idx.dtype, device=dev)
    h2d = sum(host[k].numel() * host[k].element_size() for k in names) + host_scales.numel() * 4
    d2h = host_out.numel() * 2 + host_lse.numel() * 4 + host_idx.numel() * 4

    def step():
        for k in names:
            dev_in[k].copy_(host[k], non_blocking=True)
        dev_scales.copy_(host_scales, non_blocking=True)
        dsa.dsa_forward(dims, dev_in["q_idx"], dev_in["w"], dev_in["k_idx"], dev_scales, dev_in["lengths"],
                        cfg.topk, dev_in["q"], dev_in["kv"], idx, out, lse, ws.buf, stream)
        host_out.copy_(out, non_blocking=True)
        host_lse.copy_(lse, non_blocking=True)
        host_idx.copy_(idx, non_blocking=True)

    steps = max(1, min(args.steps, args.e2e_steps))
    step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(a.elapsed_time(b), dev)
    ws.check()
    return {"value": aggregate_value(cfg.batch * cfg.n_q, steps, world, ms), "unit": UNIT, "steps": steps,
            "ms_per_step": ms / steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pinned": pinned}


def run_e2e_decode(args, cfg, dsa, dims, g, scales, ws, dev, stream, world):
    """A decode step end to end through the public API, as a serving loop runs it: the caches
    (indexer keys, their scales and the latent rows) stay resident on the device; every step
    uploads the new queries' inputs and the lengths from pinned host memory and reads back out,
    lse and idx. Successive steps are independent request batches, so they pipeline: a step's
    inputs go up on a copy stream while the step before computes and the one before that comes
    back on a second copy stream, through a ring of device buffers. Appending the new token's own
    cache rows belongs to the caller's cache management and is not part of this path."""
    B = cfg.batch
    q_side = ["q_idx", "w", "q", "lengths"]
    NS = 3                                               # device buffer slots
    try:
        host = {n: torch.empty(g[n].shape, dtype=g[n].dtype, pin_memory=True) for n in q_side}
        host_qs = torch.empty((B * cfg.n_q,), dtype=torch.float32, pin_memory=True)
        host_out = torch.empty((B, cfg.n_q, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, pin_memory=True)
        host_lse = torch.empty((B, cfg.n_q, cfg.n_heads), dtype=torch.float32, pin_memory=True)
        host_idx = torch.empty((B, cfg.n_q, cfg.topk), dtype=torch.int32, pin_memory=True)
    except RuntimeError:
        return {"value": None, "unit": DECODE_UNIT, "note": "pinned host allocation failed"}
    for n in q_side:
        host[n].copy_(g[n])
    host_qs.copy_(scales[:B * cfg.n_q])
    # per slot: the query side, the scales (key scales resident, query scales rewritten per step)
    # and the outputs
    slot = [dict({n: torch.empty_like(g[n]) for n in q_side}, scales=scales.clone(),
                 out=torch.empty(host_out.shape, dtype=host_out.dtype, device=dev),
                 lse=torch.empty(host_lse.shape, dtype=host_lse.dtype, device=dev),
                 idx=torch.empty(host_idx.shape, dtype=host_idx.dtype, device=dev)) for _ in range(NS)]
    h2d = sum(host[n].numel() * host[n].element_size() for n in q_side) + host_qs.numel() * 4
    d2h = host_out.numel() * 2 + host_lse.numel() * 4 + host_idx.numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    prev = {"comp": [None] * NS, "d2h": [None] * NS, "n": 0}

    def step():
        sl = prev["n"] % NS
        prev["n"] += 1
        bufs = slot[sl]
        with torch.cuda.stream(s_in):
            if prev["comp"][sl] is not None:
                s_in.wait_event(prev["comp"][sl])          # the slot's inputs are no longer read
            for n in q_side:
                bufs[n].copy_(host[n], non_blocking=True)
            bufs["scales"][:B * cfg.n_q].copy_(host_qs, non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(s_in)
        stream.wait_event(ready)
        if prev["d2h"][sl] is not None:
            stream.wait_event(prev["d2h"][sl])             # the slot's outputs have been read back
        dsa.dsa_forward(dims, bufs["q_idx"], bufs["w"], g["k_idx"], bufs["scales"], bufs["lengths"], cfg.topk,
                        bufs["q"], g["kv"], bufs["idx"], bufs["out"], bufs["lse"], ws.buf, stream)
        done = torch.cuda.Event()
        done.record(stream)
        prev["comp"][sl] = done
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            host_out.copy_(bufs["out"], non_blocking=True)
            host_lse.copy_(bufs["lse"], non_blocking=True)
            host_idx.copy_(bufs["idx"], non_blocking=True)
            back = torch.cuda.Event()
            back.record(s_out)
            prev["d2h"][sl] = back

    steps = max(3, args.steps)
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(steps):
        step()
    b.record(s_out)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(a.elapsed_time(b), dev)
    ws.check()
    return {"value": aggregate_value(B * cfg.n_q, steps, world, ms), "unit": DECODE_UNIT, "steps": steps,
            "ms_per_step": ms / steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "pinned": True,
            "caches": "resident on the device (uploaded once, outside the timed region)",
            "streams": "h2d / compute / d2h overlapped across steps (independent request batches)"}


def run_e2e(args, cfg, dsa, dims, g, scales, ws, dev, stream, world):
    """The step end to end through the public API: inputs from pinned host memory, results read back.

    A prefill sequence (B = 1) runs as query chunks so that transfers overlap compute: the key-side
    inputs (k_idx, latent_kv, key scales) go up first, then each chunk's query-side inputs go up on a
    copy stream, its dsa_forward runs on the compute stream and its out, lse and idx come back on a
    second copy stream, through a ring of device buffers. A chunk of queries [i0, i1) is the call with
    n_q = i1 - i0 and lengths = i1, the query positions the header defines; it computes exactly what
    the whole call computes for those queries.
    """
    if cfg.is_decode:
        return run_e2e_decode(args, cfg, dsa, dims, g, scales, ws, dev, stream, world)
    if cfg.batch != 1 or args.e2e_chunk <= 0:
        return run_e2e_whole(args, cfg, dsa, dims, g, scales, ws, dev, stream, world)
    L, H, dv, k = cfg.max_len, cfg.n_heads, cfg.d_v, cfg.topk
    C = min(args.e2e_chunk, cfg.n_q)
    starts = list(range(0, cfg.n_q, C))
    NS = 3                                               # device buffer slots
    q_side = ["q_idx", "w", "q"]
    try:
        host = {n: torch.empty(g[n].shape, dtype=g[n].dtype, pin_memory=True) for n in q_side + ["k_idx", "kv"]}
        host_scales = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
        host_out = torch.empty((1, cfg.n_q, H, dv), dtype=torch.bfloat16, pin_memory=True)
        host_lse = torch.empty((1, cfg.n_q, H), dtype=torch.float32, pin_memory=True)
        host_idx = torch.empty((1, cfg.n_q, k), dtype=torch.int32, pin_memory=True)
    except RuntimeError:
        return {"value": None, "unit": UNIT, "note": "pinned host allocation failed"}
    for n in host:
        host[n].copy_(g[n])
    host_scales.copy_(scales)
    nq = cfg.n_q
    # device: key side once, query side and outputs per slot
    d_kidx, d_kv = torch.empty_like(g["k_idx"]), torch.empty_like(g["kv"])
    d_kscale = torch.empty(L, dtype=torch.float32, device=dev)
    # query-side tensors as [n_q, row] (B = 1): a chunk is a row range
    hrow = {n: host[n].view(nq, -1) for n in q_side}
    slot = [dict({n: torch.empty((C, hrow[n].shape[1]), dtype=hrow[n].dtype, device=dev) for n in q_side},
                 scales=torch.empty(C + L, dtype=torch.float32, device=dev),
                 out=torch.empty((C, H * dv), dtype=torch.bfloat16, device=dev),
                 lse=torch.empty((C, H), dtype=torch.float32, device=dev),
                 idx=torch.empty((C, k), dtype=torch.int32, device=dev)) for _ in range(NS)]
    hout, hlse, hidx = host_out.view(nq, -1), host_lse.view(nq, -1), host_idx.view(nq, -1)
    ends = torch.tensor([min(i0 + C, nq) + (L - nq) for i0 in starts], dtype=torch.int32, device=dev)
    chunk_dims = {}
    for i0 in starts:
        c = min(C, nq - i0)
        if c not in chunk_dims:
            chunk_dims[c] = dsa.make_dims(1, c, L, cfg.n_idx_heads, cfg.idx_dim, H, cfg.d_latent, cfg.d_rope,
                                          cfg.softmax_scale)
    ws_c = dsa.Workspace.create(chunk_dims[C], k, device=dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d = (sum(host[n].numel() * host[n].element_size() for n in host) + host_scales.numel() * 4)
    d2h = host_out.numel() * 2 + host_lse.numel() * 4 + host_idx.numel() * 4

    def ev():
        return torch.cuda.Event()

    prev = {"keys_free": None, "comp": [None] * NS, "d2h": [None] * NS}

    def step():
        with torch.cuda.stream(s_in):
            if prev["keys_free"] is not None:
                s_in.wait_event(prev["keys_free"])
            d_kidx.copy_(host["k_idx"], non_blocking=True)
            d_kv.copy_(host["kv"], non_blocking=True)
            d_kscale.copy_(host_scales[nq:], non_blocking=True)
        last = None
        for ci, i0 in enumerate(starts):
            c, sl = min(C, nq - i0), ci % NS
            bufs = slot[sl]
            with torch.cuda.stream(s_in):
                if prev["comp"][sl] is not None:
                    s_in.wait_event(prev["comp"][sl])      # the slot's inputs are no longer read
                for n in q_side:
                    bufs[n][:c].copy_(hrow[n][i0:i0 + c], non_blocking=True)
                bufs["scales"][:c].copy_(host_scales[i0:i0 + c], non_blocking=True)
                bufs["scales"][c:c + L].copy_(d_kscale, non_blocking=True)
                ready = ev()
                ready.record(s_in)
            stream.wait_event(ready)
            if prev["d2h"][sl] is not None:
                stream.wait_event(prev["d2h"][sl])         # the slot's outputs have been read back
            dsa.dsa_forward(chunk_dims[c], bufs["q_idx"][:c], bufs["w"][:c], d_kidx, bufs["scales"][:c + L],
                            ends[ci:ci + 1], k, bufs["q"][:c], d_kv, bufs["idx"][:c], bufs["out"][:c],
                            bufs["lse"][:c], ws_c.buf, stream)
            done = ev()
            done.record(stream)
            prev["comp"][sl] = done
            last = done
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                hout[i0:i0 + c].copy_(bufs["out"][:c], non_blocking=True)
                hlse[i0:i0 + c].copy_(bufs["lse"][:c], non_blocking=True)
                hidx[i0:i0 + c].copy_(bufs["idx"][:c], non_blocking=True)
                back = ev()
                back.record(s_out)
                prev["d2h"][sl] = back
        prev["keys_free"] = last

    steps = max(1, min(args.steps, args.e2e_steps))
    step()
    torch.cuda.synchronize(dev)
    ws_c.check()
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(steps):
        step()
    b.record(s_out)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(a.elapsed_time(b), dev)
    ws_c.check()
    return {"value": aggregate_value(cfg.batch * cfg.n_q, steps, world, ms), "unit": UNIT, "steps": steps,
            "ms_per_step": ms / steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "pinned": True,
            "chunk_queries": C, "streams": "h2d / compute / d2h overlapped"}


def torchrun_command(n: int, argv, port: int):
    """The command that runs bench.py with ``argv`` as n ranks on this node (127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def relaunch_under_torchrun(n: int, argv) -> int:
    cmd = torchrun_command(n, argv, _free_port())
    # the ranks' process group times out well before this last bound
    return subprocess.call(["timeout", "-k", "60", "3600", *cmd])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 10; decode: 1000, so clocks are sampled during the timed region)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_128k", choices=["tiny", "prefill_4k", "prefill_32k", "prefill_128k", "decode"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--print-ranks", action="store_true",
                    help="print each rank's RANK/LOCAL_RANK/WORLD_SIZE as JSON and exit (checks the launch)")
    ap.add_argument("--e2e-chunk", type=int, default=4096,
                    help="queries per dsa_forward call in the e2e measurement (0 = one call per step)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--stage", default="all", choices=["all", "indexer", "attention"],
                    help="time one stage only (profiling); the line then reports that stage")
    ap.add_argument("--seq-len", type=int, default=0, help="override L of a prefill workload (profiling)")
    ap.add_argument("--chunk-queries", type=int, default=0,
                    help="prefill: time the call for the last N queries only (profiling a long context small)")
    ap.add_argument("--attn-mode", default="sparse", choices=["sparse", "masked"],
                    help="attention stage: the sparse kernel, or the masked dense mode (max_len <= 16384)")
    ap.add_argument("--with-loss", action="store_true",
                    help="the step also computes the indexer-alignment KL loss (selection with scores, attention, "
                         "loss)")
    ap.add_argument("--shard", default="sequences", choices=["sequences", "rows"],
                    help="N>1: one sequence per rank (weak scaling), or one sequence's query rows split over "
                         "the ranks with an all-gather of the key-side caches per step (strong scaling)")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: run this same command under torchrun
        return relaunch_under_torchrun(args.gpus, sys.argv[1:])
    if args.print_ranks:
        print(json.dumps({k: os.environ.get(k) for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR")}),
              flush=True)
        return 0
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    cfg = synthetic.config(args.workload)
    if args.steps is None:
        args.steps = 1000 if cfg.is_decode and args.impl == "ours" else 10
    if args.seq_len:
        import dataclasses
        cfg = dataclasses.replace(cfg, n_q=args.seq_len, max_len=args.seq_len, name=f"prefill_L{args.seq_len}",
                                  description=f"causal prefill L={args.seq_len}, k=2048")
    if args.stage != "all" or args.with_loss or args.attn_mode != "sparse" or args.chunk_queries:
        args.no_e2e = True
        args.no_cpu_baseline = True
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, cfg, world)

    sharded = args.shard == "rows" and not cfg.is_decode
    if world > 1 or sharded:
        import datetime
        if world == 1:                                   # a one-rank group runs the same sharded code
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(_free_port()))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    res = run_sharded(args, cfg, rank, world, local_rank) if sharded else run_ours(args, cfg, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(report(args, cfg, res, world)), flush=True)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def report(args, cfg, res, world):
    peaks = _peaks()
    sh = res.get("shard")
    # row sharding: rank 0's rows set the per-stage work (the job's time is the slowest rank's)
    if sh:
        w = _work_rows(cfg, *sh["rank0_rows"])
    elif getattr(args, "chunk_queries", 0):
        w = _work_rows(cfg, cfg.max_len - args.chunk_queries, cfg.max_len)
    else:
        w = _work(cfg, rank_seed(args.seed, 0))
    metric, unit = _metric(cfg)
    ms_step = res["total_ms"] / args.steps
    idx_ms = statistics.mean(res["idx_ms"])
    att_ms = statistics.mean(res["att_ms"])
    fp8_peak = 2.0 * peaks["bf16_sustained"]          # nominal fp8:bf16 ratio 2 (4.5 : 2.25 PF)
    stages = {}
    if cfg.is_decode:
        # one query per sequence: both stages stream their inputs once, so HBM bounds them
        hbm = {"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s", "peak_note": f"{peaks['source']} HBM copy"}
        if args.stage in ("all", "indexer"):
            stages["indexer_topk"] = dict(hbm, ms=idx_ms, us=idx_ms * 1e3,
                                          achieved=w["indexer_bytes"] / (idx_ms / 1e3) / 1e9,
                                          bytes=w["indexer_bytes"],
                                          tflops_fp8=w["indexer_flop"] / (idx_ms / 1e3) / 1e12)
        if args.stage in ("all", "attention"):
            stages["sparse_mla_attn"] = dict(hbm, ms=att_ms, us=att_ms * 1e3,
                                             achieved=w["attn_bytes"] / (att_ms / 1e3) / 1e9,
                                             bytes=w["attn_bytes"],
                                             tflops_bf16=w["attn_flop"] / (att_ms / 1e3) / 1e12)
    else:
        if args.stage in ("all", "indexer"):
            stages["indexer_topk"] = {"ms": idx_ms, "bound": "tensor",
                                      "achieved": w["indexer_flop"] / (idx_ms / 1e3) / 1e12, "peak": fp8_peak,
                                      "unit": "TFLOP/s",
                                      "peak_note": f"fp8 = 2 x {peaks['source']} sustained bf16 "
                                                   f"{peaks['bf16_sustained']}"}
        if args.stage in ("all", "attention"):
            stages["sparse_mla_attn"] = {"ms": att_ms, "bound": "tensor",
                                         "achieved": w["attn_flop"] / (att_ms / 1e3) / 1e12,
                                         "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
                                         "peak_note": f"{peaks['source']} sustained bf16",
                                         "gather_GBps": w["attn_gather_bytes"] / (att_ms / 1e3) / 1e9}
            if getattr(args, "attn_mode", "sparse") == "masked":
                stages["sparse_mla_attn"]["mode"] = ("masked dense (whole 64-row blocks of each causal prefix; "
                                                     "work counted over the selected rows only)")
    if res.get("loss_ms"):
        # indexer-alignment loss: the logits of every selected row again (2 x 128 heads x 576 dims per row)
        # plus the gather of its latent row; bf16 tensor-bound in principle, like the attention's logits half
        loss_ms = statistics.mean(res["loss_ms"])
        stages["indexer_kl_loss"] = {"ms": loss_ms, "bound": "tensor",
                                     "achieved": w["sel_rows"] * 2 * cfg.n_heads * cfg.d_qk / (loss_ms / 1e3) / 1e12,
                                     "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
                                     "peak_note": f"{peaks['source']} sustained bf16",
                                     "gather_GBps": w["attn_gather_bytes"] / (loss_ms / 1e3) / 1e9}
    for k, st in stages.items():
        st["frac"] = st["achieved"] / st["peak"]
    dom = max(stages, key=lambda k: stages[k]["ms"])
    ds = stages[dom]
    roofline = {"kernel": dom, "bound": ds["bound"], "achieved": ds["achieved"], "peak": ds["peak"],
                "unit": ds["unit"], "frac": ds["frac"],
                "traffic": _traffic("indexer" if dom == "indexer_topk" else "attention", cfg.name)}
    if cfg.is_decode:
        lo, hi = cfg.len_range
        conf = {"workload": f"{cfg.description}; H_I={cfg.n_idx_heads} d_I={cfg.idx_dim} FP8 e4m3, "
                            f"H={cfg.n_heads}, d_qk={cfg.d_qk}, d_v={cfg.d_v}, bf16",
                "global_batch": cfg.batch * world, "seq_len": cfg.max_len, "lengths": f"U[{lo},{hi}] (seeded)",
                "topk": cfg.topk,
                "parallelism": f"{world} x {cfg.batch} independent sequences, one group per GPU (no data-path "
                               f"collective)",
                "l2": "caches larger than L2 (latent rows alone are %.1f GB)"
                      % (cfg.batch * cfg.max_len * cfg.d_qk * 2 / 1e9)}
    else:
        conf = {"workload": f"{cfg.name}: {cfg.description}; H_I={cfg.n_idx_heads} d_I={cfg.idx_dim} FP8 e4m3, "
                            f"H={cfg.n_heads}, d_qk={cfg.d_qk}, d_v={cfg.d_v}, bf16",
                "global_batch": cfg.batch * world, "seq_len": cfg.max_len, "topk": cfg.topk,
                "parallelism": f"{world} independent sequences, one per GPU (no data-path collective)",
                "l2": "inputs larger than L2 (q alone is %.1f GB)" % (cfg.n_q * cfg.n_heads * cfg.d_qk * 2 / 1e9)}
    if sh:
        value = cfg.batch * cfg.n_q * args.steps / (res["total_ms"] / 1e3)      # one sequence per step
        sizes = [r1 - r0 for r0, r1 in sh["parts"]]
        conf["global_batch"] = cfg.batch
        conf["parallelism"] = (f"query rows of one sequence over {world} GPUs (rows per rank {sizes}, balanced by "
                               f"causal work); one all-gather of the key-side caches per step")
        key_bytes = cfg.max_len * (cfg.idx_dim + 4 + cfg.d_qk * 2)
        stages["allgather"] = {"ms": statistics.mean(res["gather_ms"]), "bytes": key_bytes,
                               "note": "rank 0's view; every rank receives the whole key side"}
    else:
        n_tok = getattr(args, "chunk_queries", 0) or cfg.batch * cfg.n_q
        value = aggregate_value(n_tok, args.steps, world, res["total_ms"])
        if getattr(args, "chunk_queries", 0):
            conf["workload"] += f" -- the call for its last {args.chunk_queries} queries only"
    line = {
        "metric": metric, "value": value,
        "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong" if sh else "weak", "vs_baseline": None,
        "dtype": "fp8e4m3+bf16 (fp32 accumulate)",
        "data": "synthetic", "config": conf,
        "roofline": roofline, "stages": stages,
        "gpu_launches": res.get("launches_per_step", len(stages)) * args.steps,
        "clocks": res["clocks"], "e2e": res["e2e"],
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = (cpu_baseline_decode if cfg.is_decode else cpu_baseline)(cfg, args.seed,
                                                                                         args.cpu_budget)
    return line


def run_reference(args, cfg, world):
    """The fp64 oracle as the reference arm: each step is a bounded sample of the workload."""
    metric, unit = _metric(cfg)
    total, threads = 0.0, 1
    if cfg.is_decode:
        order = [int(i) for i in np.random.default_rng(args.seed + 7).permutation(cfg.batch)]
        per_step = 1
        pos = 0
        for _ in range(args.warmup):
            _oracle_decode(cfg, args.seed, order[pos % cfg.batch:pos % cfg.batch + 1])
            pos += 1
        for _ in range(args.steps):
            dt, threads = _oracle_decode(cfg, args.seed, order[pos % cfg.batch:pos % cfg.batch + 1])
            total += dt
            pos += 1
        sample = (f"{per_step} seeded random sequence per step of the {cfg.name} workload, full path (fp64 index "
                  f"scores over its cached keys, stable sort, fp64 attention)")
    else:
        rows_all = _shuffled_rows(cfg, 100000, args.seed + 7)
        per_step = 4
        cache = None
        pos = 0
        for _ in range(args.warmup):
            _, _, cache = _oracle_rows(cfg, args.seed, rows_all[pos:pos + per_step], cache)
            pos += per_step
        for _ in range(args.steps):
            dt, threads, cache = _oracle_rows(cfg, args.seed, rows_all[pos:pos + per_step], cache)
            total += dt
            pos += per_step
        sample = (f"{per_step} seeded uniformly-random query rows per step of the {cfg.name} workload, full path "
                  f"per row (fp64 index scores, stable sort, fp64 attention)")
    value = per_step * args.steps / total
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": _workload_name(cfg), "global_batch": cfg.batch,
                       "seq_len": cfg.max_len, "topk": cfg.topk, "parallelism": "CPU oracle, rank 0 only"},
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
