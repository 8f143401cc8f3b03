"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle, on B200.

Index sets: exact except near-ties (oracle score within 1e-3 of the k-th score).
Attention: max-abs 1e-2, relative L2 5e-3, both over the oracle's index sets and over the
GPU's own. Sizes: every row at L=512 and L=4096, seeded samples at 32K and 128K (the
workloads' own shapes), all 64 sequences of the decode batch.
"""
import numpy as np
import pytest
import torch

import synthetic
from tests.dsa_cases import RowOracle, check_selection, compare_attention, report_near_ties

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_long_indexer_b200")


def _inputs(cfg, seed, device="cuda", gen_device=None):
    g = synthetic.gen_all(cfg, seed, gen_device or device)
    return {k: v.to(device) for k, v in g.items()}


def _run_forward(cfg, g, return_idx=True):
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    idx, out, lse = dsa.forward(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"], g["lengths"],
                                cfg.topk, g["q"], g["kv"], ws, return_idx=return_idx)
    torch.cuda.synchronize()
    ws.check()
    return idx, out, lse


def _rows_to_host(t, rows):
    """t[b, i] for the listed (b, i), gathered on the device first, as float64/int numpy."""
    if not rows:
        return np.zeros((0,) + tuple(t.shape[2:]))
    bi = torch.tensor([b for b, _ in rows], device=t.device)
    ii = torch.tensor([i for _, i in rows], device=t.device)
    sel = t[bi, ii]
    return sel.cpu().numpy() if sel.dtype == torch.int32 else sel.double().cpu().numpy()


def _check_rows(cfg, seed, rows, idx, out, lse, ro=None, attn_rows=None, name=None):
    """Selections of ``rows`` against the oracle (near-ties allowed), and the attention of
    ``attn_rows`` (default: all of them) against the oracle's attention over the GPU's own sets.
    Returns {(b, i): the oracle's exact selection} for reuse."""
    ro = ro or RowOracle(cfg, seed)
    idx_h = _rows_to_host(idx, rows)
    stats, sets = [], {}
    for r, (b, i) in enumerate(rows):
        sel_o, scores = ro.indexer(b, i)
        sets[(b, i)] = sel_o
        stats.append(check_selection(idx_h[r], scores, cfg.topk, ro.pos(b, i)))
    report_near_ties(name or cfg.name, len(rows), stats)
    a_rows = [x for x in rows if attn_rows is None or x in attn_rows]
    if a_rows:
        out_h, lse_h = _rows_to_host(out, a_rows), _rows_to_host(lse, a_rows)
        pos = {x: r for r, x in enumerate(rows)}
        ref = [ro.attention(b, i, idx_h[pos[(b, i)]]) for (b, i) in a_rows]
        compare_attention(out_h, lse_h, np.stack([r[0] for r in ref]), np.stack([r[1] for r in ref]))
    return sets


def _attention_on_oracle_sets(cfg, g, sets, ro, out=None, lse=None):
    """The attention kernel fed the oracle's own selections (the other rows select nothing),
    compared with the oracle's attention over the same sets, row by row."""
    idx = torch.full((cfg.batch, cfg.n_q, cfg.topk), -1, dtype=torch.int32)
    for (b, i), s in sets.items():
        idx[b, i, :len(s)] = torch.from_numpy(np.asarray(s, dtype=np.int32))
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    if out is None:
        out, lse = dsa.sparse_mla_attn(dims, g["q"], g["kv"], idx.cuda(), cfg.topk, ws)
    else:                                   # reuse the caller's output buffers (128K: 17 GB)
        dsa.dsa_sparse_mla_attn(dims, g["q"], g["kv"], idx.cuda(), cfg.topk, out, lse, ws.buf)
    torch.cuda.synchronize()
    ws.check()
    rows = sorted(sets)
    ref = [ro.attention(b, i, sets[(b, i)]) for (b, i) in rows]
    compare_attention(_rows_to_host(out, rows), _rows_to_host(lse, rows), np.stack([r[0] for r in ref]),
                      np.stack([r[1] for r in ref]))


# ----------------------------------------------------------------------------- tiny (all rows)
def test_tiny_forward_all_rows():
    cfg = synthetic.config("tiny")
    g = _inputs(cfg, 1, gen_device="cpu")
    idx, out, lse = _run_forward(cfg, g)
    _check_rows(cfg, 1, [(0, i) for i in range(cfg.n_q)], idx, out, lse)


def test_tiny_attention_on_oracle_sets():
    cfg = synthetic.config("tiny")
    g = _inputs(cfg, 2, gen_device="cpu")
    ro = RowOracle(cfg, 2)
    _attention_on_oracle_sets(cfg, g, {(0, i): ro.indexer(0, i)[0] for i in range(cfg.n_q)}, ro)


# ----------------------------------------------------------------------------- 4K (all rows)
def test_prefill_4k_indexer_all_rows_attention_sampled():
    cfg = synthetic.config("prefill_4k")
    g = _inputs(cfg, 3)
    idx, out, lse = _run_forward(cfg, g)
    rows = [(0, i) for i in range(cfg.n_q)]
    attn = set((0, i) for i in synthetic.sample_rows(cfg.n_q, 192, 3, extra=list(range(8)) + [cfg.n_q - 1]))
    _check_rows(cfg, 3, rows, idx, out, lse, attn_rows=attn)


def test_prefill_4k_attention_on_oracle_sets():
    cfg = synthetic.config("prefill_4k")
    g = _inputs(cfg, 4)
    ro = RowOracle(cfg, 4)
    rows = synthetic.sample_rows(cfg.n_q, 96, 4, extra=[0, 1, 2047, 2048, cfg.n_q - 1])
    _attention_on_oracle_sets(cfg, g, {(0, i): ro.indexer(0, i)[0] for i in rows}, ro)


# ----------------------------------------------------------------------------- 32K / 128K (sampled rows)
def test_prefill_32k_sampled_rows():
    """512 seeded rows plus the first and last 64: selections and attention over the GPU's sets,
    then the attention kernel fed the oracle's sets of the same rows."""
    cfg = synthetic.config("prefill_32k")
    g = _inputs(cfg, 5)
    idx, out, lse = _run_forward(cfg, g)
    rows = synthetic.sample_rows(cfg.n_q, 512, 5, extra=list(range(64)) + list(range(cfg.n_q - 64, cfg.n_q)))
    ro = RowOracle(cfg, 5)
    sets = _check_rows(cfg, 5, [(0, i) for i in rows], idx, out, lse, ro=ro)
    _attention_on_oracle_sets(cfg, g, sets, ro, out=out, lse=lse)


def test_prefill_128k_sampled_rows():
    """256 seeded rows (plus the first and last): selections, attention over the GPU's sets and
    over the oracle's sets, at the metric's workload."""
    cfg = synthetic.config("prefill_128k")
    g = _inputs(cfg, 6)
    idx, out, lse = _run_forward(cfg, g)
    rows = synthetic.sample_rows(cfg.n_q, 256, 6, extra=[0, cfg.n_q - 1])
    ro = RowOracle(cfg, 6)
    sets = _check_rows(cfg, 6, [(0, i) for i in rows], idx, out, lse, ro=ro)
    del idx
    _attention_on_oracle_sets(cfg, g, sets, ro, out=out, lse=lse)
    del g, out, lse
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- decode (all sequences)
def test_decode_all_sequences():
    cfg = synthetic.config("decode")
    g = _inputs(cfg, 7)
    idx, out, lse = _run_forward(cfg, g)
    ro = RowOracle(cfg, 7)
    sets = _check_rows(cfg, 7, [(b, 0) for b in range(cfg.batch)], idx, out, lse, ro=ro)
    _attention_on_oracle_sets(cfg, g, sets, ro, out=out, lse=lse)
    del g
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- edge cases
def test_equal_scores_select_the_lowest_positions():
    cfg = synthetic.config("tiny", n_q=300, max_len=300, topk=64)
    g = _inputs(cfg, 8, gen_device="cpu")
    g["w"].zero_()                                   # every index score is exactly 0
    idx, out, lse = _run_forward(cfg, g)
    idx_h = idx.cpu().numpy()[0]
    for i in range(cfg.n_q):
        n = min(cfg.topk, i + 1)
        assert sorted(idx_h[i, :n].tolist()) == list(range(n))
        assert (idx_h[i, n:] == -1).all()


def test_sampled_threshold_falls_back_to_the_exact_pass():
    """Queries long enough for the sampled threshold (>= 64 key tiles). In every other block of
    four queries all index scores are 0 (w = 0): the sample phase then drops candidates that tie
    for their position, so those items must be rerun exactly and keep the lowest 2048
    positions; the other items keep their sampled selection, checked against the oracle."""
    cfg = synthetic.config("prefill_4k", n_q=9000, max_len=9000)
    g = {}
    g["q_idx"], g["q_scale"] = synthetic.gen_q_idx(cfg, 17, "cuda")
    g["k_idx"], g["k_scale"] = synthetic.gen_k_idx(cfg, 17, "cuda")
    g["w"] = synthetic.gen_w(cfg, 17, "cuda")
    zero = torch.arange(cfg.n_q, device="cuda") // 4 % 2 == 0
    g["w"][zero] = 0
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    idx = dsa.indexer_topk(dims, g["q_idx"].view(1, cfg.n_q, cfg.n_idx_heads, cfg.idx_dim),
                           g["w"].view(1, cfg.n_q, -1), g["k_idx"], g["q_scale"], g["k_scale"],
                           synthetic.lengths(cfg, 17).cuda(), cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    idx_h = idx.cpu().numpy()[0]
    zero_h = zero.cpu().numpy()
    for i in range(8000, cfg.n_q):                   # positions of at least 8064 use the sample phase
        if zero_h[i]:
            assert sorted(idx_h[i, :cfg.topk].tolist()) == list(range(cfg.topk)), f"row {i}"
    ro = RowOracle(cfg, 17)
    rows = [i for i in synthetic.sample_rows(cfg.n_q, 40, 17, extra=[8063, 8064, 8999]) if not zero_h[i]]
    stats = []
    for j, i in enumerate(rows):
        _, scores = ro.indexer(0, i)
        stats.append(check_selection(idx_h[i], scores, cfg.topk, i))
    report_near_ties("prefill L=9000, sampled threshold", len(rows), stats)


def test_decode_equal_scores_merge_by_position():
    # every index score is 0, so each sequence keeps its lowest min(k, len) positions; with
    # lengths spanning one to three 8192-key chunks, the merge must resolve the ties across
    # chunk lists by position, and a sequence shorter than k keeps every key
    cfg = synthetic.config("decode", batch=4, max_len=20000, len_range=(100, 20000))
    g = _inputs(cfg, 12)
    g["w"].zero_()
    lens = [100, 2048, 9000, 20000]
    g["lengths"] = torch.tensor(lens, dtype=torch.int32, device="cuda")
    idx, out, lse = _run_forward(cfg, g)
    idx_h = idx.cpu().numpy()
    for b, n_b in enumerate(lens):
        n = min(cfg.topk, n_b)
        assert sorted(idx_h[b, 0, :n].tolist()) == list(range(n))
        assert (idx_h[b, 0, n:] == -1).all()


def test_decode_repeated_keys_cut_ties_by_position():
    """Cached index keys repeat with period 97, so each sequence's scores take 97 values, each
    held by many positions: the k-th score is shared by more positions than places remain,
    and the selection must keep the lowest of them. The oracle ranks the same way (score,
    then position), so the selected sets must be equal; the premise (the k-th score well
    apart from the scores next to it, its group split) is checked on the oracle's scores first."""
    period = 97
    cfg = synthetic.config("decode", batch=3, max_len=30000, len_range=(100, 30000))
    g = _inputs(cfg, 21)
    lens = [30000, 12345, 4100]
    g["lengths"] = torch.tensor(lens, dtype=torch.int32, device="cuda")
    rep = torch.arange(cfg.max_len, device="cuda") % period
    g["k_idx"] = g["k_idx"][:, rep].contiguous()
    g["k_scale"] = g["k_scale"][:, rep].contiguous()
    idx, out, lse = _run_forward(cfg, g)
    idx_h = idx.cpu().numpy()
    ro = RowOracle(cfg, 21, lengths=torch.tensor(lens))
    for b, n_b in enumerate(lens):
        kc, ks = synthetic.gen_k_idx(cfg, 21, b=b, s_range=range(0, period))
        rep_h = np.arange(n_b) % period
        ro._keys[b] = (kc.numpy()[rep_h], ks.numpy()[rep_h])
        sel_o, scores = ro.indexer(b, 0)
        distinct = np.unique(scores)[::-1]
        assert len(distinct) == period
        kth = np.sort(scores)[::-1][cfg.topk - 1]
        at = int(np.flatnonzero(distinct == kth)[0])
        gaps = np.array([distinct[at - 1] - kth, kth - distinct[at + 1]])
        assert (gaps > 1e-4 * np.max(np.abs(distinct))).all()             # far above fp32 rounding
        assert (scores > kth).sum() < cfg.topk < (scores >= kth).sum()       # the k-th group is split
        assert sorted(idx_h[b, 0].tolist()) == sorted(sel_o.tolist()), f"sequence {b}"


def test_decode_select_falls_back_when_the_sample_misleads():
    """The decode select guesses a threshold from a 1/16 sample of the row: the key slots at
    positions p with p mod 4096 < 256. Here the first 300 sampled positions carry the row's best
    key at twice its scale, so the sample's r-th key (r ~ 200) is one of them and only those 300
    keys reach it, fewer than k. The select must notice and run over the whole row; the result
    is checked against the oracle on the same modified inputs."""
    cfg = synthetic.config("decode", batch=2, max_len=40000, len_range=(4096, 40000))
    g = _inputs(cfg, 25)
    lens = [40000, 30000]
    g["lengths"] = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ro = RowOracle(cfg, 25, lengths=torch.tensor(lens))
    strong = {}
    for b, n_b in enumerate(lens):
        _, sc = ro.indexer(b, 0)
        best = int(np.argmax(sc))
        assert sc[best] > 0
        s = np.flatnonzero(np.arange(n_b) % 4096 < 256)[:300]
        kc, ks = (a.copy() for a in ro.keys(b))
        kc[s], ks[s] = kc[best], ks[best] * 2
        ro._keys[b] = (kc, ks)
        st = torch.from_numpy(s).cuda()
        g["k_idx"][b, st] = g["k_idx"][b, best].clone()
        g["k_scale"][b, st] = g["k_scale"][b, best].clone() * 2
        strong[b] = set(s.tolist())
    idx, out, lse = _run_forward(cfg, g)
    _check_rows(cfg, 25, [(0, 0), (1, 0)], idx, out, lse, ro=ro, name="decode, misleading sample")
    idx_h = idx.cpu().numpy()
    for b in range(cfg.batch):
        assert strong[b] <= set(idx_h[b, 0].tolist())


def test_decode_rows_longer_than_one_select_cluster():
    """Decode rows of more than 131072 keys take the per-chunk partial top-k and its merge
    instead of the whole-row select; checked against the oracle like the decode workload."""
    cfg = synthetic.config("decode", batch=2, max_len=140000, len_range=(4096, 140000))
    g = _inputs(cfg, 23)
    lens = torch.tensor([140000, 70001], dtype=torch.int32)
    g["lengths"] = lens.cuda()
    idx, out, lse = _run_forward(cfg, g)
    ro = RowOracle(cfg, 23, lengths=lens)
    _check_rows(cfg, 23, [(0, 0), (1, 0)], idx, out, lse, ro=ro, name="decode, rows of 140000 keys")


@pytest.mark.parametrize("topk", [1, 7, 2048])
def test_topk_extremes(topk):
    cfg = synthetic.config("tiny", n_q=260, max_len=260, topk=topk)
    g = _inputs(cfg, 9, gen_device="cpu")
    idx, out, lse = _run_forward(cfg, g)
    _check_rows(cfg, 9, [(0, i) for i in range(cfg.n_q)], idx, out, lse, name=f"tiny L=260 k={topk}")


def test_ragged_batch_prefill_with_empty_sequence():
    cfg = synthetic.config("tiny", batch=3, n_q=200, max_len=200, topk=32)
    g = _inputs(cfg, 10, gen_device="cpu")
    lengths = torch.tensor([200, 37, 0], dtype=torch.int32)
    g["lengths"] = lengths.cuda()
    idx, out, lse = _run_forward(cfg, g)
    ro = RowOracle(cfg, 10, lengths=lengths)
    rows = [(b, i) for b in range(3) for i in range(cfg.n_q)]
    _check_rows(cfg, 10, rows, idx, out, lse, ro=ro, name="tiny ragged batch of 3")
    # queries before the start of a short sequence select nothing: out = 0, lse = -inf
    assert (idx[2] == -1).all() and (out[2] == 0).all() and torch.isinf(lse[2]).all()


def test_attention_skips_padding_and_reports_out_of_range():
    cfg = synthetic.config("tiny", n_q=64, max_len=64, topk=16)
    g = _inputs(cfg, 11, gen_device="cpu")
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    sets = torch.full((1, cfg.n_q, cfg.topk), -1, dtype=torch.int32)
    sets[0, 1, [0, 5, 9]] = torch.tensor([0, 1, -1 + 1], dtype=torch.int32)   # 0, 1, 0 (duplicate)
    sets[0, 2, 3] = 2
    out, lse = dsa.sparse_mla_attn(dims, g["q"], g["kv"], sets.cuda(), cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    ro = RowOracle(cfg, 11)
    for i in (1, 2):
        o, l = ro.attention(0, i, sets[0, i].tolist())
        compare_attention(out.float().cpu().numpy()[0, i:i + 1], lse.cpu().numpy()[0, i:i + 1], o[None], l[None])
    assert (out[0, 0] == 0).all() and torch.isinf(lse[0, 0]).all()
    sets[0, 3, 0] = cfg.max_len + 5                  # outside [0, max_len): skipped and reported
    dsa.sparse_mla_attn(dims, g["q"], g["kv"], sets.cuda(), cfg.topk, ws)
    st, _ = dsa.dsa_get_device_status(ws.buf)
    assert st == dsa.DSA_ERR_INDEX_RANGE
    assert dsa.dsa_get_device_status(ws.buf)[0] == dsa.DSA_OK    # cleared by the read


def test_attention_masked_leading_blocks():
    """Index rows whose first 64-entry blocks hold no attended entry (padding or entries past
    max_len), an all-padding row, and padding scattered through a row: masked entries are
    skipped wherever they appear, with no NaN, and an entry past max_len is reported."""
    cfg = synthetic.config("tiny", n_q=9, max_len=300, topk=256)
    g = _inputs(cfg, 16, gen_device="cpu")
    r = np.random.default_rng(16)
    k, L = cfg.topk, cfg.max_len
    rows = np.full((cfg.n_q, k), -1, dtype=np.int32)

    def valid(n):
        return r.integers(0, L, size=n).astype(np.int32)

    rows[0, 64:84] = valid(20)                      # block 0 all padding
    rows[1, 130:170] = valid(40)                    # blocks 0-1 and half of block 2 padding
    rows[2, :64] = L + 7                            # block 0 entirely past max_len (reported)
    rows[2, 64:94] = valid(30)
    # row 3: all padding -> out = 0, lse = -inf
    m = r.random(k) < 0.4                           # padding scattered, block 0 all padding
    m[:64] = False
    rows[4, m] = valid(int(m.sum()))
    rows[5, 192:] = valid(64)                       # only the last block attended
    rows[6, :3] = valid(3)                          # block 0 partly attended (then padding)
    rows[7] = valid(k)                              # every entry attended
    rows[8, 63] = valid(1)[0]                       # one attended entry, the last of block 0
    rows[8, 64:128] = L + 1                         # then a block past max_len
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    out, lse = dsa.sparse_mla_attn(dims, g["q"], g["kv"], torch.from_numpy(rows).reshape(1, cfg.n_q, k).cuda(),
                                   cfg.topk, ws)
    torch.cuda.synchronize()
    st, _ = dsa.dsa_get_device_status(ws.buf)
    assert st == dsa.DSA_ERR_INDEX_RANGE
    ro = RowOracle(cfg, 16)
    out_h, lse_h = out.double().cpu().numpy()[0], lse.cpu().numpy()[0]
    assert not np.isnan(out_h).any() and not np.isnan(lse_h).any()
    for i in range(cfg.n_q):
        kept = [int(x) for x in rows[i] if 0 <= x < L]
        o, l = ro.attention(0, i, kept)
        compare_attention(out_h[i], lse_h[i], o, l)
    assert (out_h[3] == 0).all() and np.isneginf(lse_h[3]).all()


def test_general_fp8_scales_tiny_forward():
    """FP8 inputs quantised with scale = amax/448 (not a power of two), so the kernel's fp32
    folding of the query scale into the head weights and its key-scale multiply round."""
    cfg = synthetic.config("tiny", fp8_scale="amax")
    g = _inputs(cfg, 13, gen_device="cpu")
    m, _ = np.frexp(g["k_scale"].double().cpu().numpy())
    assert (m != 0.5).mean() > 0.9
    idx, out, lse = _run_forward(cfg, g)
    _check_rows(cfg, 13, [(0, i) for i in range(cfg.n_q)], idx, out, lse, name="tiny, amax/448 scales")


def test_general_fp8_scales_prefill_4k_indexer():
    cfg = synthetic.config("prefill_4k", fp8_scale="amax")
    g = {}
    g["q_idx"], g["q_scale"] = synthetic.gen_q_idx(cfg, 14)
    g["k_idx"], g["k_scale"] = synthetic.gen_k_idx(cfg, 14)
    g["w"] = synthetic.gen_w(cfg, 14)
    g = {n: v.cuda() for n, v in g.items()}
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    idx = dsa.indexer_topk(dims, g["q_idx"].view(1, cfg.n_q, cfg.n_idx_heads, cfg.idx_dim), g["w"],
                           g["k_idx"], g["q_scale"], g["k_scale"], synthetic.lengths(cfg, 14).cuda(), cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    rows = synthetic.sample_rows(cfg.n_q, 768, 14, extra=[0, 1, 2046, 2047, 2048, 2049, cfg.n_q - 1])
    _check_rows(cfg, 14, [(0, i) for i in rows], idx, None, None, attn_rows=set(),
                name="prefill_4k, amax/448 scales")


def test_row_sharded_chunks_match_the_oracle():
    """The query-row sharding of one sequence over three ranks, run here as the three ranks'
    chunk calls on one GPU (n_q = r1 - r0, lengths = r1, the whole key side): sampled rows of
    every part, and each part's first and last row, against the oracle at their positions."""
    from sparse_attention_long_indexer_b200 import shard
    cfg = synthetic.config("prefill_4k")
    seed = 15
    g = _inputs(cfg, seed)
    ro = RowOracle(cfg, seed)
    parts = shard.row_partition(cfg.max_len, 3, cfg.topk)
    assert all(r1 > r0 for r0, r1 in parts)
    k_scale = g["k_scale"].reshape(-1)
    for rank in range(3):
        c = shard.chunk_call(parts, rank)
        r0 = c.row0
        dims_c = dsa.make_dims(1, c.n_q, cfg.max_len, cfg.n_idx_heads, cfg.idx_dim, cfg.n_heads, cfg.d_latent,
                               cfg.d_rope, cfg.softmax_scale)
        ws = dsa.Workspace.create(dims_c, cfg.topk)
        idx = torch.empty((1, c.n_q, cfg.topk), dtype=torch.int32, device="cuda")
        out = torch.empty((1, c.n_q, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((1, c.n_q, cfg.n_heads), dtype=torch.float32, device="cuda")
        scales = torch.cat([g["q_scale"].reshape(-1)[r0:r0 + c.n_q], k_scale]).contiguous()
        dsa.dsa_forward(dims_c, g["q_idx"][:, r0:r0 + c.n_q].contiguous(), g["w"][:, r0:r0 + c.n_q].contiguous(),
                        g["k_idx"], scales, torch.tensor([c.length], dtype=torch.int32, device="cuda"), cfg.topk,
                        g["q"][:, r0:r0 + c.n_q].contiguous(), g["kv"], idx, out, lse, ws.buf)
        torch.cuda.synchronize()
        ws.check()
        local = sorted(set(synthetic.sample_rows(c.n_q, 40, seed + rank, extra=[0, c.n_q - 1])))
        idx_h = _rows_to_host(idx, [(0, i) for i in local])
        out_h = _rows_to_host(out, [(0, i) for i in local])
        lse_h = _rows_to_host(lse, [(0, i) for i in local])
        stats, refs = [], []
        for j, i in enumerate(local):
            t = r0 + i                                   # the row's position in the whole sequence
            _, scores = ro.indexer(0, t)
            stats.append(check_selection(idx_h[j], scores, cfg.topk, t))
            refs.append(ro.attention(0, t, idx_h[j]))
        report_near_ties("prefill_4k, 3 row shards", len(local), stats)
        compare_attention(out_h, lse_h, np.stack([x[0] for x in refs]), np.stack([x[1] for x in refs]))


def test_empty_problem_is_a_no_op():
    cfg = synthetic.config("tiny", batch=0)
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    e = torch.empty(0, device="cuda")
    dsa.dsa_forward(dims, e, e, e, e, e, cfg.topk, e, e, None, e, e, ws.buf)
    ws.check()


# ----------------------------------------------------------------------------- query chunks
def test_query_chunks_match_one_call():
    """A prefill sequence run as query chunks [i0, i1) (n_q = i1 - i0, lengths = i1) gives what one
    call over all queries gives, query by query (the e2e measurement runs the step this way)."""
    cfg = synthetic.config("prefill_4k")
    g = _inputs(cfg, 5)
    idx, out, lse = _run_forward(cfg, g)
    L, C = cfg.max_len, 1024
    c_idx, c_out, c_lse = torch.empty_like(idx), torch.empty_like(out), torch.empty_like(lse)
    dims_c = dsa.make_dims(1, C, L, cfg.n_idx_heads, cfg.idx_dim, cfg.n_heads, cfg.d_latent, cfg.d_rope,
                           cfg.softmax_scale)
    ws = dsa.Workspace.create(dims_c, cfg.topk)
    q_scale = g["q_scale"].reshape(-1)
    k_scale = g["k_scale"].reshape(-1).float()
    for i0 in range(0, cfg.n_q, C):
        scales = torch.cat([q_scale[i0:i0 + C].float(), k_scale]).contiguous()
        lengths = torch.tensor([i0 + C], dtype=torch.int32, device="cuda")
        o_i, o_o, o_l = (torch.empty((1, C, cfg.topk), dtype=torch.int32, device="cuda"),
                         torch.empty((1, C, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device="cuda"),
                         torch.empty((1, C, cfg.n_heads), dtype=torch.float32, device="cuda"))
        dsa.dsa_forward(dims_c, g["q_idx"][:, i0:i0 + C].contiguous(), g["w"][:, i0:i0 + C].contiguous(), g["k_idx"],
                        scales, lengths, cfg.topk, g["q"][:, i0:i0 + C].contiguous(), g["kv"], o_i, o_o, o_l, ws.buf)
        c_idx[:, i0:i0 + C], c_out[:, i0:i0 + C], c_lse[:, i0:i0 + C] = o_i, o_o, o_l
    torch.cuda.synchronize()
    ws.check()
    # the same index sets; their order within a row is unspecified (candidate appends from four warps
    # interleave), and it sets the summation order and where the softmax rescales, so out may differ
    # by the rounding of P and of the sums: within the parity tolerances of the attention
    assert torch.equal(torch.sort(idx, dim=-1).values, torch.sort(c_idx, dim=-1).values)
    a, b = out.float(), c_out.float()
    assert (a - b).abs().max().item() <= 1e-2
    assert ((a - b).norm() / a.norm()).item() <= 5e-3
    assert (lse - c_lse).abs().max().item() <= 2e-3
