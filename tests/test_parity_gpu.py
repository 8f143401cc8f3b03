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
from tests.dsa_cases import RowOracle, check_selection, compare_attention

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


def _check_rows(cfg, seed, rows, idx, out, lse, ro=None, attn_rows=None):
    ro = ro or RowOracle(cfg, seed)
    idx_h = idx.cpu().numpy()
    out_h = out.float().cpu().numpy()
    lse_h = lse.cpu().numpy()
    ties = 0
    att_gpu, att_ref, lse_gpu, lse_ref = [], [], [], []
    for (b, i) in rows:
        sel_o, scores = ro.indexer(b, i)
        ties += check_selection(idx_h[b, i], scores, cfg.topk, ro.pos(b, i))
        if attn_rows is None or (b, i) in attn_rows:
            o, l = ro.attention(b, i, idx_h[b, i])          # oracle attention over the GPU's own set
            att_gpu.append(out_h[b, i]); att_ref.append(o)
            lse_gpu.append(lse_h[b, i]); lse_ref.append(l)
    if att_gpu:
        compare_attention(np.stack(att_gpu), np.stack(lse_gpu), np.stack(att_ref), np.stack(lse_ref))
    return ties


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
    sets = np.full((1, cfg.n_q, cfg.topk), -1, dtype=np.int32)
    for i in range(cfg.n_q):
        s, _ = ro.indexer(0, i)
        sets[0, i, :len(s)] = s
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    out, lse = dsa.sparse_mla_attn(dims, g["q"], g["kv"], torch.from_numpy(sets).cuda(), cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    ref = [ro.attention(0, i, sets[0, i]) for i in range(cfg.n_q)]
    compare_attention(out.float().cpu().numpy()[0], lse.cpu().numpy()[0], np.stack([r[0] for r in ref]),
                      np.stack([r[1] for r in ref]))


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
    sets = np.full((1, cfg.n_q, cfg.topk), -1, dtype=np.int32)
    for i in rows:
        s, _ = ro.indexer(0, i)
        sets[0, i, :len(s)] = s
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    out, lse = dsa.sparse_mla_attn(dims, g["q"], g["kv"], torch.from_numpy(sets).cuda(), cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    ref = [ro.attention(0, i, sets[0, i]) for i in rows]
    compare_attention(out.float().cpu().numpy()[0, rows], lse.cpu().numpy()[0, rows],
                      np.stack([r[0] for r in ref]), np.stack([r[1] for r in ref]))


# ----------------------------------------------------------------------------- 32K / 128K (sampled rows)
def test_prefill_32k_sampled_rows():
    cfg = synthetic.config("prefill_32k")
    g = _inputs(cfg, 5)
    idx, out, lse = _run_forward(cfg, g)
    rows = synthetic.sample_rows(cfg.n_q, 512, 5, extra=list(range(64)) + list(range(cfg.n_q - 64, cfg.n_q)))
    attn = set((0, i) for i in rows[::4])
    _check_rows(cfg, 5, [(0, i) for i in rows], idx, out, lse, attn_rows=attn)


def test_prefill_128k_sampled_rows():
    cfg = synthetic.config("prefill_128k")
    g = _inputs(cfg, 6)
    idx, out, lse = _run_forward(cfg, g)
    rows = synthetic.sample_rows(cfg.n_q, 256, 6, extra=[0, cfg.n_q - 1])
    attn = set((0, i) for i in rows[::4])
    _check_rows(cfg, 6, [(0, i) for i in rows], idx, out, lse, attn_rows=attn)
    del g, idx, out, lse
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- decode (all sequences)
def test_decode_all_sequences():
    cfg = synthetic.config("decode")
    g = _inputs(cfg, 7)
    idx, out, lse = _run_forward(cfg, g)
    _check_rows(cfg, 7, [(b, 0) for b in range(cfg.batch)], idx, out, lse)
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


@pytest.mark.parametrize("topk", [1, 7, 2048])
def test_topk_extremes(topk):
    cfg = synthetic.config("tiny", n_q=260, max_len=260, topk=topk)
    g = _inputs(cfg, 9, gen_device="cpu")
    idx, out, lse = _run_forward(cfg, g)
    _check_rows(cfg, 9, [(0, i) for i in range(cfg.n_q)], idx, out, lse)


def test_ragged_batch_prefill_with_empty_sequence():
    cfg = synthetic.config("tiny", batch=3, n_q=200, max_len=200, topk=32)
    g = _inputs(cfg, 10, gen_device="cpu")
    lengths = torch.tensor([200, 37, 0], dtype=torch.int32)
    g["lengths"] = lengths.cuda()
    idx, out, lse = _run_forward(cfg, g)
    ro = RowOracle(cfg, 10, lengths=lengths)
    rows = [(b, i) for b in range(3) for i in range(cfg.n_q)]
    _check_rows(cfg, 10, rows, idx, out, lse, ro=ro)
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
