"""The indexer-alignment loss forward (dsa_indexer_kl_loss) and the index scores of the selected
entries (dsa_indexer_topk_scores) against the oracle, on B200.

Tolerances. Index scores: the kernel computes each score in fp32 from the decoded inputs, the
oracle in fp64: |difference| <= 1e-5 x (|I| + RMS of the row). Loss: the kernel's target uses the
attention's own lse (fp32, from bf16-rounded weights) and fp32 arithmetic throughout, so each
query's term may differ from the fp64 oracle by |d| <= 2e-3 + 2e-3 x |KL|.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.dsa_cases import RowOracle, check_selection, u16

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_long_indexer_b200")

KL_ABS, KL_REL = 2e-3, 2e-3


def _oracle_kl(cfg, seed, ro, b, i, idx_row, scores_all):
    """Oracle term of query (b, i) over the entries of idx_row, with the oracle's fp64 scores."""
    t = b * cfg.n_q + i
    qb = u16(synthetic.gen_q(cfg, seed, tokens=[t])[0])
    idx_row = np.asarray(idx_row, dtype=np.int64)
    valid = idx_row[(idx_row >= 0) & (idx_row < cfg.max_len)]
    if valid.size == 0:
        return 0.0
    kvb = u16(synthetic.gen_kv(cfg, seed, b=b, positions=range(0, int(valid.max()) + 1)))
    return oracle.indexer_kl_row(qb, kvb, valid, scores_all[valid], cfg.softmax_scale)


def _run(cfg, g, idx=None, scores=None):
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    if idx is None:
        idx, scores = dsa.indexer_topk_scores(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"],
                                              g["lengths"], cfg.topk, ws)
    out, lse = dsa.sparse_mla_attn(dims, g["q"], g["kv"], idx, cfg.topk, ws)
    loss = dsa.indexer_kl_loss(dims, g["q"], g["kv"], idx, scores, lse, cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    return idx, scores, loss


def _check_kl(got, ref):
    assert math.isfinite(got), got
    assert abs(got - ref) <= KL_ABS + KL_REL * abs(ref), (got, ref)


def test_index_scores_of_the_selection_match_the_oracle():
    cfg = synthetic.config("tiny")
    seed = 31
    g = {k: v.cuda() for k, v in synthetic.gen_all(cfg, seed, "cpu").items()}
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    idx, scores = dsa.indexer_topk_scores(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"],
                                          g["lengths"], cfg.topk, ws)
    idx_plain = dsa.indexer_topk(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"], g["lengths"],
                                 cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    assert torch.equal(torch.sort(idx, -1).values, torch.sort(idx_plain, -1).values)
    ro = RowOracle(cfg, seed)
    idx_h, sc_h = idx.cpu().numpy()[0], scores.cpu().numpy()[0]
    for i in range(cfg.n_q):
        _, ref = ro.indexer(0, i)
        check_selection(idx_h[i], ref, cfg.topk, i)
        n = min(cfg.topk, i + 1)
        rms = math.sqrt(float(np.mean(ref ** 2)))
        np.testing.assert_allclose(sc_h[i, :n], ref[idx_h[i, :n]], rtol=0, atol=1e-5 * (np.abs(ref).max() + rms))
        assert np.isneginf(sc_h[i, n:]).all()


def test_decode_index_scores_match_the_oracle():
    cfg = synthetic.config("decode", batch=6, max_len=30000, len_range=(1000, 30000))
    seed = 32
    g = synthetic.gen_all(cfg, seed, "cuda")
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    idx, scores = dsa.indexer_topk_scores(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"],
                                          g["lengths"], cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    ro = RowOracle(cfg, seed)
    for b in range(cfg.batch):
        _, ref = ro.indexer(b, 0)
        row, sc = idx[b, 0].cpu().numpy(), scores[b, 0].cpu().numpy()
        check_selection(row, ref, cfg.topk, ro.pos(b, 0))
        n = min(cfg.topk, ro.pos(b, 0) + 1)
        rms = math.sqrt(float(np.mean(ref ** 2)))
        np.testing.assert_allclose(sc[:n], ref[row[:n]], rtol=0, atol=1e-5 * (np.abs(ref).max() + rms))
        assert np.isneginf(sc[n:]).all()


def test_kl_loss_tiny_all_rows_over_the_gpu_selection():
    cfg = synthetic.config("tiny")
    seed = 33
    g = {k: v.cuda() for k, v in synthetic.gen_all(cfg, seed, "cpu").items()}
    idx, _, loss = _run(cfg, g)
    ro = RowOracle(cfg, seed)
    idx_h, loss_h = idx.cpu().numpy()[0], loss.cpu().numpy()[0]
    for i in range(cfg.n_q):
        _, scores_all = ro.indexer(0, i)
        _check_kl(float(loss_h[i]), _oracle_kl(cfg, seed, ro, 0, i, idx_h[i], scores_all))


def test_kl_loss_prefill_4k_sampled_rows_and_the_oracles_sets():
    cfg = synthetic.config("prefill_4k")
    seed = 34
    g = synthetic.gen_all(cfg, seed, "cuda")
    idx, _, loss = _run(cfg, g)
    ro = RowOracle(cfg, seed)
    rows = synthetic.sample_rows(cfg.n_q, 48, seed, extra=[0, 1, 2047, 2048, cfg.n_q - 1])
    idx_h, loss_h = idx.cpu().numpy()[0], loss.cpu().numpy()[0]
    sets = np.full((1, cfg.n_q, cfg.topk), -1, dtype=np.int32)
    sc = np.full((1, cfg.n_q, cfg.topk), -np.inf, dtype=np.float32)
    refs = {}
    for i in rows:
        sel, scores_all = ro.indexer(0, i)
        _check_kl(float(loss_h[i]), _oracle_kl(cfg, seed, ro, 0, i, idx_h[i], scores_all))
        sets[0, i, :len(sel)] = sel
        sc[0, i, :len(sel)] = scores_all[sel]
        refs[i] = _oracle_kl(cfg, seed, ro, 0, i, sel, scores_all)
    # the loss kernel fed the oracle's own selections and scores
    _, _, loss_o = _run(cfg, g, idx=torch.from_numpy(sets).cuda(), scores=torch.from_numpy(sc).cuda())
    loss_o = loss_o.cpu().numpy()[0]
    for i in rows:
        _check_kl(float(loss_o[i]), refs[i])


def test_kl_loss_dense_warmup_term_and_empty_rows():
    # every position 0..t selected (k >= L): the dense warm-up term; rows past the sequence select nothing
    cfg = synthetic.config("tiny", batch=2, n_q=100, max_len=100, topk=128)
    seed = 35
    g = {k: v.cuda() for k, v in synthetic.gen_all(cfg, seed, "cpu").items()}
    g["lengths"] = torch.tensor([100, 0], dtype=torch.int32, device="cuda")
    idx, _, loss = _run(cfg, g)
    idx_h, loss_h = idx.cpu().numpy(), loss.cpu().numpy()
    ro = RowOracle(cfg, seed, lengths=torch.tensor([100, 0]))
    for i in range(cfg.n_q):
        assert sorted(idx_h[0, i, :i + 1].tolist()) == list(range(i + 1))
        _, scores_all = ro.indexer(0, i)
        _check_kl(float(loss_h[0, i]), _oracle_kl(cfg, seed, ro, 0, i, np.arange(i + 1), scores_all))
    assert (loss_h[1] == 0).all()
