"""The masked dense mode of the attention (dsa_masked_mqa_attn) against the oracle, on B200.

Each query attends densely over its positions 0 .. e-1 (e = one past its last valid index) with
the positions its index row does not list masked out. The oracle is the masked dense attention
written out (dense softmax over the prefix, masked logits at -inf); tolerances as for the sparse
attention (max-abs 1e-2, relative L2 5e-3 per query row, lse 2e-3). The sparse kernel on the same
index rows must agree within the same bounds.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.dsa_cases import RowOracle, compare_attention, u16

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_long_indexer_b200")


def _oracle_masked(cfg, seed, rows, idx_h, b=0):
    """Oracle masked dense attention of the listed query rows over their index rows."""
    outs, lses = [], []
    for i, row in zip(rows, idx_h):
        valid = sorted({int(x) for x in row if 0 <= x < cfg.max_len})
        t = b * cfg.n_q + i
        qb = u16(synthetic.gen_q(cfg, seed, tokens=[t])[0])
        if not valid:
            o, l = oracle.masked_dense_mqa_attention(oracle.decode_bf16(qb), np.zeros((0, cfg.d_qk)),
                                                     np.zeros(0, bool), cfg.d_v, cfg.softmax_scale)
        else:
            e = valid[-1] + 1
            kvb = u16(synthetic.gen_kv(cfg, seed, b=b, positions=range(0, e)))
            mask = np.zeros(e, bool)
            mask[valid] = True
            o, l = oracle.masked_dense_mqa_attention(oracle.decode_bf16(qb), oracle.decode_bf16(kvb), mask, cfg.d_v,
                                                     cfg.softmax_scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def _both_modes(cfg, g, idx):
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    out_m, lse_m = dsa.masked_mqa_attn(dims, g["q"], g["kv"], idx, cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    out_s, lse_s = dsa.sparse_mla_attn(dims, g["q"], g["kv"], idx, cfg.topk, ws)
    torch.cuda.synchronize()
    ws.check()
    return out_m, lse_m, out_s, lse_s


@pytest.mark.parametrize("seed", [21, 22])
def test_masked_mode_tiny_all_rows_on_the_oracle_sets(seed):
    cfg = synthetic.config("tiny")
    g = {k: v.cuda() for k, v in synthetic.gen_all(cfg, seed, "cpu").items()}
    ro = RowOracle(cfg, seed)
    sets = np.full((1, cfg.n_q, cfg.topk), -1, dtype=np.int32)
    for i in range(cfg.n_q):
        s, _ = ro.indexer(0, i)
        sets[0, i, :len(s)] = s
    idx = torch.from_numpy(sets).cuda()
    out_m, lse_m, out_s, lse_s = _both_modes(cfg, g, idx)
    rows = list(range(cfg.n_q))
    ref_o, ref_l = _oracle_masked(cfg, seed, rows, sets[0])
    compare_attention(out_m.double().cpu().numpy()[0], lse_m.cpu().numpy()[0], ref_o, ref_l)
    # the same numbers as the sparse kernel over the same sets, within the attention tolerances
    compare_attention(out_m.double().cpu().numpy()[0], lse_m.cpu().numpy()[0], out_s.double().cpu().numpy()[0],
                      lse_s.cpu().numpy()[0])


def test_masked_mode_prefill_4k_on_the_indexers_sets():
    cfg = synthetic.config("prefill_4k")
    seed = 23
    g = synthetic.gen_all(cfg, seed, "cuda")
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    idx = dsa.indexer_topk(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"], g["lengths"],
                           cfg.topk, ws)
    out_m, lse_m, out_s, lse_s = _both_modes(cfg, g, idx)
    rows = synthetic.sample_rows(cfg.n_q, 96, seed, extra=[0, 1, 63, 64, 2047, 2048, 3000, cfg.n_q - 1])
    sel = torch.tensor(rows, device="cuda")
    idx_h = idx[0, sel].cpu().numpy()
    ref_o, ref_l = _oracle_masked(cfg, seed, rows, idx_h)
    compare_attention(out_m[0, sel].double().cpu().numpy(), lse_m[0, sel].cpu().numpy(), ref_o, ref_l)
    # every row against the sparse kernel on the same sets
    a, b = out_m.float(), out_s.float()
    assert (a - b).abs().max().item() <= 1e-2
    assert ((a - b).norm() / b.norm()).item() <= 5e-3
    assert (lse_m - lse_s).abs().max().item() <= 2e-3


def test_masked_mode_padding_range_duplicates_and_empty_rows():
    cfg = synthetic.config("tiny", n_q=8, max_len=300, topk=256)
    seed = 24
    g = {k: v.cuda() for k, v in synthetic.gen_all(cfg, seed, "cpu").items()}
    r = np.random.default_rng(seed)
    rows = np.full((cfg.n_q, cfg.topk), -1, dtype=np.int32)
    rows[0, 64:84] = r.integers(0, 300, 20)          # leading padding
    rows[1, :64] = cfg.max_len + 3                   # a block past max_len (reported), then valid
    rows[1, 64:100] = r.integers(0, 300, 36)
    # row 2: all padding -> out = 0, lse = -inf
    rows[3, :10] = 17                                # one position listed ten times: attended once
    rows[3, 10] = 299                                # the last position of the cache
    rows[4] = r.integers(0, 300, cfg.topk)           # many duplicates
    rows[5, 200] = 0                                 # only position 0
    rows[6, ::3] = r.integers(0, 64, len(rows[6, ::3]))   # all within the first block
    rows[7, 5] = 130                                 # extent inside the third block
    idx = torch.from_numpy(rows).reshape(1, cfg.n_q, cfg.topk).cuda()
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    out, lse = dsa.masked_mqa_attn(dims, g["q"], g["kv"], idx, cfg.topk, ws)
    torch.cuda.synchronize()
    st, _ = dsa.dsa_get_device_status(ws.buf)
    assert st == dsa.DSA_ERR_INDEX_RANGE
    ref_o, ref_l = _oracle_masked(cfg, seed, list(range(cfg.n_q)), rows)
    out_h, lse_h = out.double().cpu().numpy()[0], lse.cpu().numpy()[0]
    assert not np.isnan(out_h).any()
    for i in range(cfg.n_q):
        compare_attention(out_h[i], lse_h[i], ref_o[i], ref_l[i])
    assert (out_h[2] == 0).all() and np.isneginf(lse_h[2]).all()


def test_masked_mode_refuses_long_caches():
    cfg = synthetic.config("prefill_4k", n_q=1, max_len=20000, batch=1)
    dims = dsa.dims_for(cfg)
    ws = dsa.Workspace.create(dims, cfg.topk)
    q = torch.zeros((1, 1, 128, 576), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 20000, 576), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1, 1, cfg.topk), dtype=torch.int32, device="cuda")
    out = torch.empty((1, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_masked_mqa_attn(dims, q, kv, idx, cfg.topk, out, lse, ws.buf)
    assert e.value.status == dsa.DSA_ERR_UNSUPPORTED
