"""Pins of the CPU oracle to things other than itself (CPU only, no GPU).

Each test ties one oracle function to a library routine, a closed form, an
invariant or a brute force, chosen so that a plausible slip (ReLU applied after
the head sum, a dropped weight, a transposed operand, a wrong tie rule, a
missing scale, softmax over the wrong axis) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic

rng = np.random.default_rng(1234)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- decoders
def test_e4m3_decode_matches_torch_on_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9


def test_e4m3_decode_applies_per_row_scale():
    codes = rng.integers(0, 256, size=(5, 7), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0
    scale = np.array([0.5, 2.0, 3.0, 1e-3, 7.25])
    assert np.array_equal(oracle.decode_e4m3(codes, scale), oracle.decode_e4m3(codes) * scale[:, None])


def test_bf16_decode_matches_torch_on_all_codes():
    bits = np.arange(65536, dtype=np.uint16)
    ours = oracle.decode_bf16(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ----------------------------------------------------------------------------- index score
def _rand_indexer(H=6, d=9, n=40):
    return rng.standard_normal((H, d)), rng.standard_normal(H), rng.standard_normal((n, d))


def test_index_score_odd_part_is_linear():
    # ReLU(x) - ReLU(-x) = x, so I(q) - I(-q) = sum_j w_j (q_j . k) = (w^T q) . k.
    q, w, k = _rand_indexer()
    lhs = oracle.index_scores(q, w, k) - oracle.index_scores(-q, w, k)
    rhs = k @ (w @ q)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_index_score_even_part_is_weighted_abs():
    # ReLU(x) + ReLU(-x) = |x|, computed here key by key with explicit loops.
    q, w, k = _rand_indexer(H=3, d=4, n=6)
    lhs = oracle.index_scores(q, w, k) + oracle.index_scores(-q, w, k)
    for s in range(k.shape[0]):
        acc = 0.0
        for j in range(q.shape[0]):
            acc += w[j] * abs(sum(q[j, d] * k[s, d] for d in range(q.shape[1])))
        assert abs(lhs[s] - acc) < 1e-12


def test_index_score_relu_is_per_head_not_after_sum():
    q = np.array([[1.0, 0.0], [-1.0, 0.0]])     # head dots +1 and -1 against k=(1,0)
    k = np.array([[1.0, 0.0]])
    w = np.array([1.0, 1.0])
    assert oracle.index_scores(q, w, k)[0] == 1.0     # ReLU(1)+ReLU(-1) = 1, not ReLU(0) = 0
    assert oracle.index_scores(q, np.array([2.0, 5.0]), k)[0] == 2.0


def test_index_score_nonnegative_for_nonnegative_weights():
    q, w, k = _rand_indexer(H=16, d=32, n=500)
    assert (oracle.index_scores(q, np.abs(w), k) >= 0).all()


def test_index_score_single_head_unit_weight_is_relu_dot():
    q, _, k = _rand_indexer(H=1, d=7, n=30)
    got = oracle.index_scores(q, np.ones(1), k)
    for s in range(k.shape[0]):
        assert got[s] == pytest.approx(max(0.0, float(np.dot(q[0], k[s]))), abs=1e-13)


def test_index_score_linear_in_weights_and_scale_homogeneous():
    q, w1, k = _rand_indexer()
    w2 = rng.standard_normal(w1.shape)
    np.testing.assert_allclose(oracle.index_scores(q, w1 + w2, k),
                               oracle.index_scores(q, w1, k) + oracle.index_scores(q, w2, k), atol=1e-12)
    np.testing.assert_allclose(oracle.index_scores(2.5 * q, w1, 0.75 * k),
                               2.5 * 0.75 * oracle.index_scores(q, w1, k), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- selection
@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (20, 20), (20, 25), (64, 10), (300, 64)])
def test_topk_matches_brute_force_sort_with_ties(n, k):
    scores = rng.integers(-4, 5, size=n).astype(np.float64)     # many exact ties
    expect = [s for _, s in sorted((-scores[s], s) for s in range(n))][: min(k, n)]
    assert oracle.select_topk(scores, k).tolist() == expect


def test_topk_ties_go_to_lower_position():
    assert oracle.select_topk(np.zeros(10), 4).tolist() == [0, 1, 2, 3]
    assert sorted(oracle.select_topk(np.array([1.0, 3.0, 3.0, 2.0, 3.0]), 2).tolist()) == [1, 2]


def _tiny_row_inputs(cfg, seed, pos):
    q_codes, q_scale = synthetic.gen_q_idx(cfg, seed, tokens=[pos])
    w = synthetic.gen_w(cfg, seed, tokens=[pos])
    k_codes, k_scale = synthetic.gen_k_idx(cfg, seed, b=0)
    return (q_codes[0].numpy(), float(q_scale[0]), w[0].view(torch.int16).numpy().view(np.uint16),
            k_codes.numpy(), k_scale.numpy())


def _finite_e4m3_codes(r, shape):
    c = r.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 0x01                    # S.1111.111 is NaN: use the neighbouring code
    return c


@pytest.mark.parametrize("pos", [11, 8, 0])
def test_indexer_row_applies_each_tokens_scale(pos):
    # One query against 12 keys, each key with its own scale (neither uniform nor a power of two)
    # and a query scale != 1: the real value of a code is code x its token's scale. Decoded here
    # with torch's own float8_e4m3fn / bfloat16 casts and summed with explicit loops:
    #     I[s] = sum_j w_j * max(0, sum_d (q_code[j,d] * s_q) * (k_code[s,d] * s_k[s]))
    H, d, n, topk = 3, 5, 12, 4
    r = np.random.default_rng(77 + pos)
    q_codes, k_codes = _finite_e4m3_codes(r, (H, d)), _finite_e4m3_codes(r, (n, d))
    q_scale = 0.3716
    k_scale = r.uniform(0.05, 3.0, size=n)
    w_bits = torch.tensor(r.standard_normal(H), dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy()
    w_bits = w_bits.view(np.uint16)
    tq = torch.from_numpy(q_codes).view(torch.float8_e4m3fn).double().tolist()
    tk = torch.from_numpy(k_codes).view(torch.float8_e4m3fn).double().tolist()
    tw = torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16).double().tolist()
    expect = []
    for s in range(pos + 1):
        acc = 0.0
        for j in range(H):
            dot = 0.0
            for e in range(d):
                dot += (tq[j][e] * q_scale) * (tk[s][e] * float(k_scale[s]))
            acc += tw[j] * max(0.0, dot)
        expect.append(acc)
    idx, scores = oracle.indexer_topk_row(q_codes, q_scale, w_bits, k_codes, k_scale, pos, topk)
    assert scores.shape == (pos + 1,)
    np.testing.assert_allclose(scores, expect, rtol=1e-12, atol=1e-300)
    brute = [s for _, s in sorted((-expect[s], s) for s in range(pos + 1))][: min(topk, pos + 1)]
    assert idx.tolist() == brute


def test_selection_is_causal_and_counts_min_k_pos():
    cfg = synthetic.config("tiny")
    for pos in [0, 1, 5, 63, 64, 65, 200, 511]:
        idx, scores = oracle.indexer_topk_row(*_tiny_row_inputs(cfg, 3, pos), pos, cfg.topk)
        assert len(idx) == min(cfg.topk, pos + 1)
        assert idx.max() <= pos and idx.min() >= 0
        assert len(set(idx.tolist())) == len(idx)
        assert scores.shape == (pos + 1,)
        # every unselected key scores no higher than every selected one
        if pos + 1 > cfg.topk:
            rest = np.setdiff1d(np.arange(pos + 1), idx)
            assert scores[rest].max() <= scores[idx].min()


# ----------------------------------------------------------------------------- attention
def _dense_mqa_sdpa(q, kv, d_v, tau):
    """torch SDPA in float64, causal, every head sharing one K (all dims) and V (latent)."""
    L, H, _ = q.shape
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                     # [1, H, L, dqk]
    kt = torch.from_numpy(kv)[None, None].expand(1, H, L, kv.shape[1])
    vt = torch.from_numpy(kv[:, :d_v])[None, None].expand(1, H, L, d_v)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=tau)
    return out[0].permute(1, 0, 2).numpy()


def test_sparse_attention_with_all_rows_selected_is_dense_causal_mqa():
    L, H, dqk, dv = 37, 5, 12, 8
    q = rng.standard_normal((L, H, dqk))
    kv = rng.standard_normal((L, dqk))
    tau = 1.0 / math.sqrt(dqk)
    ref = _dense_mqa_sdpa(q, kv, dv, tau)
    for t in range(L):
        out, _ = oracle.sparse_mla_attention(q[t], kv[: t + 1], dv, tau)
        np.testing.assert_allclose(out, ref[t], rtol=1e-11, atol=1e-12)


def test_attention_weights_sum_to_one_and_lse_is_logsumexp():
    from scipy.special import logsumexp
    H, m, dqk, dv = 4, 19, 10, 6
    q = rng.standard_normal((H, dqk)) * 3.0
    kv = rng.standard_normal((m, dqk))
    kv[:, :dv] = 1.0                                   # V = ones  =>  out = sum_s p_s = 1
    out, lse = oracle.sparse_mla_attention(q, kv, dv, 0.7)
    np.testing.assert_allclose(out, 1.0, rtol=1e-13)
    np.testing.assert_allclose(lse, logsumexp(0.7 * q @ kv.T, axis=1), rtol=1e-13, atol=1e-13)


def test_attention_closed_forms():
    H, dqk, dv = 3, 6, 4
    kv = rng.standard_normal((9, dqk))
    q = rng.standard_normal((H, dqk))
    out, lse = oracle.sparse_mla_attention(q, kv[:1], dv, 0.3)       # one row: out = its latent
    np.testing.assert_allclose(out, np.broadcast_to(kv[0, :dv], (H, dv)), rtol=1e-14)
    np.testing.assert_allclose(lse, 0.3 * q @ kv[0], rtol=1e-14)
    out, lse = oracle.sparse_mla_attention(np.zeros((H, dqk)), kv, dv, 0.3)   # equal logits: mean
    np.testing.assert_allclose(out, np.broadcast_to(kv[:, :dv].mean(0), (H, dv)), rtol=1e-13)
    np.testing.assert_allclose(lse, math.log(9.0), rtol=1e-14)
    out, lse = oracle.sparse_mla_attention(q, kv[:0], dv, 0.3)        # nothing selected
    assert (out == 0).all() and np.isneginf(lse).all()


def test_attention_ignores_order_and_padding():
    bits = (rng.integers(0, 1 << 15, size=(30, 8)) & 0x3FFF).astype(np.uint16)   # finite bf16
    qb = (rng.integers(0, 1 << 15, size=(2, 8)) & 0x3FFF).astype(np.uint16)
    a = oracle.sparse_mla_attn_row(qb, bits, [3, 7, 11, 2], 5, 0.5)
    b = oracle.sparse_mla_attn_row(qb, bits, [-1, 11, 2, -1, 7, 3, -1], 5, 0.5)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-13)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-13)


def test_full_path_reduces_to_dense_attention_when_k_covers_the_prefix():
    cfg = synthetic.config("tiny", n_q=40, max_len=40)      # topk = 64 >= pos+1 for every query
    seed = 11
    g = synthetic.gen_all(cfg, seed)
    qb = g["q"][0].view(torch.int16).numpy().view(np.uint16)
    kvb = g["kv"][0].view(torch.int16).numpy().view(np.uint16)
    tau = cfg.softmax_scale
    ref = _dense_mqa_sdpa(oracle.decode_bf16(qb), oracle.decode_bf16(kvb), cfg.d_v, tau)
    for t in range(cfg.n_q):
        idx, out, lse, _ = oracle.dsa_row(
            g["q_idx"][0, t].numpy(), float(g["q_scale"][0, t]),
            g["w"][0, t].view(torch.int16).numpy().view(np.uint16),
            g["k_idx"][0].numpy(), g["k_scale"][0].numpy(), qb[t], kvb, t, cfg.topk, cfg.d_v, tau)
        assert sorted(idx.tolist()) == list(range(t + 1))
        np.testing.assert_allclose(out, ref[t], rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- page constants
def test_page_constants_fix_128k_as_131072_and_k_2048():
    g = json.load(open(os.path.join(GOLDEN, "page_constants.json")))

    def rounds_to(x, printed, digits):
        return float(f"{x:.{digits}g}") == printed

    for ctx, ok in [(131072, True), (128000, False)]:
        dw, sp = g["dense_warmup"], g["sparse_training"]
        a = rounds_to(dw["steps"] * dw["seqs_per_step"] * ctx, dw["tokens_printed"], dw["printed_digits"])
        b = rounds_to(sp["steps"] * sp["seqs_per_step"] * ctx, sp["tokens_printed"], sp["printed_digits"])
        assert (a and b) == ok
    assert synthetic.config("prefill_128k").max_len == 131072
    for name in ["prefill_4k", "prefill_32k", "prefill_128k", "decode"]:
        assert synthetic.config(name).topk == g["topk"]["value"]


# ----------------------------------------------------------------------------- indexer alignment loss
def test_head_sum_target_brute_force():
    # a[s] = sum_h softmax_s(tau q_h . kv_s), p = a / sum(a): explicit loops with math.exp
    H, m, d = 4, 7, 5
    q = rng.standard_normal((H, d)) * 2.0
    kv = rng.standard_normal((m, d))
    tau = 0.61
    a = [0.0] * m
    for h in range(H):
        z = [tau * sum(q[h, e] * kv[s, e] for e in range(d)) for s in range(m)]
        zmax = max(z)
        ex = [math.exp(v - zmax) for v in z]
        tot = sum(ex)
        for s in range(m):
            a[s] += ex[s] / tot
    expect = [x / sum(a) for x in a]
    np.testing.assert_allclose(oracle.attention_head_sum_target(q, kv, tau), expect, rtol=1e-12)
    assert abs(sum(a) - H) < 1e-12                   # each head's weights sum to one


def test_head_sum_target_single_head_is_softmax():
    from scipy.special import softmax
    q = rng.standard_normal((1, 6))
    kv = rng.standard_normal((9, 6))
    np.testing.assert_allclose(oracle.attention_head_sum_target(q, kv, 0.4), softmax(0.4 * (kv @ q[0])), rtol=1e-12)


def test_indexer_kl_matches_scipy_entropy():
    from scipy.special import softmax
    from scipy.stats import entropy
    for m in (1, 2, 17, 300):
        p = rng.random(m) ** 3
        p /= p.sum()
        scores = rng.standard_normal(m) * 4.0
        assert oracle.indexer_kl(p, scores) == pytest.approx(entropy(p, softmax(scores)), rel=1e-11, abs=1e-13)


def test_indexer_kl_closed_forms():
    p = rng.random(11)
    p /= p.sum()
    assert abs(oracle.indexer_kl(p, np.log(p) + 3.7)) < 1e-13          # scores = ln p + c: zero
    assert oracle.indexer_kl(np.full(5, 0.2), np.full(5, -2.5)) == pytest.approx(0.0, abs=1e-15)
    x, y, a = 1.3, -0.4, 0.3                                           # two points
    sig = 1.0 / (1.0 + math.exp(-(x - y)))
    two = a * math.log(a / sig) + (1 - a) * math.log((1 - a) / (1 - sig))
    assert oracle.indexer_kl(np.array([a, 1 - a]), np.array([x, y])) == pytest.approx(two, rel=1e-13)
    s = rng.standard_normal(6)                                         # one-hot target: -ln q_0
    lse = math.log(sum(math.exp(v) for v in s))
    assert oracle.indexer_kl(np.eye(6)[0], s) == pytest.approx(lse - s[0], rel=1e-13)


def test_indexer_kl_is_nonnegative():
    for _ in range(50):
        m = int(rng.integers(1, 40))
        p = rng.random(m)
        p /= p.sum()
        assert oracle.indexer_kl(p, rng.standard_normal(m) * 3.0) >= -1e-15


def _kl_row_inputs(H=3, n=12, d=8):
    qb = torch.tensor(rng.standard_normal((H, d)), dtype=torch.float32).to(torch.bfloat16)
    kvb = torch.tensor(rng.standard_normal((n, d)), dtype=torch.float32).to(torch.bfloat16)
    u16 = lambda t: t.view(torch.int16).numpy().view(np.uint16)           # noqa: E731
    return u16(qb), u16(kvb), qb.double().numpy(), kvb.double().numpy()


def test_indexer_kl_row_brute_force_over_the_selected_set():
    # sparse stage: per-head softmax over the selected rows only, head sum, L1 normalisation,
    # KL against the softmax of the selected rows' index scores -- all with explicit loops
    qb, kvb, q, kv = _kl_row_inputs()
    H, d = q.shape
    idx = [7, 2, 9, 4, 11]
    sc = rng.standard_normal(len(idx)) * 2.0
    tau = 0.35
    a = [0.0] * len(idx)
    for h in range(H):
        z = [tau * sum(q[h, e] * kv[s, e] for e in range(d)) for s in idx]
        ex = [math.exp(v) for v in z]
        for j in range(len(idx)):
            a[j] += ex[j] / sum(ex)
    p = [x / sum(a) for x in a]
    lse = math.log(sum(math.exp(v) for v in sc))
    expect = sum(p[j] * (math.log(p[j]) - (sc[j] - lse)) for j in range(len(idx)))
    assert oracle.indexer_kl_row(qb, kvb, idx, sc, tau) == pytest.approx(expect, rel=1e-12)


def test_indexer_kl_row_ignores_padding_and_order():
    qb, kvb, _, _ = _kl_row_inputs()
    idx = np.array([3, 8, 0, 5])
    sc = rng.standard_normal(4)
    base = oracle.indexer_kl_row(qb, kvb, idx, sc, 0.5)
    perm = np.array([2, 0, 3, 1])
    padded_idx = np.array([-1, 3, -1, 8, 0, -1, 5])
    padded_sc = np.array([9.0, sc[0], -7.0, sc[1], sc[2], 5.0, sc[3]])
    assert oracle.indexer_kl_row(qb, kvb, idx[perm], sc[perm], 0.5) == pytest.approx(base, rel=1e-12)
    assert oracle.indexer_kl_row(qb, kvb, padded_idx, padded_sc, 0.5) == pytest.approx(base, rel=1e-12)
    assert oracle.indexer_kl_row(qb, kvb, [-1, -1], [0.0, 1.0], 0.5) == 0.0


def test_head_sum_target_matches_attention_weights_from_lse():
    # p[s] = (1/H) sum_h exp(tau q_h . kv_s - lse_h), lse from the attention oracle
    qb, kvb, q, kv = _kl_row_inputs(H=5, n=9)
    _, lse = oracle.sparse_mla_attention(q, kv, 4, 0.3)
    a = np.exp(0.3 * (q @ kv.T) - lse[:, None]).sum(0) / q.shape[0]
    np.testing.assert_allclose(oracle.attention_head_sum_target(q, kv, 0.3), a, rtol=1e-12)


# ----------------------------------------------------------------------------- masked dense mode
def test_masked_dense_attention_matches_sdpa_with_a_boolean_mask():
    # every query of a short causal prefill, its mask a random subset of 0..t (never empty):
    # torch scaled_dot_product_attention in float64 with the mask as attn_mask
    L, H, dqk, dv = 23, 3, 10, 6
    q = rng.standard_normal((L, H, dqk))
    kv = rng.standard_normal((L, dqk))
    tau = 0.37
    masks = np.tril(rng.random((L, L)) < 0.6)
    masks[np.arange(L), rng.integers(0, np.arange(L) + 1)] = True
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(kv)[None, None].expand(1, H, L, dqk)
    vt = torch.from_numpy(kv[:, :dv])[None, None].expand(1, H, L, dv)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(masks), scale=tau)
    ref = ref[0].permute(1, 0, 2).numpy()
    for t in range(L):
        out, _ = oracle.masked_dense_mqa_attention(q[t], kv[: t + 1], masks[t, : t + 1], dv, tau)
        np.testing.assert_allclose(out, ref[t], rtol=1e-11, atol=1e-12)


def test_masked_dense_attention_equals_sparse_attention_over_the_mask():
    H, n, dqk, dv = 4, 30, 8, 5
    q = rng.standard_normal((H, dqk)) * 2.0
    kv = rng.standard_normal((n, dqk))
    mask = rng.random(n) < 0.3
    mask[7] = True
    out_d, lse_d = oracle.masked_dense_mqa_attention(q, kv, mask, dv, 0.45)
    out_s, lse_s = oracle.sparse_mla_attention(q, kv[mask], dv, 0.45)
    np.testing.assert_allclose(out_d, out_s, rtol=1e-12)
    np.testing.assert_allclose(lse_d, lse_s, rtol=1e-12)
    out_e, lse_e = oracle.masked_dense_mqa_attention(q, kv, np.zeros(n, dtype=bool), dv, 0.45)
    assert (out_e == 0).all() and np.isneginf(lse_e).all()
