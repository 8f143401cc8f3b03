"""CPU oracle for the DeepSeek Sparse Attention (DSA) forward path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import, call
or execute anything under ``oracle/``. The product path (the C ABI library and
its Python binding) never does, and shares no code with this file: the two
meet only in the seeded input generator (``synthetic``), which holds no step of
the method.

Plain, slow and written to be checked by eye: numpy in float64, one library
primitive per step (matrix product, stable sort, exp/log), no blocking, fusion
or reordering. It works on the exact real values the kernels see: the FP8 E4M3
codes and bf16 bit patterns are decoded here from their definitions (not with
torch), scales applied multiplicatively.

Sources (the text of web pages summarising the DeepSeek-V3.2-Exp report):
  [blog]  "節前發版：Deepseek v3.2 exp" (hdetylss.com), sections "Lightning
          indexer Step 1", "Step 2", "在MLA下實例化DSA";
  [news]  "DeepSeek 发布新模型 V3.2-Exp：基于DSA稀疏注意力机制的长上下文优化"
          (gamebaike.com), bullets 闪电索引器 / 细粒度Token选择机制 / MLA架构集成;
  [v3.2]  the DeepSeek-V3.2 article on jiuyingxinxi.com (ReLU, FP8, MQA mode).
The printed formulas lost their symbols in extraction; the readings taken where
the text is silent are listed with each function.

Pins (tests/test_oracle_pins.py, CPU only) tie each function to something other
than itself: the E4M3 and bf16 decoders to torch's own casts on all codes; the
index score to the identity I(q) - I(-q) = (sum_j w_j q_j) . k (ReLU(x) - ReLU(-x)
= x), to nonnegativity for w >= 0 and to the one-head / unit-weight special
case; the per-query driver's application of the per-token FP8 scales to a
brute-force loop over torch-decoded codes with non-uniform, non-power-of-two key
scales and a query scale other than one; the selection to a brute-force sort on tiny rows and to causality; the
attention to torch's scaled_dot_product_attention in float64 when every
preceding token is selected (k >= pos+1), to weights summing to one, to the
one-row and equal-logit closed forms and to scipy's logsumexp; the
indexer-alignment loss to explicit loops (per-head softmax, head sum, L1
normalisation, KL), to scipy's softmax and relative entropy, to its closed forms
(zero for scores = ln p + c, two points, one-hot) and to Gibbs' inequality, and
its per-query term to padding and order invariance; the masked dense mode to
torch's scaled_dot_product_attention in float64 with a boolean mask and to the
sparse attention over the unmasked rows. The pages print no worked example,
so no pin uses a printed value; every function here is pinned by the checks
above, and the values at the production shapes rest on them.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "decode_e4m3", "decode_bf16", "index_scores", "select_topk", "sparse_mla_attention",
    "indexer_topk_row", "sparse_mla_attn_row", "dsa_row",
    "attention_head_sum_target", "indexer_kl", "indexer_kl_row", "masked_dense_mqa_attention",
]


# ----------------------------------------------------------------------------- input decoding
def _e4m3_table() -> np.ndarray:
    """All 256 OCP FP8 E4M3 ("fn" variant) code values: 1 sign, 4 exponent (bias 7),
    3 mantissa bits; exponent 0 is subnormal (m/8 * 2**-6); S.1111.111 is NaN; no infinities."""
    t = np.empty(256, dtype=np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            t[code] = np.nan
        elif e == 0:
            t[code] = s * (m / 8.0) * 2.0 ** -6
        else:
            t[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


_E4M3 = _e4m3_table()


def decode_e4m3(codes: np.ndarray, scale=None) -> np.ndarray:
    """FP8 E4M3 codes (uint8) -> float64, times a per-row scale if given.

    The indexer runs on FP8 inputs ([blog] section "Lightning indexer"; [news]
    bullet 闪电索引器). Reading: one fp32 scale per token, applied
    multiplicatively to the decoded code.
    """
    x = _E4M3[np.asarray(codes, dtype=np.uint8)]
    if scale is not None:
        x = x * np.asarray(scale, dtype=np.float64).reshape(x.shape[:-1] + (1,))
    return x


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64: the upper half of an IEEE binary32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):      # signalling-NaN patterns stay NaN
        return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- the three stages
def index_scores(q_t: np.ndarray, w_t: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Lightning-indexer scores of one query token against ``keys``.

    I[s] = sum_j w[j] * ReLU(q[j] . k[s])  over the indexer heads j.

    [blog] section "Lightning indexer", Step 1: the score of the query token
    against a preceding token sums, over the (few) indexer heads, a head weight
    w taken from the query token times ReLU of the dot product of that head's
    query vector (from the query token) with the key (from the preceding
    token); ReLU was picked for throughput. [v3.2] also names ReLU. Reading:
    the activation is ReLU, not the GELU that [news] names once; w is used as
    given (no extra constant, no softmax over heads).

    q_t: [H_I, d_I]; w_t: [H_I]; keys: [n, d_I]  ->  [n]
    """
    dots = q_t @ keys.T                       # [H_I, n]: q[j] . k[s]
    return w_t @ np.maximum(dots, 0.0)        # sum_j w[j] * ReLU(.)


def select_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Positions of the k largest scores (all of them if fewer than k exist).

    [blog] section "Lightning indexer", Step 2: only the tokens with the k
    highest index scores are kept; k = 2048 per query ([blog] training Step 2,
    sparse stage; [news] bullet 稀疏训练阶段).
    Reading: ties go to the lower position (the pages give no tie rule).
    Returned in rank order (best first); the kernels' order is unspecified.
    """
    n = scores.shape[0]
    order = np.lexsort((np.arange(n), -scores))   # primary: score descending, then position
    return order[: min(k, n)]


def sparse_mla_attention(q_t: np.ndarray, kv_sel: np.ndarray, d_v: int, tau: float):
    """Attention of one query token's heads over the selected latent rows (MLA, MQA mode).

    For every head h: z[s] = tau * q[h] . kv[s] (over all d_qk = latent+rope dims),
    p = softmax_s(z), out[h] = sum_s p[s] * kv[s, :d_v], lse[h] = ln sum_s exp(z[s]).

    [blog] section "Lightning indexer", Step 2, and section "在MLA下實例化DSA":
    the attention output is computed between the query token and the selected
    entries only; DSA is built on MLA's MQA mode, where one latent vector per
    token is shared by every query head ([news] bullet MLA架构集成). Readings: the
    value is the d_v-dim compressed latent (not the RoPE part); tau is the given
    softmax scale (1/sqrt(d_qk) in every workload here); lse is in natural log and
    includes tau. With no selected row: out = 0, lse = -inf.

    q_t: [H, d_qk]; kv_sel: [m, d_qk]  ->  out [H, d_v], lse [H]
    """
    H = q_t.shape[0]
    if kv_sel.shape[0] == 0:
        return np.zeros((H, d_v)), np.full(H, -np.inf)
    z = tau * (q_t @ kv_sel.T)                # [H, m]
    zmax = z.max(axis=1)
    e = np.exp(z - zmax[:, None])
    l = e.sum(axis=1)
    out = (e @ kv_sel[:, :d_v]) / l[:, None]
    lse = zmax + np.log(l)
    return out, lse


# ----------------------------------------------------------------------------- per-query drivers
def indexer_topk_row(q_codes, q_scale, w_bits, k_codes, k_scale, pos: int, topk: int):
    """Selected positions for the query at position ``pos`` (causal: keys 0..pos).

    Causality: only preceding tokens are candidates ([blog] section "Lightning
    indexer", Step 1; [news] bullet 闪电索引器). Readings: the query token itself
    is a candidate (s <= pos); with fewer than k candidates all pos+1 are
    selected. Returns (idx int64 in
    rank order, scores of keys 0..pos).
    """
    if pos < 0:
        return np.zeros(0, dtype=np.int64), np.zeros(0)
    q = decode_e4m3(q_codes, np.full(q_codes.shape[0], q_scale))
    w = decode_bf16(w_bits)
    k = decode_e4m3(k_codes[: pos + 1], k_scale[: pos + 1])
    scores = index_scores(q, w, k)
    return select_topk(scores, topk).astype(np.int64), scores


def sparse_mla_attn_row(q_bits, kv_bits, idx, d_v: int, tau: float):
    """Attention for one query over the rows named in ``idx`` (entries < 0 are padding)."""
    sel = np.asarray(idx, dtype=np.int64)
    sel = sel[sel >= 0]
    return sparse_mla_attention(decode_bf16(q_bits), decode_bf16(kv_bits[sel]), d_v, tau)


def dsa_row(q_codes, q_scale, w_bits, k_codes, k_scale, q_bits, kv_bits, pos, topk, d_v, tau):
    """The whole forward path for one query: indexer -> top-k -> sparse MLA attention."""
    idx, scores = indexer_topk_row(q_codes, q_scale, w_bits, k_codes, k_scale, pos, topk)
    out, lse = sparse_mla_attn_row(q_bits, kv_bits, idx, d_v, tau)
    return idx, out, lse, scores


# ----------------------------------------------------------------------------- indexer alignment loss
def attention_head_sum_target(q_t: np.ndarray, kv_rows: np.ndarray, tau: float) -> np.ndarray:
    """Target distribution of the indexer-alignment loss for one query token.

    a[s] = sum_h softmax_s(tau * q[h] . kv[s]) over the rows given, then p = a / sum_s a[s].

    [blog] section "訓練", Step 1 (dense warm-up): for the t-th query token the main
    attention scores are summed over all heads and the sum is L1-normalised along the
    sequence, giving the target distribution; [news] bullet 密集预热阶段 (sum, then L1
    normalisation along the sequence dimension). Reading: the "attention scores" are the
    softmax weights of each head (logits summed over heads could be negative and have no
    L1-normalised distribution); the logits are those of the MQA-mode attention, all
    d_qk dims of the shared latent row, scaled by tau.

    q_t: [H, d_qk]; kv_rows: [m, d_qk] (m >= 1)  ->  [m], summing to 1
    """
    z = tau * (q_t @ kv_rows.T)               # [H, m]
    e = np.exp(z - z.max(axis=1, keepdims=True))
    a = (e / e.sum(axis=1, keepdims=True)).sum(axis=0)   # sum over heads of each head's weights
    return a / np.abs(a).sum()                # L1 normalisation along the sequence


def indexer_kl(p: np.ndarray, scores: np.ndarray) -> float:
    """KL(p || softmax(scores)) = sum_s p[s] * (ln p[s] - ln softmax(scores)[s]), 0 ln 0 = 0.

    [blog] section "訓練", Step 1: a KL-divergence loss between the target distribution and
    the indexer's output is the indexer's training objective; the indexer's distribution is
    the softmax of its index scores over the same positions. [news] bullet 密集预热阶段
    (KL散度损失). Natural logarithm.
    """
    m = scores.max()
    log_q = scores - (m + np.log(np.exp(scores - m).sum()))
    nz = p > 0
    return float(np.sum(p[nz] * (np.log(p[nz]) - log_q[nz])))


def indexer_kl_row(q_bits, kv_bits, idx, index_scores_sel, tau: float) -> float:
    """The loss term of one query over the positions in ``idx`` (entries < 0 are padding).

    Sparse training stage: [blog] section "訓練", Step 2, and [news] bullet 稀疏训练阶段 --
    the indexer stays aligned with the main attention distribution, but only over the
    selected token set S_t. Readings: in that stage the main attention attends to S_t only,
    so its per-head weights are the softmax over S_t (the weights the sparse attention
    uses), and the indexer's distribution is the softmax of its scores over S_t. Passing all
    positions 0..t as ``idx`` gives the dense warm-up term. ``index_scores_sel[j]`` is the
    index score of position idx[j] (same order; padding entries ignored). With no valid
    position the term is 0.
    """
    idx = np.asarray(idx, dtype=np.int64)
    keep = idx >= 0
    sel = idx[keep]
    if sel.size == 0:
        return 0.0
    p = attention_head_sum_target(decode_bf16(q_bits), decode_bf16(kv_bits[sel]), tau)
    return indexer_kl(p, np.asarray(index_scores_sel, dtype=np.float64)[keep])


# ----------------------------------------------------------------------------- masked dense mode
def masked_dense_mqa_attention(q_t: np.ndarray, kv_prefix: np.ndarray, mask: np.ndarray, d_v: int, tau: float):
    """Dense attention of one query over every row of ``kv_prefix`` (positions 0..pos), with the
    logits of rows where ``mask`` is False set to -inf before the softmax.

    [news] bullet 实际服务部署: for short-sequence prefill the deployment uses a masked mode that
    emulates the effect of DSA. Reading: the mask is the top-k selection of the query, so the
    result equals the attention over the selected rows (MQA mode, as in
    ``sparse_mla_attention``), computed densely over the causal prefix. With no row unmasked:
    out = 0, lse = -inf.

    q_t: [H, d_qk]; kv_prefix: [pos+1, d_qk]; mask: [pos+1] bool  ->  out [H, d_v], lse [H]
    """
    H = q_t.shape[0]
    mask = np.asarray(mask, dtype=bool)
    if not mask.any():
        return np.zeros((H, d_v)), np.full(H, -np.inf)
    z = tau * (q_t @ kv_prefix.T)             # [H, pos+1], every causal row
    z = np.where(mask[None, :], z, -np.inf)
    zmax = z.max(axis=1)
    e = np.exp(z - zmax[:, None])             # exp(-inf) = 0 for masked rows
    l = e.sum(axis=1)
    out = (e @ kv_prefix[:, :d_v]) / l[:, None]
    return out, zmax + np.log(l)
