/*
 * dsa.h -- C ABI of the DeepSeek Sparse Attention (DSA) forward path for NVIDIA B200 (sm_100a).
 *
 * The path has three stages, restated from web summaries of the DeepSeek-V3.2-Exp report
 * ("節前發版：Deepseek v3.2 exp", sections "Lightning indexer" Step 1 / Step 2 and
 * "在MLA下實例化DSA"; "DeepSeek 发布新模型 V3.2-Exp：基于DSA稀疏注意力机制的长上下文优化",
 * bullets 闪电索引器 / 细粒度Token选择机制 / MLA架构集成):
 *
 *   1. lightning indexer: for query token t and every preceding token s <= pos(t),
 *        I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s])      (few heads j, FP8 inputs)
 *   2. fine-grained selection: the k positions with the largest I[t,.] (k = 2048 in the pages)
 *   3. attention of the query's heads over the selected tokens only, in MLA's MQA mode:
 *      one latent row per token (512-d compressed latent | 64-d RoPE part) is the key of
 *      every head, and its first d_latent dims are the value.
 *
 * Conventions (all calls):
 *  - Every tensor pointer is DEVICE memory owned by the caller, contiguous row-major, in the
 *    layout stated beside it. The library allocates no memory and never frees caller memory.
 *  - Calls are asynchronous on `stream`. Errors the host can see (bad sizes, null or
 *    misaligned pointers, a too-small workspace, unsupported dims) return before any launch.
 *    Errors found on the device (a time-bounded wait that ran out, an index outside
 *    [0, max_len)) are written into the status word at the start of `ws` and read back with
 *    dsa_get_device_status(), which also clears them.
 *  - Query i of sequence b sits at position pos = lengths[b] - n_q + i (prefill: n_q = max_len
 *    = L, so pos = i; decode: n_q = 1, so pos = lengths[b] - 1). A query attends to positions
 *    0..pos of its own sequence (causal, the token itself included). Queries with pos < 0
 *    select nothing.
 *  - Supported dims: n_idx_heads <= 64, idx_dim <= 128 (multiple of 16), n_heads <= 128,
 *    d_latent <= 512 (multiple of 8), d_rope <= 64 (multiple of 8), 1 <= topk <= 2048.
 *    The production dims (64, 128, 128, 512, 64) run directly; smaller ones are zero-padded
 *    to them inside the workspace (exact: padded heads have weight 0, padded dims are 0).
 *    Anything else returns DSA_ERR_UNSUPPORTED.
 *  - One workspace may not be used by two calls that overlap on the device.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dsa_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, negative size, n_q > max_len, ... */
  DSA_ERR_UNSUPPORTED = 2,    /* dims outside the supported set, or no sm_100 device */
  DSA_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed (launch, memset, ...) */
  DSA_ERR_DEVICE_TIMEOUT = 4, /* device: a bounded wait inside a kernel ran out */
  DSA_ERR_INDEX_RANGE = 5,    /* device: an index outside [0, max_len) reached the attention */
  DSA_ERR_WORKSPACE = 6       /* ws is NULL, misaligned or smaller than dsa_workspace_bytes() */
} dsa_status;

/* Problem dims. Prefill: n_q = max_len = L. Decode: n_q = 1, max_len = cache capacity. */
typedef struct {
  int32_t batch;         /* B, sequences */
  int32_t n_q;           /* queries per sequence (the last n_q positions of each sequence) */
  int32_t max_len;       /* key/cache rows per sequence (row stride of k_idx and latent_kv) */
  int32_t n_idx_heads;   /* H_I, indexer heads (64 in the workloads) */
  int32_t idx_dim;       /* d_I, indexer head dim (128) */
  int32_t n_heads;       /* H, attention heads sharing one latent row (128) */
  int32_t d_latent;      /* d_c, compressed latent = value dim (512) */
  int32_t d_rope;        /* d_r, decoupled RoPE part of the key (64) */
  float softmax_scale;   /* tau, multiplies q . kv before the softmax (1/sqrt(d_c+d_r)) */
} dsa_dims;

/* Bytes of workspace the calls below need for these dims and top-k (256-byte aligned
 * pointer required). Returns 0 for invalid dims. Pure host function. */
size_t dsa_workspace_bytes(const dsa_dims* dims, int32_t topk);

/* Zeroes the status word at the start of `ws` (asynchronously on `stream`). Call once
 * after allocating a workspace; dsa_get_device_status() clears it afterwards. */
dsa_status dsa_workspace_init(void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Stages 1+2: lightning-indexer scores and the causal top-k per query.
 *   q_idx   FP8 E4M3 [B, n_q, n_idx_heads, idx_dim]      (16-byte aligned)
 *   w       bf16     [B, n_q, n_idx_heads]               per-query head weights
 *   k_idx   FP8 E4M3 [B, max_len, idx_dim]               (16-byte aligned)
 *   scales  fp32     [B*n_q] q scales, then [B*max_len] k scales: the real value of an FP8
 *           code is code * scale of its token. Scales must be positive and finite.
 *   lengths int32    [B] valid keys per sequence, 0 <= lengths[b] <= max_len (device memory)
 *   out_idx int32    [B, n_q, topk]: positions s <= pos of the min(topk, pos+1) largest
 *           scores of each query, in unspecified order, then -1 padding. Ties between equal
 *           scores go to the lower position.
 * Prefill (n_q > 1) never stores the L x L score matrix: scores stream from the tensor cores
 * into a running per-query selection in shared memory. Decode (n_q = 1) with max_len <= 131072
 * writes each sequence's single score row (4 B per key) to the workspace and selects from it;
 * longer decode rows keep a partial top-k per 8192-key chunk in the workspace and merge them.
 */
dsa_status dsa_indexer_topk(const dsa_dims* dims, const void* q_idx, const void* w, const void* k_idx,
                            const float* scales, const int32_t* lengths, int32_t topk, int32_t* out_idx,
                            void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * dsa_indexer_topk that also returns the index score of every selected position:
 *   out_scores fp32 [B, n_q, topk]  out_scores[b,i,j] = I[t, out_idx[b,i,j]] as the kernel computed
 *              it in fp32 from the decoded inputs (scales applied); -inf where out_idx is -1.
 * out_scores may be NULL (then identical to dsa_indexer_topk). The scores feed the indexer's
 * alignment loss (dsa_indexer_kl_loss).
 */
dsa_status dsa_indexer_topk_scores(const dsa_dims* dims, const void* q_idx, const void* w, const void* k_idx,
                                   const float* scales, const int32_t* lengths, int32_t topk, int32_t* out_idx,
                                   float* out_scores, void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Stage 3: sparse MLA attention (MQA mode) over the selected rows.
 *   q         bf16  [B, n_q, n_heads, d_latent + d_rope]  (16-byte aligned)
 *   latent_kv bf16  [B, max_len, d_latent + d_rope]       (16-byte aligned) one row per token
 *   idx       int32 [B, n_q, topk] positions in the query's own sequence; entries < 0 are
 *             padding and are skipped wherever they appear; entries >= max_len are skipped
 *             and reported as DSA_ERR_INDEX_RANGE. Duplicates are attended twice.
 *   out       bf16  [B, n_q, n_heads, d_latent]  softmax(tau * q . kv) weighted sum of the
 *             rows' first d_latent dims, per head
 *   lse       fp32  [B, n_q, n_heads]  natural-log log-sum-exp of tau * q . kv (-inf, with
 *             out = 0, for a query with no valid index)
 */
dsa_status dsa_sparse_mla_attn(const dsa_dims* dims, const void* q, const void* latent_kv, const int32_t* idx,
                               int32_t topk, void* out, float* lse, void* ws, size_t ws_bytes,
                               dsa_stream_t stream);

/*
 * Stage 3 in the masked dense mode, for short prefill: the same result as dsa_sparse_mla_attn
 * (same arguments and layouts), computed as dense attention of each query over its positions
 * 0 .. e-1 (e = one past its last valid index) with every position the index row does not
 * list masked out. "DeepSeek 发布新模型 V3.2-Exp：基于DSA稀疏注意力机制的长上下文优化", bullet
 * 实际服务部署: short-sequence prefill uses a masked mode that emulates DSA. The key rows are
 * read as whole 64-row blocks (TMA tile copies) instead of gathered row by row.
 * Differences from dsa_sparse_mla_attn: a position listed twice is attended once; every latent
 * row the blocks touch (positions 0 .. 64*ceil(e/64)-1 of the query's sequence) must hold
 * finite values, since a masked row still enters the weighted sum with weight zero.
 * Requires max_len <= 16384 (else DSA_ERR_UNSUPPORTED). Uses workspace for one bitmap row per
 * query (included in dsa_workspace_bytes for such dims).
 */
dsa_status dsa_masked_mqa_attn(const dsa_dims* dims, const void* q, const void* latent_kv, const int32_t* idx,
                               int32_t topk, void* out, float* lse, void* ws, size_t ws_bytes,
                               dsa_stream_t stream);

/*
 * Forward of the indexer-alignment loss, one term per query. "節前發版：Deepseek v3.2 exp",
 * section "訓練", Step 1 / Step 2, and "DeepSeek 发布新模型 V3.2-Exp：...", bullets 密集预热阶段
 * / 稀疏训练阶段: the target distribution sums the main attention over all heads and
 * L1-normalises it along the sequence; the loss is the KL divergence from it to the softmax of
 * the index scores, both over the query's selected entries in the sparse stage:
 *   a_s = sum_h exp(tau * q_h . kv_s - lse_h),  p_s = a_s / sum_s a_s,
 *   loss[t] = sum_s p_s * (ln p_s - ln softmax_s(I_s))          (natural log)
 * over the valid entries s of idx[t] (< 0 padding; >= max_len reported as DSA_ERR_INDEX_RANGE
 * and skipped). Passing every position 0..t of a query (topk >= t+1) gives the dense warm-up term.
 *   q, latent_kv, idx  as for dsa_sparse_mla_attn
 *   idx_scores  fp32 [B, n_q, topk]  the index score of each entry (dsa_indexer_topk_scores)
 *   lse         fp32 [B, n_q, n_heads]  the lse output of dsa_sparse_mla_attn on the same idx
 *   loss        fp32 [B, n_q]  the per-query term (0 for a query with no valid entry); the
 *               training objective is its sum over the queries.
 */
dsa_status dsa_indexer_kl_loss(const dsa_dims* dims, const void* q, const void* latent_kv, const int32_t* idx,
                               const float* idx_scores, const float* lse, int32_t topk, float* loss, void* ws,
                               size_t ws_bytes, dsa_stream_t stream);

/*
 * The whole forward path: dsa_indexer_topk then dsa_sparse_mla_attn on the same stream.
 * out_idx may be NULL, in which case the selection lives only in the workspace.
 */
dsa_status dsa_forward(const dsa_dims* dims, const void* q_idx, const void* w, const void* k_idx,
                       const float* scales, const int32_t* lengths, int32_t topk, const void* q,
                       const void* latent_kv, int32_t* out_idx, void* out, float* lse, void* ws,
                       size_t ws_bytes, dsa_stream_t stream);

/*
 * Decode selection without a workspace, for callers that cannot allocate device memory
 * for a call (serving runtimes that plan every buffer ahead and forbid allocation on the
 * request path, plugin interfaces that pass a kernel only its inputs and outputs, loops
 * where cudaMalloc's implicit synchronisation is not acceptable). The pages have no
 * counterpart: this is a deployment variant of dsa_indexer_topk for n_q = 1.
 *
 * Same inputs, output and selection rule as dsa_indexer_topk with n_q = 1 and the
 * production dims (64 indexer heads of dim 128). Its scratch -- the exact top-k list of
 * every (sequence, 8192-key chunk) pair before the merge -- lives in a file-scope device
 * array of the library (16 MiB + 4 KiB, held by every GPU that loads the library until the
 * process exits), so the call allocates nothing and needs no workspace.
 *   status  optional device pointer to 2 uint32 words: a device-side error (see dsa_status)
 *           is recorded there, first error wins; the caller zeroes and reads it. May be NULL,
 *           but then a device-side error goes unreported: after a bounded wait that ran out,
 *           the selection of the sequences that were not finished is incomplete without notice.
 * Limits: batch * ceil(max_len / 8192) <= 1024 and topk <= 2048, else DSA_ERR_UNSUPPORTED
 * (also for n_q != 1 or other dims). The first call on a device looks up the array's device
 * address; make that first call before any stream capture. All calls on one device share
 * the one array: two calls whose executions overlap on the GPU (for example on different
 * streams) race and corrupt each other's results.
 */
dsa_status dsa_indexer_topk_decode_noalloc(const dsa_dims* dims, const void* q_idx, const void* w,
                                           const void* k_idx, const float* scales, const int32_t* lengths,
                                           int32_t topk, int32_t* out_idx, uint32_t* status, dsa_stream_t stream);

/* Synchronises `stream`, returns the first device-side error recorded in `ws` since the
 * last call (DSA_OK if none) and clears it. `detail`, if non-NULL, receives a location tag. */
dsa_status dsa_get_device_status(void* ws, dsa_stream_t stream, uint32_t* detail);

/*
 * Test setting for failure detection: the time budget of every bounded wait in the indexer's
 * pipeline (dsa_indexer_topk*, forward's first stage), in ns; 0 restores the default of 2 s.
 * Process-wide, read at each launch. With a budget too short for the pipeline's handshakes a
 * launch stops early: its waits record DSA_ERR_DEVICE_TIMEOUT in the status word, every role
 * ends, the teardown still lets in-flight copies and MMAs land (under their own fixed budget),
 * and the selection written is incomplete. Not for production use.
 */
dsa_status dsa_set_wait_budget_ns(uint64_t ns);

/* Static description of a status code. Never NULL. */
const char* dsa_status_string(dsa_status status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
