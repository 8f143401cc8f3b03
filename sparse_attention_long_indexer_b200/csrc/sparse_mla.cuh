// Sparse MLA attention in MQA mode over the selected latent rows, for sm_100a.
//
// For one query token t with H = 128 heads and its selected rows S_t (from the indexer):
//   z[h,s] = tau * q[t,h,:] . kv[s,:]    (576 = 512 latent + 64 RoPE dims)
//   out[t,h,:] = sum_s softmax_s(z[h,.]) * kv[s, :512],   lse[t,h] = ln sum_s exp z[h,s]
// ("節前發版：Deepseek v3.2 exp", section "Lightning indexer" Step 2 and section
// "在MLA下實例化DSA": attention runs only over the selected entries, and in MLA's MQA mode
// every query head shares the one latent vector of each token).
//
// B200 design. The fp32 output accumulator of one query (128 heads x 512 dims) is 256 KB,
// all of one SM's tensor memory, so each query runs on a pair of CTAs (a 2-CTA cluster) and
// every product is a 2-SM tcgen05 MMA (cta_group::2) issued from the even CTA:
//  * logits: M = 128 heads (CTA r supplies heads 64r..64r+63), N = 64 selected rows (CTA r
//    supplies block rows 32r..32r+31), K = 576. The hardware shares the halves and each CTA
//    receives the logits of its own 64 heads for all 64 rows, folded in TMEM as 128 lanes x
//    32 columns (lane m: rows 0..31 of head m, lane 64+m: rows 32..63); three such buffers.
//    Dims 0..319 of Q come from TMEM (A operand, duplicated over both lane halves), dims
//    320..575 from shared memory.
//  * output: M = 128 heads, N = 256 latent dims per instruction (two instructions), K = 64
//    rows: A = P (bf16, this CTA's heads, two buffers) in shared memory, B = the rows' latent
//    dims with CTA r supplying dims 256i + 128r .. +127. Each CTA accumulates all 512 dims of
//    its 64 heads (TMEM: 256 columns; lane m / 64+m hold the low / high 128 dims of each
//    instruction).
//  * per 64-row block, CTA r gathers its 32 rows completely (logits operand, a 3-stage ring
//    freed by the logits MMA) and all 64 rows' dims it supplies to the output product (a
//    2-stage ring freed by the output MMA), with 16-byte cp.async into 128-byte-swizzled
//    stages; two groups of four producer warps run the two rings independently. Rows are
//    read straight from the query's index row, one block ahead; padding and out-of-range
//    entries are gathered as zero rows and masked in the softmax.
//  * softmax: one thread per TMEM lane holds half a row (32 logits); the two halves of a row
//    exchange their maxima through tagged 64-bit shared-memory words; online softmax in the log2 domain, the
//    output rescaled only when the running max grows by more than 32 (exact: the final
//    normalisation uses the same max). P is announced with a CTA-scope arrive; the odd CTA's
//    announcements reach the even CTA through one relay thread.
//  * two issuing threads share the tensor pipe: one for the logits MMAs, one for the output
//    MMAs; the output thread hands a logits buffer back once it has seen that block's P, so
//    the logits -> softmax -> P -> logits loop spans three blocks.
// Nothing crosses between the two CTAs except through the 2-SM MMAs themselves; the pair
// synchronises through mbarriers of the even CTA (remote arrives) and commits that the MMA
// threads address to both CTAs.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dsa {

constexpr int kHeads = 128;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kBlk = 64;                 // selected rows per block
constexpr int kMaxTopk = 2048;
// The running max m2 (log2 domain) is raised, and O rescaled, only when a block's max exceeds it
// by more than this. Until then P = 2^(z - m2) <= 2^32: bf16 P and the fp32 O and row sum have
// the exponent range of fp32, so nothing overflows unless |kv| > 2^80, and the final
// normalisation divides by the row sum taken against the same m2, so the result is unchanged.
// A rescale waits for the previous block's output MMAs, a stall of the whole pipeline, so it
// should be rare: with a bound of 8, random logits with a spread of several units trigger it in
// a sizeable fraction of blocks for some warp.
constexpr float kLazyRescale = 32.0f;

struct AttnCfg {
  static constexpr int SB_STAGES = 3;                    // own rows, all dims (logits operand)
  static constexpr int VR_STAGES = 2;                    // all rows, this CTA's output dims
  static constexpr int SB_ATOM = 32 * 128;               // 32 rows x 128 B
  static constexpr int SB_BYTES = 9 * SB_ATOM;           // own 32 rows x 576 dims
  static constexpr int VR_ATOM = kBlk * 128;             // 64 rows x 128 B
  static constexpr int VR_BYTES = 4 * VR_ATOM;           // 64 rows x this CTA's 256 output dims
  static constexpr int Q_TMEM_DIMS = 320;                // dims 0..319 of q in TMEM, the rest in smem
  static constexpr int QS_ATOMS = (kDqk - Q_TMEM_DIMS) / 64;
  static constexpr int QS_BYTES = QS_ATOMS * 64 * 128;   // 64 heads x dims 384..575
  static constexpr int P_BYTES = 64 * 128;               // 64 heads x 64 rows bf16
  static constexpr int P_BUFS = 2;                       // P of consecutive blocks (1 or 2)
  static constexpr int S_BUFS = 3;                       // TMEM logits buffers
  static constexpr int SOFTMAX_WARPS = 4;
  static constexpr int PRODUCER_WARPS = 8;               // 4 gather the logits ring, 4 the output ring
  static constexpr int GROUP_WARPS = PRODUCER_WARPS / 2;
  static constexpr int GROUP_THREADS = GROUP_WARPS * 32;
  static constexpr int MMA_WARP = SOFTMAX_WARPS + PRODUCER_WARPS;   // logits MMAs (and TMEM owner)
  static constexpr int PV_WARP = MMA_WARP + 1;                       // output MMAs
  static constexpr int THREADS = (PV_WARP + 1) * 32;
  // TMEM columns
  static constexpr uint32_t COL_O = 0, COL_S = 256, COL_Q = COL_S + 32 * S_BUFS, TMEM_COLS = 512;
  // shared memory
  static constexpr int OFF_SB = 0;
  static constexpr int OFF_VR = OFF_SB + SB_STAGES * SB_BYTES;
  static constexpr int OFF_QS = OFF_VR + VR_STAGES * VR_BYTES;
  static constexpr int OFF_P = OFF_QS + QS_BYTES;
  static constexpr int OFF_XMAX = OFF_P + P_BUFS * P_BYTES;        // 2 x 128 tagged words
  static constexpr int OFF_SCAN = OFF_XMAX + 2 * 128 * 8;
  static constexpr int OFF_INFO = OFF_SCAN + 64;
  static constexpr int OFF_BAR = OFF_INFO + 16;
  static constexpr int NUM_BARS = 45;                    // 40..44: masked-mode copy barriers
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(OFF_VR % 1024 == 0 && OFF_QS % 1024 == 0 && OFF_P % 1024 == 0, "swizzle atoms");
  static_assert(SB_BYTES % 1024 == 0 && Q_TMEM_DIMS / 2 + COL_Q <= TMEM_COLS, "layout");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(P_BUFS == 1 || P_BUFS == 2, "P buffers");
  static_assert(SB_STAGES <= 4 && VR_STAGES <= 4 && S_BUFS <= 3, "barrier slots");
  static_assert(SB_STAGES <= 3 && VR_STAGES <= 2, "masked-mode copy barriers");
};

// Masked dense mode: the longest key range whose attended positions fit the bitmap (see
// mask_rows_kernel) and the words of a bitmap row.
constexpr int kMaskMaxLen = 16384;
constexpr int kMaskMaxWords = kMaskMaxLen / 32;

struct AttnParams {
  const __nv_bfloat16* q;      // [B*n_q, 128, 576]
  const __nv_bfloat16* kv;     // [B, max_len, 576]
  const int32_t* idx;          // [B*n_q, topk]
  __nv_bfloat16* out;          // [B*n_q, 128, 512]
  float* lse;                  // [B*n_q, 128]
  uint32_t* status;
  int32_t n_q, max_len, topk, n_queries;
  float scale_log2;            // tau * log2(e)
  uint64_t wait_budget_ns;
  // masked dense mode: attended positions as a bitmap per query, and one past the last of them
  const uint32_t* mask;        // [B*n_q, mask_words]
  const int32_t* extent;       // [B*n_q]
  int32_t mask_words;
};

// Masked dense mode, first step: the attended positions of each query as a bitmap of `words`
// words (bit s%32 of word s/32), and one past the last of them. One CTA per query. Entries < 0
// are padding; entries >= max_len are reported (DSA_ERR_INDEX_RANGE) and ignored; a position
// listed twice is attended once.
__global__ void __launch_bounds__(256) mask_rows_kernel(const int32_t* __restrict__ idx, int32_t topk,
                                                        int32_t max_len, int32_t words, uint32_t* __restrict__ mask,
                                                        int32_t* __restrict__ extent, uint32_t* status) {
  __shared__ uint32_t bm[kMaskMaxWords];
  __shared__ int32_t last;
  const int32_t qi = blockIdx.x;
  for (int32_t w = threadIdx.x; w < words; w += blockDim.x) bm[w] = 0u;
  if (threadIdx.x == 0) last = -1;
  __syncthreads();
  const int32_t* row = idx + static_cast<size_t>(qi) * topk;
  int32_t mx = -1;
  for (int32_t j = threadIdx.x; j < topk; j += blockDim.x) {
    const int32_t v = __ldg(row + j);
    if (v >= max_len) {
      record_error(status, DSA_ERR_INDEX_RANGE, static_cast<uint32_t>(qi));
    } else if (v >= 0) {
      atomicOr(&bm[v >> 5], 1u << (v & 31));
      mx = max(mx, v);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) atomicMax(&last, mx);
  __syncthreads();
  uint32_t* out = mask + static_cast<size_t>(qi) * words;
  for (int32_t w = threadIdx.x; w < words; w += blockDim.x) out[w] = bm[w];
  if (threadIdx.x == 0) extent[qi] = last + 1;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void attn_drain_wait(uint32_t bar, uint32_t parity, uint64_t budget_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > budget_ns) return;
  }
}

// 2-SM MMAs (issued by one thread of the even CTA; operands at the same shared-memory
// offsets / TMEM columns in both CTAs) and commits to an mbarrier of either CTA.
__device__ __forceinline__ void mma2_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
               ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void mma2_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
               ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void commit2(uint32_t bar_cluster_addr) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster_addr)
               : "memory");
}

// kDense: the masked dense mode. Block b of a query is then its positions 64b .. 64b+63, loaded
// whole by TMA tile copies (map_kv_a: boxes of 32 rows, map_kv_b: boxes of 64 rows, both over the
// latent cache as [B * max_len rows, 576 dims]), and the softmax masks the positions that are not
// in the query's bitmap; blocks run up to the query's extent (one past its last attended position).
template <bool kDense>
__global__ void __launch_bounds__(AttnCfg::THREADS, 1) __cluster_dims__(2, 1, 1)
sparse_mla_attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kv_a,
                       const __grid_constant__ CUtensorMap map_kv_b, const AttnParams p) {
  using C = AttnCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* xmax = reinterpret_cast<uint64_t*>(smem + C::OFF_XMAX);
  int32_t* scan = reinterpret_cast<int32_t*>(smem + C::OFF_SCAN);
  int32_t* info = reinterpret_cast<int32_t*>(smem + C::OFF_INFO);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto B = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  // local barriers (both CTAs)
  auto info_full = [&](int i) { return B(0 + i); };
  auto info_empty = [&](int i) { return B(2 + i); };
  // ring barriers: stages 0..2 / 0..1 in their first slots, further stages in free slots
  auto sb_empty = [&](int s) { return s < 3 ? B(4 + s) : B(15); };         // commit: logits stage consumed
  auto vr_empty = [&](int s) { return s < 2 ? B(7 + s) : B(12 + (s - 2)); };  // commit: output stage consumed
  const uint32_t q_tma = B(9);                           // this CTA's smem part of q landed (TMA)
  const uint32_t q_empty = B(10);                        // commit: all logits MMAs of a query done
  auto s_full = [&](uint32_t i) { return B(31 + i); };   // commit: logits buffer i ready (3)
  auto p_empty = [&](uint32_t j) { return B(34 + j); };  // commit: output MMA that read P buffer j done (2)
  const uint32_t o_full = B(14);                         // commit: all output MMAs of a query done
  // barriers of the even CTA, arrived on by both CTAs
  auto sb_full2 = [&](int s) { return s < 3 ? B(19 + s) : B(16); };
  auto vr_full2 = [&](int s) { return s < 2 ? B(22 + s) : B(25 + (s - 2)); };
  const uint32_t q_full2 = B(24);
  // logits buffer i free again: arrived by the output-MMA thread once it has seen the P of the
  // block that used the buffer (the softmax reads the logits before it writes P)
  auto s_free = [&](uint32_t i) { return B(36 + i); };
  // P buffer j announced (one barrier per buffer: a warp may announce the next block before a
  // slower one has announced this one)
  auto p_full2 = [&](uint32_t j) { return j ? B(39) : B(27); };   // even CTA: its softmax warps + relay
  auto pbuf_of = [](uint32_t n) { return n % static_cast<uint32_t>(C::P_BUFS); };        // P buffer of block n
  auto puse_of = [](uint32_t n) { return (n / static_cast<uint32_t>(C::P_BUFS)) & 1u; }; // parity of its use
  auto p_local = [&](uint32_t j) { return j ? B(11) : B(30); };   // odd CTA: its softmax warps
  const uint32_t o_empty2 = B(28);
  const uint32_t mma_done = B(29);
  // masked dense mode: a stage's TMA copies landed in this CTA (local, one expect_tx arrive)
  auto sb_tma = [&](uint32_t s) { return B(40 + static_cast<int>(s)); };
  auto vr_tma = [&](uint32_t s) { return B(43 + static_cast<int>(s)); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(info_full(i), 1);
      // softmax warps + output-ring producer warps (+ the MMA thread in the even CTA)
      mbar_init(info_empty(i), C::SOFTMAX_WARPS + C::GROUP_WARPS + (leader ? 2 : 1));
    }
    for (int i = 0; i < C::VR_STAGES; ++i) {
      mbar_init(vr_empty(i), 1);
      mbar_init(vr_full2(i), 2 * C::GROUP_WARPS);
    }
    for (int i = 0; i < C::SB_STAGES; ++i) {
      mbar_init(sb_empty(i), 1);
      mbar_init(sb_full2(i), 2 * C::GROUP_WARPS);
    }
    mbar_init(q_tma, 1);
    mbar_init(q_empty, 1);
    for (uint32_t i = 0; i < static_cast<uint32_t>(C::S_BUFS); ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), 1);
    }
    for (uint32_t j = 0; j < static_cast<uint32_t>(C::P_BUFS); ++j) mbar_init(p_empty(j), 1);
    mbar_init(o_full, 1);
    mbar_init(q_full2, 2 * (1 + C::GROUP_WARPS));
    for (uint32_t j = 0; j < static_cast<uint32_t>(C::P_BUFS); ++j) {
      mbar_init(p_full2(j), C::SOFTMAX_WARPS + 1);
      mbar_init(p_local(j), C::SOFTMAX_WARPS);
    }
    mbar_init(o_empty2, 2 * C::SOFTMAX_WARPS);
    mbar_init(mma_done, 2);
    for (uint32_t i = 0; i < 3u; ++i) mbar_init(sb_tma(i), 1);
    for (uint32_t i = 0; i < 2u; ++i) mbar_init(vr_tma(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (uint32_t i = threadIdx.x; i < 256u; i += blockDim.x) xmax[i] = 0;   // exchange numbers start at 1
  if (warp == C::MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // both CTAs' barriers and TMEM exist before any remote traffic
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter wt{p.status, abort_flag, p.wait_budget_ns, 2u};
  const int32_t ncl = static_cast<int32_t>(nclusters_x());
  const int32_t cid = static_cast<int32_t>(cluster_id_x());
  // cluster address of the even CTA's copy of a local barrier (arrives from either CTA)
  const uint32_t lead_off = mapa(bar0, 0) - bar0;
  auto at_leader = [&](uint32_t local_bar) { return local_bar + lead_off; };

  if (warp >= C::SOFTMAX_WARPS && warp < C::MMA_WARP) {
    // ================================================================ producers
    // Group A (warps 4..7, one per TMEM lane quarter): index compaction, the q operand (TMA
    // part, and the TMEM part in both lane halves), and the logits ring (this CTA's 32 rows of
    // each block, all dims). Group B (warps 8..11): the output ring (all 64 rows of each block,
    // the 256 output dims this CTA supplies).
    // Each group waits for its own copies (cp.async.wait_group, one group behind) and
    // announces a stage to the even CTA per warp; the rings are independent, so a stage is
    // announced without waiting for the other ring (no cycle through the MMA order).
    const uint32_t ptid = threadIdx.x - C::SOFTMAX_WARPS * 32;
    const uint32_t pw = ptid >> 5;                     // producer warp 0..7
    const bool group_a = pw < static_cast<uint32_t>(C::GROUP_WARPS);
    const uint32_t gw = pw % C::GROUP_WARPS;           // warp in group = TMEM lane quarter (group A)
    const uint32_t gtid = ptid % C::GROUP_THREADS;
    volatile int32_t* go = scan + 8;
    uint32_t qn = 0, nsync = 0, qq = 0;
    uint32_t st = 0, ph = 0;                            // ring position (this group's ring)
    const uint32_t n_stages = group_a ? C::SB_STAGES : C::VR_STAGES;
    bool ok = true;
    auto gate = [&](uint32_t bar, uint32_t parity, uint32_t tag) -> bool {   // group A only
      if (gtid == 0) go[nsync & 1u] = (wt.wait(bar, parity, tag) && !wt.aborted()) ? 1 : 0;
      named_barrier(2, C::GROUP_THREADS);
      return go[(nsync++) & 1u] != 0;
    };
    auto warp_wait = [&](uint32_t bar, uint32_t parity, uint32_t tag) -> bool {
      uint32_t got = 1;
      if (lane == 0) got = wt.wait(bar, parity, tag) ? 1u : 0u;
      return __shfl_sync(0xffffffffu, got, 0) != 0;
    };
    for (int32_t qi = cid; qi < p.n_queries; qi += ncl, ++qn) {
      const uint32_t slot = qn & 1u, sph = (qn >> 1) & 1u;
      const int32_t* idx_row = p.idx + static_cast<size_t>(qi) * p.topk;
      int32_t total = 0;                                 // extent of the index row (see below)
      if (group_a) {
        if (!gate(info_empty(slot), sph ^ 1u, 10)) break;
        // ---- the extent of the index row: one past its last valid entry. Entries < 0 (padding)
        // and >= max_len (reported) are masked wherever they appear: their rows are gathered as
        // zeros and their logits set to -inf, so blocks are read straight from the index row.
        int32_t last = -1;
        if constexpr (kDense) {
          last = __ldg(p.extent + qi) - 1;                // blocks cover positions 0 .. extent-1
        } else {
          for (int32_t j = static_cast<int32_t>(gtid); j < p.topk; j += C::GROUP_THREADS) {
            const int32_t v = __ldg(idx_row + j);
            if (v >= p.max_len) record_error(p.status, DSA_ERR_INDEX_RANGE, static_cast<uint32_t>(qi));
            if (v >= 0 && v < p.max_len) last = j;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
        if (lane == 0) scan[gw] = last;
        named_barrier(2, C::GROUP_THREADS);
        total = 0;
#pragma unroll
        for (int w = 0; w < C::GROUP_WARPS; ++w) total = max(total, scan[w] + 1);
        if (gtid == 0) {
          info[slot] = total;
          mbar_arrive(info_full(slot));
        }
      } else {
        if (!warp_wait(info_full(slot), sph, 14)) break;
        total = info[slot];
      }
      const int32_t n_blocks = (total + kBlk - 1) / kBlk;
      if (n_blocks > 0 && ok) {
        // ---- the q operand (group A): dims Q_TMEM_DIMS.. by TMA into shared memory (thread 0),
        // dims 0..Q_TMEM_DIMS-1 into this warp's TMEM lane quarter (both lane halves hold the
        // same 64 heads)
        if (!group_a) {
        } else if (warp_wait(q_empty, (qq & 1u) ^ 1u, 12)) {
          if (ptid == 0) {
            mbar_expect_tx(q_tma, C::QS_BYTES);
            for (int a = 0; a < C::QS_ATOMS; ++a)
              tma_load_3d(sbase + C::OFF_QS + a * 8192, &map_q, q_tma, C::Q_TMEM_DIMS + 64 * a,
                          qi * kHeads + 64 * static_cast<int32_t>(rank), 0);
          }
          tc_fence_after();
          const uint32_t hl = gtid & 63u;
          const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(qi) * kHeads + 64 * rank + hl) *
                                                             kDqk);
#pragma unroll 1
          for (int c = 0; c < C::Q_TMEM_DIMS / 32; ++c) {     // 16 columns (32 dims) at a time
            uint32_t r[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 u = __ldg(qsrc + c * 4 + v);
              r[4 * v + 0] = u.x; r[4 * v + 1] = u.y; r[4 * v + 2] = u.z; r[4 * v + 3] = u.w;
            }
            tmem_st16(tmem + ((gw * 32u) << 16) + C::COL_Q + 16 * c, r);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(at_leader(q_full2));
          if (ptid == 0 && wt.wait(q_tma, qq & 1u, 13)) mbar_arrive_cluster(at_leader(q_full2));
        } else {
          ok = false;
        }
        ++qq;
        if constexpr (kDense) {
          // ---- masked dense mode: thread 0 of the group loads each block of its ring with TMA
          // tile copies into the same swizzled layout, then (one stage behind, so that two stages
          // are in flight) announces it to the even CTA for the group's four warps at once
          if (gtid == 0) {
            const int32_t row0 = (qi / p.n_q) * p.max_len;     // the sequence's first cache row
            const uint32_t bytes = group_a ? static_cast<uint32_t>(C::SB_BYTES) : static_cast<uint32_t>(C::VR_BYTES);
            int32_t pend = -1;
            uint32_t pend_ph = 0;
            int32_t inflight[2] = {-1, -1};                      // issued stages not yet waited on
            uint32_t inflight_ph[2] = {0, 0};
            auto land_and_announce = [&](int32_t stage, uint32_t par) -> bool {
              const uint32_t tb = group_a ? sb_tma(stage) : vr_tma(stage);
              if (!wt.wait(tb, par, 15)) return false;
              if (inflight[0] == stage) inflight[0] = -1;
              if (inflight[1] == stage) inflight[1] = -1;
              mbar_arrive_cluster_n(at_leader(group_a ? sb_full2(stage) : vr_full2(stage)),
                                    static_cast<uint32_t>(C::GROUP_WARPS));
              return true;
            };
            for (int32_t b = 0; b < n_blocks && ok; ++b) {
              const uint32_t empty_bar = group_a ? sb_empty(st) : vr_empty(st);
              if (!wt.wait(empty_bar, ph ^ 1u, 11)) { ok = false; break; }
              const uint32_t tb = group_a ? sb_tma(st) : vr_tma(st);
              mbar_expect_tx(tb, bytes);
              if (group_a) {
                const uint32_t dst = sbase + C::OFF_SB + st * C::SB_BYTES;
                const int32_t y = row0 + b * kBlk + 32 * static_cast<int32_t>(rank);
#pragma unroll 1
                for (int a = 0; a < 9; ++a) tma_load_3d(dst + a * C::SB_ATOM, &map_kv_a, tb, 64 * a, y, 0);
              } else {
                const uint32_t dst = sbase + C::OFF_VR + st * C::VR_BYTES;
                const int32_t y = row0 + b * kBlk;
                const int32_t x0 = 128 * static_cast<int32_t>(rank);
                tma_load_3d(dst + 0 * C::VR_ATOM, &map_kv_b, tb, x0 + 0, y, 0);
                tma_load_3d(dst + 1 * C::VR_ATOM, &map_kv_b, tb, x0 + 64, y, 0);
                tma_load_3d(dst + 2 * C::VR_ATOM, &map_kv_b, tb, x0 + 256, y, 0);
                tma_load_3d(dst + 3 * C::VR_ATOM, &map_kv_b, tb, x0 + 320, y, 0);
              }
              if (inflight[0] < 0) { inflight[0] = static_cast<int32_t>(st); inflight_ph[0] = ph; }
              else { inflight[1] = static_cast<int32_t>(st); inflight_ph[1] = ph; }
              if (pend >= 0 && !land_and_announce(pend, pend_ph)) { ok = false; break; }
              pend = static_cast<int32_t>(st);
              pend_ph = ph;
              if (++st == n_stages) { st = 0; ph ^= 1u; }
            }
            if (ok && pend >= 0 && !land_and_announce(pend, pend_ph)) ok = false;
            // after an abort, every issued copy lands before the CTA may leave
            for (int k2 = 0; k2 < 2; ++k2)
              if (inflight[k2] >= 0)
                attn_drain_wait(group_a ? sb_tma(inflight[k2]) : vr_tma(inflight[k2]), inflight_ph[k2],
                                kDrainBudgetNs);
          }
        } else {
          // ---- the ring of this group. Thread (r0, cc) copies 16-byte chunk cc of every 128-byte
          // segment of block rows r0, r0 + GROUP_THREADS/8, ...: the row indices are read once per block and each
          // copy is a constant offset from the row's base, so copies issue back to back.
          const __nv_bfloat16* kv_seq = p.kv + static_cast<size_t>(qi / p.n_q) * p.max_len * kDqk;
          const uint32_t cc = gtid & 7u, r0 = gtid >> 3;
          const int32_t own0 = 32 * static_cast<int32_t>(rank);
          const uint32_t seg0 = 128u * rank;               // group B: segments 2r, 2r+1, 4+2r, 5+2r
          // block row r of block b: its row of the latent cache, or -1 when masked (padding, past the
          // extent, or out of range); read from the index row one block ahead of its gathers
          constexpr int RS = C::GROUP_THREADS / 8;       // rows per pass
          constexpr int NRA = 32 / RS, NRB = kBlk / RS;  // rows per thread: logits ring, output ring
          auto row_of = [&](int32_t b, int32_t r) -> int32_t {
            const int32_t j = b * kBlk + r;
            const int32_t v = j < total ? __ldg(idx_row + j) : -1;
            return (v >= 0 && v < p.max_len) ? v : -1;
          };
          int32_t rows_a[NRA], rows_b[NRB];
          auto load_rows = [&](int32_t b) {
            if (group_a) {
#pragma unroll
              for (int q = 0; q < NRA; ++q) rows_a[q] = row_of(b, own0 + static_cast<int32_t>(r0) + RS * q);
            } else {
#pragma unroll
              for (int q = 0; q < NRB; ++q) rows_b[q] = row_of(b, static_cast<int32_t>(r0) + RS * q);
            }
          };
          load_rows(0);
          int32_t pending = -1;
          auto announce = [&](int32_t stage) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(at_leader(group_a ? sb_full2(stage) : vr_full2(stage)));
          };
          for (int32_t b = 0; b < n_blocks && ok; ++b) {
            const uint32_t empty_bar = group_a ? sb_empty(st) : vr_empty(st);
            if (pending >= 0) {                          // about to wait: announce the last stage first
              uint32_t free_now = 0;
              if (lane == 0) free_now = mbar_test_wait(empty_bar, ph ^ 1u) ? 1u : 0u;
              if (!__shfl_sync(0xffffffffu, free_now, 0)) {
                cp_async_wait<0>();
                announce(pending);
                pending = -1;
              }
            }
            if (!warp_wait(empty_bar, ph ^ 1u, 11)) { ok = false; break; }
            if (group_a) {
              const uint32_t dst0 = sbase + C::OFF_SB + st * C::SB_BYTES + sw128_offset(r0, cc);
#pragma unroll
              for (int q = 0; q < NRA; ++q) {
                const bool v = rows_a[q] >= 0;
                const __nv_bfloat16* src = (v ? kv_seq + static_cast<size_t>(rows_a[q]) * kDqk : p.kv) + cc * 8;
                const uint32_t n = v ? 16u : 0u;
#pragma unroll
                for (int a = 0; a < 9; ++a) cp_async_16(dst0 + q * RS * 128 + a * C::SB_ATOM, src + a * 64, n);
              }
            } else {
              const uint32_t dst0 = sbase + C::OFF_VR + st * C::VR_BYTES + sw128_offset(r0, cc);
#pragma unroll
              for (int q = 0; q < NRB; ++q) {
                const bool v = rows_b[q] >= 0;
                const __nv_bfloat16* src = (v ? kv_seq + static_cast<size_t>(rows_b[q]) * kDqk : p.kv) + seg0 + cc * 8;
                const uint32_t n = v ? 16u : 0u;
                const uint32_t d = dst0 + q * RS * 128;
                cp_async_16(d + 0 * C::VR_ATOM, src + 0, n);
                cp_async_16(d + 1 * C::VR_ATOM, src + 64, n);
                cp_async_16(d + 2 * C::VR_ATOM, src + 256, n);
                cp_async_16(d + 3 * C::VR_ATOM, src + 320, n);
              }
            }
            cp_async_commit();
            if (b + 1 < n_blocks) load_rows(b + 1);
            if (pending >= 0) {
              cp_async_wait<1>();
              announce(pending);
            }
            pending = static_cast<int32_t>(st);
            if (++st == n_stages) { st = 0; ph ^= 1u; }
          }
          cp_async_wait<0>();
          if (pending >= 0) announce(pending);
        }
      }
      if (!group_a) {                                  // info[slot] no longer read by this warp
        __syncwarp();
        if (lane == 0) mbar_arrive(info_empty(slot));
      }
    }
    cp_async_wait<0>();
  } else if (warp == C::MMA_WARP || warp == C::PV_WARP) {
    // ================================================================ MMA issuers (even CTA only)
    // Two threads feed the one tensor pipe so that each one's waits overlap the other's MMAs:
    // warp MMA_WARP issues the logits MMAs, warp PV_WARP the output MMAs. A tcgen05.commit
    // tracks the MMAs of its own thread, so each thread commits only what it issued.
    if (leader && lane == 0) {
      const bool logits = warp == C::MMA_WARP;
      constexpr uint32_t idesc_s = make_idesc(1, 1, 0, 0, 128, kBlk);
      constexpr uint32_t idesc_o = make_idesc(1, 1, 0, 1, 128, 256);
      const uint32_t peer_off = mapa(bar0, 1) - bar0;
      auto commit_both = [&](uint32_t local_bar) {
        commit2(local_bar);
        commit2(local_bar + peer_off);
      };
      uint32_t sst = 0, sph = 0, vst = 0, vph = 0, qn = 0, pb = 0, qq = 0;
      uint32_t s_i = 0, s_u = 0;                         // logits buffer, and its use count
      bool ok = true;
      for (int32_t qi = cid; qi < p.n_queries && ok; qi += ncl, ++qn) {
        const uint32_t slot = qn & 1u, iph = (qn >> 1) & 1u;
        if (!wt.wait(info_full(slot), iph, 20)) break;
        const int32_t total = info[slot];
        mbar_arrive(info_empty(slot));
        const int32_t n_blocks = (total + kBlk - 1) / kBlk;
        if (n_blocks == 0) continue;
        if (logits) {
          if (!wt.wait(q_full2, qq & 1u, 21)) break;
          for (int32_t b = 0; b < n_blocks; ++b) {
            // logits of the next block into TMEM buffer s_i from the next logits stage; the
            // buffer was last written three blocks back and is free once that block's P was seen
            if (!wt.wait(sb_full2(sst), sph, 22)) { ok = false; break; }
            if (!wt.wait(s_free(s_i), (s_u & 1u) ^ 1u, 23)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sbuf = sbase + C::OFF_SB + sst * C::SB_BYTES;
            const uint32_t d = tmem + C::COL_S + 32u * s_i;
#pragma unroll
            for (int j = 0; j < C::Q_TMEM_DIMS / 16; ++j) {      // A from TMEM
              const int dj = 16 * j;
              mma2_ts(d, tmem + C::COL_Q + 8 * j, sw128_desc(sbuf + (dj >> 6) * C::SB_ATOM + (dj & 63) * 2, 1, 1024),
                      idesc_s, j > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int j = C::Q_TMEM_DIMS / 16; j < kDqk / 16; ++j) {   // A from shared memory
              const int dj = 16 * j, dq = dj - C::Q_TMEM_DIMS;
              mma2_ss(d, sw128_desc(sbase + C::OFF_QS + (dq >> 6) * 8192 + (dq & 63) * 2, 1, 1024),
                      sw128_desc(sbuf + (dj >> 6) * C::SB_ATOM + (dj & 63) * 2, 1, 1024), idesc_s, 1u);
            }
            commit_both(s_full(s_i));
            commit_both(sb_empty(sst));
            if (++s_i == static_cast<uint32_t>(C::S_BUFS)) { s_i = 0; ++s_u; }
            if (++sst == C::SB_STAGES) { sst = 0; sph ^= 1u; }
          }
          if (!ok) break;
          commit_both(q_empty);                      // every logits MMA of the query is issued
        } else {
          for (int32_t b = 0; b < n_blocks; ++b) {
            if (!wt.wait(vr_full2(vst), vph, 26)) { ok = false; break; }
            if (!wt.wait(p_full2(pbuf_of(pb)), puse_of(pb), 24)) { ok = false; break; }
            mbar_arrive(s_free(pb % C::S_BUFS));     // the softmax is done with that logits buffer
            if (b == 0 && !wt.wait(o_empty2, (qq & 1u) ^ 1u, 25)) { ok = false; break; }
            tc_fence_after();
            const uint32_t vr = sbase + C::OFF_VR + vst * C::VR_BYTES;
            const uint32_t pbuf = sbase + C::OFF_P + pbuf_of(pb) * C::P_BYTES;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
#pragma unroll
              for (int kk = 0; kk < kBlk / 16; ++kk) {
                mma2_ss(tmem + C::COL_O + 128 * i, sw128_desc(pbuf + kk * 32, 1, 1024),
                        sw128_desc(vr + 2 * i * C::VR_ATOM + kk * 2048, C::VR_ATOM, 1024), idesc_o,
                        (b > 0 || kk > 0) ? 1u : 0u);
              }
            }
            commit_both(vr_empty(vst));
            commit_both(p_empty(pbuf_of(pb)));
            ++pb;
            if (++vst == C::VR_STAGES) { vst = 0; vph ^= 1u; }
          }
          if (!ok) break;
          commit_both(o_full);
        }
        ++qq;
      }
      tc_commit(mma_done);
      attn_drain_wait(mma_done, 0, kDrainBudgetNs);
    } else if (!leader && warp == C::MMA_WARP && lane == 0) {
      // relay of the odd CTA: its softmax warps announce P locally (a CTA-scope arrive does not
      // stall them); this thread observes that (acquire) and forwards one cluster-scope release
      // arrive to the even CTA, which by cumulativity carries the observed P stores
      uint32_t qn = 0, pb = 0;
      for (int32_t qi = cid; qi < p.n_queries; qi += ncl, ++qn) {
        const uint32_t slot = qn & 1u, iph = (qn >> 1) & 1u;
        if (!wt.wait(info_full(slot), iph, 27)) break;
        const int32_t total = info[slot];
        mbar_arrive(info_empty(slot));
        const int32_t n_blocks = (total + kBlk - 1) / kBlk;
        bool ok = true;
        for (int32_t b = 0; b < n_blocks; ++b, ++pb) {
          if (!wt.wait(p_local(pbuf_of(pb)), puse_of(pb), 28)) { ok = false; break; }
          mbar_arrive_cluster(at_leader(p_full2(pbuf_of(pb))));
        }
        if (!ok) break;
      }
    }
  } else {
    // ================================================================ softmax warps (TMEM lane = thread)
    // lane L: head 64*rank + (L % 64); logits of block rows 32*(L/64) .. +31; output dims
    // 256 i + 128 (L/64) .. +127 for i = 0, 1. Warps w and w+2 hold the two halves of the
    // same 32 heads and exchange row maxima (and, at the end, row sums) in shared memory.
    const uint32_t L = threadIdx.x;
    const uint32_t half = L >> 6;
    const uint32_t hl = L & 63u;
    const uint32_t lane_off = (warp * 32u) << 16;
    const uint32_t partner = L ^ 64u;
    uint32_t qn = 0, pb = 0, nx = 0, qd = 0;
    uint32_t s_i = 0, s_u = 0;                         // logits buffer, and its use count
    bool ok = true;
    // one float from the partner lane (the other half of the same head)
    // Each lane owns two 64-bit slots (alternating exchanges) and stores (exchange number, value)
    // in one word; the partner polls for the number it expects. A lane can reuse a slot only
    // after the partner has answered the next exchange, so no unread value is overwritten.
    auto swap_partner = [&](float mine) -> float {
      const uint32_t par = nx & 1u;
      const uint32_t tag = ++nx;
      const uint64_t word = (static_cast<uint64_t>(tag) << 32) | __float_as_uint(mine);
      asm volatile("st.volatile.shared.u64 [%0], %1;" ::"r"(sbase + C::OFF_XMAX + (par * 128u + L) * 8u), "l"(word)
                   : "memory");
      uint32_t v = 0;
      const bool okl = wt.wait_tagged(sbase + C::OFF_XMAX + (par * 128u + partner) * 8u, tag, 37, v);
      if (!__all_sync(0xffffffffu, okl)) ok = false;
      return __uint_as_float(v);
    };
    for (int32_t qi = cid; qi < p.n_queries && ok; qi += ncl, ++qn) {
      const uint32_t slot = qn & 1u, sph = (qn >> 1) & 1u;
      uint32_t got = 1;
      if (lane == 0) got = wt.wait(info_full(slot), sph, 30) ? 1u : 0u;
      if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
      const int32_t total = info[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(info_empty(slot));
      const int32_t n_blocks = (total + kBlk - 1) / kBlk;
      const size_t orow = (static_cast<size_t>(qi) * kHeads + 64 * rank + hl) * kDv;
      if (n_blocks == 0) {
        const uint4 zz = make_uint4(0, 0, 0, 0);
        for (int i = 0; i < 2; ++i)
          for (int c = 0; c < 16; ++c) reinterpret_cast<uint4*>(p.out + orow + 256 * i + 128 * half)[c] = zz;
        if (half == 0) p.lse[static_cast<size_t>(qi) * kHeads + 64 * rank + hl] = -INFINITY;
        continue;
      }
      float m2 = -INFINITY, l = 0.f;
      // validity of this half's 32 rows of a block: lane j reads entry 32*half + j of the block from
      // the index row, one block ahead, and a ballot gives the mask (bit j: row j is attended)
      const int32_t* idx_row = p.idx + static_cast<size_t>(qi) * p.topk;
      auto entry = [&](int32_t b) -> int32_t {
        const int32_t j = b * kBlk + 32 * static_cast<int32_t>(half) + static_cast<int32_t>(lane);
        return j < total ? __ldg(idx_row + j) : -1;
      };
      // masked dense mode: the bitmap word of this half of block b (bit j: position 64b + 32 half
      // + j is attended; bits at or past the extent are 0)
      const uint32_t* mask_row = kDense ? p.mask + static_cast<size_t>(qi) * p.mask_words : nullptr;
      auto mask_word = [&](int32_t b) -> uint32_t { return __ldg(mask_row + 2 * b + static_cast<int32_t>(half)); };
      int32_t e_next = kDense ? 0 : entry(0);
      uint32_t m_next = kDense ? mask_word(0) : 0u;
      for (int32_t b = 0; b < n_blocks && ok; ++b) {
        uint32_t vmask;
        if constexpr (kDense) {
          vmask = m_next;
          if (b + 1 < n_blocks) m_next = mask_word(b + 1);
        } else {
          vmask = __ballot_sync(0xffffffffu, e_next >= 0 && e_next < p.max_len);
          if (b + 1 < n_blocks) e_next = entry(b + 1);
        }
        // ---- this lane's 32 logits
        if (lane == 0) got = wt.wait(s_full(s_i), s_u & 1u, 32) ? 1u : 0u;
        if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(tmem + lane_off + C::COL_S + 32u * s_i, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (++s_i == static_cast<uint32_t>(C::S_BUFS)) { s_i = 0; ++s_u; }
        // masked logits become -inf (their P is then exactly 0); a block of all-valid rows, the
        // usual case, skips the selects. The scale is positive, so the max of the raw logits
        // times the scale is the max of the scaled ones.
        const float sc = p.scale_log2;
        if (vmask != 0xffffffffu) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (!((vmask >> j) & 1u)) sr[j] = __float_as_uint(-INFINITY);
        }
        float mraw = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) mraw = fmaxf(mraw, __uint_as_float(sr[j]));
        float mb = mraw * sc;
        mb = fmaxf(mb, swap_partner(mb));
        if (!ok) break;
        const bool need = (mb > m2 + kLazyRescale);
        float alpha = 1.0f;
        if (need) {
          alpha = (m2 == -INFINITY) ? 0.0f : ex2_approx(m2 - mb);
          m2 = mb;
          l *= alpha;
        }
        // P = 2^(s*sc - m2) in bf16 for the output product; the row sum adds the same bf16 values,
        // so the normalisation matches the weights the output product uses. While every row seen so
        // far was masked, m2 is still -inf and so is every logit of this block: the subtrahend is
        // then 0, so P = 2^-inf = 0 instead of the NaN of -inf + inf.
        const float msub = (m2 == -INFINITY) ? 0.0f : m2;
        uint32_t pk[16];
        float2 lsum2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float e0 = ex2_approx(fmaf(__uint_as_float(sr[2 * j]), sc, -msub));
          const float e1 = ex2_approx(fmaf(__uint_as_float(sr[2 * j + 1]), sc, -msub));
          const __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
          const float2 back = __bfloat1622float2(pr);
          lsum2.x += back.x;
          lsum2.y += back.y;
          pk[j] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        l += lsum2.x + lsum2.y;
        // ---- the P buffer of block pb is free once the output MMA of block pb - P_BUFS has
        // finished; a rescale of O needs the one of block pb-1 finished (it implies the earlier ones)
        const bool rescale = __any_sync(0xffffffffu, need) && b > 0;
        if (rescale && pb >= 1) {
          if (lane == 0) got = wt.wait(p_empty(pbuf_of(pb - 1)), puse_of(pb - 1), 35) ? 1u : 0u;
          if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
        } else if (pb >= static_cast<uint32_t>(C::P_BUFS)) {
          if (lane == 0) got = wt.wait(p_empty(pbuf_of(pb)), puse_of(pb) ^ 1u, 34) ? 1u : 0u;
          if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
        }
        // ---- rescale this lane's output columns if the running max moved
        if (rescale) {
          tc_fence_after();
          const float a = need ? alpha : 1.0f;
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tmem + lane_off + C::COL_O + 16 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < 16; ++v) o[v] = __float_as_uint(__uint_as_float(o[v]) * a);
            tmem_st16(tmem + lane_off + C::COL_O + 16 * c, o);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        {
          // P row hl, columns 32*half .. +31 (64 B = 4 chunks of the 128-byte swizzled row)
          const uint32_t prow = sbase + C::OFF_P + pbuf_of(pb) * C::P_BYTES;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(prow + sw128_offset(hl, 4 * half + c)),
                         "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(leader ? p_full2(pbuf_of(pb)) : p_local(pbuf_of(pb)));
        ++pb;
      }
      if (!ok) break;
      // ---- epilogue: row sum of both halves, wait for the last output MMA, normalise, store
      l += swap_partner(l);
      if (!ok) break;
      if (lane == 0) got = wt.wait(o_full, qd & 1u, 36) ? 1u : 0u;
      if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
      ++qd;
      tc_fence_after();
      const float inv = 1.0f / l;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {               // 2 instructions x 128 columns, 32 at a time
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + C::COL_O + 32 * c, o);
        tmem_wait_ld();
        uint4 pkd[4];
        uint32_t* pw32 = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          const __nv_bfloat162 pr =
              __floats2bfloat162_rn(__uint_as_float(o[2 * v]) * inv, __uint_as_float(o[2 * v + 1]) * inv);
          pw32[v] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        const int i = c >> 2, cc = c & 3;
        uint4* dst = reinterpret_cast<uint4*>(p.out + orow + 256 * i + 128 * half + 32 * cc);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = pkd[v];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(at_leader(o_empty2));
      if (half == 0) p.lse[static_cast<size_t>(qi) * kHeads + 64 * rank + hl] = (m2 + log2f(l)) * 0.69314718055994531f;
    }
  }
  // ---- teardown: every role reaches here (all waits are bounded)
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // no CTA leaves while its peer may still use its memory
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS) : "memory");
  }
}

}  // namespace dsa
