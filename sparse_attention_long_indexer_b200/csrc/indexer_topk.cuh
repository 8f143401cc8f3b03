// Lightning indexer + fine-grained top-k selection, fused, for sm_100a.
//
// Computes, for every query t and every key s <= pos(t) of its sequence,
//     I[t,s] = k_scale[s] * sum_j (w[t,j] * q_scale[t]) * ReLU(q8[t,j] . k8[s])
// (the index score of the DeepSeek-V3.2-Exp summary "節前發版：Deepseek v3.2 exp",
// section "Lightning indexer" Step 1, with the per-token FP8 scales of the inputs folded
// out of the dot product: both are positive, so this equals sum_j w * ReLU(q . k) on the
// decoded values), and keeps the k largest per query (Step 2), ties to the lower s.
//
// Design (one CTA per SM in prefill, two in decode; persistent over work items):
//  * a work item is NQ consecutive queries of one sequence and a contiguous key range;
//  * TMA brings the item's query block [NQ*64 rows x 128 B] once and streams key tiles
//    [128 keys x 128 B] through a ring of shared-memory stages (128-byte swizzle);
//  * one thread issues tcgen05.mma kind::f8f6f4 (E4M3 x E4M3 -> f32), M = 128 keys,
//    N = NQ*64 (query, head) columns, K = 128 in four steps, into one of two TMEM
//    accumulators, so the MMA of tile i+1 overlaps the epilogue of tile i;
//  * epilogue warps own one TMEM lane quarter each (a key per thread); they read the
//    64 head columns of a query, apply ReLU and the weighted head sum in fp32 registers,
//    mask s > pos(t), and note which keys beat the query's threshold; every few tiles each
//    warp appends its survivors to the query's candidate buffer in shared memory with one
//    atomic. When a buffer nears capacity, the query's warps shrink it (a histogram pass over
//    the candidates' key range) or select exactly k, which raises the threshold. The L x L
//    score matrix is never written anywhere.
//  * prefill items cover a query block's whole causal key range and write the final
//    indices; decode items (one query per sequence) cover a key chunk and write an exact
//    partial top-k to the workspace, merged by `merge_partials_kernel`.
//  * sampled threshold (prefill items of at least kSpecMinTiles key tiles, top-k >= kSpecMinTopk):
//    the item first visits every kSampleStride-th key tile (a stratified sample of its keys)
//    and selects the sample's r ~ 1.5 k / kSampleStride best; the r-th score becomes the
//    admission threshold for the other tiles, which then follow in position order. About 1.5 k
//    keys of the whole range score at least that, so the candidate buffers rarely need a shrink
//    afterwards. The threshold is a guess, so the item checks it: if a query ends with fewer
//    than k candidates, or its sample phase had to cut a group of equal keys too large to keep
//    (the sample phase otherwise keeps every key tied with its r-th), the item is queued and a
//    second launch reruns the queued items with the exact streaming threshold. Thresholds in a sampled item never exclude ties (the stream is
//    not in position order), so the final selection settles ties by position as always.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kIdxHeads = 64;     // H_I (padded)
constexpr int kIdxDim = 128;      // d_I (padded), one 128-byte row per head / key
constexpr int kKeyTile = 128;     // keys per MMA tile (M)
constexpr int kDecodeChunk = 8192;  // keys per decode work item
constexpr int kSampleStride = 16;   // sampled threshold: the sample is every 16th key tile
constexpr int kSpecMinTiles = 64;   // ... for items with at least this many key tiles
constexpr int kSpecMinTopk = 1024;  // ... and at least this top-k (the sample's rank is ~ 3 k / 32)
constexpr int kSampleLimit = 2048;  // candidate count above which the sample phase shrinks its buffer

template <int NQ>
struct IdxCfg {
  static constexpr int N = NQ * kIdxHeads;                 // accumulator columns per tile
  static constexpr int NBUF = (NQ == 2) ? 4 : 2;           // TMEM accumulators (NBUF * N <= 512)
  static constexpr int HALVES = 1;                         // one MMA of N = NQ * 64 per K step
  // few warps: registers for the head weights and all 64 head columns at once
  static constexpr bool WIDE = NQ <= 2;
  static constexpr int CAND = (NQ == 2) ? 6144 : 3584;     // candidate capacity per query
  static constexpr int NH = N / HALVES;                    // MMA N
  static constexpr int EPI_WARPS = 4 * NQ;                 // a query per group of 4 lane-quarter warps
  static constexpr int EPI_THREADS = EPI_WARPS * 32;
  static constexpr int GROUP_THREADS = 128;                // the threads of one query
  static constexpr int PRODUCER_WARP = EPI_WARPS;
  static constexpr int MMA_WARP = EPI_WARPS + 1;
  // prefill: the producer and MMA warps and two idle warps form a fifth warpgroup, which gives
  // registers to the four epilogue warpgroups with setmaxnreg (launched at LAUNCH_REGS each:
  // the producer warpgroup drops to AUX_REGS, the epilogue warpgroups rise to EPI_REGS)
  static constexpr bool REG_SPLIT = NQ == 4;
  static constexpr int AUX_WARPS = REG_SPLIT ? 4 : 2;
  static constexpr int THREADS = (EPI_WARPS + AUX_WARPS) * 32;
  static constexpr int LAUNCH_REGS = 96;                   // 65536 / THREADS rounded down to 8
  static constexpr int AUX_REGS = 32;
  static constexpr int EPI_REGS = 112;
  static constexpr int STAGES = (NQ == 4) ? 4 : (NQ == 2) ? 6 : 4;
  // decode (one query per item) runs two CTAs per SM, so that two items' epilogues share an SM
  static constexpr int CTAS_PER_SM = (NQ == 1) ? 2 : 1;
  static constexpr int Q_BYTES = NQ * kIdxHeads * kIdxDim;
  static constexpr int K_BYTES = kKeyTile * kIdxDim;       // 16 KB
  static constexpr int TMEM_COLS = NBUF * N;
  static constexpr int MAXPER = CAND / GROUP_THREADS;
  // key tiles between two capacity checks of a candidate buffer (each check is a named barrier
  // of the query's warps; decode chunks are short, so they check more often)
  static constexpr int SYNC = (NQ == 4) ? 8 : 4;
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_KEYS = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_POS = OFF_KEYS + NQ * CAND * 4;
  static constexpr int OFF_W = OFF_POS + NQ * CAND * 4;
  static constexpr int OFF_SEL = OFF_W + NQ * kIdxHeads * 4;
  static constexpr int OFF_QST = OFF_SEL + NQ * static_cast<int>(sizeof(SelectScratch));
  static constexpr int OFF_BAR = (OFF_QST + 5 * 4 * NQ + 16 + 7) & ~7;
  static constexpr int NUM_BARS = 2 * STAGES + 2 + 8 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(CAND % GROUP_THREADS == 0 && MAXPER <= 64, "candidate buffer must split evenly");
  static_assert(CAND - SYNC * kKeyTile >= 2048, "a checked buffer must hold the largest k");
  static_assert(kSampleLimit + SYNC * kKeyTile <= CAND, "sample-phase limit");
  static_assert(NBUF * HALVES <= 4 && TMEM_COLS <= 512, "accumulators");
  static_assert(THREADS <= 1024 && NQ <= 4, "block shape");
  // setmaxnreg.inc waits until the registers the block was launched with can serve it, so the
  // split must fit in THREADS x LAUNCH_REGS (the host checks the compiled count at launch)
  static_assert(!REG_SPLIT || (THREADS * LAUNCH_REGS <= 65536 &&
                               EPI_WARPS * 32 * EPI_REGS + AUX_WARPS * 32 * AUX_REGS <= THREADS * LAUNCH_REGS),
                "register split");
  static_assert(Q_BYTES % 1024 == 0 && K_BYTES % 1024 == 0, "swizzle atoms");
};

struct IndexerParams {
  const uint8_t* q_idx;     // [B, n_q, 64, 128] e4m3 (padded dims)
  const __nv_bfloat16* w;   // [B, n_q, 64]
  const float* q_scale;     // [B*n_q]
  const float* k_scale;     // [B*max_len]
  const int32_t* lengths;   // [B]
  int32_t* out_idx;         // prefill: [B, n_q, topk]
  float* out_scores;        // optional, prefill: [B, n_q, topk] index score of each selected position
  uint32_t* part_keys;      // decode: [B, n_chunks, topk]
  int32_t* part_pos;        // decode: [B, n_chunks, topk]
  int32_t* part_count;      // decode: [B, n_chunks]
  // decode, score-only: when set, every key's order-preserving score goes to key_rows
  // [B, max_len] (positions the query sees) and no selection is made here
  uint32_t* key_rows;
  uint32_t* status;
  int32_t batch, n_q, max_len, topk, n_chunks;
  int32_t n_items;
  uint64_t wait_budget_ns;
  // sampled threshold (prefill): spec enables it; items whose guess fails are queued here
  int32_t spec;
  uint32_t* redo_flag;          // [n_items] 1 once the item is queued
  int32_t* redo_list;           // [n_items] queued items
  uint32_t* redo_count;         // entries in redo_list (zeroed by the host before the launch)
  // exact pass over queued items: item j of this launch is item_list[j], j < *item_count
  const int32_t* item_list;
  const uint32_t* item_count;
};

// Bounded wait that ignores the abort flag: used at teardown to let in-flight copies and
// MMAs land before shared memory / TMEM are released. Gives up silently after the budget.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t budget_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > budget_ns) return;
  }
}

// Work item u -> (sequence, first query, key start, key end (exclusive), #tiles, sample tiles).
struct Item {
  int32_t b, i0, s_begin, s_end, ntiles, len, n_s;
};

// Key tile visited at step t of an item: with a sample phase (n_s > 0) steps 0..n_s-1 visit
// tiles 0, 16, 32, ... and the later steps the other tiles in increasing order.
__device__ __forceinline__ int32_t tile_at(const Item& it, int32_t t) {
  if (it.n_s == 0) return t;
  if (t < it.n_s) return t * kSampleStride;
  const int32_t j = t - it.n_s;
  return j + j / (kSampleStride - 1) + 1;
}

// The sample's rank r: about 1.5 k scaled to the sampled fraction of the tiles.
__device__ __forceinline__ uint32_t sample_rank(int32_t topk, const Item& it) {
  return static_cast<uint32_t>((3 * topk * it.n_s + 2 * it.ntiles - 1) / (2 * it.ntiles));
}

// Item index of round `round` of this CTA, false when the CTA has no more items.
__device__ __forceinline__ bool item_at(const IndexerParams& p, int32_t round, int32_t cta, int32_t G, int32_t& u);

template <int NQ>
__device__ __forceinline__ Item make_item(const IndexerParams& p, int32_t u) {
  Item it;
  if (NQ == 1) {  // decode: key chunks of one query per sequence
    it.b = u / p.n_chunks;
    const int32_t c = u - it.b * p.n_chunks;
    it.i0 = 0;
    int32_t len = __ldg(p.lengths + it.b);
    len = min(max(len, 0), p.max_len);
    it.len = len;
    const int32_t pos = len - p.n_q;          // the single query (i = 0)
    it.s_begin = c * kDecodeChunk;
    it.s_end = min(it.s_begin + kDecodeChunk, pos + 1);
  } else {        // prefill: longest query blocks first
    const int32_t nqb = (p.n_q + NQ - 1) / NQ;
    const int32_t qb = nqb - 1 - u / p.batch;
    it.b = u - (u / p.batch) * p.batch;
    it.i0 = qb * NQ;
    int32_t len = __ldg(p.lengths + it.b);
    len = min(max(len, 0), p.max_len);
    it.len = len;
    const int32_t last_i = min(it.i0 + NQ, p.n_q) - 1;
    const int32_t max_pos = len - p.n_q + last_i;
    it.s_begin = 0;
    it.s_end = max_pos + 1;
  }
  const int32_t span = it.s_end - it.s_begin;
  it.ntiles = span > 0 ? (span + kKeyTile - 1) / kKeyTile : 0;
  it.n_s = (NQ > 1 && p.spec && it.ntiles >= kSpecMinTiles && p.topk >= kSpecMinTopk)
               ? (it.ntiles + kSampleStride - 1) / kSampleStride
               : 0;
  return it;
}

// Item sequence of CTA `cta` among `G`: snake order over rounds.
__device__ __forceinline__ int32_t item_of(int32_t round, int32_t cta, int32_t G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

__device__ __forceinline__ bool item_at(const IndexerParams& p, int32_t round, int32_t cta, int32_t G, int32_t& u) {
  const int32_t j = item_of(round, cta, G);
  if (p.item_list == nullptr) {
    u = j;
    return j < p.n_items;
  }
  if (j >= static_cast<int32_t>(__ldg(p.item_count))) return false;
  u = __ldg(p.item_list + j);
  return true;
}

template <int NQ>
__global__ void __launch_bounds__(IdxCfg<NQ>::THREADS, IdxCfg<NQ>::CTAS_PER_SM)
indexer_topk_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const IndexerParams p) {
  using C = IdxCfg<NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint32_t* cand_keys = reinterpret_cast<uint32_t*>(smem + C::OFF_KEYS);
  int32_t* cand_pos = reinterpret_cast<int32_t*>(smem + C::OFF_POS);
  float* wq = reinterpret_cast<float*>(smem + C::OFF_W);
  SelectScratch* sel = reinterpret_cast<SelectScratch*>(smem + C::OFF_SEL);
  uint32_t* q_count = reinterpret_cast<uint32_t*>(smem + C::OFF_QST);
  uint32_t* q_thr = q_count + NQ;
  uint32_t* q_strict = q_thr + NQ;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto k_full = [&](int s) { return bar0 + 8u * s; };
  auto k_empty = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  const uint32_t q_full = bar0 + 8u * (2 * C::STAGES);
  const uint32_t q_empty = q_full + 8;
  // accumulator buffer b, half h (queries 2h, 2h+1 of a 4-query block)
  auto acc_full = [&](uint32_t b, uint32_t h) { return q_full + 16 + 8u * (b * C::HALVES + h); };
  auto acc_empty = [&](uint32_t b, uint32_t h) { return q_full + 48 + 8u * (b * C::HALVES + h); };
  const uint32_t mma_done = q_full + 80;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (uint32_t b = 0; b < static_cast<uint32_t>(C::NBUF); ++b)
      for (uint32_t h = 0; h < static_cast<uint32_t>(C::HALVES); ++h) {
        mbar_init(acc_full(b, h), 1);
        mbar_init(acc_empty(b, h), C::EPI_WARPS / C::HALVES);
      }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  const int32_t G = gridDim.x;
  const int32_t cta = blockIdx.x;
  if ((NQ == 1 && p.part_count != nullptr) || (NQ > 1 && p.spec && p.item_list == nullptr)) {
    // Per-item words that only this CTA writes start at zero here, before the barrier. Decode
    // with partial lists: slot u belongs to item u, so a slot this CTA never reaches (after an
    // aborted wait) reads as empty in the merge instead of holding an earlier call's count.
    // (Score-only decode has no per-item words.) Sampled prefill: item u's queued flag.
    for (int32_t r = static_cast<int32_t>(threadIdx.x);; r += static_cast<int32_t>(blockDim.x)) {
      const int32_t u = item_of(r, cta, G);
      if (u >= p.n_items) break;
      if (NQ == 1) p.part_count[u] = 0;
      else p.redo_flag[u] = 0u;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter wt{p.status, abort_flag, p.wait_budget_ns, 1u};

  if (warp >= static_cast<uint32_t>(C::EPI_WARPS)) {
    // producer, MMA issuer and (prefill) two idle warps: one warpgroup, which hands registers
    // to the epilogue warpgroups
    if constexpr (C::REG_SPLIT) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::AUX_REGS));
  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&map_q);
      prefetch_tensormap(&map_k);
      uint32_t stage = 0, phase = 0, qph = 0;
      uint32_t used = 0, last_par = 0, q_out = 0;  // per stage: issued at least once / parity of last issue
      for (int32_t r = 0;; ++r) {
        int32_t u;
        if (!item_at(p, r, cta, G, u) || wt.aborted()) break;
        const Item it = make_item<NQ>(p, u);
        if (it.ntiles == 0) continue;
        if (!wt.wait(q_empty, qph ^ 1u, 1)) break;
        q_out = 1u | (qph << 1);
        qph ^= 1u;
        mbar_expect_tx(q_full, C::Q_BYTES);
        tma_load_3d(sbase + C::OFF_Q, &map_q, q_full, 0, it.i0 * kIdxHeads, it.b);
        bool ok = true;
        for (int32_t t = 0; t < it.ntiles; ++t) {
          if (!wt.wait(k_empty(stage), phase ^ 1u, 2)) { ok = false; break; }
          mbar_expect_tx(k_full(stage), C::K_BYTES);
          tma_load_3d(sbase + C::OFF_K + stage * C::K_BYTES, &map_k, k_full(stage), 0,
                      it.s_begin + tile_at(it, t) * kKeyTile, it.b);
          used |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // drain: every issued copy must have landed before the CTA may exit. Waiting on a
      // completed phase returns at once; after an abort this bounds the in-flight copies.
      for (int s = 0; s < C::STAGES; ++s)
        if (used & (1u << s)) drain_wait(k_full(s), (last_par >> s) & 1u, kDrainBudgetNs);
      if (q_out & 1u) drain_wait(q_full, (q_out >> 1) & 1u, kDrainBudgetNs);
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(0, 0, 0, 0, kKeyTile, C::NH);
      uint32_t stage = 0, phase = 0, qph = 0, g = 0;
      for (int32_t r = 0;; ++r) {
        int32_t u;
        if (!item_at(p, r, cta, G, u) || wt.aborted()) break;
        const Item it = make_item<NQ>(p, u);
        if (it.ntiles == 0) continue;
        if (!wt.wait(q_full, qph, 4)) break;
        qph ^= 1u;
        bool ok = true;
        for (int32_t t = 0; t < it.ntiles; ++t, ++g) {
          const uint32_t buf = g % C::NBUF, acc_ph = (g / C::NBUF) & 1u;
          if (!wt.wait(k_full(stage), phase, 5)) { ok = false; break; }
          const uint32_t a_base = sbase + C::OFF_K + stage * C::K_BYTES;
          // one MMA group per query pair, each announced on its own, so the two epilogue
          // halves run staggered by half a tile
#pragma unroll
          for (uint32_t h = 0; h < static_cast<uint32_t>(C::HALVES); ++h) {
            if (!wt.wait(acc_empty(buf, h), acc_ph ^ 1u, 6)) { ok = false; break; }
            tc_fence_after();
            const uint32_t b_base = sbase + C::OFF_Q + h * C::NH * kIdxDim;
#pragma unroll
            for (int kk = 0; kk < kIdxDim / 32; ++kk) {
              const uint64_t ad = sw128_desc(a_base + kk * 32, 1, 1024);
              const uint64_t bd = sw128_desc(b_base + kk * 32, 1, 1024);
              mma_f8_ss(tmem + buf * C::N + h * C::NH, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            tc_commit(acc_full(buf, h));
          }
          if (!ok) break;
          tc_commit(k_empty(stage));
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        tc_commit(q_empty);
        if (!ok) break;
      }
      // drain: all MMAs complete before TMEM is released
      tc_commit(mma_done);
      drain_wait(mma_done, 0, kDrainBudgetNs);
    }
  }
  } else {
    if constexpr (C::REG_SPLIT) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::EPI_REGS));
    // ------------------------------------------------------------- epilogue warps
    // Warps 4q .. 4q+3 own query q of the block, one TMEM lane quarter (32 keys) each; the
    // four run as a group with their own named barrier (1 + q), candidate buffer and select
    // scratch, so queries never wait for one another except through the shared accumulator.
    // Named barriers (bar.sync) cannot time out, so every warp of a group takes the same path
    // through them: mbarrier waits are done by lane 0 and broadcast, and the decision to stop
    // after an abort is a snapshot taken by one thread of the group between two barriers.
    const uint32_t q = warp >> 2;
    const uint32_t half = q / (NQ / C::HALVES);
    const uint32_t quarter = warp & 3u;
    const uint32_t gtid = threadIdx.x & (C::GROUP_THREADS - 1);
    const uint32_t bar_id = 1u + q;
    const uint32_t lane_base = (quarter * 32u) << 16;
    SelectScratch* gsel = sel + q;
    volatile uint32_t* snap = q_strict + NQ + 2 * q;     // two parity slots per group
    uint32_t* cq_keys = cand_keys + q * C::CAND;
    int32_t* cq_pos = cand_pos + q * C::CAND;
    uint32_t g = 0, nsync = 0;
    // One barrier per step: thread 0 of the group publishes the abort flag as it sees it into
    // a parity slot before the barrier and the group reads that slot after it. A slot is
    // rewritten two steps later, after every thread of the group has read it.
    auto uniform_stop = [&]() -> bool {
      if (gtid == 0) snap[nsync & 1u] = (*abort_flag != 0) ? 1u : 0u;
      named_barrier(bar_id, C::GROUP_THREADS);
      return snap[(nsync++) & 1u] != 0;
    };
    bool stop = false;
    for (int32_t r = 0; !stop; ++r) {
      int32_t u;
      if (!item_at(p, r, cta, G, u)) break;
      const Item it = make_item<NQ>(p, u);
      const int32_t i = it.i0 + static_cast<int32_t>(q);
      const bool q_valid = NQ == 1 || i < p.n_q;
      // per-query setup: head weights with the query's scale folded in
      if (gtid < static_cast<uint32_t>(kIdxHeads)) {
        float v = 0.f;
        if (q_valid) {
          const size_t qt = static_cast<size_t>(it.b) * p.n_q + i;
          v = __bfloat162float(p.w[qt * kIdxHeads + gtid]) * __ldg(p.q_scale + qt);
        }
        wq[q * kIdxHeads + gtid] = v;
      }
      if (gtid == 0) {
        q_count[q] = 0;
        q_thr[q] = 0;
        q_strict[q] = 0;
      }
      named_barrier(bar_id, C::GROUP_THREADS);
      // the query's admission threshold, changed only by a capacity check; kept in registers
      uint32_t thr_r = 0, strict_r = 0;
      const int32_t qpos = q_valid ? it.len - p.n_q + i : -1;
      const float4* w4 = reinterpret_cast<const float4*>(wq + q * kIdxHeads);
      // with few epilogue warps the query's head weights stay in registers for the whole item
      float2 wr[C::WIDE ? kIdxHeads / 2 : 1];
      if constexpr (C::WIDE) {
#pragma unroll
        for (int h = 0; h < kIdxHeads / 2; ++h) wr[h] = reinterpret_cast<const float2*>(wq + q * kIdxHeads)[h];
      }
      const float* ks_row = p.k_scale + static_cast<size_t>(it.b) * p.max_len;
      const int32_t s_lane = it.s_begin + static_cast<int32_t>(quarter * 32 + lane);
      // this lane's key at step t; the next step's key and its scale are fetched one step ahead
      // (address clamped to the item's range: the scale of a key outside it is never used)
      auto key_at = [&](int32_t t) -> int32_t { return s_lane + tile_at(it, t) * kKeyTile; };
      auto scale_at = [&](int32_t s) -> float { return __ldg(ks_row + max(min(s, it.s_end - 1), 0)); };
      int32_t s_next = key_at(0);
      float ks_next = scale_at(s_next);
      // a sampled item may drop candidates that tie with the sample's selection for their
      // position; its queries are then rerun exactly
      bool sample_tie = false;
      const uint32_t lanes_below = (1u << lane) - 1u;
      for (int32_t t = 0; t < it.ntiles; ++t, ++g) {
        const uint32_t buf = g % C::NBUF, acc_ph = (g / C::NBUF) & 1u;
        const int32_t s = s_next;
        const float ks = ks_next;
        s_next = key_at(t + 1);
        ks_next = scale_at(s_next);
        const bool in_range = s < it.s_end;
        // every lane waits (no divergent branch); the warp then runs the collective TMEM loads
        const bool ok = __all_sync(0xffffffffu, wt.wait(acc_full(buf, half), acc_ph, 8)) != 0;
        bool pass = false;
        uint32_t key = 0;
        if (ok) {
          tc_fence_after();
          const uint32_t col = buf * C::N + q * kIdxHeads;
          // sum_j w'_j * ReLU(x_j): packed fp32x2 FMAs over 4 independent accumulator pairs (head
          // h goes to pair 2*((h/4)&1) + ((h/2)&1), the same in both forms below)
          float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
          if constexpr (C::WIDE) {
            // all 64 head columns in one go, weights from registers
            uint32_t x[64];
            tmem_ld32(tmem + lane_base + col, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
            tmem_ld32(tmem + lane_base + col + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty(buf, half));
#pragma unroll
            for (int h = 0; h < kIdxHeads; h += 4) {
              const float2 r01 = make_float2(fmaxf(__uint_as_float(x[h + 0]), 0.f), fmaxf(__uint_as_float(x[h + 1]), 0.f));
              const float2 r23 = make_float2(fmaxf(__uint_as_float(x[h + 2]), 0.f), fmaxf(__uint_as_float(x[h + 3]), 0.f));
              const int c = (h / 4) & 1;
              acc[2 * c] = __ffma2_rn(wr[h / 2], r01, acc[2 * c]);
              acc[2 * c + 1] = __ffma2_rn(wr[h / 2 + 1], r23, acc[2 * c + 1]);
            }
          } else {
          // the 64 head columns come in two loads of 32 (fewer live registers), and the
          // accumulator is released after the second
          uint32_t x[32];
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            tmem_ld32(tmem + lane_base + col + 32 * part, x);
            tmem_wait_ld();
            if (part == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(acc_empty(buf, half));
            }
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
              const float4 wv = w4[(32 * part + h) / 4];
              const float2 r01 = make_float2(fmaxf(__uint_as_float(x[h + 0]), 0.f), fmaxf(__uint_as_float(x[h + 1]), 0.f));
              const float2 r23 = make_float2(fmaxf(__uint_as_float(x[h + 2]), 0.f), fmaxf(__uint_as_float(x[h + 3]), 0.f));
              const int c = (h / 4) & 1;
              acc[2 * c] = __ffma2_rn(make_float2(wv.x, wv.y), r01, acc[2 * c]);
              acc[2 * c + 1] = __ffma2_rn(make_float2(wv.z, wv.w), r23, acc[2 * c + 1]);
            }
          }
          }
          const float score =
              (((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y))) * ks;
          key = score_key(score);
          const bool valid = in_range && s <= qpos;
          if (NQ == 1 && p.key_rows != nullptr) {
            if (valid) p.key_rows[static_cast<size_t>(it.b) * p.max_len + s] = key;
          } else {
            pass = valid && (key > thr_r || (key == thr_r && strict_r == 0));
          }
        }
        // this tile's passes go into the buffer at once: one ballot, and one atomic for a warp
        // with any pass (after the first few tiles most warps have none)
        const uint32_t passed = __ballot_sync(0xffffffffu, pass);
        if (passed != 0u) {
          uint32_t base = 0;
          if (lane == 0) base = atomicAdd(&q_count[q], static_cast<uint32_t>(__popc(passed)));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (pass) {
            const uint32_t at = base + static_cast<uint32_t>(__popc(passed & lanes_below));
            cq_keys[at] = key;
            cq_pos[at] = s;
          }
        }
        // capacity check every C::SYNC tiles: between two checks at most C::SYNC * 128
        // candidates arrive, and a check leaves at most CAND - C::SYNC * 128 (also at the
        // end of a sample phase)
        const bool boundary = t + 1 == it.n_s;
        if (t % C::SYNC != C::SYNC - 1 && t + 1 != it.ntiles && !boundary) continue;
        if (uniform_stop()) { stop = true; break; }
        if (NQ == 1 && p.key_rows != nullptr) continue;
        uint32_t n = q_count[q];
        // the sample phase selects the sample's r best, under a lower capacity limit
        const bool sampling = t < it.n_s;
        const uint32_t tgt = sampling ? sample_rank(p.topk, it) : static_cast<uint32_t>(p.topk);
        const uint32_t limit = sampling ? static_cast<uint32_t>(kSampleLimit)
                                        : static_cast<uint32_t>(C::CAND - C::SYNC * kKeyTile);
        // Beyond the cheap shrink, a check may keep the tgt best with every candidate tied with
        // the tgt-th (the sample phase: a tie dropped there could still belong to the final
        // top-k; and the end of the sample phase, whose r-th key becomes the threshold), or
        // select exactly tgt, cutting ties by position (streaming, or a sample-phase tie group
        // too large to keep, after which the item is rerun exactly).
        bool keep = boundary, exact = false;
        if (n > limit) {
          uint32_t thr = 0;
          const uint32_t m = shrink_candidates<C::GROUP_THREADS, C::MAXPER>(cq_keys, cq_pos, n, tgt, gsel, gtid,
                                                                            bar_id, &thr);
          // more when the shrink freed less than half of the usable space
          if (m > (limit + tgt) / 2) {
            keep = keep || sampling;
            exact = !sampling;
          }
          if (gtid == 0) {
            q_count[q] = m;
            q_thr[q] = thr;
            q_strict[q] = 0;
          }
          named_barrier(bar_id, C::GROUP_THREADS);
          thr_r = q_thr[q];
          strict_r = 0;
          n = q_count[q];
        }
        if (keep && n > tgt) {
          uint32_t kept = 0;
          const uint32_t v =
              select_keep_ge<C::GROUP_THREADS, C::MAXPER>(cq_keys, cq_pos, n, tgt, gsel, gtid, bar_id, &kept);
          if (kept > (limit + tgt) / 2) {
            exact = true;
          } else if (gtid == 0) {
            q_count[q] = kept;
            q_thr[q] = max(v, thr_r);
            q_strict[q] = 0;
          }
          named_barrier(bar_id, C::GROUP_THREADS);
          thr_r = q_thr[q];
          n = exact ? kept : q_count[q];
        }
        if (exact) {
          bool tied = false;
          const uint32_t vk =
              select_exact<C::GROUP_THREADS, C::MAXPER>(cq_keys, cq_pos, n, tgt, gsel, gtid, bar_id, &tied);
          if (sampling && tied) sample_tie = true;
          if (gtid == 0) {
            q_count[q] = tgt;
            q_thr[q] = vk;
            // a strict threshold relies on later keys having larger positions: only in
            // position order
            q_strict[q] = it.n_s == 0 ? 1u : 0u;
          }
          named_barrier(bar_id, C::GROUP_THREADS);
          thr_r = q_thr[q];
          strict_r = q_strict[q];
        }
      }
      if (stop) break;
      // ---- finish the query: exact k, then write
      if (q_valid && !(NQ == 1 && p.key_rows != nullptr)) {
        uint32_t n = q_count[q];
        // a sampled item whose threshold kept fewer than k candidates, or dropped ties in its
        // sample phase, is queued for the exact pass (which rewrites all its queries)
        if (it.n_s > 0 && (n < static_cast<uint32_t>(p.topk) || sample_tie) && gtid == 0) {
          if (atomicExch(p.redo_flag + u, 1u) == 0u) p.redo_list[atomicAdd(p.redo_count, 1u)] = u;
        }
        if (n > static_cast<uint32_t>(p.topk)) {
          select_exact<C::GROUP_THREADS, C::MAXPER>(cq_keys, cq_pos, n, static_cast<uint32_t>(p.topk), gsel, gtid,
                                                    bar_id);
          n = p.topk;
        }
        if (NQ == 1) {
          const size_t slot = static_cast<size_t>(it.b) * p.n_chunks + (it.s_begin / kDecodeChunk);
          for (uint32_t j = gtid; j < n; j += C::GROUP_THREADS) {
            p.part_keys[slot * p.topk + j] = cq_keys[j];
            p.part_pos[slot * p.topk + j] = cq_pos[j];
          }
          if (gtid == 0) p.part_count[slot] = static_cast<int32_t>(n);
        } else {
          const size_t row = (static_cast<size_t>(it.b) * p.n_q + i) * p.topk;
          int32_t* dst = p.out_idx + row;
          for (uint32_t j = gtid; j < static_cast<uint32_t>(p.topk); j += C::GROUP_THREADS)
            dst[j] = j < n ? cq_pos[j] : -1;
          if (p.out_scores != nullptr) {
            float* sdst = p.out_scores + row;
            for (uint32_t j = gtid; j < static_cast<uint32_t>(p.topk); j += C::GROUP_THREADS)
              sdst[j] = j < n ? key_score(cq_keys[j]) : -INFINITY;
          }
        }
      }
      named_barrier(bar_id, C::GROUP_THREADS);
    }
  }
  // ---- teardown: every role reaches here (all waits are bounded)
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Decode: merge the per-chunk exact top-k lists of one sequence into its final top-k.
// One CTA per sequence; candidates are read from the workspace (L2-resident).
struct MergeParams {
  const uint32_t* part_keys;
  const int32_t* part_pos;
  const int32_t* part_count;
  int32_t* out_idx;        // [B, n_q(=1), topk]
  int32_t n_chunks, topk;
  float* out_scores;       // optional [B, n_q(=1), topk]
};

template <int T>
__global__ void __launch_bounds__(T) merge_partials_kernel(const MergeParams p) {
  __shared__ SelectScratch sc;
  __shared__ uint32_t s_count[1024 + 1];
  __shared__ uint32_t s_lo[T / 32], s_hi[T / 32];
  const uint32_t tid = threadIdx.x, lane = tid & 31u;
  const int32_t b = blockIdx.x;
  const size_t base_slot = static_cast<size_t>(b) * p.n_chunks;
  // a count never exceeds topk; the clamp keeps every read inside its slot regardless
  for (int32_t c = tid; c < p.n_chunks; c += T)
    s_count[c] = min(static_cast<uint32_t>(max(p.part_count[base_slot + c], 0)), static_cast<uint32_t>(p.topk));
  __syncthreads();
  uint32_t n = 0;
  for (int32_t c = 0; c < p.n_chunks; ++c) n += s_count[c];
  const uint32_t k = static_cast<uint32_t>(p.topk);
  int32_t* dst = p.out_idx + static_cast<size_t>(b) * p.topk;
  // fn(key, pos, has) for every candidate, in warp-uniform rounds (has = false past a list's end)
  auto for_each = [&](auto&& fn) {
    for (int32_t c = 0; c < p.n_chunks; ++c) {
      const uint32_t* kk = p.part_keys + (base_slot + c) * p.topk;
      const int32_t* pp = p.part_pos + (base_slot + c) * p.topk;
      for (uint32_t j0 = 0; j0 < s_count[c]; j0 += T) {
        const uint32_t j = j0 + tid;
        const bool has = j < s_count[c];
        fn(has ? kk[j] : 0u, has ? pp[j] : 0, has);
      }
    }
  };
  uint32_t vk = 0, plim = 0xFFFFFFFFu;
  if (n > k) {
    // ---- key passes over an adaptive range: 256 bins over [min, max] of the candidates, then
    // over the chosen bin, until the bin holding the k-th key is taken whole or is one value
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for_each([&](uint32_t key, int32_t, bool has) {
      if (has) {
        lo = min(lo, key);
        hi = max(hi, key);
      }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      s_lo[tid >> 5] = lo;
      s_hi[tid >> 5] = hi;
    }
    __syncthreads();
    for (int w = 0; w < T / 32; ++w) {
      lo = min(lo, s_lo[w]);
      hi = max(hi, s_hi[w]);
    }
    uint32_t rem = k, shift = bin_shift(hi - lo), a_lo = lo, a_hi = hi;
    bool ties = false;
    while (true) {
      for (uint32_t i = tid; i < 256; i += T) sc.hist[i] = 0;
      __syncthreads();
      for_each([&](uint32_t key, int32_t, bool has) {
        if (has && key >= a_lo && key <= a_hi) atomicAdd(&sc.hist[(key - a_lo) >> shift], 1u);
      });
      __syncthreads();
      if (tid < 32) scan_bins<true>(&sc, rem);
      __syncthreads();
      const uint32_t bin = sc.bin, above = sc.above, cnt = sc.cnt;
      __syncthreads();                                  // scan results read before the next pass
      rem -= above;
      const uint32_t blo = a_lo + (bin << shift);
      if (cnt == rem) {                                 // the whole bin is in: keys >= blo
        vk = blo;
        break;
      }
      if (shift == 0) {                                 // one key value, more items than places
        vk = blo;
        ties = true;
        break;
      }
      a_hi = bin_end(blo, shift, a_hi);
      a_lo = blo;
      shift = shift > 8u ? shift - 8u : 0u;
    }
    if (ties) {
      // ---- position passes among the candidates equal to vk: keep the rem lowest positions
      uint32_t pprefix = 0, pmask = 0, prem = rem;
      for (int ps = 24; ps >= 0; ps -= 8) {
        for (uint32_t i = tid; i < 256; i += T) sc.hist[i] = 0;
        __syncthreads();
        for_each([&](uint32_t key, int32_t pos, bool has) {
          const uint32_t pu = static_cast<uint32_t>(pos);
          if (has && key == vk && (pu & pmask) == pprefix) atomicAdd(&sc.hist[(pu >> ps) & 255u], 1u);
        });
        __syncthreads();
        if (tid < 32) scan_pick<false>(&sc, prem);
        __syncthreads();
        prem -= sc.above;
        pprefix |= sc.bin << ps;
        pmask |= 0xFFu << ps;
        __syncthreads();
      }
      plim = pprefix;
    } else {
      plim = 0xFFFFFFFFu;                               // every candidate equal to vk is kept
    }
  }
  // ---- write the kept positions, one atomic per warp and round
  if (tid == 0) sc.out_count = 0;
  __syncthreads();
  const bool all = n <= k;
  for_each([&](uint32_t key, int32_t ps, bool has) {
    const bool keep = has && (all || key > vk || (key == vk && static_cast<uint32_t>(ps) <= plim));
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    uint32_t base = 0;
    if (lane == 0 && m) base = atomicAdd(&sc.out_count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    const uint32_t at = base + __popc(m & ((1u << lane) - 1u));
    if (keep && at < k) {
      dst[at] = ps;
      if (p.out_scores != nullptr) p.out_scores[static_cast<size_t>(b) * p.topk + at] = key_score(key);
    }
  });
  __syncthreads();
  for (uint32_t j = min(sc.out_count, k) + tid; j < k; j += T) {
    dst[j] = -1;
    if (p.out_scores != nullptr) p.out_scores[static_cast<size_t>(b) * p.topk + j] = -INFINITY;
  }
}

}  // namespace dsa
