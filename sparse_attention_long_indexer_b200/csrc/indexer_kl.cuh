// Indexer-alignment loss (KL divergence) forward for sm_100a.
//
// For query token t with its selected entries S_t (an index row), the index score I_s of each
// entry and the per-head log-sum-exp lse_h of the attention over S_t:
//   a_s  = sum_h exp(tau * q_h . kv_s - lse_h)      the head sum of the attention weights
//   p_s  = a_s / sum_s a_s                          L1 normalisation over S_t
//   KL_t = sum_s p_s * (ln p_s - I_s + LSE_I),      LSE_I = ln sum_s exp(I_s)
// ("節前發版：Deepseek v3.2 exp", section "訓練", Step 1 and Step 2: the target distribution sums
// the main attention over the heads and L1-normalises it along the sequence; the indexer's
// training objective is the KL divergence to the softmax of its scores, over the selected set
// in the sparse stage). With sum_s p_s = 1 the term is S1/A - ln A - S2/A + LSE_I with
// A = sum a_s, S1 = sum a_s ln a_s, S2 = sum a_s I_s, accumulated block by block.
//
// B200 design (one CTA per SM, persistent over queries, no cluster):
//  * logits: tcgen05.mma kind::f16 (bf16), M = 128 heads with q in TMEM (the A operand, 288
//    columns per lane = the 576 dims of that head), N = 64 selected rows gathered into shared
//    memory (B operand, K-major, 128-byte swizzle, 9 atoms of 64 dims), K = 576 in 36 steps,
//    into one of three 64-column TMEM buffers;
//  * four producer warps gather the rows of each 64-entry block with 16-byte cp.async into a
//    three-stage ring (padding and out-of-range entries become zero rows and are masked);
//  * four math warps, one thread per head (its TMEM lane): e = 2^(z * tau log2 e - lse_h log2 e)
//    for the 64 rows, a butterfly reduction over the 32 lanes of the warp gives each lane the
//    head sum of one row, and the four warps' partial sums meet in shared memory, where warp 0
//    accumulates A, S1, S2 and the online log-sum-exp of the index scores;
//  * the loss kernel reads the attention's lse, so the attention must have run on the same
//    index rows first.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "sparse_mla.cuh"

namespace dsa {

struct KlCfg {
  static constexpr int BLK = 64;                       // selected rows per block (MMA N)
  static constexpr int STAGES = 3;
  static constexpr int ATOM = BLK * 128;               // 64 rows x 64 dims (128 B)
  static constexpr int STAGE_BYTES = 9 * ATOM;         // 64 rows x 576 dims
  static constexpr int MATH_WARPS = 4;
  static constexpr int PRODUCER_WARPS = 4;
  static constexpr int PRODUCER_THREADS = PRODUCER_WARPS * 32;
  static constexpr int MMA_WARP = MATH_WARPS + PRODUCER_WARPS;
  static constexpr int THREADS = (MMA_WARP + 1) * 32;
  static constexpr uint32_t COL_Q = 0, COL_D = 288, D_BUFS = 3, TMEM_COLS = 512;
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_PART = OFF_STAGE + STAGES * STAGE_BYTES;          // [2][4 warps][64] fp32
  static constexpr int OFF_INFO = OFF_PART + 2 * MATH_WARPS * BLK * 4;       // [2] extents
  static constexpr int OFF_SCAN = OFF_INFO + 16;                              // per-warp scan / snapshots
  static constexpr int OFF_BAR = OFF_SCAN + 64;       // scan: 4 maxima, 2+2+2 parity slots
  static constexpr int NUM_BARS = 2 * STAGES + 2 * D_BUFS + 2 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(STAGE_BYTES % 1024 == 0 && OFF_PART % 16 == 0, "layout");
  static_assert(COL_D + D_BUFS * BLK <= TMEM_COLS, "TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct KlParams {
  const __nv_bfloat16* q;       // [B*n_q, 128, 576]
  const __nv_bfloat16* kv;      // [B, max_len, 576]
  const int32_t* idx;           // [B*n_q, topk]
  const float* scores;          // [B*n_q, topk] index score of each entry
  const float* lse;             // [B*n_q, 128] natural-log lse of the attention over the same rows
  float* loss;                  // [B*n_q] per-query KL term
  uint32_t* status;
  int32_t n_q, max_len, topk, n_queries;
  float scale_log2;             // tau * log2(e)
  uint64_t wait_budget_ns;
};

__device__ __forceinline__ void kl_drain_wait(uint32_t bar, uint32_t parity, uint64_t budget_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > budget_ns) return;
  }
}

__global__ void __launch_bounds__(KlCfg::THREADS, 1) indexer_kl_kernel(const KlParams p) {
  using C = KlCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* part = reinterpret_cast<float*>(smem + C::OFF_PART);
  int32_t* info = reinterpret_cast<int32_t*>(smem + C::OFF_INFO);
  int32_t* scan = reinterpret_cast<int32_t*>(smem + C::OFF_SCAN);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto B = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  auto full = [&](uint32_t s) { return B(static_cast<int>(s)); };                       // producers (4 warps)
  auto empty = [&](uint32_t s) { return B(C::STAGES + static_cast<int>(s)); };          // commit
  auto d_full = [&](uint32_t j) { return B(2 * C::STAGES + static_cast<int>(j)); };     // commit
  auto d_empty = [&](uint32_t j) { return B(2 * C::STAGES + C::D_BUFS + static_cast<int>(j)); };  // math (4)
  const uint32_t q_full = B(2 * C::STAGES + 2 * C::D_BUFS);                              // math (4)
  const uint32_t q_empty = q_full + 8;                                                   // commit
  auto info_full = [&](uint32_t i) { return q_full + 16 + 8u * i; };                    // producers (1)
  auto info_empty = [&](uint32_t i) { return q_full + 32 + 8u * i; };                   // math 4 + MMA 1
  const uint32_t mma_done = q_full + 48;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < static_cast<uint32_t>(C::STAGES); ++s) {
      mbar_init(full(s), C::PRODUCER_WARPS);
      mbar_init(empty(s), 1);
    }
    for (uint32_t j = 0; j < C::D_BUFS; ++j) {
      mbar_init(d_full(j), 1);
      mbar_init(d_empty(j), C::MATH_WARPS);
    }
    mbar_init(q_full, C::MATH_WARPS);
    mbar_init(q_empty, 1);
    for (uint32_t i = 0; i < 2; ++i) {
      mbar_init(info_full(i), 1);
      mbar_init(info_empty(i), C::MATH_WARPS + 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter wt{p.status, abort_flag, p.wait_budget_ns, 3u};
  const int32_t G = gridDim.x, cta = blockIdx.x;

  if (warp >= static_cast<uint32_t>(C::MATH_WARPS) && warp < static_cast<uint32_t>(C::MMA_WARP)) {
    // ================================================================ producers
    const uint32_t gtid = threadIdx.x - C::MATH_WARPS * 32;
    const uint32_t gw = gtid >> 5;
    volatile int32_t* go = scan + 8;
    uint32_t nsync = 0, qn = 0, st = 0, ph = 0;
    bool ok = true;
    // group-uniform bounded wait: thread 0 waits, the group reads its verdict after a barrier
    auto gate = [&](uint32_t bar, uint32_t parity, uint32_t tag) -> bool {
      if (gtid == 0) go[nsync & 1u] = (wt.wait(bar, parity, tag) && !wt.aborted()) ? 1 : 0;
      named_barrier(2, C::PRODUCER_THREADS);
      return go[(nsync++) & 1u] != 0;
    };
    const uint32_t cc = gtid & 7u, r0 = gtid >> 3;      // 16-byte chunk, first row (rows r0 + 16 i)
    for (int32_t qi = cta; qi < p.n_queries; qi += G, ++qn) {
      const uint32_t slot = qn & 1u, sph = (qn >> 1) & 1u;
      if (!gate(info_empty(slot), sph ^ 1u, 40)) break;
      const int32_t* idx_row = p.idx + static_cast<size_t>(qi) * p.topk;
      int32_t last = -1;                                // one past the last valid entry = extent
      for (int32_t j = static_cast<int32_t>(gtid); j < p.topk; j += C::PRODUCER_THREADS) {
        const int32_t v = __ldg(idx_row + j);
        if (v >= p.max_len) record_error(p.status, DSA_ERR_INDEX_RANGE, static_cast<uint32_t>(qi));
        if (v >= 0 && v < p.max_len) last = j;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
      if (lane == 0) scan[gw] = last;
      named_barrier(2, C::PRODUCER_THREADS);
      int32_t total = 0;
#pragma unroll
      for (int w = 0; w < C::PRODUCER_WARPS; ++w) total = max(total, scan[w] + 1);
      named_barrier(2, C::PRODUCER_THREADS);            // scan[] read before the next query writes it
      if (gtid == 0) {
        info[slot] = total;
        mbar_arrive(info_full(slot));
      }
      const int32_t n_blocks = (total + C::BLK - 1) / C::BLK;
      const __nv_bfloat16* kv_seq = p.kv + static_cast<size_t>(qi / p.n_q) * p.max_len * kDqk;
      int32_t pending = -1;
      auto announce = [&](int32_t stage) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(full(static_cast<uint32_t>(stage)));
      };
      for (int32_t b = 0; b < n_blocks && ok; ++b) {
        uint32_t got = 1;
        if (lane == 0) got = wt.wait(empty(st), ph ^ 1u, 41) ? 1u : 0u;
        if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
        const uint32_t dst0 = sbase + C::OFF_STAGE + st * C::STAGE_BYTES;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t r = r0 + 16u * i;
          const int32_t e = b * C::BLK + static_cast<int32_t>(r);
          const int32_t v = e < total ? __ldg(idx_row + e) : -1;
          const bool valid = v >= 0 && v < p.max_len;
          const __nv_bfloat16* src = (valid ? kv_seq + static_cast<size_t>(v) * kDqk : p.kv) + cc * 8;
          const uint32_t dst = dst0 + sw128_offset(r, cc);
#pragma unroll
          for (int a = 0; a < 9; ++a) cp_async_16(dst + a * C::ATOM, src + a * 64, valid ? 16u : 0u);
        }
        cp_async_commit();
        if (pending >= 0) {
          cp_async_wait<1>();
          announce(pending);
        }
        pending = static_cast<int32_t>(st);
        if (++st == static_cast<uint32_t>(C::STAGES)) { st = 0; ph ^= 1u; }
      }
      cp_async_wait<0>();
      if (pending >= 0) announce(pending);
    }
    cp_async_wait<0>();
  } else if (warp == C::MMA_WARP) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(1, 1, 0, 0, 128, C::BLK);
      uint32_t st = 0, ph = 0, qn = 0, nb = 0, qq = 0;    // qq: queries with at least one block
      bool ok = true;
      for (int32_t qi = cta; qi < p.n_queries && ok; qi += G, ++qn) {
        const uint32_t slot = qn & 1u, iph = (qn >> 1) & 1u;
        if (!wt.wait(info_full(slot), iph, 42)) break;
        const int32_t total = info[slot];
        mbar_arrive(info_empty(slot));
        const int32_t n_blocks = (total + C::BLK - 1) / C::BLK;
        if (n_blocks == 0) continue;
        if (!wt.wait(q_full, qq & 1u, 43)) break;
        ++qq;
        for (int32_t b = 0; b < n_blocks; ++b, ++nb) {
          const uint32_t j = nb % C::D_BUFS, dph = (nb / C::D_BUFS) & 1u;
          if (!wt.wait(full(st), ph, 44)) { ok = false; break; }
          if (!wt.wait(d_empty(j), dph ^ 1u, 45)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sb = sbase + C::OFF_STAGE + st * C::STAGE_BYTES;
#pragma unroll
          for (int k = 0; k < kDqk / 16; ++k) {
            const int dk = 16 * k;
            mma_bf16_ts(tmem + C::COL_D + C::BLK * j, tmem + C::COL_Q + 8 * k,
                        sw128_desc(sb + (dk >> 6) * C::ATOM + (dk & 63) * 2, 1, 1024), idesc, k > 0 ? 1u : 0u);
          }
          tc_commit(d_full(j));
          tc_commit(empty(st));
          if (++st == static_cast<uint32_t>(C::STAGES)) { st = 0; ph ^= 1u; }
        }
        tc_commit(q_empty);                         // every MMA reading this query's q issued
      }
      tc_commit(mma_done);
      kl_drain_wait(mma_done, 0, kDrainBudgetNs);
    }
  } else {
    // ================================================================ math warps (thread = head)
    const uint32_t h = threadIdx.x;                     // 0..127: head and TMEM lane
    const uint32_t lane_off = (warp * 32u) << 16;
    volatile int32_t* snap = scan + 4;
    uint32_t nsync = 0, qn = 0, nb = 0, qq = 0;
    // one barrier per step for the four math warps: warp 0's lane 0 publishes the abort flag into
    // a parity slot before the barrier, every warp reads it after, so all stop together
    auto uniform_stop = [&]() -> bool {
      if (threadIdx.x == 0) snap[nsync & 1u] = (*abort_flag != 0) ? 1 : 0;
      named_barrier(1, C::MATH_WARPS * 32);
      return snap[(nsync++) & 1u] != 0;
    };
    const float sc = p.scale_log2;
    volatile int32_t* go = scan + 12;
    for (int32_t qi = cta; qi < p.n_queries; qi += G, ++qn) {
      const uint32_t slot = qn & 1u, sph = (qn >> 1) & 1u;
      // one thread waits for the query's extent and the four warps read its verdict after a
      // barrier, so they all take the same number of blocks (and barriers) or all stop
      if (threadIdx.x == 0) go[nsync & 1u] = (wt.wait(info_full(slot), sph, 46) && !wt.aborted()) ? 1 : 0;
      named_barrier(1, C::MATH_WARPS * 32);
      if (go[(nsync++) & 1u] == 0) break;
      const int32_t total = info[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(info_empty(slot));
      uint32_t got = 1;
      const int32_t n_blocks = (total + C::BLK - 1) / C::BLK;
      if (n_blocks == 0) {
        if (threadIdx.x == 0) p.loss[qi] = 0.f;
        continue;
      }
      // ---- this query's q into TMEM (lane h: head h, columns 0..287 = dims 0..575), once the
      // previous query's MMAs are done reading it
      if (qq > 0) {
        if (lane == 0) got = wt.wait(q_empty, (qq - 1) & 1u, 47) ? 1u : 0u;
        got = __shfl_sync(0xffffffffu, got, 0);
      }
      ++qq;
      if (got) {
        tc_fence_after();
        const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(qi) * kHeads + h) * kDqk);
#pragma unroll 1
        for (int c = 0; c < kDqk / 32; ++c) {        // 16 columns (32 dims) per store
          uint32_t r[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = __ldg(qsrc + c * 4 + v);
            r[4 * v + 0] = u.x; r[4 * v + 1] = u.y; r[4 * v + 2] = u.z; r[4 * v + 3] = u.w;
          }
          tmem_st16(tmem + lane_off + C::COL_Q + 16 * c, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full);
      }
      const float lse2 = __ldg(p.lse + static_cast<size_t>(qi) * kHeads + h) * 1.4426950408889634f;
      const int32_t* idx_row = p.idx + static_cast<size_t>(qi) * p.topk;
      const float* sc_row = p.scores + static_cast<size_t>(qi) * p.topk;
      // warp 0 accumulates A, S1, S2 and the online LSE of the index scores (two rows per lane)
      float acc_a = 0.f, acc_s1 = 0.f, acc_s2 = 0.f, lse_m = -INFINITY, lse_z = 0.f;
      bool stop = false;
      for (int32_t b = 0; b < n_blocks; ++b, ++nb) {
        const uint32_t j = nb % C::D_BUFS, dph = (nb / C::D_BUFS) & 1u;
        // validity of the block's 64 entries (bit r: entry b*64 + r attended)
        const int32_t e0 = b * C::BLK + static_cast<int32_t>(lane), e1 = e0 + 32;
        const int32_t v0 = e0 < total ? __ldg(idx_row + e0) : -1;
        const int32_t v1 = e1 < total ? __ldg(idx_row + e1) : -1;
        const bool ok0 = v0 >= 0 && v0 < p.max_len, ok1 = v1 >= 0 && v1 < p.max_len;
        const uint32_t vm0 = __ballot_sync(0xffffffffu, ok0), vm1 = __ballot_sync(0xffffffffu, ok1);
        if (lane == 0) got = wt.wait(d_full(j), dph, 48) ? 1u : 0u;
        got = __shfl_sync(0xffffffffu, got, 0);
        float e[64];
        if (got) {
          tc_fence_after();
          uint32_t z[64];
          tmem_ld32(tmem + lane_off + C::COL_D + C::BLK * j, *reinterpret_cast<uint32_t(*)[32]>(&z[0]));
          tmem_ld32(tmem + lane_off + C::COL_D + C::BLK * j + 32, *reinterpret_cast<uint32_t(*)[32]>(&z[32]));
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(d_empty(j));
#pragma unroll
          for (int r = 0; r < 64; ++r) {
            const bool valid = ((r < 32 ? vm0 : vm1) >> (r & 31)) & 1u;
            e[r] = valid ? ex2_approx(fmaf(__uint_as_float(z[r]), sc, -lse2)) : 0.f;
          }
        } else {
#pragma unroll
          for (int r = 0; r < 64; ++r) e[r] = 0.f;
        }
        // butterfly over the warp's 32 heads: afterwards lane i holds the sum of row i (e[0]) and of
        // row 32 + i (e[32])
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float* v = e + 32 * half;
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
            for (int k = 0; k < o; ++k) {
              const bool upper = (lane & static_cast<uint32_t>(o)) != 0;
              const float send = upper ? v[k] : v[k + o];
              const float keep = upper ? v[k + o] : v[k];
              v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
          }
        }
        float* pb = part + (nb & 1u) * (C::MATH_WARPS * C::BLK);
        pb[warp * C::BLK + lane] = e[0];
        pb[warp * C::BLK + 32 + lane] = e[32];
        stop = uniform_stop();                          // also orders the partial sums
        if (stop) break;
        if (warp == 0) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int r = 32 * half + static_cast<int>(lane);
            const float a = pb[r] + pb[C::BLK + r] + pb[2 * C::BLK + r] + pb[3 * C::BLK + r];
            if (half == 0 ? ok0 : ok1) {
              const float is = __ldg(sc_row + (half == 0 ? e0 : e1));
              acc_a += a;
              if (a > 0.f) acc_s1 += a * __logf(a);
              acc_s2 += a * is;
              if (is > lse_m) {
                lse_z = lse_z * __expf(lse_m - is) + 1.f;
                lse_m = is;
              } else {
                lse_z += __expf(is - lse_m);
              }
            }
          }
        }
      }
      if (stop) break;
      if (warp == 0) {
        // combine the lanes: sums, and the log-sum-exp through (max, scaled sum)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          acc_a += __shfl_xor_sync(0xffffffffu, acc_a, o);
          acc_s1 += __shfl_xor_sync(0xffffffffu, acc_s1, o);
          acc_s2 += __shfl_xor_sync(0xffffffffu, acc_s2, o);
          const float m2 = __shfl_xor_sync(0xffffffffu, lse_m, o);
          const float z2 = __shfl_xor_sync(0xffffffffu, lse_z, o);
          const float mm = fmaxf(lse_m, m2);
          lse_z = (lse_m == -INFINITY ? 0.f : lse_z * __expf(lse_m - mm)) + (m2 == -INFINITY ? 0.f : z2 * __expf(m2 - mm));
          lse_m = mm;
        }
        if (lane == 0) {
          const float lse_i = lse_m + __logf(lse_z);
          p.loss[qi] = acc_a > 0.f ? (acc_s1 - acc_s2) / acc_a - __logf(acc_a) + lse_i : 0.f;
        }
      }
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

}  // namespace dsa
