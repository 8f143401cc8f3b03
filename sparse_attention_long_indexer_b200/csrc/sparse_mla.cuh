// Sparse MLA attention in MQA mode over the selected latent rows, for sm_100a.
//
// For one query token t with H = 128 heads and its selected rows S_t (from the indexer):
//   z[h,s] = tau * q[t,h,:] . kv[s,:]    (576 = 512 latent + 64 RoPE dims)
//   out[t,h,:] = sum_s softmax_s(z[h,.]) * kv[s, :512],   lse[t,h] = ln sum_s exp z[h,s]
// ("節前發版：Deepseek v3.2 exp", section "Lightning indexer" Step 2 and section
// "在MLA下實例化DSA": attention runs only over the selected entries, and in MLA's MQA mode
// every query head shares the one latent vector of each token).
//
// B200 design. The fp32 output accumulator of one query, 128 heads x 512 dims, is 256 KB:
// all of one SM's tensor memory. So each query runs on a cluster of two CTAs (two SMs):
//  * CTA r keeps output columns [256r, 256r+256) in TMEM (256 columns) and the query's
//    dims [288r, 288r+288) in TMEM (144 columns, the A operand of the QK^T MMA);
//  * per block of 64 selected rows, CTA r gathers the dims it needs (r=0: [0,288), r=1:
//    [256,576)) with 16-byte cp.async into a 128-byte-swizzled stage, and computes the
//    partial logits S_r = Q[:,dims_r] . K[:,dims_r]^T on tcgen05 (kind::f16, A from TMEM);
//  * the two fp32 partials are swapped through distributed shared memory and summed in a
//    fixed order, so both CTAs hold bit-identical logits and take identical softmax steps;
//  * P (bf16) goes to TMEM and O_r += P . V[:, 256r:256r+256] runs on tcgen05 with the same
//    stage read as an MN-major operand; the softmax is online in the log2 domain, rescaling
//    O only when the running max grows by more than 8 (exact: the final division uses the
//    same stale max).
// Each gathered row is thus shared by all 128 heads as a dense [128 x d] x [d x 64] product.
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

struct AttnCfg {
  static constexpr int STAGES = 3;
  static constexpr int ATOMS = 5;                        // 5 x 64 dims per stage row
  static constexpr int ATOM_BYTES = kBlk * 128;          // 8 KB
  static constexpr int STAGE_BYTES = ATOMS * ATOM_BYTES; // 40 KB
  static constexpr int X_BYTES = kHeads * kBlk * 4;      // 32 KB partial logits
  static constexpr int SOFTMAX_WARPS = 4;                // warp w owns TMEM lanes 32w..32w+31
  static constexpr int PRODUCER_WARPS = 4;
  static constexpr int PRODUCER_THREADS = PRODUCER_WARPS * 32;
  static constexpr int MMA_WARP = SOFTMAX_WARPS + PRODUCER_WARPS;
  static constexpr int THREADS = (MMA_WARP + 1) * 32;
  // TMEM columns
  static constexpr uint32_t COL_O = 0, COL_S = 256, COL_P = 320, COL_Q = 352, TMEM_COLS = 512;
  // shared memory
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_X = OFF_STAGE + STAGES * STAGE_BYTES;
  static constexpr int OFF_SEL = OFF_X + 2 * X_BYTES;
  static constexpr int OFF_SCAN = OFF_SEL + kMaxTopk * 4;
  static constexpr int OFF_INFO = OFF_SCAN + 64;   // scan: 4 warp sums + 2 go slots
  static constexpr int OFF_BAR = OFF_INFO + 16;
  static constexpr int NUM_BARS = 2 * STAGES + 7 + 2 + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
};

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
};

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

__global__ void __launch_bounds__(AttnCfg::THREADS, 1) __cluster_dims__(2, 1, 1)
sparse_mla_attn_kernel(const AttnParams p) {
  using C = AttnCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int32_t* sel = reinterpret_cast<int32_t*>(smem + C::OFF_SEL);
  int32_t* scan = reinterpret_cast<int32_t*>(smem + C::OFF_SCAN);
  int32_t* info = reinterpret_cast<int32_t*>(smem + C::OFF_INFO);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto kv_full = [&](int s) { return bar0 + 8u * s; };
  auto kv_empty = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  const uint32_t s_full = bar0 + 8u * (2 * C::STAGES);
  const uint32_t s_empty = s_full + 8, p_full = s_full + 16, p_empty = s_full + 24;
  const uint32_t q_full = s_full + 32, q_empty = s_full + 40, o_empty = s_full + 48;
  auto info_full = [&](int i) { return s_full + 56 + 8u * i; };
  auto info_empty = [&](int i) { return s_full + 72 + 8u * i; };
  auto x_full = [&](int i) { return s_full + 88 + 8u * i; };
  auto x_empty = [&](int i) { return s_full + 104 + 8u * i; };
  const uint32_t mma_done = s_full + 120;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(kv_full(s), C::PRODUCER_THREADS);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, C::SOFTMAX_WARPS);
    mbar_init(p_full, C::SOFTMAX_WARPS);
    mbar_init(p_empty, 1);
    mbar_init(q_full, C::SOFTMAX_WARPS);
    mbar_init(q_empty, 1);
    mbar_init(o_empty, C::SOFTMAX_WARPS);
    for (int i = 0; i < 2; ++i) {
      mbar_init(info_full(i), 1);
      mbar_init(info_empty(i), 1 + C::SOFTMAX_WARPS);
      mbar_init(x_full(i), kHeads);     // arrived by the peer's 128 softmax threads
      mbar_init(x_empty(i), kHeads);
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
  cluster_sync();            // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter wt{p.status, abort_flag, p.wait_budget_ns, 2u};
  const int32_t ncl = static_cast<int32_t>(nclusters_x());
  const int32_t cid = static_cast<int32_t>(cluster_id_x());
  const int32_t a0 = 256 * static_cast<int32_t>(rank);          // first dim of this CTA's stage rows

  if (warp >= C::SOFTMAX_WARPS && warp < C::MMA_WARP) {
    // ================================================================ producers: index list + gathers
    // bar.sync cannot time out, so all producer threads take the same path through named
    // barrier 2: thread 0 alone waits on mbarriers and publishes the go / stop decision in
    // a parity slot that every thread reads after the barrier.
    const uint32_t ptid = threadIdx.x - C::SOFTMAX_WARPS * 32;
    volatile int32_t* go = scan + 8;                  // two parity slots
    const int32_t nch = rank == 0 ? 36 : 40;          // 16-byte chunks per gathered row
    const int32_t per = (p.topk + C::PRODUCER_THREADS - 1) / C::PRODUCER_THREADS;
    uint32_t stage = 0, phase = 0, qn = 0, nsync = 0;
    auto gate = [&](uint32_t bar, uint32_t parity, uint32_t tag) -> bool {
      if (ptid == 0) go[nsync & 1u] = wt.wait(bar, parity, tag) ? 1 : 0;
      named_barrier(2, C::PRODUCER_THREADS);
      return go[(nsync++) & 1u] != 0;
    };
    for (int32_t qi = cid; qi < p.n_queries; qi += ncl, ++qn) {
      const uint32_t slot = qn & 1u, sph = (qn >> 1) & 1u;
      if (!gate(info_empty(slot), sph ^ 1u, 10)) break;
      // compact the valid entries of the index row, preserving their order
      const int32_t* row = p.idx + static_cast<size_t>(qi) * p.topk;
      const int32_t j0 = min(static_cast<int32_t>(ptid) * per, p.topk), j1 = min(j0 + per, p.topk);
      int32_t cnt = 0;
      for (int32_t j = j0; j < j1; ++j) {
        const int32_t v = __ldg(row + j);
        if (v >= p.max_len) record_error(p.status, DSA_ERR_INDEX_RANGE, static_cast<uint32_t>(qi));
        cnt += (v >= 0 && v < p.max_len) ? 1 : 0;
      }
      int32_t incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (static_cast<int32_t>(lane) >= o) incl += v;
      }
      if (lane == 31) scan[ptid >> 5] = incl;
      named_barrier(2, C::PRODUCER_THREADS);
      int32_t base = incl - cnt, total = 0;
      for (uint32_t w = 0; w < C::PRODUCER_WARPS; ++w) {
        const int32_t v = scan[w];
        if (w < (ptid >> 5)) base += v;
        total += v;
      }
      for (int32_t j = j0; j < j1; ++j) {
        const int32_t v = __ldg(row + j);
        if (v >= 0 && v < p.max_len) sel[base++] = v;
      }
      named_barrier(2, C::PRODUCER_THREADS);
      if (ptid == 0) {
        info[slot] = total;
        mbar_arrive(info_full(slot));
      }
      const int32_t n_blocks = (total + kBlk - 1) / kBlk;
      const size_t kv_seq = static_cast<size_t>(qi / p.n_q) * p.max_len;
      int32_t pending_stage = -1;
      bool ok = true;
      for (int32_t b = 0; b < n_blocks; ++b) {
        if (!gate(kv_empty(stage), phase ^ 1u, 11)) { ok = false; break; }
        const uint32_t st = sbase + C::OFF_STAGE + stage * C::STAGE_BYTES;
        for (int32_t i = ptid; i < kBlk * nch; i += C::PRODUCER_THREADS) {
          const int32_t r = i / nch, ch = i - r * nch;
          const int32_t j = b * kBlk + r;
          const bool valid = j < total;
          const __nv_bfloat16* src = p.kv;
          if (valid) src = p.kv + (kv_seq + sel[j]) * kDqk + a0 + ch * 8;
          const uint32_t dst = st + (ch >> 3) * C::ATOM_BYTES + sw128_offset(r, ch & 7);
          cp_async_16(dst, src, valid ? 16u : 0u);
        }
        cp_async_commit();
        if (pending_stage >= 0) {
          cp_async_wait<1>();
          fence_proxy_async_smem();
          mbar_arrive(kv_full(pending_stage));
        }
        pending_stage = static_cast<int32_t>(stage);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      cp_async_wait<0>();
      if (pending_stage >= 0) {
        fence_proxy_async_smem();
        mbar_arrive(kv_full(pending_stage));
      }
      if (!ok) break;
    }
    cp_async_wait<0>();
  } else if (warp == C::MMA_WARP) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc(1, 1, 0, 0, 128, kBlk);
      constexpr uint32_t idesc_pv = make_idesc(1, 1, 0, 1, 128, 256);
      uint32_t stage = 0, phase = 0, qn = 0, sb = 0, pb = 0, qq = 0;
      for (int32_t qi = cid; qi < p.n_queries; qi += ncl, ++qn) {
        const uint32_t slot = qn & 1u, sph = (qn >> 1) & 1u;
        if (!wt.wait(info_full(slot), sph, 20)) break;
        const int32_t total = info[slot];
        mbar_arrive(info_empty(slot));
        const int32_t n_blocks = (total + kBlk - 1) / kBlk;
        if (n_blocks == 0) continue;
        if (!wt.wait(q_full, qq & 1u, 21)) break;
        bool ok = true;
        // logits of block 0, then per block: logits of block b+1, then P.V of block b
        const uint32_t s_stage = stage, s_phase = phase;
        auto do_s = [&](uint32_t stg, uint32_t ph) -> bool {
          if (!wt.wait(kv_full(stg), ph, 22)) return false;
          if (!wt.wait(s_empty, (sb & 1u) ^ 1u, 23)) return false;
          tc_fence_after();
          const uint32_t st = sbase + C::OFF_STAGE + stg * C::STAGE_BYTES;
#pragma unroll
          for (int j = 0; j < 18; ++j) {
            const int dj = (rank == 0 ? 0 : 32) + 16 * j;
            const uint32_t addr = st + (dj >> 6) * C::ATOM_BYTES + (dj & 63) * 2;
            mma_bf16_ts(tmem + C::COL_S, tmem + C::COL_Q + 8 * j, sw128_desc(addr, 1, 1024), idesc_s,
                        j > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
          ++sb;
          return true;
        };
        if (!do_s(s_stage, s_phase)) break;
        for (int32_t b = 0; b < n_blocks; ++b) {
          const uint32_t cur_stage = stage;
          uint32_t nstage = stage + 1, nphase = phase;
          if (nstage == C::STAGES) { nstage = 0; nphase ^= 1u; }
          if (b + 1 < n_blocks) {
            if (!do_s(nstage, nphase)) { ok = false; break; }
          }
          if (!wt.wait(p_full, pb & 1u, 24)) { ok = false; break; }
          if (b == 0 && !wt.wait(o_empty, (qq & 1u) ^ 1u, 25)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = sbase + C::OFF_STAGE + cur_stage * C::STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk) {
            mma_bf16_ts(tmem + C::COL_O, tmem + C::COL_P + 8 * kk,
                        sw128_desc(st + kk * 2048, C::ATOM_BYTES, 1024), idesc_pv, (b > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(kv_empty(cur_stage));
          tc_commit(p_empty);
          ++pb;
          stage = nstage;
          phase = nphase;
        }
        tc_commit(q_empty);
        ++qq;
        if (!ok) break;
      }
      tc_commit(mma_done);
      attn_drain_wait(mma_done, 0, p.wait_budget_ns);
    }
  } else {
    // ================================================================ softmax / epilogue warps (thread = head)
    const uint32_t h = threadIdx.x;                  // 0..127, TMEM lane h
    const uint32_t lane_off = (warp * 32u) << 16;
    const uint32_t xpeer = mapa(sbase + C::OFF_X, peer);
    const uint32_t xfull_peer0 = mapa(x_full(0), peer);
    const uint32_t xempty_peer0 = mapa(x_empty(0), peer);
    const float* xloc = reinterpret_cast<const float*>(smem + C::OFF_X);
    uint32_t qn = 0, sb = 0, pb = 0, qq = 0, xb = 0;
    bool ok = true;
    for (int32_t qi = cid; qi < p.n_queries && ok; qi += ncl, ++qn) {
      const uint32_t slot = qn & 1u, sph = (qn >> 1) & 1u;
      uint32_t got = 1;
      if (lane == 0) got = wt.wait(info_full(slot), sph, 30) ? 1u : 0u;
      if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
      const int32_t total = info[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(info_empty(slot));
      const int32_t n_blocks = (total + kBlk - 1) / kBlk;
      __nv_bfloat16* orow = p.out + (static_cast<size_t>(qi) * kHeads + h) * kDv + 256 * rank;
      if (n_blocks == 0) {
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int c = 0; c < 32; ++c) reinterpret_cast<uint4*>(orow)[c] = z;
        if (rank == 0) p.lse[static_cast<size_t>(qi) * kHeads + h] = -INFINITY;
        continue;
      }
      // ---- Q[:, 288r : 288r+288] -> TMEM columns COL_Q.. (A operand of the logits MMA)
      if (lane == 0) got = wt.wait(q_empty, (qq & 1u) ^ 1u, 31) ? 1u : 0u;
      if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
      tc_fence_after();
      {
        const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(qi) * kHeads + h) * kDqk +
                                                           288 * rank);
#pragma unroll 1
        for (int c = 0; c < 9; ++c) {          // 9 x 16 columns = 288 bf16
          uint32_t r[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = __ldg(qsrc + c * 4 + v);
            r[4 * v + 0] = u.x; r[4 * v + 1] = u.y; r[4 * v + 2] = u.z; r[4 * v + 3] = u.w;
          }
          tmem_st16(tmem + lane_off + C::COL_Q + 16 * c, r);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
      ++qq;
      float m2 = -INFINITY, l = 0.f;
      for (int32_t b = 0; b < n_blocks; ++b) {
        // ---- partial logits from TMEM
        if (lane == 0) got = wt.wait(s_full, sb & 1u, 32) ? 1u : 0u;
        if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(tmem + lane_off + C::COL_S, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tmem + lane_off + C::COL_S + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty);
        ++sb;
        // ---- swap partials with the peer CTA (distributed shared memory)
        const uint32_t xs = xb & 1u, xph = (xb >> 1) & 1u;
        ++xb;
        if (!wt.wait<true>(x_empty(xs), xph ^ 1u, 33)) { ok = false; break; }
        {
          const uint32_t rowaddr = xpeer + xs * C::X_BYTES + h * 256u;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            st_cluster_v4(rowaddr + ((c ^ (h & 15u)) << 4), __uint_as_float(sr[4 * c]), __uint_as_float(sr[4 * c + 1]),
                          __uint_as_float(sr[4 * c + 2]), __uint_as_float(sr[4 * c + 3]));
          }
        }
        mbar_arrive_cluster(xfull_peer0 + 8u * xs);
        if (!wt.wait<true>(x_full(xs), xph, 34)) { ok = false; break; }
        float z[64];
        {
          const float* rowp = xloc + xs * (C::X_BYTES / 4) + h * 64u;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float4 o = *reinterpret_cast<const float4*>(rowp + ((c ^ (h & 15u)) << 2));
            const float m0 = __uint_as_float(sr[4 * c]), m1 = __uint_as_float(sr[4 * c + 1]);
            const float m2_ = __uint_as_float(sr[4 * c + 2]), m3 = __uint_as_float(sr[4 * c + 3]);
            // fixed order (rank-0 partial + rank-1 partial): both CTAs get identical sums
            z[4 * c + 0] = rank == 0 ? m0 + o.x : o.x + m0;
            z[4 * c + 1] = rank == 0 ? m1 + o.y : o.y + m1;
            z[4 * c + 2] = rank == 0 ? m2_ + o.z : o.z + m2_;
            z[4 * c + 3] = rank == 0 ? m3 + o.w : o.w + m3;
          }
        }
        mbar_arrive_cluster(xempty_peer0 + 8u * xs);
        // ---- online softmax (log2 domain), lazy rescale
        const int32_t nvalid = min(kBlk, total - b * kBlk);
        float mb = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          z[j] = (j < nvalid) ? z[j] * p.scale_log2 : -INFINITY;
          mb = fmaxf(mb, z[j]);
        }
        const bool need = (mb > m2 + 8.0f);
        float alpha = 1.0f;
        if (need) {
          alpha = (m2 == -INFINITY) ? 0.0f : ex2_approx(m2 - mb);
          m2 = mb;
          l *= alpha;
        }
        uint32_t pk[32];
        float lsum = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __nv_bfloat162 pr = __floats2bfloat162_rn(ex2_approx(z[2 * j] - m2), ex2_approx(z[2 * j + 1] - m2));
          const float2 back = __bfloat1622float2(pr);
          lsum += back.x + back.y;
          pk[j] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        l += lsum;
        // ---- P -> TMEM (and rescale O) once the previous P.V has finished
        if (b > 0) {
          if (lane == 0) got = wt.wait(p_empty, (pb & 1u), 35) ? 1u : 0u;
          if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
          ++pb;
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
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
          }
        }
        tmem_st16(tmem + lane_off + C::COL_P, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
        tmem_st16(tmem + lane_off + C::COL_P + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      // ---- epilogue: wait for the last P.V, normalise, store
      if (lane == 0) got = wt.wait(p_empty, (pb & 1u), 36) ? 1u : 0u;
      if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
      ++pb;
      tc_fence_after();
      const float inv = 1.0f / l;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + C::COL_O + 32 * c, o);
        tmem_wait_ld();
        uint4 pkd[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          const __nv_bfloat162 pr =
              __floats2bfloat162_rn(__uint_as_float(o[2 * v]) * inv, __uint_as_float(o[2 * v + 1]) * inv);
          pw[v] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = pkd[v];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      if (rank == 0) p.lse[static_cast<size_t>(qi) * kHeads + h] = (m2 + log2f(l)) * 0.69314718055994531f;
    }
  }
  // ---- teardown: every role reaches here (all waits are bounded)
  tc_fence_before();
  __syncthreads();
  cluster_sync();            // no CTA leaves while its peer may still touch its shared memory
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace dsa
