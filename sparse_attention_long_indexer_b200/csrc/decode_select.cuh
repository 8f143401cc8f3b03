// Decode top-k: the exact k best keys of one query per sequence, from its full row of keys.
//
// DeepSeek-V3.2 article, DSA section (top-k selector): each query keeps the k tokens with
// the highest index scores among the tokens before it. In decode there is one query per
// sequence, so its index scores form one row of at most max_len values. The indexer kernel
// writes that row as order-preserving keys (`score_key`) and this kernel selects from it;
// the row (4 bytes a token) is written and read back through L2, against 132 bytes a token
// of cached indexer keys that the scoring pass streams from HBM.
//
// One cluster of kSelCluster CTAs per sequence; CTA c owns the row's positions
// [c * kSelSlice, (c + 1) * kSelSlice), thread j the positions base + j + kSelThreads * i.
// Each pass streams the CTA's keys again (from L2, where the row was just written): small
// CTAs that all fit on the GPU at once beat keeping the row in registers, which would need
// most of the register file per sequence. Histogram passes (256 bins: the top 8 bits first,
// then a shrinking range, as in select.cuh) find the bin of the k-th key; the CTAs add up
// their histograms through distributed shared memory, so every CTA takes the same
// decisions. Keys equal to the k-th are resolved by further passes over their positions
// (lowest first).
//
// Before that, a guess: the r-th best key of a 1/16 sample of the row (r ~ 1.5 k scaled to
// the sample, as in the indexer's prefill items) is very likely below the k-th key. One stream
// over the row keeps every key at or above it in shared memory (about 1.5 k for the whole
// row), and when no CTA overflowed and at least k keys made it, the passes run over those
// candidates only; otherwise they run over the whole row.
//
// Ranking matches select.cuh: key descending, then position ascending. The output row holds
// min(k, n) positions (in no particular order) followed by -1.
#pragma once
#include <cstdint>

#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kSelCluster = 8;                                  // CTAs per sequence
constexpr int kSelThreads = 256;
constexpr int kSelPer = 64;                                     // positions per thread
constexpr int kSelSlice = kSelThreads * kSelPer;                // positions per CTA
constexpr int kSelMaxLen = kSelCluster * kSelSlice;             // 131072 positions per row
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelBatch = 16;                                   // loads in flight per thread
static_assert(kSelPer % kSelBatch == 0, "whole batches per thread");
constexpr int kSelSampleEvery = 16;                             // the sample: every 16th key slot
constexpr int kSelSamples = kSelPer / kSelSampleEvery;          // sampled slots per thread
constexpr int kSelCap = 4096;                                   // candidates per CTA (sampled path)

struct DecodeSelectParams {
  const uint32_t* keys;     // [B, max_len] order-preserving keys, positions < n valid
  const int32_t* lengths;   // [B]; the query sits at position len - 1 and sees n = len keys
  int32_t* out_idx;         // [B, topk]
  float* out_scores;        // optional [B, topk]
  int32_t max_len, topk;
};

struct DecodeSelectSmem {
  uint32_t lhist[2][256];           // this CTA's histogram (double-buffered across passes)
  SelectScratch sc;                 // the cluster's histogram and the scan result
  uint32_t taken;                   // keys this CTA writes (read by the CTAs of higher rank)
  uint32_t n_sample, n_cand;        // this CTA's sampled keys and candidates (read by all CTAs)
  uint32_t wred[kSelWarps];
  uint32_t out_ctr;
  uint32_t cand_n;                  // candidates appended (may pass kSelCap: then none is trusted)
  uint32_t cand_key[kSelCap];
  int32_t cand_pos[kSelCap];
};

// Sum over the CTAs of ranks below `rank` of the smem word at `local`.
__device__ __forceinline__ uint32_t cluster_prefix(uint32_t local, uint32_t rank) {
  uint32_t s = 0;
  for (uint32_t r = 0; r < rank; ++r) s += ld_cluster_u32(mapa(local, r));
  return s;
}

// The value v(key, pos) of the rank-`rem` item among those with act(key, pos), over the
// cluster: histogram passes over [a_lo, a_hi] (bins descending when kDesc, else ascending).
// Returns with `v` the lower (kDesc) or upper (ascending) edge of the last bin and rem the
// number of items still needed from it; `whole` when the bin's items are all needed.
// `pb` carries the histogram buffer parity across calls.
template <bool kDesc, typename Fn>
__device__ __forceinline__ void cluster_select(Fn&& for_items, uint32_t a_lo, uint32_t a_hi, uint32_t shift,
                                               uint32_t& rem, uint32_t& v, bool& whole, DecodeSelectSmem& sm,
                                               uint32_t& pb) {
  const uint32_t tid = threadIdx.x;
  while (true) {
    for_items([&](uint32_t x, bool act) {
      act = act && x >= a_lo && x <= a_hi;
      if (__any_sync(0xffffffffu, act)) hist_add(sm.lhist[pb], act ? (x - a_lo) >> shift : 0u, act);
    });
    cluster_sync();   // this pass's histograms are complete; last pass's were read by all
    if (tid < 256) {
      sm.lhist[pb ^ 1u][tid] = 0u;
      uint32_t s = 0;
#pragma unroll
      for (int r = 0; r < kSelCluster; ++r) s += ld_cluster_u32(mapa(smem_u32(&sm.lhist[pb][tid]), r));
      sm.sc.hist[tid] = s;
    }
    pb ^= 1u;
    __syncthreads();
    if (tid < 32) scan_bins<kDesc>(&sm.sc, rem);
    __syncthreads();
    const uint32_t bin = sm.sc.bin, above = sm.sc.above, cnt = sm.sc.cnt;
    rem -= above;
    const uint32_t blo = a_lo + (bin << shift), bhi = bin_end(blo, shift, a_hi);
    if (cnt == rem || shift == 0) {   // the whole bin is needed, or it holds a single value
      v = kDesc ? blo : bhi;
      whole = cnt == rem;
      return;
    }
    a_lo = blo;
    a_hi = bhi;
    shift = shift > 8u ? shift - 8u : 0u;
  }
}

__global__ void __cluster_dims__(kSelCluster, 1, 1) __launch_bounds__(kSelThreads, 4)
decode_select_kernel(const DecodeSelectParams p) {
  __shared__ DecodeSelectSmem sm;
  const uint32_t tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const uint32_t rank = cluster_ctarank();
  const int32_t b = static_cast<int32_t>(blockIdx.x / kSelCluster);
  const int32_t n = min(max(__ldg(p.lengths + b), 0), p.max_len);   // keys 0 .. len - 1
  const uint32_t k = static_cast<uint32_t>(p.topk);
  const int32_t base = static_cast<int32_t>(rank) * kSelSlice + static_cast<int32_t>(tid);
  const uint32_t* row = p.keys + static_cast<size_t>(b) * p.max_len;
  int32_t* out = p.out_idx + static_cast<size_t>(b) * p.topk;
  float* outs = p.out_scores == nullptr ? nullptr : p.out_scores + static_cast<size_t>(b) * p.topk;
  // fn(key, pos, valid) for this thread's positions, in warp-uniform steps. The keys come in
  // batches, each loaded while the one before is processed (fn holds warp votes and shared
  // atomics, which would otherwise keep every load behind the last key's work); batches past
  // the row's end for the whole CTA are skipped.
  const int32_t cta_base = static_cast<int32_t>(rank) * kSelSlice;
  auto load_batch = [&](int i0, uint32_t(&kb)[kSelBatch]) {
#pragma unroll
    for (int j = 0; j < kSelBatch; ++j) {
      const int32_t pos = base + (i0 + j) * kSelThreads;
      kb[j] = pos < n ? __ldcg(row + pos) : 0u;
    }
  };
  auto for_keys = [&](auto&& fn) {
    if (cta_base >= n) return;                          // the same for every thread of the CTA
    uint32_t kb[kSelBatch], kn[kSelBatch];
    load_batch(0, kb);
#pragma unroll
    for (int i0 = 0; i0 < kSelPer; i0 += kSelBatch) {
      const bool more = i0 + kSelBatch < kSelPer && cta_base + (i0 + kSelBatch) * kSelThreads < n;
      if (more) load_batch(i0 + kSelBatch, kn);
#pragma unroll
      for (int j = 0; j < kSelBatch; ++j) {
        const int32_t pos = base + (i0 + j) * kSelThreads;
        fn(kb[j], pos, pos < n);
      }
      if (!more) break;
#pragma unroll
      for (int j = 0; j < kSelBatch; ++j) kb[j] = kn[j];
    }
  };

  if (static_cast<uint32_t>(n) <= k) {
    // every key is selected: position j goes to slot j, the rest of the row is padding
    for_keys([&](uint32_t key, int32_t pos, bool valid) {
      if (valid) {
        out[pos] = pos;
        if (outs != nullptr) outs[pos] = key_score(key);
      }
    });
    if (rank == 0)
      for (uint32_t j = static_cast<uint32_t>(n) + tid; j < k; j += kSelThreads) {
        out[j] = -1;
        if (outs != nullptr) outs[j] = -INFINITY;
      }
    return;   // no distributed shared memory was touched
  }

  for (uint32_t t = tid; t < 512u; t += kSelThreads) (&sm.lhist[0][0])[t] = 0u;
  if (tid == 0) sm.cand_n = 0;
  __syncthreads();
  uint32_t pb = 0;
  auto block_total = [&](uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) sm.wred[warp] = v;
    __syncthreads();
    uint32_t t = 0;
    for (int w = 0; w < kSelWarps; ++w) t += sm.wred[w];
    return t;
  };

  // The exact top-k of the items that for_items(fn) visits (fn(key, pos, valid), warp-uniform),
  // written to the output row. Every key at least as good as the k-th must be among the items.
  auto select_and_write = [&](auto&& for_items) {
    // ---- the k-th key: first over the top 8 bits of the key, then within the chosen bin
    uint32_t rem = k, vk = 0;
    bool take_all = false;
    cluster_select<true>(
        [&](auto&& add) { for_items([&](uint32_t key, int32_t, bool valid) { add(key, valid); }); }, 0u,
        0xFFFFFFFFu, 24u, rem, vk, take_all, sm, pb);
    // ---- keys equal to vk when only rem of them fit: the rem lowest positions
    uint32_t vp = 0xFFFFFFFFu;   // ties at positions <= vp are taken
    if (!take_all) {
      const uint32_t span = static_cast<uint32_t>(n - 1);
      bool whole = false;
      cluster_select<false>(
          [&](auto&& add) {
            for_items(
                [&](uint32_t key, int32_t pos, bool valid) { add(static_cast<uint32_t>(pos), valid && key == vk); });
          },
          0u, span, bin_shift(span), rem, vp, whole, sm, pb);
    }
    // ---- write: CTA offsets by a prefix over ranks, warp slots by one shared atomic per warp
    auto taken = [&](uint32_t key, int32_t pos, bool valid) {
      return valid && (key > vk || (key == vk && static_cast<uint32_t>(pos) <= vp));
    };
    uint32_t mine = 0;
    for_items([&](uint32_t key, int32_t pos, bool valid) { mine += taken(key, pos, valid) ? 1u : 0u; });
    const uint32_t total = block_total(mine);
    if (tid == 0) {
      sm.taken = total;
      sm.out_ctr = 0;
    }
    cluster_sync();
    const uint32_t offset = cluster_prefix(smem_u32(&sm.taken), rank);
    cluster_sync();   // no CTA leaves while another may still read its shared memory
    for_items([&](uint32_t key, int32_t pos, bool valid) {
      const bool t = taken(key, pos, valid);
      const uint32_t m = __ballot_sync(0xffffffffu, t);
      if (m == 0u) return;
      uint32_t at = 0;
      if (lane == 0) at = atomicAdd(&sm.out_ctr, static_cast<uint32_t>(__popc(m)));
      at = __shfl_sync(0xffffffffu, at, 0);
      if (t) {
        const uint32_t j = offset + at + static_cast<uint32_t>(__popc(m & ((1u << lane) - 1u)));
        if (j < k) {             // exactly k are taken; the bound keeps every store in the row
          out[j] = pos;
          if (outs != nullptr) outs[j] = key_score(key);
        }
      }
    });
  };

  // ---- sampled threshold: the r-th best of a 1/16 sample (key slots 0, 16, 32, 48 of every
  // thread), r ~ 1.5 k scaled to the sample, is a guess at a key below the k-th. One stream over
  // the row keeps every key at or above it in shared memory, and the exact selection runs over
  // those few candidates. If some CTA's candidates overflow, or fewer than k keys reach the
  // guess, the selection runs over the whole row instead (the decision is the cluster's).
  uint32_t skey[kSelSamples];
  uint32_t n_mine = 0;
#pragma unroll
  for (int q = 0; q < kSelSamples; ++q) {
    const int32_t pos = base + q * kSelSampleEvery * kSelThreads;
    skey[q] = pos < n ? __ldcg(row + pos) : 0u;
    n_mine += pos < n ? 1u : 0u;
  }
  const uint32_t n_cta = block_total(n_mine);
  if (tid == 0) sm.n_sample = n_cta;
  cluster_sync();
  uint32_t n_s = 0;
#pragma unroll
  for (int r = 0; r < kSelCluster; ++r) n_s += ld_cluster_u32(mapa(smem_u32(&sm.n_sample), static_cast<uint32_t>(r)));
  const uint64_t r_s = (3ull * k * n_s + 2ull * static_cast<uint64_t>(n) - 1ull) / (2ull * static_cast<uint64_t>(n));
  if (r_s >= 1 && r_s < n_s) {
    uint32_t rem = static_cast<uint32_t>(r_s), vs = 0;
    bool whole = false;
    cluster_select<true>(
        [&](auto&& add) {
#pragma unroll
          for (int q = 0; q < kSelSamples; ++q) add(skey[q], base + q * kSelSampleEvery * kSelThreads < n);
        },
        0u, 0xFFFFFFFFu, 24u, rem, vs, whole, sm, pb);
    // at least r sampled keys are >= vs; keep every key of the row at or above it
    for_keys([&](uint32_t key, int32_t pos, bool valid) {
      const bool c = valid && key >= vs;
      const uint32_t m = __ballot_sync(0xffffffffu, c);
      if (m == 0u) return;
      uint32_t at = 0;
      if (lane == 0) at = atomicAdd(&sm.cand_n, static_cast<uint32_t>(__popc(m)));
      at = __shfl_sync(0xffffffffu, at, 0);
      if (c) {
        const uint32_t j = at + static_cast<uint32_t>(__popc(m & ((1u << lane) - 1u)));
        if (j < static_cast<uint32_t>(kSelCap)) {
          sm.cand_key[j] = key;
          sm.cand_pos[j] = pos;
        }
      }
    });
    __syncthreads();
    if (tid == 0) sm.n_cand = sm.cand_n;
    cluster_sync();
    uint32_t total = 0;
    bool over = false;
#pragma unroll
    for (int r = 0; r < kSelCluster; ++r) {
      const uint32_t c = ld_cluster_u32(mapa(smem_u32(&sm.n_cand), static_cast<uint32_t>(r)));
      total += c;
      over = over || c > static_cast<uint32_t>(kSelCap);
    }
    if (!over && total >= k) {
      // every key at least as good as the k-th is >= vs, so it is a candidate
      const uint32_t c = sm.cand_n;   // <= kSelCap, the same for every thread of the CTA
      select_and_write([&](auto&& fn) {
        for (uint32_t j0 = 0; j0 < c; j0 += kSelThreads) {
          const uint32_t j = j0 + tid;
          const bool v = j < c;
          fn(v ? sm.cand_key[j] : 0u, v ? sm.cand_pos[j] : 0, v);
        }
      });
      return;
    }
  }
  select_and_write(for_keys);
}

}  // namespace dsa
