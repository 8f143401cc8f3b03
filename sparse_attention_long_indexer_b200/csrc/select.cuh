// Exact top-k selection over (key, position) candidates held in shared memory.
//
// Keys are order-preserving 32-bit images of fp32 scores (larger score <=> larger key);
// ranking is by key descending, then by position ascending (equal scores go to the lower
// position). `select_exact` keeps exactly k of n > k candidates in place: an 8-bit MSB-first
// radix select finds the k-th key v, a second radix select over positions resolves the
// items equal to v, and one pass compacts. All `T` threads of the calling group execute it
// together; synchronisation uses named barrier `bar_id`.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace dsa {

// Order-preserving map of an fp32 score to uint32 (-0 is folded into +0 first).
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelectScratch {
  uint32_t hist[256];
  uint32_t bin;     // chosen digit
  uint32_t above;   // items strictly above the chosen bin (among the active prefix)
  uint32_t out_count;
  uint32_t pad;
};

// Adds 1 to hist[bin] for every lane with `active`, one shared atomic per distinct bin in
// the warp (candidates cluster in few bins, so per-lane atomics would serialise).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t key = active ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, key);
  if (active && lane == static_cast<uint32_t>(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
}

// Warp 0 scans hist (bins descending when kDescending, else ascending) and publishes the bin
// where the running count first reaches `rem`, with the count before it.
template <bool kDescending>
__device__ __forceinline__ void scan_pick(SelectScratch* sc, uint32_t rem) {
  const uint32_t lane = threadIdx.x & 31;
  uint32_t loc[8];
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t bin = kDescending ? (255u - 8u * lane - i) : (8u * lane + i);
    loc[i] = sc->hist[bin];
    sum += loc[i];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= (uint32_t)o) incl += v;
  }
  uint32_t excl = incl - sum;
  if (excl < rem && rem <= incl) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (excl + loc[i] >= rem) {
        sc->bin = kDescending ? (255u - 8u * lane - i) : (8u * lane + i);
        sc->above = excl;
        break;
      }
      excl += loc[i];
    }
  }
}

// Keeps exactly k of the n candidates (n > k). Returns the k-th key; afterwards only
// candidates strictly better than (that key, any larger position) may be added.
template <int T, int MAXPER>
__device__ uint32_t select_exact(uint32_t* keys, int32_t* pos, uint32_t n, uint32_t k, SelectScratch* sc,
                                 uint32_t tid, uint32_t bar_id) {
  // ---- phase 1: the k-th largest key
  uint32_t prefix = 0, mask = 0, rem = k, n_eq = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (uint32_t i = tid; i < 256; i += T) sc->hist[i] = 0;
    named_barrier(bar_id, T);
    for (uint32_t i0 = 0; i0 < n; i0 += T) {      // uniform trip count: hist_add is warp-collective
      const uint32_t i = i0 + tid;
      const uint32_t key = i < n ? keys[i] : 0u;
      hist_add(sc->hist, (key >> shift) & 255u, i < n && (key & mask) == prefix);
    }
    named_barrier(bar_id, T);
    if (tid < 32) scan_pick<true>(sc, rem);
    named_barrier(bar_id, T);
    uint32_t bin = sc->bin;
    rem -= sc->above;
    n_eq = sc->hist[bin];
    prefix |= bin << shift;
    mask |= 0xFFu << shift;
    named_barrier(bar_id, T);
  }
  const uint32_t vk = prefix;
  // ---- phase 2: among the n_eq items equal to vk keep the rem lowest positions
  uint32_t plim = 0xFFFFFFFFu;
  if (rem < n_eq) {
    uint32_t pprefix = 0, pmask = 0, prem = rem;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (uint32_t i = tid; i < 256; i += T) sc->hist[i] = 0;
      named_barrier(bar_id, T);
      for (uint32_t i0 = 0; i0 < n; i0 += T) {
        const uint32_t i = i0 + tid;
        const uint32_t p = i < n ? static_cast<uint32_t>(pos[i]) : 0u;
        hist_add(sc->hist, (p >> shift) & 255u, i < n && keys[i] == vk && (p & pmask) == pprefix);
      }
      named_barrier(bar_id, T);
      if (tid < 32) scan_pick<false>(sc, prem);
      named_barrier(bar_id, T);
      prem -= sc->above;
      pprefix |= sc->bin << shift;
      pmask |= 0xFFu << shift;
      named_barrier(bar_id, T);
    }
    plim = pprefix;
  }
  // ---- phase 3: compact in place (every item is read before any is written)
  uint32_t rk[MAXPER];
  int32_t rp[MAXPER];
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    uint32_t i = tid + j * T;
    rk[j] = 0;
    rp[j] = -1;
    if (i < n) {
      rk[j] = keys[i];
      rp[j] = pos[i];
    }
  }
  if (tid == 0) sc->out_count = 0;
  named_barrier(bar_id, T);
  const uint32_t lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    bool keep = (rp[j] >= 0) && (tid + j * T < n) &&
                (rk[j] > vk || (rk[j] == vk && static_cast<uint32_t>(rp[j]) <= plim));
    uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (m) {
      uint32_t base = 0;
      uint32_t leader = __ffs(m) - 1;
      if (lane == leader) base = atomicAdd(&sc->out_count, __popc(m));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (keep) {
        uint32_t at = base + __popc(m & ((1u << lane) - 1u));
        keys[at] = rk[j];
        pos[at] = rp[j];
      }
    }
  }
  named_barrier(bar_id, T);
  return vk;
}

// Cheap shrink used while streaming: keeps every candidate whose key is at least the lower
// edge of the histogram bin holding the k-th largest key, bins splitting the current key
// range [min, max] into 256 equal intervals. At least k candidates stay (typically k plus a
// few), and everything dropped is strictly below k kept ones, so the returned threshold is
// non-strict: later candidates equal to it must still be admitted. Returns the new count;
// `*thr_out` receives the threshold.
template <int T, int MAXPER>
__device__ uint32_t shrink_candidates(uint32_t* keys, int32_t* pos, uint32_t n, uint32_t k, SelectScratch* sc,
                                      uint32_t tid, uint32_t bar_id, uint32_t* thr_out) {
  const uint32_t lane = threadIdx.x & 31;
  uint32_t rk[MAXPER];
  int32_t rp[MAXPER];
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    const uint32_t i = tid + j * T;
    rk[j] = 0;
    rp[j] = -1;
    if (i < n) {
      rk[j] = keys[i];
      rp[j] = pos[i];
      lo = min(lo, rk[j]);
      hi = max(hi, rk[j]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  for (uint32_t i = tid; i < 256; i += T) sc->hist[i] = 0;
  if (tid == 0) {
    sc->bin = 0xFFFFFFFFu;   // running min
    sc->above = 0u;          // running max
  }
  named_barrier(bar_id, T);
  if (lane == 0) {
    atomicMin(&sc->bin, lo);
    atomicMax(&sc->above, hi);
  }
  named_barrier(bar_id, T);
  lo = sc->bin;
  hi = sc->above;
  const uint32_t range = hi - lo;
  const uint32_t shift = range < 256u ? 0u : (32u - __clz(range)) - 8u;
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) hist_add(sc->hist, (rk[j] - lo) >> shift, rp[j] >= 0);
  named_barrier(bar_id, T);
  if (tid < 32) scan_pick<true>(sc, k);
  named_barrier(bar_id, T);
  const uint32_t thr = lo + (sc->bin << shift);
  if (tid == 0) sc->out_count = 0;
  named_barrier(bar_id, T);
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    const bool keep = rp[j] >= 0 && rk[j] >= thr;
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (m) {
      uint32_t base = 0;
      const uint32_t leader = __ffs(m) - 1;
      if (lane == leader) base = atomicAdd(&sc->out_count, __popc(m));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (keep) {
        const uint32_t at = base + __popc(m & ((1u << lane) - 1u));
        keys[at] = rk[j];
        pos[at] = rp[j];
      }
    }
  }
  named_barrier(bar_id, T);
  *thr_out = thr;
  return sc->out_count;
}

}  // namespace dsa
