// Exact top-k selection over (key, position) candidates held in shared memory.
//
// Keys are order-preserving 32-bit images of fp32 scores (larger score <=> larger key);
// ranking is by key descending, then by position ascending (equal scores go to the lower
// position). `select_exact` keeps exactly k of n > k candidates in place: histogram passes
// over a shrinking key range find the bin holding the k-th key (down to a single key value
// if needed), passes over positions resolve the items equal to it, and one pass compacts.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace dsa {

// Order-preserving map of an fp32 score to uint32 (-0 is folded into +0 first).
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of score_key: the fp32 score a key was made from.
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct SelectScratch {
  uint32_t hist[256];
  uint32_t bin;     // chosen digit
  uint32_t above;   // items strictly above the chosen bin (among the active prefix)
  uint32_t out_count;
  uint32_t cnt;     // items in the chosen bin
  uint32_t wlo[8];  // per-warp minima / maxima of a group reduction
  uint32_t whi[8];
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

// ------------------------------------------------------------------ register-resident selection
// The candidates of a group are read once into registers (thread tid holds items tid + j*T);
// histogram passes bin them over an adaptive key range with plain shared-memory atomics, and
// the survivors are written back with one atomic per warp. All T threads of the group call
// these together; synchronisation uses named barrier `bar_id`.

template <int T, int MAXPER>
__device__ __forceinline__ void load_candidates(const uint32_t* keys, const int32_t* pos, uint32_t n, uint32_t tid,
                                                uint32_t (&rk)[MAXPER], int32_t (&rp)[MAXPER]) {
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    const uint32_t i = tid + j * T;
    rk[j] = i < n ? keys[i] : 0u;
    rp[j] = i < n ? pos[i] : -1;
  }
}

// Upper edge of the bin starting at b of width 2^shift, clamped to hi.
__device__ __forceinline__ uint32_t bin_end(uint32_t b, uint32_t shift, uint32_t hi) {
  const uint64_t e = static_cast<uint64_t>(b) + ((1ull << shift) - 1ull);
  return e < hi ? static_cast<uint32_t>(e) : hi;
}

// Smallest shift that brings a value range below 256 bins.
__device__ __forceinline__ uint32_t bin_shift(uint32_t range) { return range < 256u ? 0u : (32u - __clz(range)) - 8u; }

// Group-wide min / max of v(j) over the items with act(j).
template <int T, int MAXPER, typename Act, typename Val>
__device__ __forceinline__ void group_minmax(Act act, Val v, SelectScratch* sc, uint32_t tid, uint32_t bar_id,
                                             uint32_t& lo, uint32_t& hi) {
  lo = 0xFFFFFFFFu;
  hi = 0u;
#pragma unroll
  for (int j = 0; j < MAXPER; ++j)
    if (act(j)) {
      lo = min(lo, v(j));
      hi = max(hi, v(j));
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if ((threadIdx.x & 31) == 0) {
    sc->wlo[tid >> 5] = lo;
    sc->whi[tid >> 5] = hi;
  }
  named_barrier(bar_id, T);
#pragma unroll
  for (int w = 0; w < T / 32; ++w) {
    lo = min(lo, sc->wlo[w]);
    hi = max(hi, sc->whi[w]);
  }
}

// Warp 0 scans hist (descending or ascending bins) for the bin where the running count
// first reaches `rem`; publishes the bin, the count before it and its own count.
template <bool kDescending>
__device__ __forceinline__ void scan_bins(SelectScratch* sc, uint32_t rem) {
  const uint32_t lane = threadIdx.x & 31;
  uint32_t loc[8];
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t bin = kDescending ? (255u - 8u * lane - i) : (8u * lane + i);
    loc[i] = sc->hist[bin];
    sum += loc[i];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= static_cast<uint32_t>(o)) incl += v;
  }
  uint32_t excl = incl - sum;
  if (excl < rem && rem <= incl) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (excl + loc[i] >= rem) {
        sc->bin = kDescending ? (255u - 8u * lane - i) : (8u * lane + i);
        sc->above = excl;
        sc->cnt = loc[i];
        break;
      }
      excl += loc[i];
    }
  }
}

// One histogram pass over the items with act(j), bin b(j) < 256.
template <bool kDescending, int T, int MAXPER, typename Act, typename Bin>
__device__ __forceinline__ void hist_pass(Act act, Bin b, uint32_t rem, SelectScratch* sc, uint32_t tid,
                                          uint32_t bar_id, uint32_t& bin, uint32_t& above, uint32_t& cnt) {
  for (uint32_t i = tid; i < 256; i += T) sc->hist[i] = 0;
  named_barrier(bar_id, T);
#pragma unroll
  for (int j = 0; j < MAXPER; ++j)
    if (act(j)) atomicAdd(&sc->hist[b(j)], 1u);
  named_barrier(bar_id, T);
  if (tid < 32) scan_bins<kDescending>(sc, rem);
  named_barrier(bar_id, T);
  bin = sc->bin;
  above = sc->above;
  cnt = sc->cnt;
}

// Writes the kept register items to the front of keys/pos (any order), one atomic per warp.
// Every thread must have loaded its items before the group's last barrier.
template <int T, int MAXPER, typename Keep>
__device__ __forceinline__ void compact_candidates(uint32_t* keys, int32_t* pos, const uint32_t (&rk)[MAXPER],
                                                   const int32_t (&rp)[MAXPER], Keep keep, SelectScratch* sc,
                                                   uint32_t bar_id) {
  static_assert(MAXPER <= 64, "keep mask");
  const uint32_t lane = threadIdx.x & 31;
  uint64_t mask = 0;
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < MAXPER; ++j)
    if (rp[j] >= 0 && keep(rk[j], rp[j])) {
      mask |= 1ull << j;
      ++c;
    }
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= static_cast<uint32_t>(o)) incl += v;
  }
  uint32_t base = 0;
  if (lane == 31) base = atomicAdd(&sc->out_count, incl);
  base = __shfl_sync(0xffffffffu, base, 31);
  uint32_t at = base + incl - c;
#pragma unroll
  for (int j = 0; j < MAXPER; ++j)
    if (mask & (1ull << j)) {
      keys[at] = rk[j];
      pos[at] = rp[j];
      ++at;
    }
  named_barrier(bar_id, T);
}

// Key passes over the items held in registers: narrows an adaptive range down to the bin that
// holds the k-th largest key. Returns the bin's lower edge and `rem`, the places left for the
// items at or above it once the items above the bin are counted; `ties` says that the bin is a
// single key value holding more items than places.
struct KthKey {
  uint32_t value;
  uint32_t rem;
  bool ties;
};

template <int T, int MAXPER>
__device__ __forceinline__ KthKey kth_key(const uint32_t (&rk)[MAXPER], const int32_t (&rp)[MAXPER], uint32_t k,
                                          SelectScratch* sc, uint32_t tid, uint32_t bar_id) {
  uint32_t lo, hi;
  group_minmax<T, MAXPER>([&](int j) { return rp[j] >= 0; }, [&](int j) { return rk[j]; }, sc, tid, bar_id, lo, hi);
  uint32_t rem = k, shift = bin_shift(hi - lo), a_lo = lo, a_hi = hi;
  while (true) {
    uint32_t bin, above, cnt;
    hist_pass<true, T, MAXPER>([&](int j) { return rp[j] >= 0 && rk[j] >= a_lo && rk[j] <= a_hi; },
                               [&](int j) { return (rk[j] - a_lo) >> shift; }, rem, sc, tid, bar_id, bin, above, cnt);
    rem -= above;
    const uint32_t blo = a_lo + (bin << shift);
    if (cnt == rem) return KthKey{blo, rem, false};   // the whole bin is in: keys >= blo are exactly k
    if (shift == 0) return KthKey{blo, rem, true};    // one key value, more items than places
    a_hi = bin_end(blo, shift, a_hi);
    a_lo = blo;
    shift = shift > 8u ? shift - 8u : 0u;
  }
}

// Keeps exactly k of the n candidates (n > k): the k largest keys, equal keys ranked by the
// lower position. Returns a threshold key t such that any later candidate with a key <= t
// (and, being later, a larger position) cannot enter the top k. `*tied` (if given) is set when
// candidates equal to the k-th key were dropped for their position.
template <int T, int MAXPER>
__device__ uint32_t select_exact(uint32_t* keys, int32_t* pos, uint32_t n, uint32_t k, SelectScratch* sc,
                                 uint32_t tid, uint32_t bar_id, bool* tied = nullptr) {
  uint32_t rk[MAXPER];
  int32_t rp[MAXPER];
  load_candidates<T, MAXPER>(keys, pos, n, tid, rk, rp);
  if (tid == 0) sc->out_count = 0;
  const KthKey kth = kth_key<T, MAXPER>(rk, rp, k, sc, tid, bar_id);
  if (tied != nullptr) *tied = kth.ties;
  if (!kth.ties) {
    const uint32_t thr = kth.value;
    compact_candidates<T, MAXPER>(keys, pos, rk, rp, [&](uint32_t key, int32_t) { return key >= thr; }, sc, bar_id);
    return thr;
  }
  // ---- position passes among the items equal to vk: keep the rem lowest positions
  const uint32_t vk = kth.value;
  uint32_t rem = kth.rem;
  uint32_t plo, phi;
  group_minmax<T, MAXPER>([&](int j) { return rp[j] >= 0 && rk[j] == vk; },
                          [&](int j) { return static_cast<uint32_t>(rp[j]); }, sc, tid, bar_id, plo, phi);
  uint32_t pshift = bin_shift(phi - plo), p_lo = plo, p_hi = phi, plim = phi;
  while (true) {
    uint32_t bin, below, cnt;
    hist_pass<false, T, MAXPER>(
        [&](int j) {
          const uint32_t pu = static_cast<uint32_t>(rp[j]);
          return rp[j] >= 0 && rk[j] == vk && pu >= p_lo && pu <= p_hi;
        },
        [&](int j) { return (static_cast<uint32_t>(rp[j]) - p_lo) >> pshift; }, rem, sc, tid, bar_id, bin, below, cnt);
    rem -= below;
    const uint32_t pb = p_lo + (bin << pshift);
    const uint32_t pe = bin_end(pb, pshift, p_hi);
    if (cnt == rem || pshift == 0) {  // positions are distinct: a one-position bin holds one item
      plim = pe;
      break;
    }
    p_lo = pb;
    p_hi = pe;
    pshift = pshift > 8u ? pshift - 8u : 0u;
  }
  compact_candidates<T, MAXPER>(
      keys, pos, rk, rp,
      [&](uint32_t key, int32_t ps) { return key > vk || (key == vk && static_cast<uint32_t>(ps) <= plim); }, sc,
      bar_id);
  return vk;
}

// Keeps every candidate whose key is at least the k-th largest key value v (ties at v all
// stay, so k or more remain) and returns v, or the lower edge of a bin that holds exactly the
// k largest keys. `*kept` receives the number of candidates kept.
template <int T, int MAXPER>
__device__ uint32_t select_keep_ge(uint32_t* keys, int32_t* pos, uint32_t n, uint32_t k, SelectScratch* sc,
                                   uint32_t tid, uint32_t bar_id, uint32_t* kept) {
  uint32_t rk[MAXPER];
  int32_t rp[MAXPER];
  load_candidates<T, MAXPER>(keys, pos, n, tid, rk, rp);
  if (tid == 0) sc->out_count = 0;
  const uint32_t v = kth_key<T, MAXPER>(rk, rp, k, sc, tid, bar_id).value;
  compact_candidates<T, MAXPER>(keys, pos, rk, rp, [&](uint32_t key, int32_t) { return key >= v; }, sc, bar_id);
  *kept = sc->out_count;
  return v;
}

// Cheap shrink used while streaming: one histogram pass over the candidates' key range
// [min, max] in 256 equal bins keeps every candidate at or above the lower edge of the bin
// holding the k-th largest key. At least k candidates stay, and everything dropped is below
// k kept ones, so the returned threshold is non-strict: later candidates equal to it must
// still be admitted. Returns the new count; `*thr_out` receives the threshold.
template <int T, int MAXPER>
__device__ uint32_t shrink_candidates(uint32_t* keys, int32_t* pos, uint32_t n, uint32_t k, SelectScratch* sc,
                                      uint32_t tid, uint32_t bar_id, uint32_t* thr_out) {
  uint32_t rk[MAXPER];
  int32_t rp[MAXPER];
  load_candidates<T, MAXPER>(keys, pos, n, tid, rk, rp);
  if (tid == 0) sc->out_count = 0;
  uint32_t lo, hi;
  group_minmax<T, MAXPER>([&](int j) { return rp[j] >= 0; }, [&](int j) { return rk[j]; }, sc, tid, bar_id, lo, hi);
  const uint32_t shift = bin_shift(hi - lo);
  uint32_t bin, above, cnt;
  hist_pass<true, T, MAXPER>([&](int j) { return rp[j] >= 0; }, [&](int j) { return (rk[j] - lo) >> shift; }, k, sc,
                             tid, bar_id, bin, above, cnt);
  const uint32_t thr = lo + (bin << shift);
  compact_candidates<T, MAXPER>(keys, pos, rk, rp, [&](uint32_t key, int32_t) { return key >= thr; }, sc, bar_id);
  *thr_out = thr;
  return above + cnt;
}

}  // namespace dsa
