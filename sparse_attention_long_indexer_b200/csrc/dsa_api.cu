// C ABI of the DSA forward path (declared in include/dsa.h): host-side validation,
// workspace layout, tensor-map encoding and kernel launches. No memory is allocated here;
// all scratch lives in the caller's workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "dsa.h"
#include "indexer_topk.cuh"
#include "decode_select.cuh"
#include "sparse_mla.cuh"
#include "indexer_kl.cuh"

namespace dsa {

// ----------------------------------------------------------------------------- padding kernels
// Copies rows of [heads_src x dims_src] into [heads_dst x dims_dst], zero elsewhere. Source dim
// d < split maps to d; split <= d < dims_src maps to d - split + hi_off (the RoPE part of a
// latent row lands at 512); used for inputs whose dims are below the production ones.
template <typename T>
__global__ void pad_rows_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t rows, int heads_src,
                                int dims_src, int heads_dst, int dims_dst, int split, int hi_off) {
  const int64_t per_row = static_cast<int64_t>(heads_dst) * dims_dst;
  const int64_t total = rows * per_row;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / per_row;
    const int64_t rem = e - r * per_row;
    const int hd = static_cast<int>(rem / dims_dst);
    const int dd = static_cast<int>(rem - static_cast<int64_t>(hd) * dims_dst);
    int ds = -1;
    if (hd < heads_src) {
      if (dd < split) ds = dd;
      else if (dd >= hi_off && dd - hi_off < dims_src - split) ds = dd - hi_off + split;
    }
    dst[e] = ds >= 0 ? src[(r * heads_src + hd) * dims_src + ds] : T(0);
  }
}

// Inverse: takes the first heads_dst x dims_dst of each [heads_src x dims_src] row.
template <typename T>
__global__ void unpad_rows_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t rows, int heads_src,
                                  int dims_src, int heads_dst, int dims_dst) {
  const int64_t per_row = static_cast<int64_t>(heads_dst) * dims_dst;
  const int64_t total = rows * per_row;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / per_row;
    const int64_t rem = e - r * per_row;
    const int hd = static_cast<int>(rem / dims_dst);
    const int dd = static_cast<int>(rem - static_cast<int64_t>(hd) * dims_dst);
    dst[e] = src[(r * heads_src + hd) * dims_src + dd];
  }
}

// Sets columns [cols_from, cols) of each of `rows` rows of width `cols` to `v`.
template <typename T>
__global__ void fill_cols_kernel(T* __restrict__ dst, int64_t rows, int cols_from, int cols, T v) {
  const int64_t per = cols - cols_from;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < rows * per;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / per;
    dst[r * cols + cols_from + (e - r * per)] = v;
  }
}

}  // namespace dsa

using namespace dsa;

namespace {

// An NVTX range over a scope: each call and each stage it launches shows up by name in a profiler
// timeline (`ncu --nvtx --nvtx-include ...` can filter on them). Header-only NVTX3: without a tool
// attached the calls do nothing.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr uint64_t kWaitBudgetNs = 2000000000ull;   // 2 s per bounded wait
// budget of the indexer's pipeline waits (dsa_set_wait_budget_ns, a test setting)
std::atomic<uint64_t> g_indexer_wait_ns{kWaitBudgetNs};
constexpr size_t kAlign = 256;
constexpr int kPrefillNQ = 4;                       // queries per prefill indexer work item
constexpr int kMergeThreads = 1024;                  // decode merge: one CTA per sequence

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Prefill items long enough for the indexer's sampled threshold exist (see indexer_topk.cuh).
bool sampled_threshold(const dsa_dims& d, int32_t topk) {
  return d.n_q > 1 && topk >= kSpecMinTopk && d.max_len >= kSpecMinTiles * kKeyTile;
}

bool is_production(const dsa_dims& d) {
  return d.n_idx_heads == kIdxHeads && d.idx_dim == kIdxDim && d.n_heads == kHeads && d.d_latent == kDv &&
         d.d_rope == kDqk - kDv;
}

dsa_status check_dims(const dsa_dims* d, int32_t topk) {
  if (d == nullptr) return DSA_ERR_INVALID_ARG;
  if (d->batch < 0 || d->n_q < 0 || d->max_len < 0) return DSA_ERR_INVALID_ARG;
  if (d->n_q > d->max_len) return DSA_ERR_INVALID_ARG;
  if (topk < 1) return DSA_ERR_INVALID_ARG;
  if (!(std::isfinite(d->softmax_scale))) return DSA_ERR_INVALID_ARG;
  if (d->n_idx_heads < 1 || d->idx_dim < 1 || d->n_heads < 1 || d->d_latent < 1 || d->d_rope < 0)
    return DSA_ERR_INVALID_ARG;
  if (topk > kMaxTopk) return DSA_ERR_UNSUPPORTED;
  if (d->n_idx_heads > kIdxHeads || d->idx_dim > kIdxDim || d->idx_dim % 16 != 0) return DSA_ERR_UNSUPPORTED;
  if (d->n_heads > kHeads || d->d_latent > kDv || d->d_latent % 8 != 0) return DSA_ERR_UNSUPPORTED;
  if (d->d_rope > kDqk - kDv || d->d_rope % 8 != 0) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->batch) * d->max_len > (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (d->n_q == 1 && (d->max_len + kDecodeChunk - 1) / kDecodeChunk > 1024) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

// Workspace regions, each 256-byte aligned.
struct Layout {
  size_t status = 0;                     // 256 B: status word + detail
  size_t key_rows = 0;                   // decode: every key of the row (max_len <= kSelMaxLen)
  size_t part_keys = 0, part_pos = 0, part_count = 0;   // decode beyond that: partial top-k
  size_t redo_flag = 0, redo_list = 0, redo_count = 0;  // prefill items queued for the exact pass
  size_t idx = 0;                        // forward's selection when out_idx == NULL
  size_t mask = 0, extent = 0;           // masked dense mode: bitmap rows and extents
  int32_t mask_words = 0;
  size_t q_idx = 0, w = 0, k_idx = 0, q = 0, kv = 0, out = 0, lse = 0;  // padded copies
  size_t total = 0;
  int32_t n_chunks = 0;
  bool padded = false;
};

Layout make_layout(const dsa_dims& d, int32_t topk) {
  Layout L;
  size_t off = 0;
  L.status = off;
  off += kAlign;
  const int64_t T = static_cast<int64_t>(d.batch) * d.n_q;
  const int64_t K = static_cast<int64_t>(d.batch) * d.max_len;
  if (d.n_q == 1) {
    L.n_chunks = (d.max_len + kDecodeChunk - 1) / kDecodeChunk;
    if (d.max_len <= kSelMaxLen) {
      L.key_rows = off; off = align_up(off + static_cast<size_t>(K) * 4);
    } else {
      const size_t slots = static_cast<size_t>(d.batch) * L.n_chunks;
      L.part_keys = off; off = align_up(off + slots * topk * 4);
      L.part_pos = off; off = align_up(off + slots * topk * 4);
      L.part_count = off; off = align_up(off + slots * 4);
    }
  }
  if (sampled_threshold(d, topk)) {
    const size_t items = static_cast<size_t>(d.batch) * ((d.n_q + kPrefillNQ - 1) / kPrefillNQ);
    L.redo_flag = off; off = align_up(off + items * 4);
    L.redo_list = off; off = align_up(off + items * 4);
    L.redo_count = off; off = align_up(off + 4);
  }
  L.idx = off; off = align_up(off + static_cast<size_t>(T) * topk * 4);
  if (d.max_len <= kMaskMaxLen) {
    L.mask_words = 2 * ((d.max_len + kBlk - 1) / kBlk);      // two words per 64-row block
    L.mask = off; off = align_up(off + static_cast<size_t>(T) * L.mask_words * 4);
    L.extent = off; off = align_up(off + static_cast<size_t>(T) * 4);
  }
  L.padded = !is_production(d);
  if (L.padded) {
    L.q_idx = off; off = align_up(off + static_cast<size_t>(T) * kIdxHeads * kIdxDim);
    L.w = off; off = align_up(off + static_cast<size_t>(T) * kIdxHeads * 2);
    L.k_idx = off; off = align_up(off + static_cast<size_t>(K) * kIdxDim);
    L.q = off; off = align_up(off + static_cast<size_t>(T) * kHeads * kDqk * 2);
    L.kv = off; off = align_up(off + static_cast<size_t>(K) * kDqk * 2);
    L.out = off; off = align_up(off + static_cast<size_t>(T) * kHeads * kDv * 2);
    L.lse = off; off = align_up(off + static_cast<size_t>(T) * kHeads * 4);
  }
  L.total = off;
  return L;
}

struct DeviceInfo {
  int sms = 0;
  bool sm100 = false;
  // the prefill indexer moves registers between warpgroups with setmaxnreg, which is sound only
  // for the register count its split was computed for
  bool indexer_regs_ok = false;
};

DeviceInfo device_info() {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return {};
  std::lock_guard<std::mutex> g(mu);
  if (!have[dev]) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cache[dev].sms = sms;
    cache[dev].sm100 = (major == 10 && minor == 0);
    // per-device kernel attributes (dynamic shared memory above 48 KB)
    cudaFuncSetAttribute(indexer_topk_kernel<kPrefillNQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         IdxCfg<kPrefillNQ>::SMEM_BYTES);
    cudaFuncSetAttribute(indexer_topk_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         IdxCfg<1>::SMEM_BYTES);
    cudaFuncSetAttribute(sparse_mla_attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         AttnCfg::SMEM_BYTES);
    cudaFuncSetAttribute(sparse_mla_attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         AttnCfg::SMEM_BYTES);
    cudaFuncSetAttribute(indexer_kl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, KlCfg::SMEM_BYTES);
    cudaFuncAttributes fa{};
    cache[dev].indexer_regs_ok = cudaFuncGetAttributes(&fa, indexer_topk_kernel<kPrefillNQ>) == cudaSuccess &&
                                 fa.numRegs == IdxCfg<kPrefillNQ>::LAUNCH_REGS;
    have[dev] = true;
  }
  return cache[dev];
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D byte tensor [outer, rows, 128] with a 128-byte-swizzled box {128, box_rows, 1}.
bool encode_rows_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t outer, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {128, rows, outer};
  const cuuint64_t strides[2] = {128, rows * 128};
  const cuuint32_t box[3] = {128, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Queries as a 2-D bf16 tensor [rows = B*n_q*128 heads, 576 dims], box {64 dims, 64 heads}.
bool encode_q_bf16(CUtensorMap* map, const void* base, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDqk), rows, 1};
  const cuuint64_t strides[2] = {kDqk * 2, rows * kDqk * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Latent cache as a 3-D bf16 tensor [1, rows = B*max_len, 576 dims], box {64 dims, box_rows, 1},
// 128-byte swizzle: one box is one swizzle-atom column of box_rows rows.
bool encode_kv_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDqk), rows, 1};
  const cuuint64_t strides[2] = {kDqk * 2, rows * kDqk * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

dsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

template <typename T>
cudaError_t launch_pad(const T* src, T* dst, int64_t rows, int hs, int ds, int hd, int dd, int split, int hi_off,
                       cudaStream_t st) {
  const int64_t total = rows * hd * dd;
  if (total == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 65535));
  pad_rows_kernel<T><<<blocks, 256, 0, st>>>(src, dst, rows, hs, ds, hd, dd, split, hi_off);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fill(T* dst, int64_t rows, int cols_from, int cols, T v, cudaStream_t st) {
  const int64_t total = rows * (cols - cols_from);
  if (total <= 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 65535));
  fill_cols_kernel<T><<<blocks, 256, 0, st>>>(dst, rows, cols_from, cols, v);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_unpad(const T* src, T* dst, int64_t rows, int hs, int ds, int hd, int dd, cudaStream_t st) {
  const int64_t total = rows * hd * dd;
  if (total == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 65535));
  unpad_rows_kernel<T><<<blocks, 256, 0, st>>>(src, dst, rows, hs, ds, hd, dd);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------- indexer launch
dsa_status run_indexer(const dsa_dims& d, const uint8_t* q_idx, const __nv_bfloat16* w, const uint8_t* k_idx,
                       const float* scales, const int32_t* lengths, int32_t topk, int32_t* out_idx,
                       float* out_scores, uint8_t* ws, const Layout& L, cudaStream_t st) {
  NvtxRange range("indexer_topk");
  const DeviceInfo dev = device_info();
  IndexerParams p{};
  p.q_idx = q_idx;
  p.w = w;
  p.q_scale = scales;
  p.k_scale = scales + static_cast<size_t>(d.batch) * d.n_q;
  p.lengths = lengths;
  p.out_idx = out_idx;
  p.out_scores = out_scores;
  p.status = reinterpret_cast<uint32_t*>(ws + L.status);
  p.batch = d.batch;
  p.n_q = d.n_q;
  p.max_len = d.max_len;
  p.topk = topk;
  p.wait_budget_ns = g_indexer_wait_ns.load(std::memory_order_relaxed);
  CUtensorMap map_q, map_k;
  if (!encode_rows_u8(&map_k, k_idx, static_cast<uint64_t>(d.max_len), static_cast<uint64_t>(d.batch), kKeyTile))
    return DSA_ERR_CUDA;
  if (d.n_q == 1) {
    // decode: the chunk items score every key of the row; rows up to kSelMaxLen keys are then
    // selected whole by one cluster per sequence, longer ones keep a partial top-k per chunk
    // that a merge reduces
    const bool rows = L.key_rows != 0;
    p.n_chunks = L.n_chunks;
    if (rows) {
      p.key_rows = reinterpret_cast<uint32_t*>(ws + L.key_rows);
    } else {
      p.part_keys = reinterpret_cast<uint32_t*>(ws + L.part_keys);
      p.part_pos = reinterpret_cast<int32_t*>(ws + L.part_pos);
      p.part_count = reinterpret_cast<int32_t*>(ws + L.part_count);
    }
    p.n_items = d.batch * L.n_chunks;
    if (!encode_rows_u8(&map_q, q_idx, static_cast<uint64_t>(kIdxHeads), static_cast<uint64_t>(d.batch),
                        kIdxHeads))
      return DSA_ERR_CUDA;
    const int grid = std::min(p.n_items, IdxCfg<1>::CTAS_PER_SM * dev.sms);
    indexer_topk_kernel<1><<<grid, IdxCfg<1>::THREADS, IdxCfg<1>::SMEM_BYTES, st>>>(map_q, map_k, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    if (rows) {
      DecodeSelectParams sp{p.key_rows, lengths, out_idx, out_scores, d.max_len, topk};
      decode_select_kernel<<<d.batch * kSelCluster, kSelThreads, 0, st>>>(sp);
    } else {
      MergeParams mp{p.part_keys, p.part_pos, p.part_count, out_idx, L.n_chunks, topk, out_scores};
      merge_partials_kernel<kMergeThreads><<<d.batch, kMergeThreads, 0, st>>>(mp);
    }
    return from_cuda(cudaGetLastError());
  }
  p.n_chunks = 0;
  p.n_items = d.batch * ((d.n_q + kPrefillNQ - 1) / kPrefillNQ);
  if (!dev.indexer_regs_ok) return DSA_ERR_UNSUPPORTED;   // a build whose register count breaks the split
  if (!encode_rows_u8(&map_q, q_idx, static_cast<uint64_t>(d.n_q) * kIdxHeads, static_cast<uint64_t>(d.batch),
                      kPrefillNQ * kIdxHeads))
    return DSA_ERR_CUDA;
  const bool spec = sampled_threshold(d, topk);
  if (spec) {
    // items whose sampled threshold fails are queued during the first launch and rerun exactly
    // by the second; the queue's length starts at zero
    p.spec = 1;
    p.redo_flag = reinterpret_cast<uint32_t*>(ws + L.redo_flag);
    p.redo_list = reinterpret_cast<int32_t*>(ws + L.redo_list);
    p.redo_count = reinterpret_cast<uint32_t*>(ws + L.redo_count);
    if (cudaMemsetAsync(p.redo_count, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  }
  const int grid = std::min(p.n_items, dev.sms);
  indexer_topk_kernel<kPrefillNQ><<<grid, IdxCfg<kPrefillNQ>::THREADS, IdxCfg<kPrefillNQ>::SMEM_BYTES, st>>>(map_q,
                                                                                                        map_k, p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  if (spec) {
    IndexerParams px = p;
    px.spec = 0;
    px.item_list = p.redo_list;
    px.item_count = p.redo_count;
    indexer_topk_kernel<kPrefillNQ><<<grid, IdxCfg<kPrefillNQ>::THREADS, IdxCfg<kPrefillNQ>::SMEM_BYTES, st>>>(
        map_q, map_k, px);
  }
  return from_cuda(cudaGetLastError());
}

dsa_status run_attention(const dsa_dims& d, const __nv_bfloat16* q, const __nv_bfloat16* kv, const int32_t* idx,
                         int32_t topk, __nv_bfloat16* out, float* lse, uint8_t* ws, const Layout& L,
                         cudaStream_t st, bool masked) {
  NvtxRange range(masked ? "masked_mqa_attn" : "sparse_mla_attn");
  const DeviceInfo dev = device_info();
  AttnParams p{};
  p.q = q;
  p.kv = kv;
  p.idx = idx;
  p.out = out;
  p.lse = lse;
  p.status = reinterpret_cast<uint32_t*>(ws + L.status);
  p.n_q = d.n_q;
  p.max_len = d.max_len;
  p.topk = topk;
  p.n_queries = d.batch * d.n_q;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.wait_budget_ns = kWaitBudgetNs;
  CUtensorMap map_q, map_a, map_b;
  if (!encode_q_bf16(&map_q, q, static_cast<uint64_t>(p.n_queries) * kHeads)) return DSA_ERR_CUDA;
  const int clusters = std::max(1, std::min(p.n_queries, dev.sms / 2));
  if (!masked) {
    sparse_mla_attn_kernel<false><<<2 * clusters, AttnCfg::THREADS, AttnCfg::SMEM_BYTES, st>>>(map_q, map_q, map_q, p);
    return from_cuda(cudaGetLastError());
  }
  // masked dense mode: the bitmap of each query's attended positions, then whole 64-row blocks
  // of its causal prefix by TMA
  p.mask = reinterpret_cast<const uint32_t*>(ws + L.mask);
  p.extent = reinterpret_cast<const int32_t*>(ws + L.extent);
  p.mask_words = L.mask_words;
  const uint64_t rows = static_cast<uint64_t>(d.batch) * d.max_len;
  if (!encode_kv_bf16(&map_a, kv, rows, 32) || !encode_kv_bf16(&map_b, kv, rows, kBlk)) return DSA_ERR_CUDA;
  mask_rows_kernel<<<p.n_queries, 256, 0, st>>>(idx, topk, d.max_len, L.mask_words,
                                                reinterpret_cast<uint32_t*>(ws + L.mask),
                                                reinterpret_cast<int32_t*>(ws + L.extent), p.status);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  sparse_mla_attn_kernel<true><<<2 * clusters, AttnCfg::THREADS, AttnCfg::SMEM_BYTES, st>>>(map_q, map_a, map_b, p);
  return from_cuda(cudaGetLastError());
}

struct Prepared {
  const uint8_t* q_idx;
  const __nv_bfloat16* w;
  const uint8_t* k_idx;
  const __nv_bfloat16* q;
  const __nv_bfloat16* kv;
};

dsa_status pad_indexer_inputs(const dsa_dims& d, const void* q_idx, const void* w, const void* k_idx, uint8_t* ws,
                              const Layout& L, cudaStream_t st, Prepared* out) {
  const int64_t T = static_cast<int64_t>(d.batch) * d.n_q, K = static_cast<int64_t>(d.batch) * d.max_len;
  if (!L.padded) {
    out->q_idx = static_cast<const uint8_t*>(q_idx);
    out->w = static_cast<const __nv_bfloat16*>(w);
    out->k_idx = static_cast<const uint8_t*>(k_idx);
    return DSA_OK;
  }
  uint8_t* pq = ws + L.q_idx;
  __nv_bfloat16* pw = reinterpret_cast<__nv_bfloat16*>(ws + L.w);
  uint8_t* pk = ws + L.k_idx;
  if (launch_pad<uint8_t>(static_cast<const uint8_t*>(q_idx), pq, T, d.n_idx_heads, d.idx_dim, kIdxHeads, kIdxDim,
                          d.idx_dim, kIdxDim, st) != cudaSuccess ||
      launch_pad<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(w), pw, T, 1, d.n_idx_heads, 1, kIdxHeads,
                                d.n_idx_heads, kIdxHeads, st) != cudaSuccess ||
      launch_pad<uint8_t>(static_cast<const uint8_t*>(k_idx), pk, K, 1, d.idx_dim, 1, kIdxDim, d.idx_dim, kIdxDim,
                          st) != cudaSuccess)
    return DSA_ERR_CUDA;
  out->q_idx = pq;
  out->w = pw;
  out->k_idx = pk;
  return DSA_OK;
}

dsa_status pad_attention_inputs(const dsa_dims& d, const void* q, const void* kv, uint8_t* ws, const Layout& L,
                                cudaStream_t st, Prepared* out) {
  const int64_t T = static_cast<int64_t>(d.batch) * d.n_q, K = static_cast<int64_t>(d.batch) * d.max_len;
  if (!L.padded) {
    out->q = static_cast<const __nv_bfloat16*>(q);
    out->kv = static_cast<const __nv_bfloat16*>(kv);
    return DSA_OK;
  }
  __nv_bfloat16* pq = reinterpret_cast<__nv_bfloat16*>(ws + L.q);
  __nv_bfloat16* pkv = reinterpret_cast<__nv_bfloat16*>(ws + L.kv);
  const int dqk = d.d_latent + d.d_rope;
  if (launch_pad<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(q), pq, T, d.n_heads, dqk, kHeads, kDqk,
                                d.d_latent, kDv, st) != cudaSuccess ||
      launch_pad<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(kv), pkv, K, 1, dqk, 1, kDqk, d.d_latent, kDv,
                                st) != cudaSuccess)
    return DSA_ERR_CUDA;
  out->q = pq;
  out->kv = pkv;
  return DSA_OK;
}

dsa_status check_ws(void* ws, size_t ws_bytes, const Layout& L) {
  if (ws == nullptr || !aligned(ws, kAlign) || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

dsa_status device_ok() {
  const DeviceInfo dev = device_info();
  if (dev.sms == 0) return DSA_ERR_CUDA;
  if (!dev.sm100) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

}  // namespace

extern "C" {

size_t dsa_workspace_bytes(const dsa_dims* dims, int32_t topk) {
  if (check_dims(dims, topk) != DSA_OK) return 0;
  return make_layout(*dims, topk).total;
}

dsa_status dsa_workspace_init(void* ws, size_t ws_bytes, dsa_stream_t stream) {
  if (ws == nullptr || !aligned(ws, kAlign) || ws_bytes < kAlign) return DSA_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(ws, 0, kAlign, reinterpret_cast<cudaStream_t>(stream)));
}

dsa_status dsa_indexer_topk_scores(const dsa_dims* dims, const void* q_idx, const void* w, const void* k_idx,
                                   const float* scales, const int32_t* lengths, int32_t topk, int32_t* out_idx,
                                   float* out_scores, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status s = check_dims(dims, topk);
  if (s != DSA_OK) return s;
  const dsa_dims& d = *dims;
  const Layout L = make_layout(d, topk);
  if ((s = check_ws(ws, ws_bytes, L)) != DSA_OK) return s;
  if (static_cast<int64_t>(d.batch) * d.n_q == 0) return DSA_OK;
  if (!q_idx || !w || !k_idx || !scales || !lengths || !out_idx) return DSA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(k_idx, 16) || !aligned(w, 2) || !aligned(scales, 4) ||
      !aligned(lengths, 4) || !aligned(out_idx, 4) || !aligned(out_scores, 4))
    return DSA_ERR_INVALID_ARG;
  if ((s = device_ok()) != DSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  Prepared pr{};
  if ((s = pad_indexer_inputs(d, q_idx, w, k_idx, wsb, L, st, &pr)) != DSA_OK) return s;
  return run_indexer(d, pr.q_idx, pr.w, pr.k_idx, scales, lengths, topk, out_idx, out_scores, wsb, L, st);
}

dsa_status dsa_indexer_topk(const dsa_dims* dims, const void* q_idx, const void* w, const void* k_idx,
                            const float* scales, const int32_t* lengths, int32_t topk, int32_t* out_idx, void* ws,
                            size_t ws_bytes, dsa_stream_t stream) {
  return dsa_indexer_topk_scores(dims, q_idx, w, k_idx, scales, lengths, topk, out_idx, nullptr, ws, ws_bytes,
                                 stream);
}

static dsa_status attention_call(const dsa_dims* dims, const void* q, const void* latent_kv, const int32_t* idx,
                                 int32_t topk, void* out, float* lse, void* ws, size_t ws_bytes, dsa_stream_t stream,
                                 bool masked) {
  dsa_status s = check_dims(dims, topk);
  if (s != DSA_OK) return s;
  const dsa_dims& d = *dims;
  const Layout L = make_layout(d, topk);
  if ((s = check_ws(ws, ws_bytes, L)) != DSA_OK) return s;
  if (static_cast<int64_t>(d.batch) * d.n_q == 0) return DSA_OK;
  if (!q || !latent_kv || !idx || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(latent_kv, 16) || !aligned(idx, 4) || !aligned(out, 16) || !aligned(lse, 4))
    return DSA_ERR_INVALID_ARG;
  if (masked && d.max_len > kMaskMaxLen) return DSA_ERR_UNSUPPORTED;
  if ((s = device_ok()) != DSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  Prepared pr{};
  if ((s = pad_attention_inputs(d, q, latent_kv, wsb, L, st, &pr)) != DSA_OK) return s;
  const int64_t T = static_cast<int64_t>(d.batch) * d.n_q;
  __nv_bfloat16* o = L.padded ? reinterpret_cast<__nv_bfloat16*>(wsb + L.out) : static_cast<__nv_bfloat16*>(out);
  float* ls = L.padded ? reinterpret_cast<float*>(wsb + L.lse) : lse;
  if ((s = run_attention(d, pr.q, pr.kv, idx, topk, o, ls, wsb, L, st, masked)) != DSA_OK) return s;
  if (L.padded) {
    if (launch_unpad<__nv_bfloat16>(o, static_cast<__nv_bfloat16*>(out), T, kHeads, kDv, d.n_heads, d.d_latent,
                                    st) != cudaSuccess ||
        launch_unpad<float>(ls, lse, T, 1, kHeads, 1, d.n_heads, st) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status dsa_sparse_mla_attn(const dsa_dims* dims, const void* q, const void* latent_kv, const int32_t* idx,
                               int32_t topk, void* out, float* lse, void* ws, size_t ws_bytes,
                               dsa_stream_t stream) {
  return attention_call(dims, q, latent_kv, idx, topk, out, lse, ws, ws_bytes, stream, false);
}

dsa_status dsa_masked_mqa_attn(const dsa_dims* dims, const void* q, const void* latent_kv, const int32_t* idx,
                               int32_t topk, void* out, float* lse, void* ws, size_t ws_bytes,
                               dsa_stream_t stream) {
  return attention_call(dims, q, latent_kv, idx, topk, out, lse, ws, ws_bytes, stream, true);
}

dsa_status dsa_indexer_kl_loss(const dsa_dims* dims, const void* q, const void* latent_kv, const int32_t* idx,
                               const float* idx_scores, const float* lse, int32_t topk, float* loss, void* ws,
                               size_t ws_bytes, dsa_stream_t stream) {
  NvtxRange range("indexer_kl_loss");
  dsa_status s = check_dims(dims, topk);
  if (s != DSA_OK) return s;
  const dsa_dims& d = *dims;
  const Layout L = make_layout(d, topk);
  if ((s = check_ws(ws, ws_bytes, L)) != DSA_OK) return s;
  if (static_cast<int64_t>(d.batch) * d.n_q == 0) return DSA_OK;
  if (!q || !latent_kv || !idx || !idx_scores || !lse || !loss) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(latent_kv, 16) || !aligned(idx, 4) || !aligned(idx_scores, 4) || !aligned(lse, 4) ||
      !aligned(loss, 4))
    return DSA_ERR_INVALID_ARG;
  if ((s = device_ok()) != DSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  Prepared pr{};
  if ((s = pad_attention_inputs(d, q, latent_kv, wsb, L, st, &pr)) != DSA_OK) return s;
  const int64_t T = static_cast<int64_t>(d.batch) * d.n_q;
  const float* lse_in = lse;
  if (L.padded) {   // the lse of the padded heads is +inf: their weights exp(z - lse) are 0
    float* pl = reinterpret_cast<float*>(wsb + L.lse);
    if (launch_pad<float>(lse, pl, T, 1, d.n_heads, 1, kHeads, d.n_heads, kHeads, st) != cudaSuccess ||
        launch_fill<float>(pl, T, d.n_heads, kHeads, INFINITY, st) != cudaSuccess)
      return DSA_ERR_CUDA;
    lse_in = pl;
  }
  const DeviceInfo dev = device_info();
  KlParams p{};
  p.q = pr.q;
  p.kv = pr.kv;
  p.idx = idx;
  p.scores = idx_scores;
  p.lse = lse_in;
  p.loss = loss;
  p.status = reinterpret_cast<uint32_t*>(wsb + L.status);
  p.n_q = d.n_q;
  p.max_len = d.max_len;
  p.topk = topk;
  p.n_queries = static_cast<int32_t>(T);
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.wait_budget_ns = kWaitBudgetNs;
  const int grid = static_cast<int>(std::min<int64_t>(T, dev.sms));
  indexer_kl_kernel<<<grid, KlCfg::THREADS, KlCfg::SMEM_BYTES, st>>>(p);
  return from_cuda(cudaGetLastError());
}

dsa_status dsa_forward(const dsa_dims* dims, const void* q_idx, const void* w, const void* k_idx,
                       const float* scales, const int32_t* lengths, int32_t topk, const void* q,
                       const void* latent_kv, int32_t* out_idx, void* out, float* lse, void* ws, size_t ws_bytes,
                       dsa_stream_t stream) {
  NvtxRange range("dsa_forward");
  dsa_status s = check_dims(dims, topk);
  if (s != DSA_OK) return s;
  const Layout L = make_layout(*dims, topk);
  if ((s = check_ws(ws, ws_bytes, L)) != DSA_OK) return s;
  int32_t* sel = out_idx != nullptr ? out_idx : reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + L.idx);
  s = dsa_indexer_topk(dims, q_idx, w, k_idx, scales, lengths, topk, sel, ws, ws_bytes, stream);
  if (s != DSA_OK) return s;
  return dsa_sparse_mla_attn(dims, q, latent_kv, sel, topk, out, lse, ws, ws_bytes, stream);
}

dsa_status dsa_get_device_status(void* ws, dsa_stream_t stream, uint32_t* detail) {
  if (ws == nullptr || !aligned(ws, kAlign)) return DSA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  if (cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  if (h[0] != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(h), st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  }
  if (detail) *detail = h[1];
  return static_cast<dsa_status>(h[0]);
}

const char* dsa_status_string(dsa_status status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported dims or device";
    case DSA_ERR_CUDA: return "CUDA call failed";
    case DSA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case DSA_ERR_INDEX_RANGE: return "an index outside [0, max_len) reached the attention";
    case DSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

int32_t dsa_version(void) { return 200; }

dsa_status dsa_set_wait_budget_ns(uint64_t ns) {
  g_indexer_wait_ns.store(ns == 0 ? kWaitBudgetNs : ns, std::memory_order_relaxed);
  return DSA_OK;
}

}  // extern "C"

// ----------------------------------------------------------------------------- decode without a workspace
// Some callers cannot allocate device memory for a call: serving runtimes that plan every
// buffer ahead and forbid allocation on the request path, plugin interfaces that hand a kernel
// only its inputs and outputs, and latency-critical loops where cudaMalloc's implicit device
// synchronisation is unacceptable. For them, the decode selection (one query per sequence)
// has a variant whose scratch -- the exact per-chunk top-k lists merged into the final
// selection -- lives in this file-scope device array instead of a caller workspace. The array
// is sized for kStaticSlots (sequence, 8192-key chunk) pairs at top-k <= 2048 (16 MiB plus the
// counts); every GPU that loads the library keeps it until the process exits.
namespace {

constexpr size_t kStaticSlots = 1024;
constexpr size_t kStaticTopk = 2048;
constexpr size_t kStaticKeysBytes = kStaticSlots * kStaticTopk * 4;
constexpr size_t kStaticBytes = 2 * kStaticKeysBytes + kStaticSlots * 4;

static __device__ __align__(256) uint8_t g_decode_scratch[kStaticBytes];

// Device address of g_decode_scratch on the current device, looked up once per device.
dsa_status static_scratch(uint8_t** out) {
  static std::mutex mu;
  static uint8_t* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return DSA_ERR_CUDA;
    addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = addr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status dsa_indexer_topk_decode_noalloc(const dsa_dims* dims, const void* q_idx, const void* w,
                                                      const void* k_idx, const float* scales, const int32_t* lengths,
                                                      int32_t topk, int32_t* out_idx, uint32_t* status,
                                                      dsa_stream_t stream) {
  dsa_status s = check_dims(dims, topk);
  if (s != DSA_OK) return s;
  const dsa_dims& d = *dims;
  if (d.n_q != 1 || !is_production(d)) return DSA_ERR_UNSUPPORTED;
  const int32_t n_chunks = (d.max_len + kDecodeChunk - 1) / kDecodeChunk;
  if (static_cast<size_t>(d.batch) * n_chunks > kStaticSlots || static_cast<size_t>(topk) > kStaticTopk)
    return DSA_ERR_UNSUPPORTED;
  if (d.batch == 0) return DSA_OK;
  if (!q_idx || !w || !k_idx || !scales || !lengths || !out_idx) return DSA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(k_idx, 16) || !aligned(w, 2) || !aligned(scales, 4) ||
      !aligned(lengths, 4) || !aligned(out_idx, 4) || (status != nullptr && !aligned(status, 4)))
    return DSA_ERR_INVALID_ARG;
  if ((s = device_ok()) != DSA_OK) return s;
  uint8_t* scratch = nullptr;
  if ((s = static_scratch(&scratch)) != DSA_OK) return s;
  const DeviceInfo dev = device_info();
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  IndexerParams p{};
  p.q_idx = static_cast<const uint8_t*>(q_idx);
  p.w = static_cast<const __nv_bfloat16*>(w);
  p.q_scale = scales;
  p.k_scale = scales + d.batch;
  p.lengths = lengths;
  p.out_idx = out_idx;
  p.status = status;
  p.batch = d.batch;
  p.n_q = 1;
  p.max_len = d.max_len;
  p.topk = topk;
  p.wait_budget_ns = kWaitBudgetNs;
  p.n_chunks = n_chunks;
  // the slots are laid out with the call's top-k as row width. The chunk kernel zeroes the
  // count of every slot of this call before it starts, and the merge reads only a slot's first
  // count entries, so an earlier call's contents are never used: a slot an aborted CTA never
  // reached counts as empty (the abort itself is reported through `status`)
  p.part_keys = reinterpret_cast<uint32_t*>(scratch);
  p.part_pos = reinterpret_cast<int32_t*>(scratch + kStaticKeysBytes);
  p.part_count = reinterpret_cast<int32_t*>(scratch + 2 * kStaticKeysBytes);
  p.n_items = d.batch * n_chunks;
  CUtensorMap map_q, map_k;
  if (!encode_rows_u8(&map_k, k_idx, static_cast<uint64_t>(d.max_len), static_cast<uint64_t>(d.batch), kKeyTile) ||
      !encode_rows_u8(&map_q, q_idx, static_cast<uint64_t>(kIdxHeads), static_cast<uint64_t>(d.batch), kIdxHeads))
    return DSA_ERR_CUDA;
  const int grid = std::min(p.n_items, IdxCfg<1>::CTAS_PER_SM * dev.sms);
  indexer_topk_kernel<1><<<grid, IdxCfg<1>::THREADS, IdxCfg<1>::SMEM_BYTES, st>>>(map_q, map_k, p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  MergeParams mp{p.part_keys, p.part_pos, p.part_count, out_idx, n_chunks, topk, nullptr};
  merge_partials_kernel<kMergeThreads><<<d.batch, kMergeThreads, 0, st>>>(mp);
  return from_cuda(cudaGetLastError());
}
