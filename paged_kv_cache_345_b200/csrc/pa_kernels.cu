// Kernels and launchers: cache append, block copy, paged decode + split-K merge.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>

#include "pa_decode.cuh"
#include "pa_decode_mma.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// Device error word: kernels OR PA_DEVERR_* bits into it; pa_device_errors
// reads and clears it.
__device__ unsigned int g_error_word = 0;

namespace {

// Unique id of the current context (0 when no context is current yet).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(ptr);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

std::mutex g_symbol_mutex;

}  // namespace

cudaError_t SymbolAddressCache::get(const void* symbol, void** out) {
  unsigned long long id = current_context_id();
  if (id != 0) {
    std::lock_guard<std::mutex> lock(g_symbol_mutex);
    for (const Entry& e : entries_)
      if (e.ctx_id == id && e.ptr) {
        *out = e.ptr;
        return cudaSuccess;
      }
  }
  void* ptr = nullptr;
  // (makes the device's primary context current if none was)
  cudaError_t e = cudaGetSymbolAddress(&ptr, symbol);
  if (e != cudaSuccess) return e;
  if (!ptr) return cudaErrorInvalidSymbol;
  id = current_context_id();
  if (id != 0) {
    std::lock_guard<std::mutex> lock(g_symbol_mutex);
    entries_[next_] = Entry{id, ptr};
    next_ = (next_ + 1) % kEntries;
  }
  *out = ptr;
  return cudaSuccess;
}

cudaError_t device_error_word(unsigned int** ptr) {
  static SymbolAddressCache cache;
  void* addr = nullptr;
  cudaError_t e = cache.get(&g_error_word, &addr);
  if (e == cudaSuccess) *ptr = static_cast<unsigned int*>(addr);
  return e;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream drains; it calls pdl_wait() before reading
// anything that kernel could have written.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ append

// One warp per token row (K and V rows of all KV heads of a token are
// contiguous both in k_new and in the cache slot): 16-byte vector copies.
__global__ void __launch_bounds__(256)
    kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                     const int64_t* __restrict__ slot_mapping, int num_tokens,
                     uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, int64_t num_slots,
                     int vec_per_row, unsigned* err) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t tok = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       tok < num_tokens; tok += warps) {
    const int64_t slot = __ldg(slot_mapping + tok);
    if (slot < 0) continue;  // padding row
    if (slot >= num_slots) {
      if (lane == 0) atomicOr(err, PA_DEVERR_SLOT);
      continue;
    }
    const uint4* ks = k_new + tok * vec_per_row;
    const uint4* vs = v_new + tok * vec_per_row;
    uint4* kd = k_cache + slot * vec_per_row;
    uint4* vd = v_cache + slot * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) {
      const uint4 a = ldg_stream(ks + v);
      const uint4 b = ldg_stream(vs + v);
      kd[v] = a;
      vd[v] = b;
    }
  }
}

cudaError_t launch_kv_append(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                             int num_tokens, void* k_cache, void* v_cache, int64_t num_slots,
                             int row_bytes, cudaStream_t stream) {
  unsigned* err = nullptr;
  cudaError_t e = device_error_word(&err);
  if (e != cudaSuccess) return e;
  const int threads = 256, warps_per_cta = threads / 32;
  int64_t ctas = (static_cast<int64_t>(num_tokens) + warps_per_cta - 1) / warps_per_cta;
  if (ctas > 148 * 16) ctas = 148 * 16;
  return launch_pdl(kv_append_kernel, dim3(static_cast<unsigned>(ctas)), dim3(threads), 0, stream,
                    static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                    slot_mapping, num_tokens, static_cast<uint4*>(k_cache),
                    static_cast<uint4*>(v_cache), num_slots, row_bytes / 16, err);
}

// One warp per token row, E4M3 caches: 16 values per lane step (32 bytes of
// bfloat16 in, 16 codes out), each divided by its KV head's scale.
__global__ void __launch_bounds__(256)
    kv_append_fp8_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                         const int64_t* __restrict__ slot_mapping, int num_tokens,
                         uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                         const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                         int64_t num_slots, int head_dim, int units_per_row, unsigned* err) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t tok = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       tok < num_tokens; tok += warps) {
    const int64_t slot = __ldg(slot_mapping + tok);
    if (slot < 0) continue;  // padding row
    if (slot >= num_slots) {
      if (lane == 0) atomicOr(err, PA_DEVERR_SLOT);
      continue;
    }
    const uint4* ks = k_new + tok * units_per_row * 2;
    const uint4* vs = v_new + tok * units_per_row * 2;
    uint4* kd = k_cache + slot * units_per_row;
    uint4* vd = v_cache + slot * units_per_row;
    for (int u = lane; u < units_per_row; u += 32) {
      const int h = u * 16 / head_dim;
      kd[u] = bf16x16_to_e4m3(ldg_stream(ks + 2 * u), ldg_stream(ks + 2 * u + 1),
                              __ldg(k_scale + h));
      vd[u] = bf16x16_to_e4m3(ldg_stream(vs + 2 * u), ldg_stream(vs + 2 * u + 1),
                              __ldg(v_scale + h));
    }
  }
}

cudaError_t launch_kv_append_fp8(const void* k_new, const void* v_new,
                                 const int64_t* slot_mapping, int num_tokens, void* k_cache,
                                 void* v_cache, const float* k_scale, const float* v_scale,
                                 int64_t num_slots, int num_kv_heads, int head_dim,
                                 cudaStream_t stream) {
  unsigned* err = nullptr;
  cudaError_t e = device_error_word(&err);
  if (e != cudaSuccess) return e;
  const int threads = 256, warps_per_cta = threads / 32;
  int64_t ctas = (static_cast<int64_t>(num_tokens) + warps_per_cta - 1) / warps_per_cta;
  if (ctas > 148 * 16) ctas = 148 * 16;
  return launch_pdl(kv_append_fp8_kernel, dim3(static_cast<unsigned>(ctas)), dim3(threads), 0,
                    stream, static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                    slot_mapping, num_tokens, static_cast<uint4*>(k_cache),
                    static_cast<uint4*>(v_cache), k_scale, v_scale, num_slots, head_dim,
                    num_kv_heads * head_dim / 16, err);
}

// -------------------------------------------------------------- copy blocks

// blockIdx.x = pair, blockIdx.y = slice of the block; 16-byte vector copies.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                       const int64_t* __restrict__ block_mapping, int num_blocks,
                       int64_t vec_per_block, unsigned* err) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t src = __ldg(block_mapping + 2 * blockIdx.x);
  const int64_t dst = __ldg(block_mapping + 2 * blockIdx.x + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, PA_DEVERR_COPY_PAIR);
    return;
  }
  const int64_t stride = static_cast<int64_t>(gridDim.y) * blockDim.x;
  for (int64_t v = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x; v < vec_per_block;
       v += stride) {
    const uint4 a = ldg_stream(k_cache + src * vec_per_block + v);
    const uint4 b = ldg_stream(v_cache + src * vec_per_block + v);
    k_cache[dst * vec_per_block + v] = a;
    v_cache[dst * vec_per_block + v] = b;
  }
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                               int num_pairs, int num_blocks, int64_t block_bytes,
                               cudaStream_t stream) {
  unsigned* err = nullptr;
  cudaError_t e = device_error_word(&err);
  if (e != cudaSuccess) return e;
  const int64_t vec = block_bytes / 16;
  const int threads = 256;
  int64_t slices = (vec + threads * 4 - 1) / (threads * 4);  // ~4 vectors per thread
  if (slices < 1) slices = 1;
  if (slices > 65535) slices = 65535;
  dim3 grid(num_pairs, static_cast<unsigned>(slices));
  return launch_pdl(copy_blocks_kernel, grid, dim3(threads), 0, stream,
                    static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), block_mapping,
                    num_blocks, vec, err);
}

// -------------------------------------------------------------- swap blocks

// Copies whole blocks between two pools (device memory or page-locked host
// memory mapped into the device's address space): blockIdx.x = pair,
// blockIdx.y = slice of the block. Plain (coherent) loads, since one side may
// be host memory reached over the bus.
__global__ void __launch_bounds__(256)
    swap_blocks_kernel(uint4* dst_k, uint4* dst_v, const uint4* src_k, const uint4* src_v,
                       const int64_t* block_mapping, int src_num_blocks, int dst_num_blocks,
                       int64_t vec_per_block, unsigned* err) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t src = block_mapping[2 * blockIdx.x];
  const int64_t dst = block_mapping[2 * blockIdx.x + 1];
  if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, PA_DEVERR_COPY_PAIR);
    return;
  }
  const int64_t stride = static_cast<int64_t>(gridDim.y) * blockDim.x;
  for (int64_t v = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x; v < vec_per_block;
       v += stride) {
    const uint4 a = src_k[src * vec_per_block + v];
    const uint4 b = src_v[src * vec_per_block + v];
    dst_k[dst * vec_per_block + v] = a;
    dst_v[dst * vec_per_block + v] = b;
  }
}

cudaError_t launch_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int64_t* block_mapping, int num_pairs, int src_num_blocks,
                               int dst_num_blocks, int64_t block_bytes, cudaStream_t stream) {
  unsigned* err = nullptr;
  cudaError_t e = device_error_word(&err);
  if (e != cudaSuccess) return e;
  const int64_t vec = block_bytes / 16;
  const int threads = 256;
  int64_t slices = (vec + threads * 4 - 1) / (threads * 4);
  if (slices < 1) slices = 1;
  if (slices > 65535) slices = 65535;
  dim3 grid(num_pairs, static_cast<unsigned>(slices));
  return launch_pdl(swap_blocks_kernel, grid, dim3(threads), 0, stream,
                    static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v),
                    static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v),
                    block_mapping, src_num_blocks, dst_num_blocks, vec, err);
}

// ------------------------------------------------------------------ decode

// cuTensorMapEncodeTiled from the driver, looked up once (also used by pa_prefill.cu).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

namespace {

// 4-D view of a cache [num_blocks][block_size][num_kv_heads][head_dim]; a box is
// `box_rows` consecutive tokens of one block for one KV head and `box_cols`
// columns (all of head_dim when 0): box_cols x 1 x box_rows x 1.
cudaError_t encode_cache_map(CUtensorMap* map, const void* base, const DecodeShape& sh,
                             int box_rows, int box_cols = 0, bool swizzle128 = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const int eb = sh.dtype == PA_BF16 ? 2 : 4;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(sh.head_dim),
                              static_cast<cuuint64_t>(sh.num_kv_heads),
                              static_cast<cuuint64_t>(sh.block_size),
                              static_cast<cuuint64_t>(sh.num_blocks)};
  const cuuint64_t row = static_cast<cuuint64_t>(sh.head_dim) * eb;
  const cuuint64_t strides[3] = {row, row * sh.num_kv_heads,
                                 row * sh.num_kv_heads * static_cast<cuuint64_t>(sh.block_size)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_cols ? box_cols : sh.head_dim), 1u,
                             static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, sh.dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   4, const_cast<void*>(base), dims, strides, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Sets a kernel's dynamic shared-memory limit once per device.
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, std::atomic<unsigned long long>& configured) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev % 64);
  if (configured.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) configured.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <typename T, int D>
cudaError_t launch_merge(const DecodeShape& sh, const DecodeParams& p, cudaStream_t stream) {
  if (sh.num_partitions <= 1 && sh.prefix_slots == 0) return cudaSuccess;
  // warps per row: enough to load every partial of a row in one batch of 8
  // per warp, at most 4
  const unsigned rows = static_cast<unsigned>(sh.num_seqs) * sh.num_heads;
  if (sh.num_partitions <= 8)
    return launch_pdl(pa_merge_kernel<T, D, 1>, dim3((rows + 3) / 4), dim3(128), 0, stream, p);
  if (sh.num_partitions <= 16)
    return launch_pdl(pa_merge_kernel<T, D, 2>, dim3((rows + 1) / 2), dim3(128), 0, stream, p);
  return launch_pdl(pa_merge_kernel<T, D, 4>, dim3(rows), dim3(128), 0, stream, p);
}

// float32 caches: CUDA-core kernel (tensor maps, exact fp32 products).
template <int D, int G>
cudaError_t launch_decode_f32(const DecodeShape& sh, const DecodeParams& p, const void* k_cache,
                              const void* v_cache, cudaStream_t stream) {
  using Cfg = DecodeConfig<float, D, G>;
  static std::atomic<unsigned long long> configured{0};
  cudaError_t e = ensure_smem(pa_decode_kernel<float, D, G>, Cfg::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  CUtensorMap kmap, vmap;
  const int box_rows = sh.block_size < Cfg::kC ? sh.block_size : Cfg::kC;
  if ((e = encode_cache_map(&kmap, k_cache, sh, box_rows)) != cudaSuccess) return e;
  if ((e = encode_cache_map(&vmap, v_cache, sh, box_rows)) != cudaSuccess) return e;
  dim3 grid(sh.num_kv_heads, sh.num_partitions, sh.num_seqs);
  pa_decode_kernel<float, D, G><<<grid, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(kmap, vmap, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_merge<float, D>(sh, p, stream);
}

// 4-D view of a cache with the dimensions ordered (column, token, head, block)
// so that a box {head_dim + 16 bytes, rows, heads, 1} lands in shared memory
// as [head][token][row + 16 bytes]; the columns past head_dim are outside the
// tensor and arrive as zeros (row padding against bank conflicts). bfloat16
// or, for E4M3 caches, bytes.
cudaError_t encode_group_map(CUtensorMap* map, const void* base, const DecodeShape& sh,
                             int box_rows, int box_heads) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const bool fp8 = sh.dtype == PA_FP8_E4M3;
  const cuuint64_t row = static_cast<cuuint64_t>(sh.head_dim) * (fp8 ? 1 : 2);
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(sh.head_dim),
                              static_cast<cuuint64_t>(sh.block_size),
                              static_cast<cuuint64_t>(sh.num_kv_heads),
                              static_cast<cuuint64_t>(sh.num_blocks)};
  const cuuint64_t strides[3] = {row * sh.num_kv_heads, row,
                                 row * sh.num_kv_heads * static_cast<cuuint64_t>(sh.block_size)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(sh.head_dim + (fp8 ? 16 : 8)),
                             static_cast<cuuint32_t>(box_rows),
                             static_cast<cuuint32_t>(box_heads), 1u};
  const cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
  const CUtensorMapDataType type =
      fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = enc(map, type, 4, const_cast<void*>(base), dims, strides,
                   box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// bfloat16 and E4M3 caches: tensor-core kernel over groups of HB KV heads.
template <int D, int G, int HB, bool FP8>
cudaError_t launch_decode_group_t(const DecodeShape& sh, const DecodeParams& p,
                                  const void* k_cache, const void* v_cache, cudaStream_t stream) {
  // stages: as many as fit ~112 KB of ring (two CTAs per SM), at most 4; E4M3
  // stages are half the size and its consumers hold more registers per byte,
  // so its ring is capped at ~64 KB for three CTAs per SM
  constexpr int kStage = 2 * GroupConfig<D, G, HB, 1, FP8>::kTensorBytes;
  constexpr int kNSfit = (FP8 ? 65536 : 114688) / kStage;
  constexpr int NS = kNSfit < 2 ? 2 : (kNSfit > 4 ? 4 : kNSfit);
  using Cfg = GroupConfig<D, G, HB, NS, FP8>;
  auto kernel = pa_decode_mma_kernel<D, G, HB, NS, FP8, true>;
  if constexpr (!FP8) {
    if (sh.contiguous) kernel = pa_decode_mma_kernel<D, G, HB, NS, false, false>;
  }
  static std::atomic<unsigned long long> configured[2] = {{0}, {0}};
  cudaError_t e = ensure_smem(kernel, Cfg::kSmemBytes, configured[sh.contiguous ? 1 : 0]);
  if (e != cudaSuccess) return e;
  CUtensorMap kmap, vmap;
  const int rows = (sh.contiguous || sh.block_size >= Cfg::kC) ? Cfg::kC : sh.block_size;
  if ((e = encode_group_map(&kmap, k_cache, sh, rows, HB)) != cudaSuccess) return e;
  if ((e = encode_group_map(&vmap, v_cache, sh, rows, HB)) != cudaSuccess) return e;
  // A work list pays where its items take more than one wave of resident
  // CTAs: the longest start first and the short ones fill the tail. When
  // every item fits in one wave the order does not matter, and the plain
  // grid (whose CTAs past a sequence's end exit at once) saves each CTA the
  // read of its item before its table read: same results either way.
  DecodeParams q = p;
  const unsigned groups = static_cast<unsigned>(sh.num_kv_heads / HB);
  if (sh.work != nullptr) {
    static std::atomic<int> per_sm{0};
    int fit = per_sm.load(std::memory_order_relaxed);
    if (fit == 0) {
      if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, kernel, Cfg::kThreads,
                                                             Cfg::kSmemBytes)) != cudaSuccess)
        return e;
      fit = fit < 1 ? 1 : fit;
      per_sm.store(fit, std::memory_order_relaxed);
    }
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    if (static_cast<int64_t>(sh.num_items) * groups <= static_cast<int64_t>(fit) * sms)
      q.work = nullptr;
  }
  // (a shared-prefix call's own partitions follow the prefix's slots; E4M3:
  // partitions slowest, see the kernel)
  const unsigned parts = static_cast<unsigned>(sh.num_partitions - sh.prefix_slots);
  const dim3 grid = q.work != nullptr ? dim3(groups, sh.num_items, 1)
                    : FP8            ? dim3(groups, sh.num_seqs, parts)
                                     : dim3(groups, parts, sh.num_seqs);
  e = launch_pdl(kernel, grid, dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, kmap, vmap, q);
  if (e != cudaSuccess) return e;
  return launch_merge<__nv_bfloat16, D>(sh, q, stream);
}

template <int D, int G, bool FP8>
cudaError_t launch_decode_group(const DecodeShape& sh, const DecodeParams& p, const void* kc,
                                const void* vc, cudaStream_t st) {
  if (sh.num_kv_heads % 4 == 0) return launch_decode_group_t<D, G, 4, FP8>(sh, p, kc, vc, st);
  if (sh.num_kv_heads % 2 == 0) return launch_decode_group_t<D, G, 2, FP8>(sh, p, kc, vc, st);
  return launch_decode_group_t<D, G, 1, FP8>(sh, p, kc, vc, st);
}

template <int D, int G>
cudaError_t launch_decode_bf16(const DecodeShape& sh, const DecodeParams& p, const void* k_cache,
                               const void* v_cache, cudaStream_t stream) {
  return launch_decode_group<D, G, false>(sh, p, k_cache, v_cache, stream);
}

// E4M3 caches: head_dim 128 only.
template <int D>
cudaError_t dispatch_fp8(const DecodeShape& sh, const DecodeParams& p, const void* kc,
                         const void* vc, cudaStream_t st) {
  if constexpr (D != 128) {
    return cudaErrorNotSupported;
  } else {
    switch (sh.num_heads / sh.num_kv_heads) {
      case 1: return launch_decode_group<D, 1, true>(sh, p, kc, vc, st);
      case 2: return launch_decode_group<D, 2, true>(sh, p, kc, vc, st);
      case 4: return launch_decode_group<D, 4, true>(sh, p, kc, vc, st);
      case 8: return launch_decode_group<D, 8, true>(sh, p, kc, vc, st);
      default: return cudaErrorNotSupported;
    }
  }
}

template <int D>
cudaError_t dispatch_group(const DecodeShape& sh, const DecodeParams& p, const void* kc,
                           const void* vc, cudaStream_t st) {
  if (sh.dtype == PA_FP8_E4M3) return dispatch_fp8<D>(sh, p, kc, vc, st);
  const bool bf = sh.dtype == PA_BF16;
  switch (sh.num_heads / sh.num_kv_heads) {
    case 1: return bf ? launch_decode_bf16<D, 1>(sh, p, kc, vc, st) : launch_decode_f32<D, 1>(sh, p, kc, vc, st);
    case 2: return bf ? launch_decode_bf16<D, 2>(sh, p, kc, vc, st) : launch_decode_f32<D, 2>(sh, p, kc, vc, st);
    case 4: return bf ? launch_decode_bf16<D, 4>(sh, p, kc, vc, st) : launch_decode_f32<D, 4>(sh, p, kc, vc, st);
    case 8: return bf ? launch_decode_bf16<D, 8>(sh, p, kc, vc, st) : launch_decode_f32<D, 8>(sh, p, kc, vc, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeShape& sh, void* out, const void* q, const void* k_cache,
                          const void* v_cache, const int32_t* block_tables,
                          const int32_t* context_lens, void* workspace, const void* k_new,
                          const void* v_new, const float* k_scale, const float* v_scale,
                          cudaStream_t stream) {
  DecodeParams p{};
  p.out = out;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.k_new = static_cast<const uint8_t*>(k_new);
  p.v_new = static_cast<const uint8_t*>(v_new);
  p.k_cache_w = static_cast<uint8_t*>(const_cast<void*>(k_cache));
  p.v_cache_w = static_cast<uint8_t*>(const_cast<void*>(v_cache));
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  const WorkspaceLayout wl = workspace_layout(sh.num_seqs, sh.num_heads, sh.num_kv_heads,
                                              sh.head_dim, sh.num_partitions);
  if (sh.num_partitions > 1) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.ws_m = reinterpret_cast<float*>(ws + wl.m_off);
    p.ws_l = reinterpret_cast<float*>(ws + wl.l_off);
    p.ws_acc = reinterpret_cast<float*>(ws + wl.acc_off);
  }
  cudaError_t e = device_error_word(&p.err);
  if (e != cudaSuccess) return e;
  p.num_seqs = sh.num_seqs;
  p.num_heads = sh.num_heads;
  p.num_kv_heads = sh.num_kv_heads;
  p.block_size = sh.block_size;
  int lg = 0;
  while ((1 << lg) < sh.block_size) ++lg;
  p.log2_block_size = lg;
  p.num_blocks = sh.num_blocks;
  p.max_blocks_per_seq = sh.max_blocks_per_seq;
  p.max_context_len = sh.max_context_len;
  p.partition_size = sh.partition_size;
  p.num_partitions = sh.num_partitions;
  p.q_scale = sh.scale * 1.4426950408889634f;  // log2(e)
  p.early_reads = sh.early_reads ? 1 : 0;
  p.first_token = sh.first_token;
  p.prefix_slots = sh.prefix_slots;
  p.work = sh.work;
  p.num_items = sh.num_items;
  switch (sh.head_dim) {
    case 64: return dispatch_group<64>(sh, p, k_cache, v_cache, stream);
    case 128: return dispatch_group<128>(sh, p, k_cache, v_cache, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace pa
