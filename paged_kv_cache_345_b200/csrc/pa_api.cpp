// C-ABI shim: argument checks on the host, then one launch per call.
// Nothing here touches device memory except through the launchers.
#include <cmath>
#include <cstdarg>
#include <algorithm>
#include <cstdio>
#include <string>
#include <vector>

#include "pa.h"
#include "pa_internal.h"
#include "pa_prefill_order.h"

namespace {

thread_local std::string g_last_error;
thread_local unsigned int g_decode_options = 0;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int elem_bytes(pa_dtype dt) { return dt == PA_FP8_E4M3 ? 1 : dt == PA_BF16 ? 2 : 4; }
// dtypes of calls that move whole rows or blocks bit for bit
bool valid_dtype(int dt) { return dt == PA_F32 || dt == PA_BF16 || dt == PA_FP8_E4M3; }
// dtypes of pa_kv_append / pa_decode / pa_decode_append (E4M3: the _fp8 calls)
bool valid_compute_dtype(int dt) { return dt == PA_F32 || dt == PA_BF16; }

int cuda_fail(const char* what, cudaError_t e) {
  return pa_fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

void pa_set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

void pa_clear_error() { g_last_error.clear(); }

int pa_fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

namespace pa {

WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int num_partitions) {
  WorkspaceLayout w{};
  if (num_partitions <= 1) return w;
  const size_t rows = static_cast<size_t>(num_seqs) * num_heads * num_partitions;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  (void)num_kv_heads;
  w.m_off = 0;
  w.l_off = w.m_off + up(rows * sizeof(float));
  w.acc_off = w.l_off + up(rows * sizeof(float));
  w.total = w.acc_off + up(rows * head_dim * sizeof(float));
  return w;
}

}  // namespace pa

extern "C" {

const char* pa_last_error(void) { return g_last_error.c_str(); }

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID: return "PA_ERR_INVALID";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_NO_BLOCKS: return "PA_ERR_NO_BLOCKS";
    case PA_ERR_DEVICE_CHECK: return "PA_ERR_DEVICE_CHECK";
    default: return "PA_ERR_UNKNOWN";
  }
}

int pa_kv_append(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                 int num_tokens, void* k_cache, void* v_cache, int num_blocks, int block_size,
                 int num_kv_heads, int head_dim, pa_dtype dtype, pa_stream_t stream) {
  if (num_tokens < 0) return pa_fail(PA_ERR_INVALID, "pa_kv_append: num_tokens < 0");
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache)
    return pa_fail(PA_ERR_INVALID, "pa_kv_append: null pointer");
  if (!valid_compute_dtype(dtype))
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_kv_append: dtype %d (E4M3 caches: pa_kv_append_fp8)",
                   dtype);
  if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_kv_append: sizes must be positive");
  const int64_t row_bytes = static_cast<int64_t>(num_kv_heads) * head_dim * elem_bytes(dtype);
  if (row_bytes % 16 != 0 || row_bytes > (1 << 30))
    return pa_fail(PA_ERR_UNSUPPORTED,
                   "pa_kv_append: num_kv_heads*head_dim*elem (%lld B) not a multiple of 16",
                   static_cast<long long>(row_bytes));
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16) || !aligned(slot_mapping, 8))
    return pa_fail(PA_ERR_INVALID, "pa_kv_append: misaligned pointer");
  const int64_t num_slots = static_cast<int64_t>(num_blocks) * block_size;
  cudaError_t e = pa::launch_kv_append(k_new, v_new, slot_mapping, num_tokens, k_cache, v_cache,
                                       num_slots, static_cast<int>(row_bytes),
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_kv_append launch", e);
}

int pa_kv_append_fp8(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                     int num_tokens, void* k_cache, void* v_cache, const float* k_scale,
                     const float* v_scale, int num_blocks, int block_size, int num_kv_heads,
                     int head_dim, pa_stream_t stream) {
  if (num_tokens < 0) return pa_fail(PA_ERR_INVALID, "pa_kv_append_fp8: num_tokens < 0");
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale)
    return pa_fail(PA_ERR_INVALID, "pa_kv_append_fp8: null pointer");
  if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_kv_append_fp8: sizes must be positive");
  if (head_dim % 16 != 0 || static_cast<int64_t>(num_kv_heads) * head_dim > (1 << 28))
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_kv_append_fp8: head_dim %d not a multiple of 16",
                   head_dim);
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16) || !aligned(slot_mapping, 8) || !aligned(k_scale, 4) ||
      !aligned(v_scale, 4))
    return pa_fail(PA_ERR_INVALID, "pa_kv_append_fp8: misaligned pointer");
  const int64_t num_slots = static_cast<int64_t>(num_blocks) * block_size;
  cudaError_t e = pa::launch_kv_append_fp8(k_new, v_new, slot_mapping, num_tokens, k_cache,
                                           v_cache, k_scale, v_scale, num_slots, num_kv_heads,
                                           head_dim, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_kv_append_fp8 launch", e);
}

int pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping, int num_pairs,
                   int num_blocks, int block_size, int num_kv_heads, int head_dim,
                   pa_dtype dtype, pa_stream_t stream) {
  if (num_pairs < 0) return pa_fail(PA_ERR_INVALID, "pa_copy_blocks: num_pairs < 0");
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_mapping)
    return pa_fail(PA_ERR_INVALID, "pa_copy_blocks: null pointer");
  if (!valid_dtype(dtype)) return pa_fail(PA_ERR_UNSUPPORTED, "pa_copy_blocks: dtype %d", dtype);
  if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_copy_blocks: sizes must be positive");
  if (num_pairs > 2147483647 / 2)
    return pa_fail(PA_ERR_INVALID, "pa_copy_blocks: too many pairs");
  const int64_t block_bytes =
      static_cast<int64_t>(block_size) * num_kv_heads * head_dim * elem_bytes(dtype);
  if (block_bytes % 16 != 0)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_copy_blocks: block bytes not a multiple of 16");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_mapping, 8))
    return pa_fail(PA_ERR_INVALID, "pa_copy_blocks: misaligned pointer");
  cudaError_t e = pa::launch_copy_blocks(k_cache, v_cache, block_mapping, num_pairs, num_blocks,
                                         block_bytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_copy_blocks launch", e);
}

int pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, int dst_num_blocks,
                   const void* src_k_cache, const void* src_v_cache, int src_num_blocks,
                   const int64_t* block_mapping, int num_pairs, int block_size, int num_kv_heads,
                   int head_dim, pa_dtype dtype, pa_stream_t stream) {
  if (num_pairs < 0) return pa_fail(PA_ERR_INVALID, "pa_swap_blocks: num_pairs < 0");
  if (num_pairs == 0) return PA_OK;
  if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !block_mapping)
    return pa_fail(PA_ERR_INVALID, "pa_swap_blocks: null pointer");
  if (!valid_dtype(dtype)) return pa_fail(PA_ERR_UNSUPPORTED, "pa_swap_blocks: dtype %d", dtype);
  if (dst_num_blocks <= 0 || src_num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_swap_blocks: sizes must be positive");
  if (num_pairs > 2147483647 / 2) return pa_fail(PA_ERR_INVALID, "pa_swap_blocks: too many pairs");
  const int64_t block_bytes =
      static_cast<int64_t>(block_size) * num_kv_heads * head_dim * elem_bytes(dtype);
  if (block_bytes % 16 != 0)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_swap_blocks: block bytes not a multiple of 16");
  if (!aligned(dst_k_cache, 16) || !aligned(dst_v_cache, 16) || !aligned(src_k_cache, 16) ||
      !aligned(src_v_cache, 16) || !aligned(block_mapping, 8))
    return pa_fail(PA_ERR_INVALID, "pa_swap_blocks: misaligned pointer");
  cudaError_t e = pa::launch_swap_blocks(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache,
                                         block_mapping, num_pairs, src_num_blocks, dst_num_blocks,
                                         block_bytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_swap_blocks launch", e);
}

unsigned int pa_set_decode_options(unsigned int options) {
  const unsigned int old = g_decode_options;
  g_decode_options = options & PA_DECODE_EARLY_CACHE_READS;
  return old;
}

namespace {
// Partition length for about `ctas_per_sm` CTAs per SM if every sequence were
// as long as max_context_len (one CTA per group of up to 4 KV heads,
// partition and sequence), 64..768 tokens, a multiple of the chunk.
int partition_for(int num_seqs, int num_kv_heads, int max_context_len, double ctas_per_sm) {
  const int groups = num_kv_heads % 4 == 0 ? num_kv_heads / 4
                     : num_kv_heads % 2 == 0 ? num_kv_heads / 2 : num_kv_heads;
  const double work = static_cast<double>(max_context_len) * (num_seqs > 0 ? num_seqs : 1) *
                      (groups > 0 ? groups : 1);
  double p = std::ceil(work / (148.0 * ctas_per_sm));
  if (p < 64) p = 64;
  if (p > 768) p = 768;
  const int c = pa::kChunkTokens;
  return (static_cast<int>(p) + c - 1) / c * c;
}
}  // namespace

int pa_decode_partition_size(int num_seqs, int num_kv_heads, int max_context_len) {
  // Two bf16 CTAs per SM are resident; aim for about five per SM over the
  // launch, so that most sequences are shorter than the longest still leaves
  // every SM a CTA (Llama-3-8B batch, 8 sequences up to 4,101 tokens: 96
  // tokens 11.8 us per layer back to back, 160 tokens 12.4 us). Partitions
  // of 64..768 tokens: long enough to amortise a CTA's start-up, short enough
  // to bound the tail (256-sequence lognormal batch: 512 -> 82 %, 768 -> 84 %,
  // 1024 -> 80 % of HBM bandwidth).
  return partition_for(num_seqs, num_kv_heads, max_context_len, 5.0);
}

static int resolve_partitions(int max_context_len, int* partition_size) {
  if (*partition_size == 0) *partition_size = pa_decode_partition_size(1, 1, 0);
  return max_context_len <= 0 ? 1 : (max_context_len + *partition_size - 1) / *partition_size;
}

size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int max_context_len, int partition_size) {
  if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
      partition_size < 0)
    return 0;
  int ps = partition_size == 0 ? pa_decode_partition_size(num_seqs, num_kv_heads, max_context_len)
                               : partition_size;
  const int np = resolve_partitions(max_context_len, &ps);
  return pa::workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, np).total;
}

// (C++ linkage inside the extern "C" block: an internal helper, also used by
// pa_decode_noalloc)
extern "C++" {
namespace pa {

int check_decode_args(const void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                      int partition_size, const void* workspace, pa_dtype dtype,
                      const float* k_scale, const float* v_scale, DecodeShape* shape) {
  if (num_seqs < 0) return pa_fail(PA_ERR_INVALID, "pa_decode: num_seqs < 0");
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return pa_fail(PA_ERR_INVALID, "pa_decode: null pointer");
  const bool fp8 = dtype == PA_FP8_E4M3;
  if (!fp8 && !valid_compute_dtype(dtype))
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: dtype %d (E4M3 caches: pa_decode_fp8)", dtype);
  if (fp8) {
    if (!k_scale || !v_scale) return pa_fail(PA_ERR_INVALID, "pa_decode_fp8: null scale");
    if (!aligned(k_scale, 4) || !aligned(v_scale, 4))
      return pa_fail(PA_ERR_INVALID, "pa_decode_fp8: misaligned scale");
    if (head_dim != 128)
      return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_fp8: head_dim %d (built: 128)", head_dim);
  }
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return pa_fail(PA_ERR_INVALID, "pa_decode: num_heads %d not a multiple of num_kv_heads %d",
                   num_heads, num_kv_heads);
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: group size %d (built: 1, 2, 4, 8)", group);
  if (head_dim != 64 && head_dim != 128)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: head_dim %d (built: 64, 128)", head_dim);
  if (!pow2(block_size) || block_size > 256)
    return pa_fail(PA_ERR_INVALID, "pa_decode: block_size %d not a power of two <= 256",
                   block_size);
  if (num_blocks <= 0 || max_blocks_per_seq <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_decode: num_blocks and max_blocks_per_seq must be > 0");
  if (max_context_len < 0 ||
      static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return pa_fail(PA_ERR_INVALID, "pa_decode: max_context_len %d outside [0, %lld]",
                   max_context_len,
                   static_cast<long long>(max_blocks_per_seq) * block_size);
  if (!std::isfinite(scale)) return pa_fail(PA_ERR_INVALID, "pa_decode: scale not finite");
  if (partition_size < 0 || partition_size % kChunkTokens != 0 ||
      partition_size > kMaxPartitionSize)
    return pa_fail(PA_ERR_INVALID, "pa_decode: partition_size %d not a multiple of %d in [0, %d]",
                   partition_size, kChunkTokens, kMaxPartitionSize);
  if (num_seqs > 65535) return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: num_seqs > 65535");
  if (num_kv_heads > 65535) return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: num_kv_heads > 65535");
  if (static_cast<int64_t>(num_blocks) * block_size * num_kv_heads * head_dim *
          elem_bytes(dtype) / 16 > (int64_t(1) << 36))
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: cache larger than 1 TiB");
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) ||
      (workspace && !aligned(workspace, 16)))
    return pa_fail(PA_ERR_INVALID, "pa_decode: misaligned pointer");

  DecodeShape& sh = *shape;
  sh = DecodeShape{};
  sh.num_seqs = num_seqs;
  sh.num_heads = num_heads;
  sh.num_kv_heads = num_kv_heads;
  sh.head_dim = head_dim;
  sh.block_size = block_size;
  sh.num_blocks = num_blocks;
  sh.max_blocks_per_seq = max_blocks_per_seq;
  sh.max_context_len = max_context_len;
  sh.partition_size = partition_size == 0
                          ? pa_decode_partition_size(num_seqs, num_kv_heads, max_context_len)
                          : partition_size;
  sh.num_partitions = resolve_partitions(max_context_len, &sh.partition_size);
  sh.scale = scale;
  sh.dtype = dtype;
  sh.early_reads = (g_decode_options & PA_DECODE_EARLY_CACHE_READS) != 0;
  if (sh.num_partitions > kMaxPartitions)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: %d partitions > %d", sh.num_partitions,
                   kMaxPartitions);
  return PA_OK;
}

}  // namespace pa
}  // extern "C++"

static int decode_common(void* out, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                         int num_heads, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                         int partition_size, void* workspace, size_t workspace_bytes,
                         pa_dtype dtype, const void* k_new, const void* v_new,
                         const float* k_scale, const float* v_scale, pa_stream_t stream) {
  if (num_seqs == 0) return PA_OK;
  pa::DecodeShape sh;
  const int st = pa::check_decode_args(out, q, k_cache, v_cache, block_tables, context_lens,
                                       num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                       num_blocks, max_blocks_per_seq, max_context_len, scale,
                                       partition_size, workspace, dtype, k_scale, v_scale, &sh);
  if (st != PA_OK) return st;
  const size_t need =
      pa::workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, sh.num_partitions).total;
  if (need > 0 && (!workspace || workspace_bytes < need))
    return pa_fail(PA_ERR_INVALID, "pa_decode: workspace %zu B < %zu B needed",
                   workspace ? workspace_bytes : size_t(0), need);
  cudaError_t e = pa::launch_decode(sh, out, q, k_cache, v_cache, block_tables, context_lens,
                                    workspace, k_new, v_new, k_scale, v_scale,
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: no kernel for this shape");
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_decode launch", e);
}

int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
              int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
              int max_blocks_per_seq, int max_context_len, float scale, int partition_size,
              void* workspace, size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream) {
  if (dtype == PA_FP8_E4M3)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode: E4M3 caches decode through pa_decode_fp8");
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                       max_context_len, scale, partition_size, workspace, workspace_bytes,
                       dtype, nullptr, nullptr, nullptr, nullptr, stream);
}

int pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                     void* k_cache, void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                     int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                     int max_context_len, float scale, int partition_size, void* workspace,
                     size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream) {
  if (dtype == PA_FP8_E4M3)
    return pa_fail(PA_ERR_UNSUPPORTED,
                   "pa_decode_append: E4M3 caches decode through pa_decode_append_fp8");
  if (num_seqs > 0 && (!k_new || !v_new))
    return pa_fail(PA_ERR_INVALID, "pa_decode_append: null k_new or v_new");
  if (num_seqs > 0 && (!aligned(k_new, 16) || !aligned(v_new, 16)))
    return pa_fail(PA_ERR_INVALID, "pa_decode_append: misaligned k_new or v_new");
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                       max_context_len, scale, partition_size, workspace, workspace_bytes,
                       dtype, k_new, v_new, nullptr, nullptr, stream);
}

int pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                  const float* k_scale, const float* v_scale, const int32_t* block_tables,
                  const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                  int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                  int max_context_len, float scale, int partition_size, void* workspace,
                  size_t workspace_bytes, pa_stream_t stream) {
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                       max_context_len, scale, partition_size, workspace, workspace_bytes,
                       PA_FP8_E4M3, nullptr, nullptr, k_scale, v_scale, stream);
}

int pa_decode_append_fp8(void* out, const void* q, const void* k_new, const void* v_new,
                         void* k_cache, void* v_cache, const float* k_scale,
                         const float* v_scale, const int32_t* block_tables,
                         const int32_t* context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks,
                         int max_blocks_per_seq, int max_context_len, float scale,
                         int partition_size, void* workspace, size_t workspace_bytes,
                         pa_stream_t stream) {
  if (num_seqs > 0 && (!k_new || !v_new))
    return pa_fail(PA_ERR_INVALID, "pa_decode_append_fp8: null k_new or v_new");
  if (num_seqs > 0 && (!aligned(k_new, 16) || !aligned(v_new, 16)))
    return pa_fail(PA_ERR_INVALID, "pa_decode_append_fp8: misaligned k_new or v_new");
  return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                       max_context_len, scale, partition_size, workspace, workspace_bytes,
                       PA_FP8_E4M3, k_new, v_new, k_scale, v_scale, stream);
}

int pa_decode_plan(const int32_t* context_lens, int num_seqs, int partition_size, int32_t* work,
                   int capacity, int* num_items) {
  if (!num_items || (num_seqs > 0 && (!context_lens || !work)))
    return pa_fail(PA_ERR_INVALID, "pa_decode_plan: null pointer");
  *num_items = 0;
  if (num_seqs < 0) return pa_fail(PA_ERR_INVALID, "pa_decode_plan: num_seqs < 0");
  if (partition_size <= 0 || partition_size % pa::kChunkTokens != 0 ||
      partition_size > pa::kMaxPartitionSize)
    return pa_fail(PA_ERR_INVALID,
                   "pa_decode_plan: partition_size %d not a multiple of %d in [%d, %d]",
                   partition_size, pa::kChunkTokens, pa::kChunkTokens, pa::kMaxPartitionSize);
  // count first: whole partitions, then one shorter last partition per
  // sequence (or the single item of an empty one)
  int64_t total = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const int L = context_lens[s];
    if (L < 0) return pa_fail(PA_ERR_INVALID, "pa_decode_plan: context_lens[%d] = %d", s, L);
    const int64_t n = L == 0 ? 1 : (static_cast<int64_t>(L) + partition_size - 1) / partition_size;
    if (n > 65535)
      return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_plan: sequence %d needs %lld partitions",
                     s, static_cast<long long>(n));
    total += n;
  }
  if (total > capacity) {
    *num_items = static_cast<int>(std::min<int64_t>(total, INT32_MAX));
    return pa_fail(PA_ERR_INVALID, "pa_decode_plan: %lld items > capacity %d",
                   static_cast<long long>(total), capacity);
  }
  // Whole partitions first, sequence by sequence; then the ragged last ones
  // (every sequence whose length is not a multiple of the partition, and the
  // empty ones), longest first, ties by sequence. The block scheduler hands
  // CTAs out in grid order, so the short ones fill the tail.
  thread_local std::vector<int64_t> ragged;
  ragged.clear();
  int64_t i = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const int L = context_lens[s];
    const int n = L == 0 ? 1 : static_cast<int>((static_cast<int64_t>(L) + partition_size - 1) /
                                                partition_size);
    const int whole = L / partition_size;
    for (int k = 0; k < whole; ++k, ++i) {
      work[2 * i] = s;
      work[2 * i + 1] = static_cast<int32_t>(static_cast<uint32_t>(n) << 16 | static_cast<uint32_t>(k));
    }
    if (whole < n) {
      const int rest = L - whole * partition_size;  // tokens of the last partition (0: empty)
      ragged.push_back((static_cast<int64_t>(partition_size - rest) << 32) | s);
    }
  }
  std::sort(ragged.begin(), ragged.end());
  for (const int64_t key : ragged) {
    const int s = static_cast<int>(key & 0xffffffff);
    const int L = context_lens[s];
    const int n = L == 0 ? 1 : static_cast<int>((static_cast<int64_t>(L) + partition_size - 1) /
                                                partition_size);
    work[2 * i] = s;
    work[2 * i + 1] = static_cast<int32_t>(static_cast<uint32_t>(n) << 16 | static_cast<uint32_t>(n - 1));
    ++i;
  }
  *num_items = static_cast<int>(i);
  return PA_OK;
}

int pa_decode_planned(void* out, const void* q, const void* k_new, const void* v_new,
                      void* k_cache, void* v_cache, const float* k_scale, const float* v_scale,
                      const int32_t* block_tables, const int32_t* context_lens,
                      const int32_t* work, int num_items, int num_seqs, int num_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      int max_blocks_per_seq, int max_context_len, float scale,
                      int partition_size, void* workspace, size_t workspace_bytes,
                      pa_dtype dtype, pa_stream_t stream) {
  if (num_seqs == 0) return PA_OK;
  if (dtype != PA_BF16 && dtype != PA_FP8_E4M3)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_planned: dtype %d (bf16 or E4M3 caches)",
                   dtype);
  if ((k_new == nullptr) != (v_new == nullptr))
    return pa_fail(PA_ERR_INVALID, "pa_decode_planned: k_new and v_new must both be set or null");
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16)))
    return pa_fail(PA_ERR_INVALID, "pa_decode_planned: misaligned k_new or v_new");
  if (dtype == PA_BF16 && (k_scale || v_scale))
    return pa_fail(PA_ERR_INVALID, "pa_decode_planned: scales given for a bf16 cache");
  if (!work || !aligned(work, 8))
    return pa_fail(PA_ERR_INVALID, "pa_decode_planned: null or misaligned work list");
  if (partition_size <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_decode_planned: partition_size must be the plan's (> 0)");
  pa::DecodeShape sh;
  const int st = pa::check_decode_args(out, q, k_cache, v_cache, block_tables, context_lens,
                                       num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                       num_blocks, max_blocks_per_seq, max_context_len, scale,
                                       partition_size, workspace, dtype, k_scale, v_scale, &sh);
  if (st != PA_OK) return st;
  const int64_t most = static_cast<int64_t>(num_seqs) * std::max(sh.num_partitions, 1);
  if (num_items < num_seqs || num_items > 65535 || num_items > most)
    return pa_fail(PA_ERR_INVALID, "pa_decode_planned: num_items %d outside [%d, %lld]",
                   num_items, num_seqs, static_cast<long long>(std::min<int64_t>(most, 65535)));
  const size_t need =
      pa::workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, sh.num_partitions).total;
  if (need > 0 && (!workspace || workspace_bytes < need))
    return pa_fail(PA_ERR_INVALID, "pa_decode_planned: workspace %zu B < %zu B needed",
                   workspace ? workspace_bytes : size_t(0), need);
  sh.work = work;
  sh.num_items = num_items;
  cudaError_t e = pa::launch_decode(sh, out, q, k_cache, v_cache, block_tables, context_lens,
                                    workspace, k_new, v_new, k_scale, v_scale,
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_planned: no kernel for this shape");
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_decode_planned launch", e);
}

// Sizes of a shared-prefix call: suffix partition size, suffix partitions,
// prefix partition size (keys) and prefix partitions.
namespace {
struct PrefixPlan {
  int suffix_part, suffix_parts, prefix_part, prefix_parts;
};

// Keys per partition of the prefix pass. Its CTAs (one per SM: KV heads x
// pairs of 128-row query tiles x key partitions) run beside the suffix
// decode, which takes the other SMs. Beside a decode that keeps HBM busy a CTA
// costs about kStartUs + (its key tiles) * kTileUs (4, 8, 16 tiles of 256
// query rows: 17, 20, 35 us); the decode about its bytes, sequences' own
// tokens taken as half the longest, at kDecodeBytesPerUs (measured beside the
// pass: the 64-sequence workload's estimate of 131 MB took ~30 us). Take the
// fewest partitions whose CTAs end within that estimate, at most a quarter of
// the SMs (that workload: 2 / 3 / 4 / 5 / 6 / 8 partitions gave 43.9 / 40.1 /
// 40.9 / 42.0 / 42.0 / 43.9 us a step; the rule takes 3).
int prefix_partition_keys(int num_seqs, int num_heads, int num_kv_heads, int prefix_len,
                          int max_context_len) {
  constexpr double kStartUs = 10.0, kTileUs = 1.6, kDecodeBytesPerUs = 4.4e6;
  constexpr int kTile = pa::kPrefillKeyTile;
  const int tok = 2 * (128 / (num_heads / num_kv_heads));  // query tokens per CTA
  const int64_t pairs = (static_cast<int64_t>(num_seqs) + tok - 1) / tok;
  const int64_t base = static_cast<int64_t>(num_kv_heads) * pairs;
  const int64_t tiles = (prefix_len + kTile - 1) / kTile;
  const int64_t rest = max_context_len > prefix_len ? max_context_len - prefix_len : 0;
  const double decode_us = static_cast<double>(num_seqs) * num_kv_heads * rest * 0.5 * 512.0 /
                           kDecodeBytesPerUs;
  int64_t max_parts = 37 / base;
  if (max_parts < 1) max_parts = 1;
  if (max_parts > tiles) max_parts = tiles;
  int64_t parts = 1;
  while (parts < max_parts &&
         kStartUs + static_cast<double>((tiles + parts - 1) / parts) * kTileUs > decode_us)
    ++parts;
  return static_cast<int>(((tiles + parts - 1) / parts) * kTile);
}

PrefixPlan plan_shared_prefix(int num_seqs, int num_heads, int num_kv_heads, int prefix_len,
                              int max_context_len, int partition_size) {
  PrefixPlan pl{};
  const int rest = max_context_len - prefix_len;
  if (partition_size == 0) {
    // the suffix decode runs on the SMs the prefix pass leaves and its end is
    // the critical path (64 sequences, suffixes of 50..1000 tokens: 208
    // tokens 41.0 us a step, 176 42.6, 304 45.5)
    pl.suffix_part = partition_for(num_seqs, num_kv_heads, rest > 0 ? rest : 0, 4.5);
  } else {
    pl.suffix_part = partition_size;
  }
  pl.suffix_parts = rest <= 0 ? 1 : (rest + pl.suffix_part - 1) / pl.suffix_part;
  pl.prefix_part =
      prefix_partition_keys(num_seqs, num_heads, num_kv_heads, prefix_len, max_context_len);
  pl.prefix_parts = (prefix_len + pl.prefix_part - 1) / pl.prefix_part;
  return pl;
}
}  // namespace

size_t pa_decode_shared_prefix_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                               int head_dim, int prefix_len, int max_context_len,
                                               int partition_size) {
  if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || prefix_len <= 0 ||
      max_context_len < prefix_len || partition_size < 0 || num_heads % num_kv_heads != 0)
    return 0;
  const PrefixPlan pl = plan_shared_prefix(num_seqs, num_heads, num_kv_heads, prefix_len,
                                           max_context_len, partition_size);
  return pa::workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim,
                              pl.prefix_parts + pl.suffix_parts)
      .total;
}

int pa_decode_shared_prefix(void* out, const void* q, const void* k_new, const void* v_new,
                            void* k_cache, void* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, int num_seqs, int num_heads,
                            int num_kv_heads, int head_dim, int block_size, int num_blocks,
                            int max_blocks_per_seq, int prefix_len, int max_context_len,
                            float scale, int partition_size, void* workspace,
                            size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream) {
  if (num_seqs == 0) return PA_OK;
  pa::DecodeShape sh;
  int st = pa::check_decode_args(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                                 num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                 max_blocks_per_seq, max_context_len, scale, partition_size,
                                 workspace, dtype, nullptr, nullptr, &sh);
  if (st != PA_OK) return st;
  if (dtype != PA_BF16 || head_dim != 128)
    return pa_fail(PA_ERR_UNSUPPORTED,
                   "pa_decode_shared_prefix: dtype %d, head_dim %d (built: bf16, 128)", dtype,
                   head_dim);
  if (block_size < 8)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_shared_prefix: block_size %d (built: 8..256)",
                   block_size);
  if (!std::isfinite(scale) || scale <= 0.0f)
    return pa_fail(PA_ERR_INVALID, "pa_decode_shared_prefix: scale must be finite and > 0");
  if (prefix_len <= 0 || prefix_len % block_size != 0 || prefix_len > max_context_len)
    return pa_fail(PA_ERR_INVALID,
                   "pa_decode_shared_prefix: prefix_len %d not a positive multiple of block_size "
                   "%d within max_context_len %d",
                   prefix_len, block_size, max_context_len);
  if ((k_new == nullptr) != (v_new == nullptr))
    return pa_fail(PA_ERR_INVALID, "pa_decode_shared_prefix: k_new and v_new go together");
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16)))
    return pa_fail(PA_ERR_INVALID, "pa_decode_shared_prefix: misaligned k_new or v_new");
  const PrefixPlan pl = plan_shared_prefix(num_seqs, num_heads, num_kv_heads, prefix_len,
                                           max_context_len, partition_size);
  sh.partition_size = pl.suffix_part;
  sh.prefix_slots = pl.prefix_parts;
  sh.num_partitions = pl.prefix_parts + pl.suffix_parts;
  sh.first_token = prefix_len;
  if (sh.num_partitions > pa::kMaxPartitions)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_shared_prefix: %d partitions > %d",
                   sh.num_partitions, pa::kMaxPartitions);
  const pa::WorkspaceLayout wl =
      pa::workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, sh.num_partitions);
  if (!workspace || workspace_bytes < wl.total)
    return pa_fail(PA_ERR_INVALID, "pa_decode_shared_prefix: workspace %zu B < %zu B needed",
                   workspace ? workspace_bytes : size_t(0), wl.total);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // 1: every sequence's query against the shared prefix, once per KV head
  cudaError_t e = pa::launch_prefix_attention(
      num_seqs, num_heads, num_kv_heads, block_size, num_blocks, max_blocks_per_seq, prefix_len,
      pl.prefix_part, scale, q, k_cache, v_cache, block_tables,
      reinterpret_cast<float*>(ws + wl.m_off), reinterpret_cast<float*>(ws + wl.l_off),
      reinterpret_cast<float*>(ws + wl.acc_off), sh.num_partitions, cs);
  if (e == cudaErrorNotSupported)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_shared_prefix: no prefix kernel for this shape");
  if (e != cudaSuccess) return cuda_fail("pa_decode_shared_prefix prefix launch", e);
  // 2, 3: each sequence's own tokens (appending its newest first), then the merge
  e = pa::launch_decode(sh, out, q, k_cache, v_cache, block_tables, context_lens, workspace,
                        k_new, v_new, nullptr, nullptr, cs);
  if (e == cudaErrorNotSupported)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_shared_prefix: no kernel for this shape");
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_decode_shared_prefix launch", e);
}

int pa_decode_contiguous(void* out, const void* q, const void* k, const void* v,
                         const int32_t* context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, int slab_len, int max_context_len,
                         float scale, int partition_size, void* workspace,
                         size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream) {
  if (num_seqs < 0) return pa_fail(PA_ERR_INVALID, "pa_decode_contiguous: num_seqs < 0");
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k || !v || !context_lens)
    return pa_fail(PA_ERR_INVALID, "pa_decode_contiguous: null pointer");
  if (dtype != PA_BF16)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: dtype %d (built: bf16)", dtype);
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return pa_fail(PA_ERR_INVALID,
                   "pa_decode_contiguous: num_heads %d not a multiple of num_kv_heads %d",
                   num_heads, num_kv_heads);
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: group size %d (built: 1, 2, 4, 8)",
                   group);
  if (head_dim != 64 && head_dim != 128)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: head_dim %d (built: 64, 128)",
                   head_dim);
  if (slab_len < 16 || slab_len > (1 << 24))
    return pa_fail(PA_ERR_INVALID, "pa_decode_contiguous: slab_len %d outside [16, 2^24]",
                   slab_len);
  if (max_context_len < 0 || max_context_len > slab_len)
    return pa_fail(PA_ERR_INVALID, "pa_decode_contiguous: max_context_len %d outside [0, %d]",
                   max_context_len, slab_len);
  if (!std::isfinite(scale)) return pa_fail(PA_ERR_INVALID, "pa_decode_contiguous: scale not finite");
  if (partition_size < 0 || partition_size % pa::kChunkTokens != 0 ||
      partition_size > pa::kMaxPartitionSize)
    return pa_fail(PA_ERR_INVALID,
                   "pa_decode_contiguous: partition_size %d not a multiple of %d in [0, %d]",
                   partition_size, pa::kChunkTokens, pa::kMaxPartitionSize);
  if (num_seqs > 65535 || num_kv_heads > 65535)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: num_seqs or num_kv_heads > 65535");
  if (static_cast<int64_t>(num_seqs) * slab_len * num_kv_heads * head_dim * 2 / 16 >
      (int64_t(1) << 36))
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: cache larger than 1 TiB");
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
      !aligned(context_lens, 4) || (workspace && !aligned(workspace, 16)))
    return pa_fail(PA_ERR_INVALID, "pa_decode_contiguous: misaligned pointer");
  pa::DecodeShape sh{};
  sh.num_seqs = num_seqs;
  sh.num_heads = num_heads;
  sh.num_kv_heads = num_kv_heads;
  sh.head_dim = head_dim;
  sh.block_size = slab_len;   // one "block" per sequence: its slab
  sh.num_blocks = num_seqs;
  sh.max_blocks_per_seq = 1;
  sh.max_context_len = max_context_len;
  sh.partition_size = partition_size == 0
                          ? pa_decode_partition_size(num_seqs, num_kv_heads, max_context_len)
                          : partition_size;
  sh.num_partitions = resolve_partitions(max_context_len, &sh.partition_size);
  sh.scale = scale;
  sh.dtype = dtype;
  sh.early_reads = (g_decode_options & PA_DECODE_EARLY_CACHE_READS) != 0;
  sh.contiguous = true;
  if (sh.num_partitions > pa::kMaxPartitions)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: %d partitions > %d",
                   sh.num_partitions, pa::kMaxPartitions);
  const size_t need =
      pa::workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, sh.num_partitions).total;
  if (need > 0 && (!workspace || workspace_bytes < need))
    return pa_fail(PA_ERR_INVALID, "pa_decode_contiguous: workspace %zu B < %zu B needed",
                   workspace ? workspace_bytes : size_t(0), need);
  cudaError_t e = pa::launch_decode(sh, out, q, k, v, nullptr, context_lens, workspace, nullptr,
                                    nullptr, nullptr, nullptr,
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: no kernel for this shape");
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_decode_contiguous launch", e);
}

// pa_prefill, and with a work list (work != null) pa_prefill_planned.
static int prefill_common(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens,
                          const int32_t* query_start, const int32_t* work, int num_items,
                          int num_seqs, int total_q, int num_heads, int num_kv_heads,
                          int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                          int max_query_len, float scale, pa_dtype dtype, pa_stream_t stream) {
  if (num_seqs < 0 || total_q < 0 || max_query_len < 0)
    return pa_fail(PA_ERR_INVALID, "pa_prefill: negative size");
  if (num_seqs == 0 || total_q == 0 || max_query_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
    return pa_fail(PA_ERR_INVALID, "pa_prefill: null pointer");
  if (dtype != PA_BF16) return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill: dtype %d (built: bf16)", dtype);
  if (head_dim != 128)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill: head_dim %d (built: 128)", head_dim);
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return pa_fail(PA_ERR_INVALID, "pa_prefill: num_heads %d not a multiple of num_kv_heads %d",
                   num_heads, num_kv_heads);
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill: group size %d (built: 1, 2, 4, 8)", group);
  if (!pow2(block_size) || block_size < 8 || block_size > 256)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill: block_size %d (built: powers of two 8..256)",
                   block_size);
  if (num_blocks <= 0 || max_blocks_per_seq <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_prefill: num_blocks and max_blocks_per_seq must be > 0");
  if (max_query_len > total_q)
    return pa_fail(PA_ERR_INVALID, "pa_prefill: max_query_len %d > total_q %d", max_query_len,
                   total_q);
  if (!std::isfinite(scale) || scale <= 0.0f)
    return pa_fail(PA_ERR_INVALID, "pa_prefill: scale must be finite and > 0");
  const int tok = 256 / group;  // query tokens per CTA
  if (static_cast<int64_t>(num_seqs) * ((max_query_len + tok - 1) / tok) * num_kv_heads >
      0x7fffffff)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill: grid too large");
  if (static_cast<int64_t>(num_blocks) * block_size * num_kv_heads * head_dim * 2 / 16 >
      (int64_t(1) << 36))
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill: cache larger than 1 TiB");
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start, 4))
    return pa_fail(PA_ERR_INVALID, "pa_prefill: misaligned pointer");
  pa::PrefillShape sh{};
  sh.num_seqs = num_seqs;
  sh.total_q = total_q;
  sh.num_heads = num_heads;
  sh.num_kv_heads = num_kv_heads;
  sh.head_dim = head_dim;
  sh.block_size = block_size;
  sh.num_blocks = num_blocks;
  sh.max_blocks_per_seq = max_blocks_per_seq;
  sh.max_query_len = max_query_len;
  sh.scale = scale;
  if (work != nullptr) {
    const int64_t most = static_cast<int64_t>(num_seqs) * ((max_query_len + tok - 1) / tok);
    if (num_items < 0 || num_items > most)
      return pa_fail(PA_ERR_INVALID, "pa_prefill_planned: num_items %d outside [0, %lld]",
                     num_items, static_cast<long long>(most));
    if (num_items == 0) return PA_OK;
    sh.work = work;
    sh.num_items = num_items;
  }
  cudaError_t e = pa::launch_prefill(sh, out, q, k_cache, v_cache, block_tables, context_lens,
                                     query_start, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill: no kernel for this shape");
  return e == cudaSuccess ? PA_OK : cuda_fail("pa_prefill launch", e);
}

int pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
               const int32_t* block_tables, const int32_t* context_lens,
               const int32_t* query_start, int num_seqs, int total_q, int num_heads,
               int num_kv_heads, int head_dim, int block_size, int num_blocks,
               int max_blocks_per_seq, int max_query_len, float scale, pa_dtype dtype,
               pa_stream_t stream) {
  return prefill_common(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                        nullptr, 0, num_seqs, total_q, num_heads, num_kv_heads, head_dim,
                        block_size, num_blocks, max_blocks_per_seq, max_query_len, scale, dtype,
                        stream);
}

int pa_prefill_plan(const int32_t* query_start, const int32_t* context_lens, int num_seqs,
                    int num_heads, int num_kv_heads, int32_t* work, int capacity,
                    int* num_items) {
  namespace po = pa::prefill_order;
  if (!num_items || (num_seqs > 0 && (!query_start || !context_lens || !work)))
    return pa_fail(PA_ERR_INVALID, "pa_prefill_plan: null pointer");
  *num_items = 0;
  if (num_seqs < 0) return pa_fail(PA_ERR_INVALID, "pa_prefill_plan: num_seqs < 0");
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return pa_fail(PA_ERR_INVALID,
                   "pa_prefill_plan: num_heads %d not a multiple of num_kv_heads %d", num_heads,
                   num_kv_heads);
  const int group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_prefill_plan: group size %d (built: 1, 2, 4, 8)",
                   group);
  const int ctok = 256 / group, keyn = pa::kPrefillKeyTile;
  // (cost, sequence, item) of every item, then longest first, ties by
  // sequence, then item: the order the kernel's own search gives
  struct Item {
    int cost, s, z;
  };
  thread_local std::vector<Item> items;
  items.clear();
  for (int s = 0; s < num_seqs; ++s) {
    const int n = query_start[s + 1] - query_start[s], L = context_lens[s];
    if (query_start[s] < 0 || n < 0 || L < n)
      return pa_fail(PA_ERR_INVALID,
                     "pa_prefill_plan: sequence %d: %d query rows from %d over %d tokens", s, n,
                     query_start[s], L);
    const int m = po::num_items(n, ctok);
    for (int z = 0; z < m; ++z) items.push_back(Item{po::cost(L, n, z, ctok, keyn), s, z});
  }
  if (static_cast<int64_t>(items.size()) > capacity) {
    *num_items = static_cast<int>(std::min<size_t>(items.size(), INT32_MAX));
    return pa_fail(PA_ERR_INVALID, "pa_prefill_plan: %zu items > capacity %d", items.size(),
                   capacity);
  }
  std::sort(items.begin(), items.end(), [](const Item& a, const Item& b) {
    return a.cost != b.cost ? a.cost > b.cost : a.s != b.s ? a.s < b.s : a.z < b.z;
  });
  for (size_t i = 0; i < items.size(); ++i) {
    work[2 * i] = items[i].s;
    work[2 * i + 1] = items[i].z;
  }
  *num_items = static_cast<int>(items.size());
  return PA_OK;
}

int pa_prefill_planned(void* out, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, const int32_t* context_lens,
                       const int32_t* query_start, const int32_t* work, int num_items,
                       int num_seqs, int total_q, int num_heads, int num_kv_heads, int head_dim,
                       int block_size, int num_blocks, int max_blocks_per_seq,
                       int max_query_len, float scale, pa_dtype dtype, pa_stream_t stream) {
  if (num_seqs > 0 && (!work || !aligned(work, 8)))
    return pa_fail(PA_ERR_INVALID, "pa_prefill_planned: null or misaligned work list");
  return prefill_common(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                        work, num_items, num_seqs, total_q, num_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                        max_query_len, scale, dtype, stream);
}

int pa_device_errors(pa_stream_t stream, unsigned int* flags) {
  unsigned int* word = nullptr;
  cudaError_t e = pa::device_error_word(&word);
  if (e != cudaSuccess) return cuda_fail("pa_device_errors: symbol", e);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int host = 0;
  if ((e = cudaMemcpyAsync(&host, word, sizeof(host), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail("pa_device_errors: read", e);
  if ((e = cudaMemsetAsync(word, 0, sizeof(unsigned int), st)) != cudaSuccess)
    return cuda_fail("pa_device_errors: clear", e);
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess)
    return cuda_fail("pa_device_errors: sync", e);
  if (flags) *flags = host;
  if (host != 0)
    return pa_fail(PA_ERR_DEVICE_CHECK, "device error word 0x%x", host);
  return PA_OK;
}

}  // extern "C"
