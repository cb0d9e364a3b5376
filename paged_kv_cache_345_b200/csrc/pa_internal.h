// Internal declarations shared by the C-ABI shim, the allocator and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime_api.h>

#include "pa.h"

// Thread-local "last error" text behind pa_last_error().
void pa_set_error(const char* fmt, ...) __attribute__((format(printf, 1, 2)));
void pa_clear_error();
// Sets the last-error text and returns `status`.
int pa_fail(int status, const char* fmt, ...) __attribute__((format(printf, 2, 3)));

namespace pa {

constexpr int kChunkTokens = 16;       // tokens per pipeline stage of the decode kernel
constexpr int kMaxPartitions = 65535;        // grid-y limit
constexpr int kMaxPartitionSize = 1 << 20;   // tokens; keeps partition * size in int range

// Sizes of one pa_decode call after validation.
struct DecodeShape {
  int num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks;
  int max_blocks_per_seq, max_context_len, partition_size, num_partitions;
  float scale;
  pa_dtype dtype;
  bool early_reads;  // PA_DECODE_EARLY_CACHE_READS for this call
  // pa_decode_contiguous: a slab of block_size (= slab length) tokens per
  // sequence, num_blocks = num_seqs, no block table
  bool contiguous;
  // pa_decode_shared_prefix's suffix pass: attend tokens from first_token on;
  // num_partitions counts the prefix_slots workspace slots before this
  // call's own partitions, and every row goes through the merge
  int first_token, prefix_slots;
  // pa_decode_planned: the device work list (num_items items) that replaces
  // the (partition, sequence) grid; null otherwise
  const int32_t* work;
  int num_items;
};

// Byte offsets of the split-K workspace regions.
struct WorkspaceLayout {
  size_t m_off, l_off, acc_off, total;
};
WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int num_partitions);

// Every host-side check of a decode call except the workspace size; fills the
// shape (partition size resolved) and returns PA_OK, or the status a call
// would return (with the last-error text set). num_seqs must be > 0.
int check_decode_args(const void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                      int partition_size, const void* workspace, pa_dtype dtype,
                      const float* k_scale, const float* v_scale, DecodeShape* shape);

// Launchers (pa_kernels.cu). Return cudaSuccess or the launch error.
cudaError_t launch_kv_append(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                             int num_tokens, void* k_cache, void* v_cache, int64_t num_slots,
                             int row_bytes, cudaStream_t stream);
// E4M3 caches: bfloat16 rows in, code of value / scale[head] stored.
cudaError_t launch_kv_append_fp8(const void* k_new, const void* v_new,
                                 const int64_t* slot_mapping, int num_tokens, void* k_cache,
                                 void* v_cache, const float* k_scale, const float* v_scale,
                                 int64_t num_slots, int num_kv_heads, int head_dim,
                                 cudaStream_t stream);
cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                               int num_pairs, int num_blocks, int64_t block_bytes,
                               cudaStream_t stream);
cudaError_t launch_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int64_t* block_mapping, int num_pairs, int src_num_blocks,
                               int dst_num_blocks, int64_t block_bytes, cudaStream_t stream);
// Returns cudaErrorNotSupported when no kernel is built for the shape.
// k_new / v_new non-null: fused append of each sequence's newest token.
// k_scale / v_scale: per-KV-head scales of an E4M3 cache (null otherwise).
cudaError_t launch_decode(const DecodeShape& sh, void* out, const void* q, const void* k_cache,
                          const void* v_cache, const int32_t* block_tables,
                          const int32_t* context_lens, void* workspace, const void* k_new,
                          const void* v_new, const float* k_scale, const float* v_scale,
                          cudaStream_t stream);
// Sizes of one pa_prefill call after validation.
struct PrefillShape {
  int num_seqs, total_q, num_heads, num_kv_heads, head_dim, block_size, num_blocks;
  int max_blocks_per_seq, max_query_len;
  float scale;
  // pa_prefill_planned: the device work list (num_items items {sequence,
  // item}) that replaces the kernel's own search; null otherwise
  const int32_t* work;
  int num_items;
};
// Causal chunked-prefill attention (pa_prefill.cu); bf16, head_dim 128.
cudaError_t launch_prefill(const PrefillShape& sh, void* out, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, const int32_t* query_start,
                           cudaStream_t stream);
// Shared-prefix decode, prefix pass (pa_prefill.cu): the num_seqs decode
// queries q [num_seqs][num_heads][128] (bf16) attend keys [0, prefix_len) read
// through the first row of block_tables, on the tcgen05 tensor cores, in
// partitions of prefix_part keys (a multiple of 64); partition k of row r is
// written to the decode workspace as slot k (ws_slots slots per row).
// Partitions are whole key tiles of the pass.
constexpr int kPrefillKeyTile = 64;
cudaError_t launch_prefix_attention(int num_seqs, int num_heads, int num_kv_heads, int block_size,
                                    int num_blocks, int max_blocks_per_seq, int prefix_len,
                                    int prefix_part, float scale, const void* q,
                                    const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, float* ws_m, float* ws_l,
                                    float* ws_acc, int ws_slots, cudaStream_t stream);

// Device error word of the current device (address in device memory).
cudaError_t device_error_word(unsigned int** ptr);

// Device address of a __device__ variable of this library in the current CUDA
// context, looked up with cudaGetSymbolAddress once per context and cached.
// The key is the context's unique id (cuCtxGetId), not the device ordinal: a
// context created later on the same device (after cudaDeviceReset, say) loads
// the library's device code again, possibly elsewhere, and gets its own lookup.
class SymbolAddressCache {
 public:
  cudaError_t get(const void* symbol, void** out);

 private:
  static constexpr int kEntries = 64;
  struct Entry {
    unsigned long long ctx_id;
    void* ptr;
  };
  Entry entries_[kEntries] = {};
  int next_ = 0;
};

}  // namespace pa
