// pa_decode_noalloc: paged decode attention with library-owned split-K scratch.
//
// pa_decode needs a device workspace for the partial results of long
// sequences, and leaves allocating it to the caller. Some callers cannot
// allocate device memory at the point where they decode: code that runs under
// a framework whose memory manager owns the whole device pool (a raw
// cudaMalloc there fails, or fragments memory the manager cannot see), code
// in a tight serving loop that must not take an allocation's implicit
// synchronisation, and plain C hosts that only receive pointers to buffers
// someone else created. For them this entry point uses a fixed scratch array
// that lives in the library's own device image instead.
//
// The array below is created when the library's device code is loaded on a
// GPU and stays there until the process exits: every GPU that loads the
// library holds these kScratchBytes, used or not. Its size caps what one call
// may ask for; a call that would need more is rejected before any launch.
// Host code cannot pass the array's name to a kernel (on the host that name
// is only a stand-in, not a device address), so the first call in each CUDA
// context looks its device address up with cudaGetSymbolAddress and keeps it
// for that context; a context made later (after cudaDeviceReset, say) loads
// the device code again and gets its own lookup.
#include "pa.h"
#include "pa_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device
static_assert(kScratchBytes == PA_DECODE_NOALLOC_SCRATCH_BYTES, "header and library disagree");

// Split-K partial maxima, sums and accumulators of pa_decode_noalloc calls.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// Device address of g_decode_scratch in the current context, looked up once per context.
int scratch_for_current_context(void** out) {
  static pa::SymbolAddressCache cache;
  const cudaError_t e = cache.get(&g_decode_scratch, out);
  if (e != cudaSuccess)
    return pa_fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress failed: %s",
                   cudaGetErrorString(e));
  return PA_OK;
}

}  // namespace

extern "C" size_t pa_decode_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" int pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int num_seqs, int num_heads,
                                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                 int max_blocks_per_seq, int max_context_len, float scale,
                                 int partition_size, pa_dtype dtype, pa_stream_t stream) {
  if (num_seqs == 0) return PA_OK;
  if (dtype == PA_FP8_E4M3)
    return pa_fail(PA_ERR_UNSUPPORTED, "pa_decode_noalloc: E4M3 caches decode through pa_decode_fp8");
  // pa_decode's own argument checks first, so that a bad argument is reported
  // as such and not as a scratch shortfall; then the scratch this call needs,
  // sized exactly as pa_decode sizes a workspace, refused before any launch if
  // it does not fit.
  pa::DecodeShape sh;
  const int checked = pa::check_decode_args(
      out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, num_kv_heads,
      head_dim, block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
      partition_size, nullptr, dtype, nullptr, nullptr, &sh);
  if (checked != PA_OK) return checked;
  const size_t need = pa::workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim,
                                           sh.num_partitions).total;
  if (need > kScratchBytes)
    return pa_fail(PA_ERR_INVALID,
                   "pa_decode_noalloc: this call needs %zu bytes of split-K scratch, the limit is "
                   "%zu; use a larger partition_size, fewer sequences per call, or pa_decode with "
                   "a workspace of your own",
                   need, kScratchBytes);
  void* scratch = nullptr;
  if (need > 0) {
    const int st = scratch_for_current_context(&scratch);
    if (st != PA_OK) return st;
  }
  // Same checks, kernels and launch as pa_decode; only the workspace differs.
  return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                   num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                   max_context_len, scale, partition_size, scratch, need > 0 ? kScratchBytes : 0,
                   dtype, stream);
}
