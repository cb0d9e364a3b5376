/*
 * pa.h — C ABI of the paged KV-cache decode path (B200, sm_100a).
 *
 * The method: the KV cache of every sequence lives in fixed-size physical
 * blocks from a shared pool; a per-sequence block table maps the sequence's
 * logical blocks (token t is in logical block t / block_size at offset
 * t % block_size) to physical block ids, and attention reads the cache
 * through that table without first copying it into contiguous memory.
 *   Sources: "Paged Attention" (klaylearn.com glossary), definition;
 *   "PagedAttention — AI Glossary" (modelrefs.com), How it works 1-5;
 *   "What is paged attention in vLLM, and why does it matter?"
 *   (interview.clozo.ai), Steps 1-4 and "Trade-offs and edge cases".
 *
 * Conventions shared by every call below.
 *   Memory. Every pointer is owned by the caller. "device" pointers are CUDA
 *   global-memory addresses on the current device; "host" pointers are CPU
 *   memory. The kernels allocate no device memory: scratch space for the
 *   split-K pass is a caller-provided workspace sized by
 *   pa_decode_workspace_bytes.
 *   Streams. Kernel calls are asynchronous on `stream` (a cudaStream_t; NULL
 *   is the legacy default stream) and never synchronise the host.
 *   Cache layout. k_cache and v_cache are each
 *   [num_blocks][block_size][num_kv_heads][head_dim], row-major, dense, in the
 *   element type `dtype`. The flat slot of (physical block b, offset o) is
 *   b * block_size + o, i.e. row `slot` of the cache viewed as
 *   [num_blocks * block_size][num_kv_heads][head_dim].
 *   Alignment. Cache, query, output, new-token and workspace pointers must be
 *   16-byte aligned; index arrays naturally aligned.
 *   Errors. Arguments are checked on the host before anything is launched;
 *   a failed check returns PA_ERR_INVALID or PA_ERR_UNSUPPORTED and launches
 *   nothing. A failed launch returns PA_ERR_CUDA. pa_last_error() gives a
 *   one-line reason for the last failure on the calling thread. Indices that
 *   live in device memory (slots, block ids, context lengths, copy pairs) are
 *   checked inside the kernels: a bad one is skipped, never dereferenced, and
 *   sets a bit of the device error word read by pa_device_errors().
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* pa_stream_t; /* identical to cudaStream_t */

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,      /* bad argument; nothing launched, no state changed   */
  PA_ERR_UNSUPPORTED = 2,  /* valid but not built: dtype, head_dim or group size */
  PA_ERR_CUDA = 3,         /* a CUDA runtime call failed                          */
  PA_ERR_NO_BLOCKS = 4,    /* the free pool cannot supply the blocks asked for    */
  PA_ERR_DEVICE_CHECK = 5  /* a kernel found a bad device-side index              */
} pa_status;

/*
 * Element types of a cache. PA_FP8_E4M3: 8-bit E4M3 codes (1 sign, 4 exponent
 * bits with bias 7, 3 mantissa bits, largest finite value 448) with one float32
 * scale per KV head: cache value = decode(code) * scale[head]. "What is paged
 * attention in vLLM, and why does it matter?" (interview.clozo.ai), "Trade-offs
 * and edge cases", fourth point: narrower cache values shrink every block. The
 * pages stop at 16-bit formats; the 8-bit format and its per-head scale are
 * this library's extension. pa_copy_blocks and pa_swap_blocks take
 * PA_FP8_E4M3 as a 1-byte element; writes and decode go through the _fp8
 * entry points below.
 */
typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2 } pa_dtype;

/* Bits of the device error word (pa_device_errors). */
#define PA_DEVERR_SLOT 0x1u       /* pa_kv_append: slot >= num_blocks * block_size       */
#define PA_DEVERR_BLOCK_ID 0x2u   /* pa_decode: table entry outside [0, num_blocks)       */
#define PA_DEVERR_CONTEXT 0x4u    /* pa_decode: context_lens[s] < 0, > max_context_len,
                                     or > max_blocks_per_seq * block_size; pa_prefill:
                                     a bad query_start range or chunk length (below)      */
#define PA_DEVERR_COPY_PAIR 0x8u  /* pa_copy_blocks: src or dst outside [0, num_blocks)  */
#define PA_DEVERR_TIMEOUT 0x10u   /* a bounded wait inside a kernel gave up               */
#define PA_DEVERR_PLAN 0x20u      /* pa_decode_planned: a work item outside the batch, or
                                     a sequence whose partition count differs from the
                                     one its items were planned with; pa_prefill_planned:
                                     an item naming a sequence outside the batch          */

/* ------------------------------------------------------------------ cache writes */

/*
 * pa_kv_append — write new tokens' K and V rows into their cache slots.
 * "Paged Attention" (klaylearn.com glossary), definition: during prefill blocks
 * are filled as prompt tokens produce K and V; during decode a new token is
 * appended into the current tail block. "What is paged attention in vLLM...",
 * Step 4: each decoding step writes the new token's keys and values into the
 * last block.
 *
 *   k_new, v_new   device, [num_tokens][num_kv_heads][head_dim], dtype.
 *   slot_mapping   device, int64 [num_tokens]: flat slot of each row; a
 *                  negative slot skips the row (padding). Slots must be
 *                  distinct; slot >= num_blocks * block_size sets
 *                  PA_DEVERR_SLOT and skips the row.
 *   k_cache, v_cache  device, written in place.
 * dtype PA_F32 or PA_BF16 (PA_FP8_E4M3 caches: pa_kv_append_fp8).
 * Rows are copied bit for bit. num_tokens == 0 is a no-op. Prefill and decode
 * use the same call (num_tokens = prompt tokens, or one per sequence).
 * Requires num_kv_heads * head_dim * element size to be a multiple of 16.
 */
int pa_kv_append(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                 int num_tokens, void* k_cache, void* v_cache, int num_blocks, int block_size,
                 int num_kv_heads, int head_dim, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_kv_append_fp8 — pa_kv_append into an E4M3 cache (PA_FP8_E4M3): each
 * bfloat16 value x of head h is stored as the E4M3 code of x / scale[h]
 * (float32 division, round to nearest, then round to nearest even into E4M3;
 * finite values beyond +-448 saturate to +-448, NaN stays NaN).
 *
 *   k_new, v_new   device, bfloat16 [num_tokens][num_kv_heads][head_dim].
 *   k_scale, v_scale  device, float32 [num_kv_heads], positive and finite.
 *   k_cache, v_cache  device, uint8 codes [num_blocks][block_size][num_kv_heads][head_dim].
 * slot_mapping, padding and error behaviour as pa_kv_append. Requires
 * num_kv_heads * head_dim to be a multiple of 16 and head_dim a multiple of 16.
 */
int pa_kv_append_fp8(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                     int num_tokens, void* k_cache, void* v_cache, const float* k_scale,
                     const float* v_scale, int num_blocks, int block_size, int num_kv_heads,
                     int head_dim, pa_stream_t stream);

/*
 * pa_copy_blocks — copy-on-write of shared blocks: for each pair,
 * block dst := block src, in both caches, bit for bit.
 * "PagedAttention — AI Glossary", How it works 5: when a shared sequence
 * diverges only the block being written is copied; "What is paged attention in
 * vLLM...", "Trade-offs and edge cases", third point.
 *
 *   block_mapping  device, int64 [num_pairs][2] = (src, dst). Sources and
 *                  destinations must be disjoint sets (the copies of one call
 *                  run concurrently). An id outside [0, num_blocks) sets
 *                  PA_DEVERR_COPY_PAIR and the pair is skipped.
 * num_pairs == 0 is a no-op.
 */
int pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping, int num_pairs,
                   int num_blocks, int block_size, int num_kv_heads, int head_dim,
                   pa_dtype dtype, pa_stream_t stream);

/*
 * pa_swap_blocks — copy whole blocks between two pools, either of which may be
 * device memory or page-locked host memory mapped for the device (e.g.
 * cudaHostAlloc / cudaHostRegister; on unified-addressing systems the host
 * pointer itself is used). For each pair: dst block := src block, K and V, bit
 * for bit. This is the data movement of preemption by swapping: "Paged
 * Attention" (klaylearn.com glossary), FAQ (move blocks to CPU memory); "What is
 * paged attention in vLLM...", Follow-up questions (blocks swapped to CPU
 * memory, later swapped back). Choosing between swapping and recomputing is
 * the caller's policy.
 *
 *   dst_k_cache, dst_v_cache  [dst_num_blocks][block_size][num_kv_heads][head_dim]
 *   src_k_cache, src_v_cache  [src_num_blocks][block_size][num_kv_heads][head_dim]
 *   block_mapping  int64 [num_pairs][2] = (src id, dst id), readable by the
 *                  device (device memory or mapped host memory). Destination
 *                  ids must be distinct; an id outside its pool sets
 *                  PA_DEVERR_COPY_PAIR and the pair is skipped.
 * One launch for all pairs; asynchronous on `stream`.
 */
int pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, int dst_num_blocks,
                   const void* src_k_cache, const void* src_v_cache, int src_num_blocks,
                   const int64_t* block_mapping, int num_pairs, int block_size, int num_kv_heads,
                   int head_dim, pa_dtype dtype, pa_stream_t stream);

/* --------------------------------------------------------------- decode attention */

/*
 * pa_decode_partition_size — the partition length (tokens) pa_decode uses when
 * passed partition_size = 0. Chosen from the grid size alone (sequences, KV
 * heads, max_context_len), never from block_size or placement, so results do
 * not depend on either. Always a multiple of 16, between 64 and 768.
 */
int pa_decode_partition_size(int num_seqs, int num_kv_heads, int max_context_len);

/*
 * pa_set_decode_options — options of the decode calls (pa_decode,
 * pa_decode_append, their _fp8 forms and pa_decode_noalloc) made later by the
 * calling host thread, until changed; returns the previous options. A CUDA
 * graph keeps the options its calls were captured with. Not from the pages:
 * a launch-scheduling option of this library.
 *
 *   PA_DECODE_EARLY_CACHE_READS  The decode kernels are launched with
 *     programmatic dependent launch, so they may start while the previous
 *     kernel on the stream drains. Normally they wait for it before reading
 *     anything. With this option they read the context lengths, the block
 *     tables and the cached K/V at once, filling their load pipelines in the
 *     previous kernel's tail, and wait only before reading q (and k_new /
 *     v_new) and before writing anything. Set it only when no kernel that can
 *     still be running when a decode call starts writes that call's cache
 *     blocks, block tables or context lengths: the usual case of a layer loop,
 *     where the kernel before attention produces q and the new K/V rows, and
 *     tables, lengths and copy-on-write copies were set up before the step's
 *     first layer. With the option and a kernel that does write them, the
 *     results are undefined.
 */
#define PA_DECODE_EARLY_CACHE_READS 0x1u
unsigned int pa_set_decode_options(unsigned int options);

/*
 * pa_decode_workspace_bytes — bytes of workspace pa_decode needs for these
 * sizes (0 when no sequence can span more than one partition).
 * partition_size = 0 means the automatic choice.
 */
size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int max_context_len, int partition_size);

/*
 * pa_decode — one decode query per sequence attends over its whole cached
 * context, reading K and V through the block table.
 * "Paged Attention" (klaylearn.com glossary), definition: the kernel computes
 * each token's logical block and offset, looks up the physical block and loads
 * the K/V from it. "PagedAttention — AI Glossary", Example: the attention
 * mathematics is unchanged, so for sequence s and query head j (KV head
 * h = j / (num_heads / num_kv_heads)):
 *     x_t = scale * dot(q[s][j], K_s[t][h]),  t < context_lens[s]
 *     out[s][j] = sum_t softmax(x)_t * V_s[t][h]
 * with K_s[t] the cache row in block block_tables[s][t / block_size] at offset
 * t % block_size. Accumulation is float32.
 *
 *   out            device, [num_seqs][num_heads][head_dim], dtype (bf16 output
 *                  is rounded to nearest even from the float32 result).
 *   q              device, [num_seqs][num_heads][head_dim], dtype.
 *   k_cache, v_cache  device, read only.
 *   block_tables   device, int32 [num_seqs][max_blocks_per_seq]; only the first
 *                  ceil(context_lens[s] / block_size) entries of a row are read.
 *   context_lens   device, int32 [num_seqs]: tokens to attend (after the
 *                  step's append). 0 gives an all-zero output row.
 *   max_context_len  host upper bound of context_lens (sizes the grid without a
 *                  device read); <= max_blocks_per_seq * block_size.
 *   partition_size tokens per split-K partition, a multiple of 16, or 0 for
 *                  pa_decode_partition_size(). A sequence longer than one
 *                  partition is split; partial results (max, sum, unnormalised
 *                  output) go to the workspace and a second kernel combines
 *                  them with a log-sum-exp rescale, in partition order.
 *   workspace      device scratch of at least pa_decode_workspace_bytes(...)
 *                  bytes (may be NULL when that is 0). Contents on entry are
 *                  ignored: it needs no clearing, before the first call or
 *                  between calls of any shape (every value the merge reads is
 *                  written by the same call first). Calls sharing one
 *                  workspace must not overlap on the GPU.
 * Supported: dtype PA_F32 or PA_BF16; head_dim 64 or 128; num_heads /
 * num_kv_heads in {1, 2, 4, 8}; block_size a power of two in [1, 256].
 * The result for a sequence depends only on its logical tokens and on
 * partition_size: physical placement and block_size do not change a bit of it.
 */
int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
              int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
              int max_blocks_per_seq, int max_context_len, float scale, int partition_size,
              void* workspace, size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_append — one whole decode step in one call: append each
 * sequence's newest token, then attend over the context including it.
 * "What is paged attention in vLLM...", Step 4: at each decoding step the
 * system writes the new token's keys and values into the last block;
 * "Paged Attention" (klaylearn.com glossary), definition: decode appends into
 * the tail block. Same result as pa_kv_append (with each new token's slot
 * taken from the block table) followed by pa_decode, without the separate
 * launch: the CTA that reads a sequence's last position writes it first.
 *
 *   k_new, v_new   device, [num_seqs][num_kv_heads][head_dim], dtype: the K
 *                  and V rows of each sequence's newest token, which sits at
 *                  position context_lens[s] - 1 (context_lens counts it). Its
 *                  slot is block_tables[s][(L - 1) / block_size] * block_size
 *                  + (L - 1) % block_size; that block must already be in the
 *                  table and not shared (copy-on-write first, pa_copy_blocks).
 *   k_cache, v_cache  device, the newest rows are written in place.
 * Everything else as pa_decode. A sequence with context_lens[s] == 0 appends
 * nothing. A table entry outside the pool sets PA_DEVERR_BLOCK_ID and the row
 * is not written.
 */
int pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                     void* k_cache, void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                     int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                     int max_context_len, float scale, int partition_size, void* workspace,
                     size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_fp8 — pa_decode over E4M3 caches: K_s[t][h] and V_s[t][h] are the
 * dequantised rows decode(code) * k_scale[h] and decode(code) * v_scale[h]
 * (see PA_FP8_E4M3); the attention arithmetic is pa_decode's.
 *
 *   out, q         device, bfloat16 [num_seqs][num_heads][head_dim].
 *   k_cache, v_cache  device, uint8 E4M3 codes, read only.
 *   k_scale, v_scale  device, float32 [num_kv_heads].
 * Products use float16 operands: E4M3 codes widen to float16 exactly, q is
 * converted from bfloat16 to float16 (exact for magnitudes in [2^-14, 65504];
 * smaller magnitudes lose low bits, larger ones overflow), softmax
 * probabilities are rounded to float16; accumulation is float32.
 * Supported: head_dim 128; num_heads / num_kv_heads in {1, 2, 4, 8};
 * block_size a power of two in [1, 256]. Everything else as pa_decode,
 * including the workspace (pa_decode_workspace_bytes) and the independence of
 * the result from block_size and placement.
 */
int pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                  const float* k_scale, const float* v_scale, const int32_t* block_tables,
                  const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                  int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                  int max_context_len, float scale, int partition_size, void* workspace,
                  size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode_append_fp8 — pa_decode_append over E4M3 caches: each sequence's
 * newest token (k_new / v_new, bfloat16 [num_seqs][num_kv_heads][head_dim]) is
 * quantised exactly as pa_kv_append_fp8 does and written at position
 * context_lens[s] - 1 through the block table, then the step attends as
 * pa_decode_fp8. Conditions on the newest token's block as pa_decode_append.
 */
int pa_decode_append_fp8(void* out, const void* q, const void* k_new, const void* v_new,
                         void* k_cache, void* v_cache, const float* k_scale,
                         const float* v_scale, const int32_t* block_tables,
                         const int32_t* context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks,
                         int max_blocks_per_seq, int max_context_len, float scale,
                         int partition_size, void* workspace, size_t workspace_bytes,
                         pa_stream_t stream);

/*
 * pa_decode_plan — host-side work list for pa_decode_planned.
 * The plain decode grid has one CTA per (partition, sequence) up to
 * max_context_len, so a batch of mixed lengths launches many CTAs that find
 * their partition past their sequence's end and exit; on the GPU each costs
 * about as much scheduling time as a short CTA with work. A serving loop
 * knows every length on the host (its block manager made the tables), so it
 * can list only the (sequence, partition) pairs that hold tokens, in the
 * order that shortens the tail of the grid: whole partitions first, then each
 * sequence's last, shorter one, longest first. "Paged Attention"
 * (klaylearn.com glossary), definition: the kernel reads a sequence's blocks
 * through its table; the split of a context into partitions and the order in
 * which they run change no result.
 *
 *   context_lens   HOST int32 [num_seqs]: the lengths the planned call will
 *                  find in its device context_lens (after the step's append).
 *   partition_size tokens per partition: a multiple of 16 in [16, 2^20], the
 *                  value the planned call is given (pa_decode_partition_size()
 *                  gives the automatic one).
 *   work           HOST int32 [capacity][2], written: item i is
 *                  {sequence, partition | (partitions of that sequence << 16)}.
 *                  A sequence of length L has max(1, ceil(L / partition_size))
 *                  items (an empty sequence one, which writes its zero rows).
 *   capacity       items work can hold; num_seqs * ceil(max length /
 *                  partition_size) (at least num_seqs) always suffices.
 *   num_items      written: the items listed.
 * Returns PA_ERR_INVALID for a null pointer, a negative length or a bad
 * partition_size, PA_ERR_UNSUPPORTED for a sequence of more than 65535
 * partitions, PA_ERR_INVALID when capacity is too small (num_items then holds
 * the capacity needed). No GPU work; thread-safe.
 */
int pa_decode_plan(const int32_t* context_lens, int num_seqs, int partition_size, int32_t* work,
                   int capacity, int* num_items);

/*
 * pa_decode_planned — pa_decode / pa_decode_append / pa_decode_fp8 /
 * pa_decode_append_fp8 on the grid of a pa_decode_plan work list: one CTA per
 * item and group of KV heads, none for partitions past a sequence's end. The
 * arithmetic is that of the unplanned call with the same partition_size, so
 * the results are bit-identical to it. When one wave of resident CTAs holds
 * every item (items x KV-head groups <= CTAs per SM x SMs), the order of the
 * list cannot shorten the tail and the call launches the plain grid instead
 * (which spares each CTA the read of its item); the list is then not read.
 *
 *   k_new, v_new   both NULL (attend only, as pa_decode) or both set (append
 *                  each newest token first, as pa_decode_append).
 *   k_scale, v_scale  E4M3 caches (dtype PA_FP8_E4M3): as pa_decode_fp8; NULL
 *                  for bfloat16 caches.
 *   work           device int32 [num_items][2] (8-byte aligned), as written by
 *                  pa_decode_plan for these context lengths and this
 *                  partition_size; read by the kernel at its start (under
 *                  PA_DECODE_EARLY_CACHE_READS before the dependent-launch
 *                  wait, like the tables).
 *   num_items      in [num_seqs, 65535].
 *   partition_size the plan's, > 0.
 *   dtype          PA_BF16 or PA_FP8_E4M3.
 * Everything else as the unplanned calls, including the workspace
 * (pa_decode_workspace_bytes with this partition_size). Where the list is
 * read: an item naming a sequence outside the batch or a partition past
 * max_context_len sets PA_DEVERR_PLAN and its CTA does nothing; a sequence
 * whose device length needs another number of partitions than its items say
 * sets PA_DEVERR_PLAN (its output is then undefined). A list that omits or
 * repeats items of a sequence while giving the right count is not detected:
 * the output of that sequence is undefined.
 */
int pa_decode_planned(void* out, const void* q, const void* k_new, const void* v_new,
                      void* k_cache, void* v_cache, const float* k_scale, const float* v_scale,
                      const int32_t* block_tables, const int32_t* context_lens,
                      const int32_t* work, int num_items, int num_seqs, int num_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      int max_blocks_per_seq, int max_context_len, float scale,
                      int partition_size, void* workspace, size_t workspace_bytes,
                      pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_shared_prefix — decode attention (optionally with the step's
 * append, as pa_decode_append) for a batch whose sequences all begin with the
 * same prefix_len tokens held in the same physical blocks: block_tables[s][0
 * .. prefix_len / block_size) are equal for every s (sequences forked from a
 * common parent, parallel sampling). "PagedAttention — AI Glossary", How it
 * works, step 4: sharers point at the same blocks; "What is paged attention in
 * vLLM...", Trade-offs and edge cases: prefix sharing. The result is the same
 * softmax attention over each sequence's whole context; only the work is
 * split:
 *   - the prefix: every sequence's query rows of a KV head against the shared
 *     keys at once, on the tcgen05 tensor cores (a dense contraction of
 *     num_seqs * group rows), each prefix block read once per call instead of
 *     once per sequence;
 *   - each sequence's own tokens [prefix_len, context_lens[s]) with the decode
 *     kernel (appending each newest token there when k_new / v_new are given);
 *   - the partial results of both combined per row with a log-sum-exp rescale.
 * Three kernels on `stream`: the prefix pass (a few SMs) and the suffix decode
 * run at the same time, the merge after both. The call waits for all earlier
 * work on the stream before it reads q, k_new or v_new or writes anything, as
 * pa_decode does; PA_DECODE_EARLY_CACHE_READS does not apply to it.
 * partition_size (0: the library's choice) sets the suffix partitions.
 *
 *   k_new, v_new   NULL (attend only) or each sequence's newest K/V row
 *                  [num_seqs][num_kv_heads][head_dim], written at position
 *                  context_lens[s] - 1, which must lie past the prefix.
 *   prefix_len     tokens shared by every sequence, a positive multiple of
 *                  block_size, <= every context_lens[s].
 *   workspace      at least pa_decode_shared_prefix_workspace_bytes(...) bytes;
 *                  contents on entry ignored.
 * Every other argument as pa_decode_append / pa_decode. Supported: bf16,
 * head_dim 128, num_heads / num_kv_heads in {1, 2, 4, 8}, block_size a power
 * of two in [8, 256], scale > 0. A context shorter than prefix_len sets
 * PA_DEVERR_CONTEXT. Within the bf16 tolerance of pa_decode on the same
 * tokens (the order of the sums differs), not bit-identical.
 */
size_t pa_decode_shared_prefix_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                               int head_dim, int prefix_len, int max_context_len,
                                               int partition_size);
int pa_decode_shared_prefix(void* out, const void* q, const void* k_new, const void* v_new,
                            void* k_cache, void* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, int num_seqs, int num_heads,
                            int num_kv_heads, int head_dim, int block_size, int num_blocks,
                            int max_blocks_per_seq, int prefix_len, int max_context_len,
                            float scale, int partition_size, void* workspace,
                            size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_contiguous — the same decode attention over a contiguous cache,
 * with no block table: the baseline that paging is measured against, not part
 * of the paged method. "What is paged attention in vLLM, and why does it
 * matter?", Trade-offs and edge cases, first point: the paged kernel pays for
 * its table reads and irregular accesses with higher attention-kernel latency
 * than a kernel over contiguous per-request caches; Steps 1-2 and
 * "PagedAttention — AI Glossary", Example: such caches reserve one slab per
 * request. Here every sequence owns one slab of slab_len token rows:
 *
 *   k, v           device, [num_seqs][slab_len][num_kv_heads][head_dim], bf16;
 *                  token t of sequence s is row t of slab s.
 *   context_lens   device, int32 [num_seqs]: tokens to attend, <= slab_len.
 *   slab_len       tokens per slab, >= 16.
 * Every other argument as pa_decode (bf16 only: dtype must be PA_BF16). The
 * kernel is pa_decode's tensor-core kernel with the table read removed and one
 * TMA box per 16 tokens; chunks and reduction order are the same, so on the
 * same tokens the output equals pa_decode's bit for bit.
 */
int pa_decode_contiguous(void* out, const void* q, const void* k, const void* v,
                         const int32_t* context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, int slab_len, int max_context_len,
                         float scale, int partition_size, void* workspace,
                         size_t workspace_bytes, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_prefill — causal attention of each sequence's newest chunk of query rows
 * over its paged context (prompt prefill, or chunked prefill on top of an
 * already-cached prefix). "Paged Attention" (klaylearn.com glossary),
 * definition: during prefill blocks are filled as prompt tokens produce K and
 * V, and attention reads the context through the block table; "What is paged
 * attention in vLLM, and why does it matter?", Steps 3-4. The chunk's own K
 * and V must already be in the cache (pa_kv_append). For sequence s with
 * L = context_lens[s] cached tokens and n = query_start[s+1] - query_start[s]
 * query rows, row i is position p = L - n + i and, for query head j
 * (KV head h = j / (num_heads / num_kv_heads)),
 *     out[row][j] = sum_{t <= p} softmax_t(scale * q[row][j] . K_s[t][h]) V_s[t][h]
 * with K_s[t] read through block_tables[s] as in pa_decode.
 *
 *   out, q         device, bf16 [total_q][num_heads][head_dim]; sequence s's
 *                  rows are query_start[s] .. query_start[s+1] - 1.
 *   query_start    device, int32 [num_seqs + 1], non-decreasing, from 0 to at
 *                  most total_q; 0 <= n <= context_lens[s] for every s, else
 *                  PA_DEVERR_CONTEXT is set and that sequence is skipped.
 *   max_query_len  host upper bound of n over the batch (sizes the grid); a
 *                  sequence with n > max_query_len sets PA_DEVERR_CONTEXT and
 *                  is skipped (its rows are not written).
 *   Everything else as pa_decode. Products in bf16 on the tensor cores
 *   (tcgen05), softmax and accumulation in fp32; softmax weights are rounded to
 *   bf16 before the product with V.
 * scale must be finite and > 0. Supported: dtype PA_BF16; head_dim 128;
 * num_heads / num_kv_heads in {1, 2, 4, 8}; block_size a power of two in
 * [8, 256]. The result does not depend on block_size or on the physical
 * placement of the blocks. Work is handed to CTAs longest first (an order
 * over all sequences' items found in the kernel); this affects speed only.
 * The grid has one CTA per KV head and work item of 256 / (num_heads /
 * num_kv_heads) query rows, sized for max_query_len rows per sequence: if
 * num_seqs * ceil(max_query_len / that) * num_kv_heads exceeds 2^31 - 1 the
 * call returns PA_ERR_UNSUPPORTED. num_seqs, total_q or max_query_len 0 is a
 * no-op; a negative one, a null pointer, a misaligned pointer (16 bytes for
 * out, q and the caches, 4 for the int32 arrays), max_query_len > total_q or
 * a scale that is not finite and > 0 returns PA_ERR_INVALID; launch failures
 * return PA_ERR_CUDA.
 */
int pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
               const int32_t* block_tables, const int32_t* context_lens,
               const int32_t* query_start, int num_seqs, int total_q, int num_heads,
               int num_kv_heads, int head_dim, int block_size, int num_blocks,
               int max_blocks_per_seq, int max_query_len, float scale, pa_dtype dtype,
               pa_stream_t stream);

/*
 * pa_prefill_plan — host-side work list for pa_prefill_planned: every work
 * item (two query tiles of one sequence's chunk, counted from the chunk's
 * end) in the order pa_prefill's CTAs find for themselves — most key tiles
 * visited first, ties by sequence, then by item — so that the kernel reads
 * its item instead of searching for it, and the grid has no CTA past the
 * last item. The host knows the chunk and context lengths of a step (the
 * serving loop made them).
 *
 *   query_start    HOST int32 [num_seqs + 1], context_lens HOST int32
 *                  [num_seqs]: the values the planned call's device arrays
 *                  hold.
 *   work           HOST int32 [capacity][2], written: {sequence, item}.
 *   capacity       num_seqs * ceil(max_query_len / (256 / group)) suffices.
 *   num_items      written: the items listed (capacity needed on
 *                  PA_ERR_INVALID for a small capacity).
 * PA_ERR_INVALID for a null pointer, negative rows or more rows than context;
 * PA_ERR_UNSUPPORTED for a group size outside {1, 2, 4, 8}. No GPU work.
 *
 * pa_prefill_planned — pa_prefill on such a list (device int32
 * [num_items][2], 8-byte aligned; num_items in [0, num_seqs *
 * ceil(max_query_len / (256 / group))]). Same results, bit for bit. An item
 * naming a sequence outside the batch sets PA_DEVERR_PLAN and its CTA does
 * nothing; one past its sequence's items does nothing. Everything else as
 * pa_prefill.
 */
int pa_prefill_plan(const int32_t* query_start, const int32_t* context_lens, int num_seqs,
                    int num_heads, int num_kv_heads, int32_t* work, int capacity,
                    int* num_items);
int pa_prefill_planned(void* out, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, const int32_t* context_lens,
                       const int32_t* query_start, const int32_t* work, int num_items,
                       int num_seqs, int total_q, int num_heads, int num_kv_heads, int head_dim,
                       int block_size, int num_blocks, int max_blocks_per_seq,
                       int max_query_len, float scale, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_noalloc — pa_decode for callers that cannot allocate device memory.
 * The pages have no counterpart: this is an interface convenience of this
 * library, not part of the method.
 *
 * Some callers cannot call cudaMalloc where they decode: their framework's
 * memory manager owns the whole device pool, their serving loop must not take
 * an allocation's implicit synchronisation, or they are plain C hosts that
 * only receive pointers to buffers made elsewhere. pa_decode_noalloc takes the
 * same arguments as pa_decode minus the workspace and keeps the split-K
 * partial results in a scratch array compiled into the library:
 *   - The array holds PA_DECODE_NOALLOC_SCRATCH_BYTES (16 MiB) on every GPU
 *     that loads the library, until the process exits.
 *   - A call whose pa_decode_workspace_bytes(...) exceeds that size returns
 *     PA_ERR_INVALID before launching anything (raise partition_size, split
 *     the batch, or use pa_decode with your own workspace).
 *   - The first call in each CUDA context (normally: on each device) looks
 *     up the array's device address (cudaGetSymbolAddress) and caches it for
 *     that context; make that first call before any stream capture. Later
 *     calls in the context do no set-up. A context created later on the same
 *     device (after cudaDeviceReset) gets its own lookup.
 *   - Arguments are checked exactly as pa_decode checks them, before the size
 *     check below: a bad argument is reported as such.
 *   - Nothing here allocates: no cudaMalloc, cudaFree or allocating library
 *     routine.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents. Nothing in it has to start at zero: each call writes every
 *     value it reads back. Calls whose kernels overlap on the GPU (different
 *     streams, or several host threads) race on the array and give wrong
 *     results; serialise them.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                      int num_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                      int partition_size, pa_dtype dtype, pa_stream_t stream);
/* Size of the scratch array behind pa_decode_noalloc, in bytes. */
size_t pa_decode_noalloc_scratch_bytes(void);

/*
 * pa_device_errors — synchronise `stream`, return the device error word
 * (PA_DEVERR_* bits set by kernels since the last call) in *flags and clear
 * it. Returns PA_ERR_DEVICE_CHECK if any bit was set, PA_OK otherwise. The
 * word is per device and shared by all streams.
 */
int pa_device_errors(pa_stream_t stream, unsigned int* flags);

/* One-line reason for the last non-OK return on this thread ("" if none). */
const char* pa_last_error(void);
/* Static name of a pa_status value. */
const char* pa_status_string(int status);

/* ---------------------------------------------------------- host block allocator */
/*
 * The pool of physical blocks: a free list (LIFO stack of ids) and a
 * reference count per block. "What is paged attention in vLLM...", Step 3:
 * the block manager keeps the table beside a pool of free blocks and a
 * reference count per block; Step 4: blocks return to the free pool when the
 * request ends. Host memory only; not thread safe (one owner thread).
 */
typedef struct pa_alloc pa_alloc;

/* New pool of num_blocks free blocks; the first allocations return 0, 1, 2, ...
 * NULL if num_blocks <= 0 or on allocation failure. */
pa_alloc* pa_alloc_create(int num_blocks);
void pa_alloc_destroy(pa_alloc* a);
/* Pop a free block into *out_id with count 1; PA_ERR_NO_BLOCKS if none. */
int pa_alloc_block(pa_alloc* a, int32_t* out_id);
/* Add a reference to an allocated block; PA_ERR_INVALID if out of range or free. */
int pa_incref(pa_alloc* a, int32_t id);
/* Drop a reference; at zero the block goes back on the free list.
 * PA_ERR_INVALID if out of range or already free. */
int pa_decref(pa_alloc* a, int32_t id);
/* Reference count of a block, or -1 if id is out of range. */
int pa_refcount(const pa_alloc* a, int32_t id);
int pa_num_free(const pa_alloc* a);
int pa_num_blocks(const pa_alloc* a);
/* Make the next allocations return ids[0], ids[1], ... ; ids must list every
 * free block exactly once (n == pa_num_free), else PA_ERR_INVALID. */
int pa_alloc_set_free_order(pa_alloc* a, const int32_t* ids, int n);

/* ---------------------------------------------------------- host block manager */
/*
 * Sequences over a pool: per-sequence block tables, allocation on demand,
 * sharing by fork, copy-on-write. Host memory only; not thread safe.
 *   "What is paged attention in vLLM...", Step 4: a new physical block is
 *   allocated only when the last one is full.
 *   "PagedAttention — AI Glossary", How it works 4-5: sequences sharing a
 *   prefix point at the same reference-counted blocks; a shared block is
 *   copied when one sharer writes into it.
 * A call that cannot get host memory returns PA_ERR_INVALID ("out of host
 * memory" in pa_last_error) and changes nothing; no C++ exception leaves the
 * library.
 */
typedef struct pa_bm pa_bm;

/* New manager owning a fresh pool (pa_alloc_create(num_blocks)). block_size > 0. */
pa_bm* pa_bm_create(int num_blocks, int block_size);
void pa_bm_destroy(pa_bm* bm);
/* The manager's pool, for the pa_alloc_* calls (owned by the manager). */
pa_alloc* pa_bm_allocator(pa_bm* bm);
int pa_bm_block_size(const pa_bm* bm);
/* New empty sequence; its id is written to *seq_id. */
int pa_bm_add_seq(pa_bm* bm, int32_t* seq_id);
/* New sequence sharing every block of `parent` (each count + 1) and its length. */
int pa_bm_fork(pa_bm* bm, int32_t parent, int32_t* child);
/* Drop the sequence's references (blocks at count 0 return to the free list);
 * the id becomes invalid. */
int pa_bm_free_seq(pa_bm* bm, int32_t seq_id);
/* Tokens in the sequence, or -1 for an unknown id. */
int pa_bm_seq_len(const pa_bm* bm, int32_t seq_id);
/* Blocks in the sequence's table, or -1 for an unknown id. */
int pa_bm_seq_num_blocks(const pa_bm* bm, int32_t seq_id);
/*
 * pa_bm_append_slots — reserve slots for counts[i] new tokens of sequence
 * seq_ids[i], for i < n, in that order (ids distinct). Writes the flat slot
 * of every new token to slot_mapping (host, int64, sum(counts) entries, in
 * order). When a sequence's first new token falls in a shared, partly filled
 * tail block, a fresh block replaces it in that sequence's table and the pair
 * (old, fresh) is written to cow_pairs (host, int64 [cow_capacity][2]); the
 * caller must run pa_copy_blocks on those pairs before writing the tokens.
 * *num_cow receives the number of pairs. All or nothing: if the pool lacks
 * the blocks, or cow_capacity is too small, returns PA_ERR_NO_BLOCKS /
 * PA_ERR_INVALID and changes nothing.
 */
int pa_bm_append_slots(pa_bm* bm, const int32_t* seq_ids, const int32_t* counts, int n,
                       int64_t* slot_mapping, int64_t* cow_pairs, int cow_capacity,
                       int* num_cow);
/*
 * pa_bm_block_tables — write the block tables of seq_ids[0..n) as rows of
 * `tables` (host, int32 [n][max_blocks_per_seq], unused entries set to 0)
 * and their lengths to context_lens (host, int32 [n]; may be NULL).
 * PA_ERR_INVALID if a sequence holds more than max_blocks_per_seq blocks.
 */
int pa_bm_block_tables(const pa_bm* bm, const int32_t* seq_ids, int n, int32_t* tables,
                       int max_blocks_per_seq, int32_t* context_lens);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
