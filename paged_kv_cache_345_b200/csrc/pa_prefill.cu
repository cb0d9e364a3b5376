// Paged causal prefill attention (chunked prefill) on the 5th-generation tensor
// cores: bf16 Q/K/V, head_dim 128, fp32 accumulation in tensor memory.
//
// What it computes ("Paged Attention", klaylearn.com glossary, definition:
// prefill fills blocks as the prompt produces K and V, and attention reads the
// context through the block table; "What is paged attention in vLLM, and why
// does it matter?", Steps 3-4): sequence s holds L = context_lens[s] tokens in
// the paged cache (the chunk's own K/V included); its n query rows are its last
// n positions, and row i (position p = L - n + i) attends keys t <= p with
// softmax(scale * q . k) weights, query head j reading KV head j / G.
//
// Layout and pipeline (one CTA = one KV head x 128 query rows x one sequence):
//  * The 128 rows are 128 / G tokens x the G query heads of the KV head
//    (row = token * G + g), so every K/V tile is loaded once for the group.
//  * Warp 0 (producer): TMA loads Q once, then per tile of 128 keys one box
//    per cache block {64 columns, min(block_size, 128) tokens} for each half of
//    head_dim, for K and for V, into a 2-stage ring. Boxes use the 128-byte
//    swizzle, which is the shared-memory operand layout of the MMA.
//  * Warp 1 (MMA): one thread issues tcgen05.mma. S_j = Q K_j^T (M 128, N 128,
//    K 128) goes to one of two tensor-memory buffers, so S_{j+1} runs while the
//    softmax warps read S_j; O += P_j V_j accumulates in tensor memory (V is
//    the MN-major operand, P the K-major one). Completion is signalled to
//    mbarriers with tcgen05.commit.
//  * Warps 2-5 (softmax): thread = row (tensor-memory lane). Per tile: load the
//    row of S, scale by scale * log2(e), mask keys past the row's position,
//    online softmax in base 2, write P (bf16) into shared memory in the swizzled
//    K-major layout, and when the row maximum grew rescale the row of O in
//    tensor memory (after the previous P V finished). The end divides by the
//    row sum and stores bf16.
//  * Results depend only on the logical key tiles, so they are bit-identical
//    across block sizes and placements.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tc.cuh"

namespace pa {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

struct PrefillParams {
  __nv_bfloat16* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;
  unsigned* err;
  int num_heads, num_kv_heads, block_size, log2_block_size, num_blocks, max_blocks_per_seq;
  int total_q;
  float q_scale;  // scale * log2(e)
};

template <int G>
struct PrefillConfig {
  static constexpr int kRows = 128;             // query rows per CTA (MMA M)
  static constexpr int kKeys = 128;             // keys per tile (MMA N of S, K of P V)
  static constexpr int kD = 128;                // head_dim
  static constexpr int kTok = kRows / G;        // query tokens per CTA
  static constexpr int kTile = kRows * kD * 2;  // one bf16 128 x 128 operand: 32 KB
  static constexpr int kHalf = kTile / 2;       // 64 columns of it: 16 KB
  static constexpr int kQ = 0, kP = kTile, kStage0 = 2 * kTile;
  static constexpr int kNS = 2;                 // K/V stages
  static constexpr int kBars = kStage0 + kNS * 2 * kTile;
  static constexpr int kSmemBytes = kBars + 256 + 1024;  // + 1024-byte alignment slack
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 512;    // S0, S1, O (128 columns each)
  static_assert(kRows % G == 0, "group must divide the row tile");
};

// mbarrier slots
enum : int { kQFull = 0, kKVFull = 1, kKVEmpty = 3, kSFull = 5, kPFull = 7, kODone = 8 };

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

template <int G>
__global__ void __launch_bounds__(PrefillConfig<G>::kThreads, 1)
    pa_prefill_kernel(const __grid_constant__ CUtensorMap q_map,
                      const __grid_constant__ CUtensorMap k_map,
                      const __grid_constant__ CUtensorMap v_map, const PrefillParams p) {
  using Cfg = PrefillConfig<G>;
  constexpr int TOK = Cfg::kTok, HALF = Cfg::kHalf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::kBars + 128);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const uint32_t q_s = smem_u32(sm + Cfg::kQ), p_s = smem_u32(sm + Cfg::kP);
  auto k_s = [&](int st) { return smem_u32(sm + Cfg::kStage0 + st * 2 * Cfg::kTile); };
  auto v_s = [&](int st) { return k_s(st) + Cfg::kTile; };

  const int h = blockIdx.x, qt = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bs = p.block_size, lg = p.log2_block_size;
  // every lane polls; the warp proceeds only if all saw the phase complete
  auto wait_all = [&](uint32_t b, uint32_t parity) {
    return __all_sync(kFullMask, mbar_wait(b, parity, p.err));
  };

  pdl_wait();  // inputs may come from the previous kernel in the stream
  pdl_launch_dependents();

  const int q0 = __ldg(p.query_start + s), q1 = __ldg(p.query_start + s + 1);
  const int L = __ldg(p.context_lens + s);
  const int n = q1 - q0;
  if (q0 < 0 || q1 > p.total_q || n < 0 || L < n ||
      static_cast<int64_t>(L) > static_cast<int64_t>(p.max_blocks_per_seq) * bs) {
    if (threadIdx.x == 0 && h == 0 && qt == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);
    return;
  }
  const int tq0 = qt * TOK;
  if (tq0 >= n) return;                      // no rows of this sequence in the tile
  const int ntok = min(TOK, n - tq0);        // valid query tokens in the tile
  const int pos0 = L - n + tq0;              // position of the tile's first token
  const int pos_last = pos0 + ntok - 1;      // <= L - 1
  const int nt = pos_last / Cfg::kKeys + 1;  // key tiles to visit
  const int32_t* trow = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;

  if (threadIdx.x == 0) {
    mbar_init(bar(kQFull), 1);
    for (int i = 0; i < Cfg::kNS; ++i) {
      mbar_init(bar(kKVFull + i), 1);   // producer arrival + TMA bytes
      mbar_init(bar(kKVEmpty + i), 1);  // MMA commit after P V of the tile
      mbar_init(bar(kSFull + i), 1);    // MMA commit after S of the tile
    }
    mbar_init(bar(kPFull), 128);        // every softmax thread
    mbar_init(bar(kODone), 1);          // MMA commit after P V
    fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_o = tmem + 256;  // O columns; S buffers at columns 0 and 128

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      mbar_arrive_expect_tx(bar(kQFull), Cfg::kTile);
      tma_load_3d(q_s, &q_map, 0, h * G, q0 + tq0, bar(kQFull));
      tma_load_3d(q_s + HALF, &q_map, 64, h * G, q0 + tq0, bar(kQFull));
    }
    const int rows = bs < Cfg::kKeys ? bs : Cfg::kKeys;  // tokens per box
    for (int j = 0; j < nt; ++j) {
      const int st = j & 1, u = j >> 1;
      if (u >= 1) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(bar(kKVEmpty + st), (u - 1) & 1, p.err);
        if (!__shfl_sync(kFullMask, ok, 0)) break;
      }
      const int key0 = j * Cfg::kKeys;
      const int nkeys = min(Cfg::kKeys, L - key0);
      const int nbox = (nkeys + rows - 1) / rows;  // boxes holding this tile's keys (<= 16)
      int blk = 0;
      if (lane < nbox) blk = __ldg(trow + ((key0 + lane * rows) >> lg));
      if (lane == 0)
        mbar_arrive_expect_tx(bar(kKVFull + st), static_cast<uint32_t>(nbox * rows * 128 * 4));
      __syncwarp();
      if (lane < nbox) {
        // an id outside the pool is flagged; TMA reads an out-of-range box as zeros
        if (static_cast<unsigned>(blk) >= static_cast<unsigned>(p.num_blocks))
          atomicOr(p.err, PA_DEVERR_BLOCK_ID);
        const int off = (key0 + lane * rows) & (bs - 1);
        const uint32_t dk = k_s(st) + lane * rows * 128, dv = v_s(st) + lane * rows * 128;
        tma_load_4d(dk, &k_map, 0, off, h, blk, bar(kKVFull + st));
        tma_load_4d(dk + HALF, &k_map, 64, off, h, blk, bar(kKVFull + st));
        tma_load_4d(dv, &v_map, 0, off, h, blk, bar(kKVFull + st));
        tma_load_4d(dv + HALF, &v_map, 64, off, h, blk, bar(kKVFull + st));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    constexpr uint32_t kIdS = tc::idesc_bf16_f32(128, 128, 0);   // B = K rows (K-major)
    constexpr uint32_t kIdPV = tc::idesc_bf16_f32(128, 128, 1);  // B = V rows (MN-major)
    auto issue_s = [&](int j) {
      const uint32_t kb = k_s(j & 1), d = tmem + (j & 1) * 128;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks >> 2) * HALF + (ks & 3) * 32;
        tc::mma_bf16(d, tc::smem_desc_sw128(q_s + off, 16, 1024),
                     tc::smem_desc_sw128(kb + off, 16, 1024), kIdS, ks > 0);
      }
      tc::commit(bar(kSFull + (j & 1)));
    };
    const bool ok = wait_all(bar(kQFull), 0) && wait_all(bar(kKVFull), 0);
    if (ok) {
      tc::fence_after_sync();
      if (lane == 0) issue_s(0);
      for (int j = 0; j < nt; ++j) {
        if (j + 1 < nt) {
          if (!wait_all(bar(kKVFull + ((j + 1) & 1)), ((j + 1) >> 1) & 1)) break;
          tc::fence_after_sync();
          if (lane == 0) issue_s(j + 1);
        }
        if (!wait_all(bar(kPFull), j & 1)) break;
        tc::fence_after_sync();
        if (lane == 0) {
          const uint32_t vb = v_s(j & 1);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_bf16(t_o, tc::smem_desc_sw128(p_s + (ks >> 2) * HALF + (ks & 3) * 32, 16, 1024),
                         tc::smem_desc_sw128(vb + ks * 2048, HALF, 1024), kIdPV, j > 0 || ks > 0);
          tc::commit(bar(kODone));
          tc::commit(bar(kKVEmpty + (j & 1)));
        }
        __syncwarp();
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int wq = warp & 3;  // this warp reaches tensor-memory lanes 32 wq .. 32 wq + 31
    const int r = wq * 32 + lane;
    const int tok = r / G, g = r - (r / G) * G;
    const int prow = tok < ntok ? pos0 + tok : pos_last;  // last visible key of this row
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float qs = p.q_scale;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      if (!wait_all(bar(kSFull + (j & 1)), (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::ld32(tmem + (j & 1) * 128 + lane_off + c * 32, sv[c]);
      tc::wait_ld();
      const int lim = prow - j * Cfg::kKeys;  // keys 0 .. lim of this tile are visible
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = c * 32 + i <= lim ? __uint_as_float(sv[c][i]) * qs : -INFINITY;
          sv[c][i] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      const float m_new = fmaxf(m_run, mx);  // finite: key 0 is visible to every row
      const float alpha = exp2f(m_run - m_new);
      // the previous P V must be done before P is rewritten or O rescaled
      if (j > 0) {
        if (!wait_all(bar(kODone), (j - 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (__any_sync(kFullMask, alpha != 1.0f)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t ov[32];
            tc::ld32(t_o + lane_off + c * 32, ov);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tc::st32(t_o + lane_off + c * 32, ov);
          }
          tc::wait_st();
        }
      }
      // P = 2^(x - m) as bf16 into the swizzled K-major tile: 16-byte chunk cc of
      // row r in half hh sits at hh * 16 KB + r * 128 + ((cc ^ (r % 8)) * 16)
      float rs = 0.0f;
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i0 = c8 * 8 + 2 * e;
          const float a = exp2f(__uint_as_float(sv[i0 >> 5][i0 & 31]) - m_new);
          const float b = exp2f(__uint_as_float(sv[(i0 + 1) >> 5][(i0 + 1) & 31]) - m_new);
          rs += a + b;
          w[e] = pack_bf16x2(a, b);
        }
        const uint32_t addr = p_s + (c8 >> 3) * HALF + r * 128 + (((c8 & 7) ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]),
                     "r"(w[2]), "r"(w[3])
                     : "memory");
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
      if (j == nt - 1) {
        // keys past the context in the last tile: stale or unwritten V rows become
        // zeros (their P is 0, but 0 * NaN would not be)
        const int nkeys = L - j * Cfg::kKeys;
        if (nkeys < Cfg::kKeys) {
          const uint32_t vb = v_s(j & 1);
          for (int i = r; i < (Cfg::kKeys - nkeys) * 16; i += 128) {
            const int row = nkeys + (i >> 4), c = i & 15;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                             vb + (c >> 3) * HALF + row * 128 + ((c & 7) << 4)),
                         "r"(0u)
                         : "memory");
          }
        }
      }
      // generic-proxy writes (P, zeroed V) before the MMA's async-proxy reads
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc::fence_before_sync();
      mbar_arrive(bar(kPFull));
    }
    if (ok && wait_all(bar(kODone), (nt - 1) & 1)) {
      tc::fence_after_sync();
      const float inv = 1.0f / l_run;
      __nv_bfloat16* dst = p.out + ((static_cast<int64_t>(q0) + tq0 + tok) * p.num_heads +
                                    h * G + g) * Cfg::kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tc::ld32(t_o + lane_off + c * 32, ov);
        tc::wait_ld();
        if (tok < ntok) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 x;
            x.x = pack_bf16x2(__uint_as_float(ov[8 * v]) * inv, __uint_as_float(ov[8 * v + 1]) * inv);
            x.y = pack_bf16x2(__uint_as_float(ov[8 * v + 2]) * inv, __uint_as_float(ov[8 * v + 3]) * inv);
            x.z = pack_bf16x2(__uint_as_float(ov[8 * v + 4]) * inv, __uint_as_float(ov[8 * v + 5]) * inv);
            x.w = pack_bf16x2(__uint_as_float(ov[8 * v + 6]) * inv, __uint_as_float(ov[8 * v + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + c * 32 + v * 8) = x;
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, Cfg::kTmemCols);
}

cudaError_t encode_q_map(CUtensorMap* map, const void* q, int total_q, int num_heads, int box_heads,
                         int box_tokens) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(num_heads),
                              static_cast<cuuint64_t>(total_q)};
  const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(num_heads) * 256};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_heads),
                             static_cast<cuuint32_t>(box_tokens)};
  const cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Cache [num_blocks][block_size][Hkv][128] viewed (column, token, head, block);
// a box is 64 columns x `rows` tokens of one head of one block, 128-byte swizzled.
cudaError_t encode_kv_map(CUtensorMap* map, const void* base, int num_blocks, int block_size,
                          int num_kv_heads, int rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t row = 256;
  const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(block_size),
                              static_cast<cuuint64_t>(num_kv_heads),
                              static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[3] = {row * num_kv_heads, row,
                                 row * num_kv_heads * static_cast<cuuint64_t>(block_size)};
  const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(rows), 1, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                   strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int G>
cudaError_t launch_prefill_g(const PrefillShape& sh, const PrefillParams& p, const void* q,
                             const void* k_cache, const void* v_cache, cudaStream_t stream) {
  using Cfg = PrefillConfig<G>;
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev % 64);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(pa_prefill_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  CUtensorMap qmap, kmap, vmap;
  const int rows = sh.block_size < Cfg::kKeys ? sh.block_size : Cfg::kKeys;
  if ((e = encode_q_map(&qmap, q, sh.total_q, sh.num_heads, G, Cfg::kTok)) != cudaSuccess) return e;
  if ((e = encode_kv_map(&kmap, k_cache, sh.num_blocks, sh.block_size, sh.num_kv_heads, rows)) !=
      cudaSuccess)
    return e;
  if ((e = encode_kv_map(&vmap, v_cache, sh.num_blocks, sh.block_size, sh.num_kv_heads, rows)) !=
      cudaSuccess)
    return e;
  const unsigned tiles = static_cast<unsigned>((sh.max_query_len + Cfg::kTok - 1) / Cfg::kTok);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sh.num_kv_heads), tiles, static_cast<unsigned>(sh.num_seqs));
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa_prefill_kernel<G>, qmap, kmap, vmap, p);
}

}  // namespace

cudaError_t launch_prefill(const PrefillShape& sh, void* out, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, const int32_t* query_start,
                           cudaStream_t stream) {
  if (sh.max_query_len <= 0 || sh.num_seqs <= 0) return cudaSuccess;
  PrefillParams p{};
  p.out = static_cast<__nv_bfloat16*>(out);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start = query_start;
  cudaError_t e = device_error_word(&p.err);
  if (e != cudaSuccess) return e;
  p.num_heads = sh.num_heads;
  p.num_kv_heads = sh.num_kv_heads;
  p.block_size = sh.block_size;
  int lg = 0;
  while ((1 << lg) < sh.block_size) ++lg;
  p.log2_block_size = lg;
  p.num_blocks = sh.num_blocks;
  p.max_blocks_per_seq = sh.max_blocks_per_seq;
  p.total_q = sh.total_q;
  p.q_scale = sh.scale * 1.4426950408889634f;  // log2(e)
  switch (sh.num_heads / sh.num_kv_heads) {
    case 1: return launch_prefill_g<1>(sh, p, q, k_cache, v_cache, stream);
    case 2: return launch_prefill_g<2>(sh, p, q, k_cache, v_cache, stream);
    case 4: return launch_prefill_g<4>(sh, p, q, k_cache, v_cache, stream);
    case 8: return launch_prefill_g<8>(sh, p, q, k_cache, v_cache, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace pa
