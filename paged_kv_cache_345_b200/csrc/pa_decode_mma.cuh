// Paged decode attention, bfloat16 cache, tensor-core inner products (sm_100a).
//
// Computes the same thing as pa_decode_kernel ("Paged Attention", klaylearn.com
// glossary, definition; "PagedAttention — AI Glossary", Example: the block
// table changes where K/V are read from, not the attention arithmetic).
//
// Why tensor cores in an HBM-bound kernel: on CUDA cores every token row costs
// 2 * G * head_dim fp32 FMAs plus cross-lane reductions, ~90 warp instructions
// per (token, KV head), about the whole issue budget an SM has per (token, KV
// head) at its share of HBM bandwidth. The G query heads of a GQA group
// against 16 K rows are a small dense contraction (G x head_dim x 16): one
// m16n8k16 MMA covers 8 x 16 x 8 of it with the group's heads as the M rows
// (zero-padded), which leaves ~8 warp instructions per (token, KV head).
//
// Why whole-block TMA boxes: measured on B200, TMA boxes of one KV head's
// 256-byte rows (16 rows per box) reach ~3 TB/s with one CTA per SM and need
// four CTAs per SM to approach the HBM roofline; one box covering a group of
// KV heads of a block (kilobytes contiguous per token) reaches ~7 TB/s with one.
//
// Layout and pipeline:
//  * CTA = (group of HB KV heads, partition, sequence): HB consumer warps (one
//    per KV head) + 1 producer warp.
//  * The producer reads the block table 32 entries at a time (one coalesced
//    load, shuffled out) and, per chunk of 16 tokens, issues one TMA box per
//    block for K and one for V: {head_dim + 8 columns, min(block_size, 16)
//    tokens, HB heads}. The 8 columns past head_dim lie outside the tensor and
//    arrive as zeros, so every row lands at a padded stride of head_dim * 2 +
//    16 bytes and ldmatrix reads of 8 consecutive rows hit 8 bank groups.
//    The tensor map orders the dimensions (column, token, head, block), so a
//    box lands as [head][token][row].
//  * Stages form a ring of NS; a stage is released once all HB warps read it.
//  * Consumer warp per chunk: S = Q K^T with m16n8k16 (A = Q rows of the
//    group, B = K rows via ldmatrix), online softmax in base 2 on the
//    accumulator fragments (row max / sum over the 4-lane quad; the reference
//    maximum moves only when a chunk exceeds it by 2^8), P converted to
//    bfloat16 in registers becomes the A operand of O += P V (B = V rows via
//    ldmatrix.trans). m, l and O stay in registers.
//  * End: a single-partition sequence writes `out`; otherwise (m, l, O) go to
//    the split-K workspace and pa_merge_kernel (launched right behind, with
//    programmatic dependent launch) combines the partitions.
//  * Chunks hold the same 16 logical tokens and are reduced in the same order
//    whatever the block size or placement, so results are bit-identical across
//    both.
//
// E4M3 (fp8) caches (FP8 = true, head_dim 128): the same pipeline moves rows
// of head_dim bytes (+16 zero bytes of padding, again from out-of-range box
// columns). No 8-bit ldmatrix transpose is used; each lane instead reads its
// operand bytes with 16-byte shared loads and widens them in registers
// (E4M3 -> float16 is exact), and the stage is released as soon as the loads
// are done. The inner products use float16 MMAs:
//  * S^T: lane (g, t) loads the 16-byte columns 2t and 2t+1 of token rows g
//    and g+8. The contraction index is permuted (the same permutation for K
//    and for Q, which is loaded to match), so each loaded 32-bit word becomes
//    the a0/a2 (row g) or a1/a3 (row g+8) register of one k-step directly.
//  * O^T: lane (g, t) loads column g (head_dim values 16g .. 16g+15) of token
//    rows 2t, 2t+1, 2t+8, 2t+9; a byte permute pairs the two tokens of each
//    A register. MMA row r of tile dt stands for head_dim index 16g + 2dt (+1
//    for r = g + 8), which the epilogue maps back.
//  * With a padded row stride of 144 bytes both load patterns touch 8
//    distinct 16-byte bank groups per quarter warp.
//  * Scores are scaled by scale * log2(e) * k_scale[head], the output by
//    v_scale[head].
#pragma once

#include <cmath>
#include <cstdint>

#include "pa_decode.cuh"
#include "pa_device.cuh"

namespace pa {

template <int D, int G, int HB, int NS, bool FP8 = false>
struct GroupConfig {
  static constexpr int kC = 16;                       // tokens per chunk / stage
  static constexpr int kRowBytes = FP8 ? D : D * 2;
  static constexpr int kRS = kRowBytes + 16;          // padded row stride in shared memory
  // One chunk of K (or V) for the group: up to 16 boxes (block_size 1) of HB
  // rows each, every box padded to a 128-byte boundary; fewer, larger boxes
  // (block_size 2..16+) always fit in the same space.
  static constexpr int kTensorBytes = kC * ((HB * kRS + 127) & ~127);
  static constexpr int kStageBytes = 2 * kTensorBytes;
  static constexpr int kThreads = (HB + 1) * 32;
  static constexpr int kRingBytes = NS * kStageBytes;
  static constexpr int kBarBytes = 2 * NS * 8;
  static constexpr int kSmemBytes = 128 + kRingBytes + kBarBytes;
  static_assert(G >= 1 && G <= 8, "group must fit the 8 real rows of an m16 tile");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
  static_assert(!FP8 || D == 128, "the E4M3 operand layout is built for head_dim 128");
};

// Bytes between consecutive TMA boxes of one chunk (rows_per_box tokens of HB
// heads each), rounded up so every box starts 128-byte aligned.
__host__ __device__ constexpr int box_stride_bytes(int hb, int rows_per_box, int rs) {
  return (hb * rows_per_box * rs + 127) & ~127;
}

// TABLE = false: the table-free variant over a contiguous cache
// [num_seqs][slab_len][num_kv_heads][head_dim] (each sequence's K/V in one
// slab, token t at row t): the same pipeline and arithmetic, but no block-table
// read, and every chunk of 16 tokens is one box at (token t, sequence s). The
// tensor map describes the slab as a "block" of slab_len tokens per sequence.
template <int D, int G, int HB, int NS, bool FP8, bool TABLE = true>
__global__ void __launch_bounds__(GroupConfig<D, G, HB, NS, FP8>::kThreads)
    pa_decode_mma_kernel(const __grid_constant__ CUtensorMap k_map,
                         const __grid_constant__ CUtensorMap v_map, const DecodeParams p) {
  using Cfg = GroupConfig<D, G, HB, NS, FP8>;
  constexpr int C = Cfg::kC, RS = Cfg::kRS, TB = Cfg::kTensorBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kRingBytes);  // full[NS], empty[NS]

  const int hg = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = p.partition_size, bs = p.block_size, lg = p.log2_block_size;
  const int rows_per_box = (!TABLE || bs >= C) ? C : bs;
  const int box_stride = box_stride_bytes(HB, rows_per_box, RS);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(bars + i), 1);        // full: producer arrive + TMA bytes
      mbar_init(smem_u32(bars + NS + i), HB);  // empty: every consumer warp releases
    }
    fence_barrier_init();
  }
  if (warp == HB && lane == 0) {  // descriptors are kernel parameters: fetch them early
    prefetch_tensormap(&k_map);
    prefetch_tensormap(&v_map);
  }
  // Inputs may come from the previous kernel in the stream. Normally every
  // thread waits for it here. Under PA_DECODE_EARLY_CACHE_READS the context
  // length, the block table and the cached K/V are read at once and the first
  // ring stages fill while that kernel drains; the waits then come right
  // before q (consumers), before the fused append reads k_new / v_new
  // (producer), and before any write.
  //
  // A shared-prefix decode (prefix_slots > 0) runs beside the prefix kernel
  // launched just before it, which waited for all earlier work before letting
  // this grid start and reads neither the rows this kernel writes nor their
  // workspace slots: no thread here waits, q and k_new / v_new are read
  // through L2, and one thread of the grid (gate) waits for the prefix kernel
  // before its CTA ends, so that the merge, which waits for this grid, also
  // finds the prefix's partial results.
  const bool early = p.early_reads != 0;
  const bool cascade = p.prefix_slots > 0;
  const bool gate = cascade && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
  if (!early && !cascade) pdl_wait();
  pdl_launch_dependents();

  // grid (head group, partition, sequence); E4M3: (head group, sequence,
  // partition) with the highest partition first, so that the long sequences'
  // full later partitions start before the many short first ones (the E4M3
  // kernel's CTAs are slower per byte, and its tail was the longer).
  // Planned calls: grid (head group, work item), item y = (sequence, partition
  // | partitions of that sequence << 16), longest items first, no empty CTAs.
  int part = FP8 ? static_cast<int>(gridDim.z - 1 - blockIdx.z) : static_cast<int>(blockIdx.y);
  int s = FP8 ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.z);
  int planned_parts = 0;
  if (p.work != nullptr) {
    const int2 it = __ldg(reinterpret_cast<const int2*>(p.work) + blockIdx.y);
    s = it.x;
    part = it.y & 0xffff;
    planned_parts = static_cast<int>(static_cast<unsigned>(it.y) >> 16);
    if (static_cast<unsigned>(s) >= static_cast<unsigned>(p.num_seqs) ||
        part >= p.num_partitions - p.prefix_slots) {
      if (threadIdx.x == 0) atomicOr(p.err, PA_DEVERR_PLAN);
      return;
    }
  }

  // Independent loads first so their latencies overlap: the context length,
  // the first 32 block-table entries of this partition (producer warp) and
  // (without early reads) the query fragments (consumer warps).
  int L = __ldg(p.context_lens + s);
  const int t0 = part * P;
  // (shared-prefix decode: the table from the first block after the prefix)
  const int32_t* trow = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq +
                        (p.first_token >> lg);
  int base = t0 >> lg, ent = 0;
  if (TABLE && warp == HB && base + lane < p.max_blocks_per_seq - (p.first_token >> lg))
    ent = __ldg(trow + base + lane);
  const int kvh = hg * HB + (warp < HB ? warp : 0);  // this consumer warp's KV head
  const int qr = lane >> 2;  // fragment row: query head of the group (rows >= G are padding)
  const int qc = lane & 3;   // fragment column pair
  const bool real_row = qr < G;
  const int64_t out_row = static_cast<int64_t>(s) * p.num_heads + kvh * G;
  uint32_t qa[D / 16][2];  // Q as the B operand (column = head of the group), 16-bit pairs
  auto load_q = [&]() {
    const uint32_t* qp = reinterpret_cast<const uint32_t*>(
        static_cast<const __nv_bfloat16*>(p.q) + (out_row + (real_row ? qr : 0)) * D);
    if constexpr (!FP8) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        qa[ks][0] = real_row ? (cascade ? __ldcg(qp + ks * 8 + qc) : __ldg(qp + ks * 8 + qc)) : 0u;
        qa[ks][1] = real_row ? (cascade ? __ldcg(qp + ks * 8 + 4 + qc) : __ldg(qp + ks * 8 + 4 + qc))
                             : 0u;
      }
    } else {
      // k-step 4kq + j covers head_dim 16 (2 qc + kq) + 4j .. +3 (b0: +0, +1; b1: +2, +3),
      // the order in which the K loads below deliver them; float16 pairs.
#pragma unroll
      for (int kq = 0; kq < D / 64; ++kq) {
        const uint4* q4 = reinterpret_cast<const uint4*>(qp) + 2 * (2 * qc + kq);
        const uint4 lo = real_row ? (cascade ? __ldcg(q4) : __ldg(q4)) : make_uint4(0, 0, 0, 0);
        const uint4 hi = real_row ? (cascade ? __ldcg(q4 + 1) : __ldg(q4 + 1)) : make_uint4(0, 0, 0, 0);
        const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          qa[4 * kq + j][0] = bf16x2_to_f16x2(w[2 * j]);
          qa[4 * kq + j][1] = bf16x2_to_f16x2(w[2 * j + 1]);
        }
      }
    }
  };
  // q may be the previous kernel's output: loaded here when everyone has
  // waited; under early reads only after the CTA barrier below, so that the
  // producer, which does not wait before its first loads, is never held back
  // by consumers that do
  const bool q_late = early && !cascade;
  if (warp < HB && !q_late) load_q();

  if (L < 0 || L > p.max_context_len ||
      static_cast<int64_t>(L) > static_cast<int64_t>(p.max_blocks_per_seq) * bs ||
      L < p.first_token) {
    if (threadIdx.x == 0 && hg == 0 && part == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);
    L = p.first_token;
  }
  L -= p.first_token;  // the tokens this kernel attends (all of them without a prefix)
  const int n_part_s = (L + P - 1) / P;
  if (p.work != nullptr && planned_parts != max(n_part_s, 1)) {
    // the plan was made for another length of this sequence: flagged, and
    // the CTA still attends what the real length asks of this partition
    if (threadIdx.x == 0) atomicOr(p.err, PA_DEVERR_PLAN);
  }
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  const bool to_merge = cascade;  // every row is left to the merge

  if (L == 0) {  // empty context: zeros for every query head of the group
    if (to_merge) {  // the prefix's partial results are the whole row
      // (a newest token to append would lie inside the shared prefix)
      if (p.k_new != nullptr && threadIdx.x == 0 && hg == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);
      if (gate && threadIdx.x == 0) pdl_wait();
      return;
    }
    if (early) pdl_wait();
    if (part == 0) {
      const int64_t first = static_cast<int64_t>(s) * p.num_heads + hg * HB * G;
      for (int e = threadIdx.x; e < HB * G * D; e += blockDim.x)
        out[first * D + e] = __float2bfloat16_rn(0.0f);
    }
    return;
  }
  if (t0 >= L) {
    if (gate && threadIdx.x == 0) pdl_wait();
    return;
  }
  const int t1 = min(t0 + P, L);
  const int nchunks = (t1 - t0 + C - 1) / C;
  __syncthreads();
  if (warp < HB && q_late) {
    pdl_wait();
    load_q();
  }

  if (warp == HB) {
    // ------------------------------------------------------------- producer
    const int lb_last = (t1 - 1) >> lg;
    for (int c = 0; c < nchunks; ++c) {
      const int st = c % NS, u = c / NS;
      if (u >= 1) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(smem_u32(bars + NS + st), (u - 1) & 1, p.err);
        if (!__shfl_sync(kFullMask, ok, 0)) break;
      }
      const int t = t0 + c * C;
      const int nvalid = min(C, t1 - t);
      if constexpr (!TABLE) {
        // table-free: one box of 16 token rows of this sequence's slab
        const uint32_t full_bar = smem_u32(bars + st);
        const uint32_t kdst = smem_u32(smem + st * Cfg::kStageBytes);
        if (lane == 0) {
          mbar_arrive_expect_tx(full_bar, 2u * HB * C * RS);
          tma_load_4d(kdst, &k_map, 0, t, hg * HB, s, full_bar);
          tma_load_4d(kdst + TB, &v_map, 0, t, hg * HB, s, full_bar);
        }
        continue;
      }
      const int lb_lo = t >> lg, lb_hi = (t + nvalid - 1) >> lg;
      if (lb_hi - base >= 32) {  // refill: the next 32 table entries, one per lane
        base = lb_lo;
        ent = (base + lane <= lb_last) ? __ldg(trow + base + lane) : 0;
      }
      if (p.k_new != nullptr && c == nchunks - 1 && t1 == L) {
        // this CTA holds the sequence's newest token: write it before reading it
        const int tn = L - 1;
        const int bn = __shfl_sync(kFullMask, ent, (tn >> lg) - base);
        if (q_late) pdl_wait();  // k_new / v_new come from the previous kernel
        if (static_cast<unsigned>(bn) < static_cast<unsigned>(p.num_blocks)) {
          if constexpr (FP8)
            append_newest_rows_fp8(p, s, bn, tn & (bs - 1), hg * HB, HB, D, lane);
          else
            append_newest_rows(p, s, bn, tn & (bs - 1), hg * HB, HB, Cfg::kRowBytes, lane);
        } else if (lane == 0)
          atomicOr(p.err, PA_DEVERR_BLOCK_ID);
      }
      const int nbox = lb_hi - lb_lo + 1;  // blocks holding valid tokens of this chunk
      const int blk = __shfl_sync(kFullMask, ent, min(lane, nbox - 1) + lb_lo - base);
      const uint32_t full_bar = smem_u32(bars + st);
      const uint32_t kdst = smem_u32(smem + st * Cfg::kStageBytes);
      if (lane == 0) mbar_arrive_expect_tx(full_bar, 2u * nbox * HB * rows_per_box * RS);
      __syncwarp();
      if (lane < nbox) {
        // an id outside the pool is flagged; TMA reads an out-of-range box as zeros
        if (static_cast<unsigned>(blk) >= static_cast<unsigned>(p.num_blocks))
          atomicOr(p.err, PA_DEVERR_BLOCK_ID);
        const int off = bs < C ? 0 : (t & (bs - 1));
        const uint32_t d = kdst + lane * box_stride;
        tma_load_4d(d, &k_map, 0, off, hg * HB, blk, full_bar);
        tma_load_4d(d + TB, &v_map, 0, off, hg * HB, blk, full_bar);
      }
    }
    if (gate && lane == 0) pdl_wait();
    return;
  }

  // --------------------------------------------------------------- consumers
  // Operands are swapped so the 16 rows of each MMA are tokens or head_dim
  // rows, and the GQA group is the 8-wide N side:
  //   S^T[token][head] = K[token][:] . Q^T[:][head]         (A = K rows, B = Q^T)
  //   O^T[d][head]    += V^T[d][token] . P^T[token][head]   (A = V^T, B = P^T)
  // Fragment coordinates: g = lane / 4 (row), t = lane % 4 (column pair).
  const int g = lane >> 2, t = lane & 3;
  float qscale = p.q_scale, vscale = 1.0f;
  if constexpr (FP8) {
    qscale *= __ldg(p.k_scale + kvh);
    vscale = __ldg(p.v_scale + kvh);
  }
  float o[D / 16][4];  // O^T fragments: (d = 16i + g (+8), head 2t (+1)); E4M3: see the top
#pragma unroll
  for (int i = 0; i < D / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.0f, 0.0f};  // heads 2t, 2t+1

  // byte offset of (token r of the chunk, 16-byte column c) of this warp's head
  const int head_off = warp * rows_per_box * RS;
  const int lgb = (!TABLE || lg >= 4) ? 4 : lg;  // log2(rows_per_box)
  auto at = [&](int r, int c) -> uint32_t {
    const int b = r >> lgb;
    return b * box_stride + head_off + (r - (b << lgb)) * RS + c * 16;
  };
  const int lrow = lane & 7, lmat = lane >> 3;  // ldmatrix: row within matrix, matrix index
  // K as A (non-transposed): matrix j = tokens (j & 1) * 8 .. +7, column chunk + (j >> 1)
  const uint32_t k_lane = at((lmat & 1) * 8 + lrow, lmat >> 1);
  // V^T as A (transposed load): matrix j = tokens (j >> 1) * 8 .. +7, column chunk + (j & 1)
  const uint32_t v_lane = at((lmat >> 1) * 8 + lrow, lmat & 1);

  for (int c = 0; c < nchunks; ++c) {
    const int st = c % NS, u = c / NS;
    if (!mbar_wait(smem_u32(bars + st), u & 1, p.err)) {
      mbar_wait(smem_u32(bars + st), u & 1, p.err);  // let an in-flight copy land
      break;
    }
    uint8_t* stage = smem + st * Cfg::kStageBytes;
    const uint32_t ks_u32 = smem_u32(stage), vs_u32 = ks_u32 + TB;
    const int nvalid = min(C, t1 - (t0 + c * C));

    // S^T: two accumulation chains (even / odd k-steps) for latency
    float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    uint4 vr[4];  // E4M3: V bytes of tokens 2t, 2t+1, 2t+8, 2t+9, head_dim 16g .. 16g+15
    if constexpr (!FP8) {
      if (nvalid < C) {
        // rows past the context hold stale bits: zero this head's V rows so 0 * stale = 0
        for (int i = lane; i < (C - nvalid) * (D / 8); i += 32) {
          const int r = nvalid + i / (D / 8), cc = i % (D / 8);
          *reinterpret_cast<uint4*>(stage + TB + at(r, cc)) = make_uint4(0, 0, 0, 0);
        }
        // order these generic-proxy writes before the next async copy into the stage
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a, ks_u32 + k_lane + ks * 32);
        mma_bf16_16816(ks & 1 ? s1 : s0, a, qa[ks][0], qa[ks][1]);
      }
    } else {
      uint4 kr[2][D / 64];  // tokens g, g+8; 16-byte columns 2t + kq
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int kq = 0; kq < D / 64; ++kq) kr[h][kq] = lds128(ks_u32 + at(g + 8 * h, 2 * t + kq));
#pragma unroll
      for (int i = 0; i < 4; ++i) vr[i] = lds128(vs_u32 + at(2 * t + (i & 1) + 8 * (i >> 1), g));
      if (nvalid < C) {  // (warp-uniform) the last chunk of a context
        // rows past the context hold stale bytes (possibly NaN codes): use zeros
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (2 * t + (i & 1) + 8 * (i >> 1) >= nvalid) vr[i] = make_uint4(0, 0, 0, 0);
      }
      // every operand byte is in registers: hand the stage back to the producer
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(bars + NS + st));
#pragma unroll
      for (int kq = 0; kq < D / 64; ++kq) {
        const uint32_t w0[4] = {kr[0][kq].x, kr[0][kq].y, kr[0][kq].z, kr[0][kq].w};
        const uint32_t w1[4] = {kr[1][kq].x, kr[1][kq].y, kr[1][kq].z, kr[1][kq].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ks = 4 * kq + j;
          uint32_t a[4];
          a[0] = e4m3x2_to_f16x2(static_cast<uint16_t>(w0[j]));
          a[1] = e4m3x2_to_f16x2(static_cast<uint16_t>(w1[j]));
          a[2] = e4m3x2_to_f16x2(static_cast<uint16_t>(w0[j] >> 16));
          a[3] = e4m3x2_to_f16x2(static_cast<uint16_t>(w1[j] >> 16));
          mma_f16_16816(ks & 1 ? s1 : s0, a, qa[ks][0], qa[ks][1]);
        }
      }
    }
    // x[0], x[1]: token g, heads 2t, 2t+1; x[2], x[3]: token g + 8
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = (s0[i] + s1[i]) * qscale;
    if (nvalid < C) {  // (warp-uniform) keys past the context take no weight
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (g + (i >> 1) * 8 >= nvalid) x[i] = -INFINITY;
    }
    // per-head (column) max over the 16 tokens: over the lane's 2 rows, then over g
    float cm0 = fmaxf(x[0], x[2]), cm1 = fmaxf(x[1], x[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      cm0 = fmaxf(cm0, __shfl_xor_sync(kFullMask, cm0, off));
      cm1 = fmaxf(cm1, __shfl_xor_sync(kFullMask, cm1, off));
    }
    // The reference maximum m moves only when a chunk's maximum exceeds it by
    // more than 2^8 (logits are base 2): the exponentials stay at most 2^8, far
    // from overflowing the fp32 sums or the 16-bit P, and O and l are rescaled
    // on few chunks instead of every one. Numerator and denominator share m,
    // so the softmax is the same whatever m is. The vote keeps the branch
    // warp-uniform (lanes with the same t hold the same heads' m).
    constexpr float kSlack = 8.0f;
    if (__any_sync(kFullMask, cm0 > m[0] + kSlack || cm1 > m[1] + kSlack)) {
      const float mn0 = fmaxf(m[0], cm0), mn1 = fmaxf(m[1], cm1);
      const float al0 = exp2_fast(m[0] - mn0), al1 = exp2_fast(m[1] - mn1);  // 0 on the 1st chunk
      m[0] = mn0;
      m[1] = mn1;
      l_part[0] *= al0;
      l_part[1] *= al1;
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al1;
        o[i][2] *= al0;
        o[i][3] *= al1;
      }
    }
    const float p0 = exp2_fast(x[0] - m[0]), p1 = exp2_fast(x[1] - m[1]);
    const float p2 = exp2_fast(x[2] - m[0]), p3 = exp2_fast(x[3] - m[1]);
    l_part[0] += p0 + p2;
    l_part[1] += p1 + p3;
    if constexpr (!FP8) {
      // P^T as B: (token 2t, 2t+1 (+8), head g) = transpose of the (token g, head 2t..) pairs
      const uint32_t b0 = movmatrix_trans(pack_bf16x2(p0, p1));
      const uint32_t b1 = movmatrix_trans(pack_bf16x2(p2, p3));
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        uint32_t a[4];
        ldmatrix_x4_trans(a, vs_u32 + v_lane + dt * 32);
        mma_bf16_16816(o[dt], a, b0, b1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(bars + NS + st));
    } else {
      const uint32_t b0 = movmatrix_trans(pack_f16x2(p0, p1));
      const uint32_t b1 = movmatrix_trans(pack_f16x2(p2, p3));
      const uint32_t v0[4] = {vr[0].x, vr[0].y, vr[0].z, vr[0].w};
      const uint32_t v1[4] = {vr[1].x, vr[1].y, vr[1].z, vr[1].w};
      const uint32_t v2[4] = {vr[2].x, vr[2].y, vr[2].z, vr[2].w};
      const uint32_t v3[4] = {vr[3].x, vr[3].y, vr[3].z, vr[3].w};
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        // head_dim 16g + 2dt (row g) and +1 (row g + 8): bytes 2(dt&1), +1 of word dt/2;
        // the byte permute puts token 2t next to 2t+1 (and 2t+8 next to 2t+9)
        const uint32_t sel = (dt & 1) ? 0x7362u : 0x5140u;
        const uint32_t x01 = prmt(v0[dt >> 1], v1[dt >> 1], sel);
        const uint32_t x89 = prmt(v2[dt >> 1], v3[dt >> 1], sel);
        uint32_t a[4];
        a[0] = e4m3x2_to_f16x2(static_cast<uint16_t>(x01));
        a[1] = e4m3x2_to_f16x2(static_cast<uint16_t>(x01 >> 16));
        a[2] = e4m3x2_to_f16x2(static_cast<uint16_t>(x89));
        a[3] = e4m3x2_to_f16x2(static_cast<uint16_t>(x89 >> 16));
        mma_f16_16816(o[dt], a, b0, b1);
      }
    }
  }

  // softmax denominators per head: sum over the 8 row groups
  float l0 = l_part[0], l1 = l_part[1];
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(kFullMask, l0, off);
    l1 += __shfl_xor_sync(kFullMask, l1, off);
  }
  const bool h0_real = 2 * t < G, h1_real = 2 * t + 1 < G;

  if constexpr (FP8) {
    // lane (g, t) holds head_dim 16g .. 16g+15 of heads 2t and 2t+1:
    // o[dt][0] / o[dt][1] at 16g + 2dt, o[dt][2] / o[dt][3] at 16g + 2dt + 1
    if (n_part_s == 1 && !to_merge) {
      const float i0 = l0 > 0.0f ? vscale / l0 : 0.0f, i1 = l1 > 0.0f ? vscale / l1 : 0.0f;
      uint32_t w0[8], w1[8];
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        w0[dt] = pack_bf16x2(o[dt][0] * i0, o[dt][2] * i0);
        w1[dt] = pack_bf16x2(o[dt][1] * i1, o[dt][3] * i1);
      }
      uint4* o0 = reinterpret_cast<uint4*>(out + (out_row + 2 * t) * D + 16 * g);
      uint4* o1 = reinterpret_cast<uint4*>(out + (out_row + 2 * t + 1) * D + 16 * g);
      if (h0_real) {
        o0[0] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
        o0[1] = make_uint4(w0[4], w0[5], w0[6], w0[7]);
      }
      if (h1_real) {
        o1[0] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
        o1[1] = make_uint4(w1[4], w1[5], w1[6], w1[7]);
      }
      return;
    }
    const int64_t w0 = (out_row + 2 * t) * p.num_partitions + p.prefix_slots + part;
    const int64_t w1 = w0 + p.num_partitions;
    float4* a0 = reinterpret_cast<float4*>(p.ws_acc + w0 * D + 16 * g);
    float4* a1 = reinterpret_cast<float4*>(p.ws_acc + w1 * D + 16 * g);
#pragma unroll
    for (int q4 = 0; q4 < D / 32; ++q4) {
      if (h0_real)
        a0[q4] = make_float4(o[2 * q4][0] * vscale, o[2 * q4][2] * vscale,
                             o[2 * q4 + 1][0] * vscale, o[2 * q4 + 1][2] * vscale);
      if (h1_real)
        a1[q4] = make_float4(o[2 * q4][1] * vscale, o[2 * q4][3] * vscale,
                             o[2 * q4 + 1][1] * vscale, o[2 * q4 + 1][3] * vscale);
    }
    if (g == 0) {
      if (h0_real) {
        p.ws_m[w0] = m[0];
        p.ws_l[w0] = l0;
      }
      if (h1_real) {
        p.ws_m[w1] = m[1];
        p.ws_l[w1] = l1;
      }
    }
    return;
  }

  if (n_part_s == 1 && !to_merge) {
    const float i0 = l0 > 0.0f ? 1.0f / l0 : 0.0f, i1 = l1 > 0.0f ? 1.0f / l1 : 0.0f;
    __nv_bfloat16* o0 = out + (out_row + 2 * t) * D + g;
    __nv_bfloat16* o1 = o0 + D;
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
      if (h0_real) {
        o0[dt * 16] = __float2bfloat16_rn(o[dt][0] * i0);
        o0[dt * 16 + 8] = __float2bfloat16_rn(o[dt][2] * i0);
      }
      if (h1_real) {
        o1[dt * 16] = __float2bfloat16_rn(o[dt][1] * i1);
        o1[dt * 16 + 8] = __float2bfloat16_rn(o[dt][3] * i1);
      }
    }
    return;
  }

  // split-K: this partition's (m, l, O) to the workspace
  {
    const int64_t w0 = (out_row + 2 * t) * p.num_partitions + p.prefix_slots + part;
    const int64_t w1 = w0 + p.num_partitions;
    float* a0 = p.ws_acc + w0 * D + g;
    float* a1 = p.ws_acc + w1 * D + g;
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
      if (h0_real) {
        a0[dt * 16] = o[dt][0];
        a0[dt * 16 + 8] = o[dt][2];
      }
      if (h1_real) {
        a1[dt * 16] = o[dt][1];
        a1[dt * 16 + 8] = o[dt][3];
      }
    }
    if (g == 0) {
      if (h0_real) {
        p.ws_m[w0] = m[0];
        p.ws_l[w0] = l0;
      }
      if (h1_real) {
        p.ws_m[w1] = m[1];
        p.ws_l[w1] = l1;
      }
    }
  }
}

}  // namespace pa
