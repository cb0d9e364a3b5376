// Paged decode attention for sm_100a: one CTA per (KV head, partition, sequence).
//
// What it computes ("Paged Attention", klaylearn.com glossary, definition;
// "PagedAttention — AI Glossary", Example): for sequence s and query head j
// with KV head h = j / G, softmax(scale * q . K_t) weighted sum of V_t over the
// sequence's cached tokens t, where token t lives in physical block
// block_tables[s][t / block_size] at offset t % block_size. Paging moves the
// cache, not the arithmetic.
//
// Design (B200):
//  * Warp-specialised CTA: NW consumer warps + 1 producer warp. The producer
//    reads the block table 32 entries at a time (one coalesced load, shuffled
//    out lane by lane) and issues TMA tensor loads of whole block rows of this
//    KV head into a per-warp ring of NS shared-memory stages. Each stage holds
//    one chunk of C = 16 tokens: K rows then V rows. Chunk c of the partition
//    goes to consumer warp c % NW. Completion is tracked by mbarriers
//    (transaction bytes), so the table lookup and the HBM latency sit behind
//    the ring.
//  * Each consumer warp keeps its own online-softmax state (running max m,
//    running sum l, unnormalised accumulator) for all G query heads of the
//    group: one K/V read serves the G heads. A K row is spread over LPR lanes
//    (16 bytes each); q.k partial sums are reduced across those lanes with an
//    exchange-halving butterfly (G - 1 + log2(LPR / G) shuffles per row
//    instead of G * log2(LPR)).
//  * Scores use base-2 exponentials: q is pre-scaled by scale * log2(e).
//  * End of the partition: the NW warps' states are merged through shared
//    memory. A sequence with one partition writes `out` directly; otherwise
//    (m, l, acc) go to the workspace and pa_reduce_kernel merges partitions.
//  * Every chunk has the same 16 logical tokens whatever block_size is, and is
//    reduced in the same order, so results are bit-identical across block
//    sizes and physical placements.
#pragma once

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "pa_device.cuh"

namespace pa {

struct DecodeParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_m;    // [S][Hq][NP]  running max (base-2 domain) per partition
  float* ws_l;    // [S][Hq][NP]  softmax denominator per partition
  float* ws_acc;  // [S][Hq][NP][D] unnormalised output per partition
  // Fused append (pa_decode_append): each sequence's newest token (position
  // context_lens[s] - 1) is written from k_new / v_new [S][Hkv][D] into the
  // caches through the block table before it is read. Null for pa_decode.
  const uint8_t* k_new;
  const uint8_t* v_new;
  uint8_t* k_cache_w;
  uint8_t* v_cache_w;
  unsigned* err;
  // E4M3 caches: cache value = code * scale, one scale per KV head [Hkv]. Null otherwise.
  const float* k_scale;
  const float* v_scale;
  int num_seqs, num_heads, num_kv_heads, block_size, log2_block_size, num_blocks;
  int max_blocks_per_seq, max_context_len, partition_size, num_partitions;
  float q_scale;  // scale * log2(e)
  // PA_DECODE_EARLY_CACHE_READS: the caller vouches that no kernel still
  // running when this call starts writes the cache, the block tables or the
  // context lengths, so they may be read before the dependent-launch wait.
  int early_reads;
  // Shared-prefix decode (pa_decode_shared_prefix): this kernel attends only
  // tokens [first_token, context_lens[s]) (first_token a multiple of the block
  // size; the table is read from block first_token / block_size on), and
  // leaves every row to the merge: its partition p goes to workspace slot
  // prefix_slots + p, slots 0 .. prefix_slots - 1 holding the prefix's
  // partial results. Both 0 for the other calls.
  int first_token, prefix_slots;
  // Planned decode (pa_decode_planned): num_items work items {sequence,
  // partition | partitions of the sequence << 16} made on the host from the
  // context lengths, one CTA per item and head group. Null otherwise.
  const int32_t* work;
  int num_items;
};


// Fused append (pa_decode_append): the producer warp of the CTA that holds a
// sequence's newest token copies that token's K and V rows for KV heads
// [h0, h0 + nh) from k_new / v_new into cache block `blk` at offset `off`,
// then orders these generic-proxy writes before the TMA reads that follow.
__device__ __forceinline__ void append_newest_rows(const DecodeParams& p, int s, int blk, int off,
                                                   int h0, int nh, int row_bytes, int lane) {
  const int64_t vec = static_cast<int64_t>(nh) * row_bytes / 16;
  const int64_t src = (static_cast<int64_t>(s) * p.num_kv_heads + h0) * row_bytes;
  const int64_t dst =
      ((static_cast<int64_t>(blk) * p.block_size + off) * p.num_kv_heads + h0) * row_bytes;
  for (int64_t i = lane; i < vec; i += 32) {
    // read at L2 (not through L1): under a shared-prefix decode these rows
    // are read without a dependent-launch wait in this kernel
    const uint4 a = __ldcg(reinterpret_cast<const uint4*>(p.k_new + src + i * 16));
    const uint4 b = __ldcg(reinterpret_cast<const uint4*>(p.v_new + src + i * 16));
    *reinterpret_cast<uint4*>(p.k_cache_w + dst + i * 16) = a;
    *reinterpret_cast<uint4*>(p.v_cache_w + dst + i * 16) = b;
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncwarp();
}

// The same for an E4M3 cache: k_new / v_new hold bfloat16 rows of head_dim
// values; each value is stored as the E4M3 code of value / scale[head].
__device__ __forceinline__ void append_newest_rows_fp8(const DecodeParams& p, int s, int blk,
                                                       int off, int h0, int nh, int head_dim,
                                                       int lane) {
  const int units = nh * head_dim / 16;  // 16 values per unit
  const int64_t src = (static_cast<int64_t>(s) * p.num_kv_heads + h0) * head_dim * 2;
  const int64_t dst =
      ((static_cast<int64_t>(blk) * p.block_size + off) * p.num_kv_heads + h0) * head_dim;
  for (int i = lane; i < units; i += 32) {
    const int h = h0 + i * 16 / head_dim;
    const uint4* ks = reinterpret_cast<const uint4*>(p.k_new + src) + 2 * i;
    const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + src) + 2 * i;
    const uint4 kc = bf16x16_to_e4m3(__ldcg(ks), __ldcg(ks + 1), __ldg(p.k_scale + h));
    const uint4 vc = bf16x16_to_e4m3(__ldcg(vs), __ldcg(vs + 1), __ldg(p.v_scale + h));
    *reinterpret_cast<uint4*>(p.k_cache_w + dst + i * 16) = kc;
    *reinterpret_cast<uint4*>(p.v_cache_w + dst + i * 16) = vc;
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncwarp();
}

template <typename T, int D, int G>
struct DecodeConfig {
  static constexpr int kElemBytes = ElemTraits<T>::kBytes;
  static constexpr int kRowBytes = D * kElemBytes;      // one token, one KV head
  static constexpr int kLPR = kRowBytes / 16;           // lanes per row
  static constexpr int kTPW = 32 / kLPR;                // rows per warp instruction
  static constexpr int kEPL = 16 / kElemBytes;          // elements per lane
  static constexpr int kC = 16;                         // tokens per chunk / stage
  static constexpr int kNI = kC / kTPW;                 // row iterations per chunk
  static constexpr int kNW = 4;                         // consumer warps
  static constexpr int kStageBytes = 2 * kC * kRowBytes;
  static constexpr int kNSraw = 98304 / (kNW * kStageBytes);
  static constexpr int kNS = kNSraw < 2 ? 2 : kNSraw;   // stages per consumer warp
  static constexpr int kThreads = (kNW + 1) * 32;
  static constexpr int kLog2G = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  static constexpr int kLog2LPR = kLPR == 8 ? 3 : kLPR == 16 ? 4 : 5;
  static constexpr int kRingBytes = kNW * kNS * kStageBytes;
  static constexpr int kBarBytes = 2 * kNW * kNS * 8;
  static constexpr int kSmemBytes = 1024 + kRingBytes + kBarBytes;  // + alignment slack
  static_assert(kRowBytes % 16 == 0 && 32 % kLPR == 0, "row must split over lanes");
  static_assert(G <= kLPR, "group larger than lanes per row");
  static_assert(kC % kTPW == 0, "chunk must be whole warp rows");
  static_assert(kNS * kStageBytes >= (2 * G + G * D) * 4, "epilogue must fit a warp's ring");
};

// Query head index held by `lane` after the exchange-halving reduction (the
// bit-reversal of the lane's low log2(G) bits); also its own inverse.
template <int LOG2G>
__device__ __forceinline__ int reversed_low_bits(int x) {
  int r = 0;
#pragma unroll
  for (int k = 0; k < LOG2G; ++k) r |= ((x >> k) & 1) << (LOG2G - 1 - k);
  return r;
}

// Sum s[0..G) over the kLPR lanes of a row. On return s[0] holds, in every
// lane, the full sum for head reversed_low_bits(lane).
template <int G, int LOG2G, int LOG2LPR>
__device__ __forceinline__ void row_reduce(float (&s)[G], int lane) {
#pragma unroll
  for (int k = 0; k < LOG2G; ++k) {
    const int nh = G >> k;
    const bool upper = (lane >> k) & 1;
#pragma unroll
    for (int i = 0; i < (G >> (k + 1)); ++i) {
      const float send = upper ? s[i] : s[i + nh / 2];
      const float keep = upper ? s[i + nh / 2] : s[i];
      s[i] = keep + __shfl_xor_sync(kFullMask, send, 1 << k);
    }
  }
#pragma unroll
  for (int k = LOG2G; k < LOG2LPR; ++k) s[0] += __shfl_xor_sync(kFullMask, s[0], 1 << k);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(DecodeConfig<T, D, G>::kThreads)
    pa_decode_kernel(const __grid_constant__ CUtensorMap k_map,
                     const __grid_constant__ CUtensorMap v_map, const DecodeParams p) {
  using Cfg = DecodeConfig<T, D, G>;
  constexpr int C = Cfg::kC, NW = Cfg::kNW, NS = Cfg::kNS, LPR = Cfg::kLPR, TPW = Cfg::kTPW;
  constexpr int EPL = Cfg::kEPL, NI = Cfg::kNI, ROW = Cfg::kRowBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kRingBytes);  // full[], then empty[]

  const int h = blockIdx.x, part = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = p.partition_size, bs = p.block_size;

  int L = __ldg(p.context_lens + s);
  if (L < 0 || L > p.max_context_len ||
      static_cast<int64_t>(L) > static_cast<int64_t>(p.max_blocks_per_seq) * bs) {
    if (threadIdx.x == 0 && h == 0 && part == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);
    L = 0;  // attend nothing: the row becomes zeros
  }
  const int t0 = part * P;
  const int n_part_s = (L + P - 1) / P;
  T* out = static_cast<T*>(p.out);
  const int64_t out_row = (static_cast<int64_t>(s) * p.num_heads + h * G);

  if (L == 0) {  // empty context: zeros, written once by partition 0
    if (part == 0)
      for (int e = threadIdx.x; e < G * D; e += blockDim.x)
        ElemTraits<T>::store(out + out_row * D + e, 0.0f);
    return;
  }
  if (t0 >= L) return;  // this sequence has fewer partitions than the grid
  const int t1 = min(t0 + P, L);
  const int nchunks = (t1 - t0 + C - 1) / C;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NW * NS; ++i) {
      mbar_init(smem_u32(bars + i), 1);            // full: producer arrive + TMA bytes
      mbar_init(smem_u32(bars + NW * NS + i), 1);  // empty: consumer warp's release
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
    }
    const int32_t* trow = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
    const int lb_last = (t1 - 1) >> p.log2_block_size;
    const bool whole_chunk_in_block = bs >= C;
    const int rows_per_box = whole_chunk_in_block ? C : bs;
    int base = -64, ent = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int w = c % NW, k = c / NW, st = k % NS;
      const int bi = w * NS + st;
      if (k >= NS) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(smem_u32(bars + NW * NS + bi), ((k / NS) - 1) & 1, p.err);
        if (!__shfl_sync(kFullMask, ok, 0)) break;
      }
      const int t = t0 + c * C;
      const int nvalid = min(C, t1 - t);
      const int lb0 = t >> p.log2_block_size;
      const int nblk = whole_chunk_in_block ? 1 : (nvalid + bs - 1) / bs;
      const uint32_t full_bar = smem_u32(bars + bi);
      const uint32_t kdst = smem_u32(smem + bi * Cfg::kStageBytes);
      const uint32_t vdst = kdst + C * ROW;
      if (p.k_new != nullptr && c == nchunks - 1 && t1 == L) {
        // this CTA holds the sequence's newest token: write it before reading it
        const int tn = L - 1;
        const int bn = __ldg(trow + (tn >> p.log2_block_size));
        if (static_cast<unsigned>(bn) < static_cast<unsigned>(p.num_blocks))
          append_newest_rows(p, s, bn, tn & (bs - 1), h, 1, ROW, lane);
        else if (lane == 0)
          atomicOr(p.err, PA_DEVERR_BLOCK_ID);
      }
      if (lane == 0) mbar_arrive_expect_tx(full_bar, 2u * nblk * rows_per_box * ROW);
      for (int b = 0; b < nblk; ++b) {
        const int lb = lb0 + b;
        if (lb - base >= 32) {  // refill: the next 32 table entries, one per lane
          base = lb;
          ent = (lb + lane <= lb_last) ? __ldg(trow + lb + lane) : 0;
        }
        const int blk = __shfl_sync(kFullMask, ent, lb - base);
        if (lane == 0) {
          // An id outside the pool is flagged; TMA reads out-of-range boxes as zeros.
          if (static_cast<unsigned>(blk) >= static_cast<unsigned>(p.num_blocks))
            atomicOr(p.err, PA_DEVERR_BLOCK_ID);
          const int off = whole_chunk_in_block ? (t & (bs - 1)) : 0;
          tma_load_4d(kdst + b * rows_per_box * ROW, &k_map, 0, h, off, blk, full_bar);
          tma_load_4d(vdst + b * rows_per_box * ROW, &v_map, 0, h, off, blk, full_bar);
        }
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int rg = lane / LPR;  // which row of a warp instruction this lane reads
  const int li = lane % LPR;  // which 16-byte piece of the row
  const int my_head = reversed_low_bits<Cfg::kLog2G>(li);

  float qf[G][EPL];
  {
    const T* qp = static_cast<const T*>(p.q) + out_row * D + li * EPL;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint4 raw = *reinterpret_cast<const uint4*>(qp + g * D);
      ElemTraits<T>::unpack(raw, qf[g]);
#pragma unroll
      for (int e = 0; e < EPL; ++e) qf[g][e] *= p.q_scale;
    }
  }

  float m[G], l[G], acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.0f;
  }
  float m_mine = -INFINITY;

  for (int k = 0;; ++k) {
    const int c = k * NW + warp;
    if (c >= nchunks) break;
    const int st = k % NS, bi = warp * NS + st;
    if (!mbar_wait(smem_u32(bars + bi), (k / NS) & 1, p.err)) {
      mbar_wait(smem_u32(bars + bi), (k / NS) & 1, p.err);  // let an in-flight copy land
      break;
    }
    const uint8_t* kst = smem + bi * Cfg::kStageBytes;
    const uint8_t* vst = kst + C * ROW;
    const int nvalid = min(C, t1 - (t0 + c * C));

    // scores of this lane's rows for head my_head (base-2 logits)
    float sc[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const uint4 raw = *reinterpret_cast<const uint4*>(kst + (i * TPW + rg) * ROW + li * 16);
      float kf[EPL];
      ElemTraits<T>::unpack(raw, kf);
      float part_sum[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a = 0.0f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) a = fmaf(qf[g][e], kf[e], a);
        part_sum[g] = a;
      }
      row_reduce<G, Cfg::kLog2G, Cfg::kLog2LPR>(part_sum, lane);
      sc[i] = (i * TPW + rg < nvalid) ? part_sum[0] : -INFINITY;
    }

    // chunk max of head my_head across this warp's rows
    float cm = sc[0];
#pragma unroll
    for (int i = 1; i < NI; ++i) cm = fmaxf(cm, sc[i]);
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(kFullMask, cm, off));
    const float m_mine_new = fmaxf(m_mine, cm);

    float ps = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      sc[i] = exp2f(sc[i] - m_mine_new);
      ps += sc[i];
    }
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) ps += __shfl_xor_sync(kFullMask, ps, off);

    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int src = reversed_low_bits<Cfg::kLog2G>(g);
      const float mg = __shfl_sync(kFullMask, m_mine_new, src);
      const float sg = __shfl_sync(kFullMask, ps, src);
      alpha[g] = exp2f(m[g] - mg);
      m[g] = mg;
      l[g] = fmaf(l[g], alpha[g], sg);
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] *= alpha[g];
    }
    m_mine = m_mine_new;

#pragma unroll
    for (int i = 0; i < NI; ++i) {
      float pg[G];
#pragma unroll
      for (int g = 0; g < G; ++g)
        pg[g] = __shfl_sync(kFullMask, sc[i], rg * LPR + reversed_low_bits<Cfg::kLog2G>(g));
      if (i * TPW + rg < nvalid) {  // rows past the context may hold stale bits
        const uint4 raw = *reinterpret_cast<const uint4*>(vst + (i * TPW + rg) * ROW + li * 16);
        float vf[EPL];
        ElemTraits<T>::unpack(raw, vf);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(pg[g], vf[e], acc[g][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(bars + NW * NS + bi));
  }

  // merge the rows of this warp (lanes with equal li, different rg)
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] += __shfl_xor_sync(kFullMask, acc[g][e], off);

  // this warp's (m, l, acc) into its own, now idle, ring region
  float* red = reinterpret_cast<float*>(smem + warp * NS * Cfg::kStageBytes);
  if (rg == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) red[2 * G + g * D + li * EPL + e] = acc[g][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      red[g] = m[g];
      red[G + g] = l[g];
    }
  }
  named_barrier(1, NW * 32);

  // merge the NW warps: thread -> (head g, element d)
  const int tid = threadIdx.x;
  const bool split = n_part_s > 1;
  for (int e = tid; e < G * D; e += NW * 32) {
    const int g = e / D, d = e - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      M = fmaxf(M, reinterpret_cast<const float*>(smem + w * NS * Cfg::kStageBytes)[g]);
    float A = 0.0f, Lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* rw = reinterpret_cast<const float*>(smem + w * NS * Cfg::kStageBytes);
      const float f = (rw[g] == -INFINITY) ? 0.0f : exp2f(rw[g] - M);
      Lsum = fmaf(f, rw[G + g], Lsum);
      A = fmaf(f, rw[2 * G + g * D + d], A);
    }
    if (!split) {
      ElemTraits<T>::store(out + (out_row + g) * D + d, Lsum > 0.0f ? A / Lsum : 0.0f);
    } else {
      const int64_t wrow = (out_row + g) * p.num_partitions + part;
      p.ws_acc[wrow * D + d] = A;
      if (d == 0) {
        p.ws_m[wrow] = M;
        p.ws_l[wrow] = Lsum;
      }
    }
  }
}


// Split-K merge, for rows (sequence, query head) with more than one partial
// result:
//   M = max_p m_p,  Lambda = sum_p l_p 2^(m_p - M),  out = sum_p 2^(m_p - M) acc_p / Lambda.
// W warps per row (1, 2 or 4, chosen on the host from the partition count),
// 4 / W rows per CTA of 4 warps: few partials need few threads, and the grid
// stays within one wave of resident CTAs. Warp w of a row takes partitions
// w, w + W, ... in batches of 8: a batch's maxima, sums and accumulator rows
// (each lane owns D / 32 columns) are loaded together (volatile loads, kept
// ahead of their uses), so a row with up to 8 W partitions costs one round
// trip; batches are folded in with an online
// rescale. With W > 1 the row's warps are combined in warp order through
// shared memory. The result depends only on the partials (deterministic).
// Launched with programmatic dependent launch.
template <typename T, int D, int W>
__global__ void __launch_bounds__(128) pa_merge_kernel(const DecodeParams p) {
  static_assert(W == 1 || W == 2 || W == 4, "warps per row");
  constexpr int E = D / 32;  // columns per lane
  constexpr int B = 8;       // partitions per warp per batch
  constexpr int R = 4 / W;   // rows per CTA
  using Vec = typename std::conditional<E == 4, float4, float2>::type;
  __shared__ float s_m[4], s_l[4], s_acc[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = warp % W;  // this warp's place among its row's warps
  const int64_t r = static_cast<int64_t>(blockIdx.x) * R + warp / W;  // s * num_heads + j
  const int s = static_cast<int>(r / p.num_heads);
  // The context length is read before the dependent-launch wait: the kernel
  // before this one is the decode kernel of the same call, which waited for all
  // earlier work before letting this kernel start (or, under
  // PA_DECODE_EARLY_CACHE_READS, the caller vouches that nothing still running
  // writes it), and neither kernel writes it. Rows without partials (flagged,
  // and without a prefix zero-filled, by the decode kernel; or written there
  // directly) are skipped.
  int np = 0;
  if (s < p.num_seqs) {
    const int L = __ldg(p.context_lens + s);
    if (!(L < 0 || L > p.max_context_len ||
          static_cast<int64_t>(L) > static_cast<int64_t>(p.max_blocks_per_seq) * p.block_size ||
          L < p.first_token)) {
      // partial results: the prefix's slots, then this row's own partitions
      np = p.prefix_slots + (L - p.first_token + p.partition_size - 1) / p.partition_size;
      if (np <= 1 && p.prefix_slots == 0) np = 0;
    }
  }
  if (W == 1 && np == 0) return;  // (W > 1: every warp reaches the barrier below)
  // The next kernel may start its launch now: whatever it reads before its
  // own wait is, by the same contract, not written here.
  pdl_launch_dependents();
  pdl_wait();  // the partials are the decode kernel's output
  const int64_t row = r * p.num_partitions;
  const float* a = p.ws_acc + row * D + lane * E;
  float Mw = -INFINITY, Lw = 0.0f, acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.0f;
  for (int q0 = wr; q0 < np; q0 += W * B) {
    float mq[B], lq[B];
    Vec vq[B];
    // no branch around the loads: a slot past the row's last partial loads
    // that partial again and is masked below
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int q = min(q0 + W * j, np - 1);
      mq[j] = ld_cg_f32(p.ws_m + row + q);
      lq[j] = ld_cg_f32(p.ws_l + row + q);
      if constexpr (E == 4)
        vq[j] = ld_cg_f32x4(a + static_cast<int64_t>(q) * D);
      else
        vq[j] = ld_cg_f32x2(a + static_cast<int64_t>(q) * D);
    }
#pragma unroll
    for (int j = 0; j < B; ++j) {
      if (q0 + W * j >= np) {
        mq[j] = -INFINITY;
        lq[j] = 0.0f;
        vq[j] = Vec{};
      }
    }
    float bm = Mw;
#pragma unroll
    for (int j = 0; j < B; ++j) bm = fmaxf(bm, mq[j]);
    const float sc = exp2f(Mw - bm);  // 0 on the first batch (Mw = -inf, bm finite)
    Lw *= sc;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= sc;
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const float w = exp2f(mq[j] - bm);  // 0 for the padding slots of a batch
      Lw = fmaf(w, lq[j], Lw);
      const float* v = reinterpret_cast<const float*>(&vq[j]);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(w, v[e], acc[e]);
    }
    Mw = bm;
  }
  if constexpr (W == 1) {
#pragma unroll
    for (int e = 0; e < E; ++e)
      ElemTraits<T>::store(static_cast<T*>(p.out) + r * D + lane * E + e, acc[e] / Lw);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) s_acc[warp][lane * E + e] = acc[e];
    if (lane == 0) {
      s_m[warp] = Mw;
      s_l[warp] = Lw;
    }
    __syncthreads();
    // the row's 32 W threads: columns t, t + 32 W, ... of the row
    const int t = threadIdx.x % (32 * W), w0 = warp - wr;
    if (np > 0) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w) M = fmaxf(M, s_m[w0 + w]);
      float f[W], lsum = 0.0f;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        f[w] = s_m[w0 + w] == -INFINITY ? 0.0f : exp2f(s_m[w0 + w] - M);
        lsum = fmaf(f[w], s_l[w0 + w], lsum);
      }
      for (int d = t; d < D; d += 32 * W) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < W; ++w) v = fmaf(f[w], s_acc[w0 + w][d], v);
        ElemTraits<T>::store(static_cast<T*>(p.out) + r * D + d, v / lsum);
      }
    }
  }
}

}  // namespace pa
