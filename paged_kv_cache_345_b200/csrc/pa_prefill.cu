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
// Layout and pipeline. One CTA = one sequence x one KV head x two query tiles
// of 128 rows (each 128 / G tokens x the G query heads of the KV head, row =
// token * G + g). Both tiles share every K/V tile, which halves the K/V bytes
// per flop: with one 128-row tile per CTA the K/V tile loads (the per-SM load
// path and its latency), not the tensor cores, set the pace. The grid counts
// tiles from each sequence's end, so the tiles that see the most keys start
// first.
//  * Warp 0 (producer): TMA loads both Q tiles once, then per tile of 64 keys
//    one box per cache block {64 columns, min(block_size, 64) tokens} for each
//    half of head_dim, for K and for V, into a 4-stage ring. Boxes use the
//    128-byte swizzle, which is the shared-memory operand layout of the MMA.
//  * Warps 1 and 10 (MMA): one thread each issues tcgen05.mma. Warp 1 issues
//    S_x = Q_x K^T (M 128, N 64, K 128) for both query tiles x into
//    double-buffered tensor memory, two key tiles ahead; warp 10 issues
//    O_x += P_x V (M 128, N 128, K 64) as each P_x becomes ready (V is the
//    MN-major operand, P the K-major one). An MMA issue blocks while the
//    tensor pipe's queue is full; with one issuer a ready P V waited behind a
//    batch of S (measured), with two it does not. Completion is signalled to
//    mbarriers with tcgen05.commit.
//  * Warps 2-5 and 6-9 (softmax, one warpgroup per query tile): thread = row
//    (tensor-memory lane). Per key tile: load the row of S, mask keys past the
//    row's position, exponentials in base 2 against a reference maximum that
//    moves only when the row maximum exceeds it by 2^8 (so O is rarely
//    rescaled; numerator and denominator share it), computed while the
//    previous P V runs; then write P (bf16) into shared memory in the swizzled
//    K-major layout and, if the reference moved, rescale the row of O in
//    tensor memory. The end divides by the row sum and stores bf16.
//  * Results depend only on the logical key tiles, so they are bit-identical
//    across block sizes and placements.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_prefill_order.h"
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
  int num_seqs, total_q, max_query_len;
  float q_scale;  // scale * log2(e)
  // Shared-prefix mode (PREFIX kernels, pa_decode_shared_prefix): the
  // total_q decode queries ([total_q][Hq][128], one "token" per sequence)
  // attend keys [0, prefix_keys) through the first table row (every sequence
  // shares those blocks), split into prefix_parts partitions of prefix_part
  // keys (a multiple of 64), no causal mask; each CTA writes fp32 partial
  // results (reference maximum m, sum l, unnormalised O) of its rows to the
  // decode split-K workspace at slot = its partition (ws_slots per row).
  int prefix_keys, prefix_part, prefix_parts, ws_slots;
  float* ws_m;
  float* ws_l;
  float* ws_acc;
  // pa_prefill_planned: work item jw is {sequence, item} (made on the host in
  // the order the search below would find); null: the kernel searches
  const int32_t* work;
};

template <int G>
struct PrefillConfig {
  static constexpr int kRows = 128;                  // rows of one query tile (MMA M)
  static constexpr int kQT = 2;                      // query tiles per CTA
  static constexpr int kKeys = 64;                   // keys per K/V tile
  static constexpr int kD = 128;                     // head_dim
  static constexpr int kTok = kRows / G;             // tokens per query tile
  static constexpr int kQBytes = kRows * kD * 2;     // a Q tile: two 64-column halves of 16 KB
  static constexpr int kQHalf = kQBytes / 2;
  static constexpr int kKVBytes = kKeys * kD * 2;    // a K or V tile: two halves of 8 KB
  static constexpr int kKVHalf = kKVBytes / 2;
  static constexpr int kNS = 4;                      // K/V stages
  static constexpr int kQ = 0, kStage0 = kQT * kQBytes;  // (P lives in tensor memory)
  static constexpr int kBars = kStage0 + kNS * 2 * kKVBytes;
  static constexpr int kSmemBytes = kBars + 256;     // the base is 1024-byte aligned
  // producer, S-MMA issuer, 2 x 4 softmax warps, P V-MMA issuer
  static constexpr int kThreads = 352;
  static constexpr uint32_t kTmemCols = 512;  // S[x][2] (64 each; P over its first 32), O[x] (128 each)
  static_assert(kRows % G == 0, "group must divide the row tile");
  static_assert(kKeys == kPrefillKeyTile, "prefix partitions are whole key tiles");
};

// mbarrier slots
// Barriers that two warps wait on with different lags come in pairs by tile
// parity ([query tile][j % 2]), so that no waiter can fall two phases behind.
enum : int {
  kQFull = 0,
  kKVFull = 1,    // [kNS]
  kKVEmpty = 5,   // [kNS]: a commit of each MMA issuer
  kSFull = 9,     // [query tile][j % 2]
  kPFull = 13,    // [query tile][j % 2]
  kODone = 17,    // [query tile][j % 2]: P V of tile j done (its P read, O updated)
  kNumBars = 21
};
constexpr int kTmemSlotOffset = 192;  // after the barriers

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// 2^x by the MUFU unit (approximate; results below 2^-126 flush to 0, -inf gives 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Longest-first order over at most kOrderMaxSeqs sequences; larger batches
// take their items pair by pair across the sequences.
constexpr int kOrderMaxSeqs = 256;

// The work item (sequence *s, item *z) of work index j in longest-first
// order: items sorted by cost (key tiles visited) downward, then by sequence,
// then by z. Every lane of the warp returns the same answer. Each lane holds
// sequences lane, lane + 32, ... (PER of them); the search finds the cost
// level c with count(c + 1) <= j < count(c), count(c) = items costing at
// least c, then the item among those costing exactly c. *bad tells whether
// any sequence has unusable arguments (it then has no items). Returns false
// when j is past the last item.
template <int PER, int CTOK, int KEYN>
__device__ __forceinline__ bool work_item(const PrefillParams& p, int S, int j, int lane, int* s,
                                          int* z, bool* bad) {
  namespace po = prefill_order;
  constexpr int LG = CTOK == 32 ? 5 : CTOK == 64 ? 6 : CTOK == 128 ? 7 : 8;
  static_assert((1 << LG) == CTOK, "query rows per item must be a power of two");
  po::ItemCosts q[PER];
  bool any_bad = false;
  int cmax = 0;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int t = lane + 32 * k;
    q[k] = po::ItemCosts{0, 0, 0};
    if (t < S) {
      const int q0 = __ldg(p.query_start + t), q1 = __ldg(p.query_start + t + 1);
      const int L = __ldg(p.context_lens + t);
      if (po::chunk_ok(q0, q1, L, p.total_q, p.max_query_len,
                       static_cast<int64_t>(p.max_blocks_per_seq) * p.block_size))
        q[k] = po::item_costs(L, q1 - q0, CTOK, KEYN);
      else
        any_bad = true;
    }
    cmax = max(cmax, q[k].top);
  }
  *bad = __any_sync(kFullMask, any_bad);
  auto count = [&](int c) {
    int acc = 0;
#pragma unroll
    for (int k = 0; k < PER; ++k) acc += po::items_at_least(q[k], c, LG, KEYN);
    return __reduce_add_sync(kFullMask, acc);
  };
  cmax = __reduce_max_sync(kFullMask, cmax);
  if (cmax == 0 || j >= count(1)) return false;
  int lo = 1, hi = cmax + 1;  // count(lo) > j >= count(hi)
  while (hi - lo > 1) {       // at most 31 rounds: cmax < 2^31
    const int mid = lo + ((hi - lo) >> 1);
    if (count(mid) > j) lo = mid;
    else hi = mid;
  }
  int o = j - count(lo + 1);  // rank among the items costing exactly lo
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int above = po::items_at_least(q[k], lo + 1, LG, KEYN);
    const int e = po::items_at_least(q[k], lo, LG, KEYN) - above;
    int incl = e;  // inclusive prefix over the lanes: sequences 32k .. 32k + lane
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(kFullMask, incl, d);
      if (lane >= d) incl += v;
    }
    const int here = __shfl_sync(kFullMask, incl, 31);
    if (o < here) {
      const int src = __ffs(__ballot_sync(kFullMask, incl > o)) - 1;
      *z = __shfl_sync(kFullMask, above + o - (incl - e), src);
      *s = 32 * k + src;
      return true;
    }
    o -= here;
  }
  if (lane == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);  // unreachable when the counts agree
  return false;
}

template <int G, bool PREFIX = false>
__global__ void __launch_bounds__(PrefillConfig<G>::kThreads, 1)
    pa_prefill_kernel(const __grid_constant__ CUtensorMap q_map,
                      const __grid_constant__ CUtensorMap k_map,
                      const __grid_constant__ CUtensorMap v_map, const PrefillParams p) {
  using Cfg = PrefillConfig<G>;
  constexpr int TOK = Cfg::kTok, QHALF = Cfg::kQHalf, KVHALF = Cfg::kKVHalf, KEYN = Cfg::kKeys;
  constexpr int NS = Cfg::kNS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::kBars + kTmemSlotOffset);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto q_s = [&](int x) { return smem_u32(sm + Cfg::kQ + x * Cfg::kQBytes); };
  auto k_s = [&](int st) { return smem_u32(sm + Cfg::kStage0 + st * 2 * Cfg::kKVBytes); };
  auto v_s = [&](int st) { return k_s(st) + Cfg::kKVBytes; };

  // one-dimensional grid: KV head fastest, then the work index
  const int h = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.num_kv_heads));
  const int jw = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.num_kv_heads));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bs = p.block_size, lg = p.log2_block_size;
  // every lane polls; the warp proceeds only if all saw the phase complete
  auto wait_all = [&](uint32_t b, uint32_t parity) {
    return __all_sync(kFullMask, mbar_wait(b, parity, p.err));
  };

  pdl_wait();  // inputs may come from the previous kernel in the stream
  pdl_launch_dependents();

  constexpr int CTOK = Cfg::kQT * TOK;  // tokens per CTA
  const int S = p.num_seqs;
  // this CTA's query rows (tokens tq0 .. of the chunk [q0, q0 + n)) and keys
  // [key_lo, L), of which the last visible to any row is pos_last
  int s = 0, z = 0, q0 = 0, n = 0, L = 0, tq0 = 0, pos_last = 0, nt = 0, key_lo = 0, kpart = 0;
  const int32_t* trow = p.block_tables;
  if constexpr (PREFIX) {
    // grid: KV head fastest, then the key partition, then the pair of query tiles
    kpart = jw % p.prefix_parts;
    z = jw / p.prefix_parts;
    n = p.total_q;
    tq0 = z * CTOK;
    key_lo = kpart * p.prefix_part;
    L = min(key_lo + p.prefix_part, p.prefix_keys);
    if (tq0 >= n || key_lo >= L) return;
    pos_last = L - 1;
    nt = (L - key_lo + KEYN - 1) / KEYN;
  } else {
    if (p.work != nullptr) {
      const int2 it = __ldg(reinterpret_cast<const int2*>(p.work) + jw);
      s = it.x;
      z = it.y;
      if (static_cast<unsigned>(s) >= static_cast<unsigned>(S) || z < 0) {
        if (threadIdx.x == 0) atomicOr(p.err, PA_DEVERR_PLAN);
        return;
      }
    } else if (S <= kOrderMaxSeqs) {
      bool bad = false, found;
      if (S <= 32) found = work_item<1, CTOK, KEYN>(p, S, jw, lane, &s, &z, &bad);
      else if (S <= 64) found = work_item<2, CTOK, KEYN>(p, S, jw, lane, &s, &z, &bad);
      else if (S <= 128) found = work_item<4, CTOK, KEYN>(p, S, jw, lane, &s, &z, &bad);
      else found = work_item<8, CTOK, KEYN>(p, S, jw, lane, &s, &z, &bad);
      // a sequence with unusable arguments (among them n above the host bound,
      // whose rows would lie outside the grid) gets no items: flagged once
      if (bad && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);
      if (!found) return;
    } else {
      s = jw % S;
      z = jw / S;
    }
    q0 = __ldg(p.query_start + s);
    const int q1 = __ldg(p.query_start + s + 1);
    L = __ldg(p.context_lens + s);
    n = q1 - q0;
    if (!prefill_order::chunk_ok(q0, q1, L, p.total_q, p.max_query_len,
                                 static_cast<int64_t>(p.max_blocks_per_seq) * bs)) {
      if (threadIdx.x == 0 && h == 0 && z == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);
      return;
    }
    const int npairs = prefill_order::num_items(n, CTOK);
    if (z >= npairs) return;  // no rows of this sequence here
    tq0 = (npairs - 1 - z) * CTOK;
    const int ntok_all = min(CTOK, n - tq0);
    pos_last = L - n + tq0 + ntok_all - 1;  // <= L - 1
    nt = pos_last / KEYN + 1;               // key tiles to visit
    trow = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
  }
  if (smem_u32(sm) & 1023) {                         // the swizzled operand layout needs this
    if (threadIdx.x == 0) atomicOr(p.err, PA_DEVERR_CONTEXT);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(kQFull), 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar(kKVFull + i), 1);   // producer arrival + TMA bytes
      mbar_init(bar(kKVEmpty + i), 2);  // commits of both MMA issuers (S, then P V)
    }
    for (int i = 0; i < 2 * Cfg::kQT; ++i) {
      mbar_init(bar(kSFull + i), 1);    // MMA commit after S of the tile
      mbar_init(bar(kPFull + i), 128);  // every thread of the softmax warpgroup
      mbar_init(bar(kODone + i), 1);    // commit after P V of the tile
    }
    fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  auto t_s = [&](int x, int b) { return tmem + (2 * x + b) * KEYN; };
  auto t_o = [&](int x) { return tmem + 4 * KEYN + x * 128; };

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      mbar_arrive_expect_tx(bar(kQFull), Cfg::kQT * Cfg::kQBytes);
      for (int x = 0; x < Cfg::kQT; ++x) {
        tma_load_3d(q_s(x), &q_map, 0, h * G, q0 + tq0 + x * TOK, bar(kQFull));
        tma_load_3d(q_s(x) + QHALF, &q_map, 64, h * G, q0 + tq0 + x * TOK, bar(kQFull));
      }
    }
    const int rows = bs < KEYN ? bs : KEYN;  // tokens per box
    for (int j = 0; j < nt; ++j) {
      const int st = j % NS, u = j / NS;
      if (u >= 1) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(bar(kKVEmpty + st), (u - 1) & 1, p.err);
        if (!__shfl_sync(kFullMask, ok, 0)) break;
      }
      const int key0 = key_lo + j * KEYN;
      const int nkeys = min(KEYN, L - key0);
      const int nbox = (nkeys + rows - 1) / rows;  // boxes holding this tile's keys (<= 8)
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
        tma_load_4d(dk + KVHALF, &k_map, 64, off, h, blk, bar(kKVFull + st));
        tma_load_4d(dv, &v_map, 0, off, h, blk, bar(kKVFull + st));
        tma_load_4d(dv + KVHALF, &v_map, 64, off, h, blk, bar(kKVFull + st));
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- S = Q K^T MMAs
    // A tcgen05.mma issue blocks while the tensor pipe's queue is full, so the
    // S and P V MMAs come from two warps: a ready P V never waits behind a
    // batch of S. Tile j + 2's S reuses the tensor-memory buffers of tile j once
    // both P V of tile j are done: P is stored over the S it was computed from.
    constexpr uint32_t kIdS = tc::idesc_bf16_f32(128, KEYN, 0);  // B = K rows (K-major)
    auto issue_s = [&](int j) {  // S_x = Q_x K_j^T for both query tiles
      const uint32_t kb = k_s(j % NS);
#pragma unroll
      for (int x = 0; x < Cfg::kQT; ++x) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks & 3) * 32;
          tc::mma_bf16(t_s(x, j & 1), tc::smem_desc_sw128(q_s(x) + (ks >> 2) * QHALF + off, 16, 1024),
                       tc::smem_desc_sw128(kb + (ks >> 2) * KVHALF + off, 16, 1024), kIdS, ks > 0);
        }
        tc::commit(bar(kSFull + 2 * x + (j & 1)));
      }
      tc::commit(bar(kKVEmpty + j % NS));  // K of tile j read (first of two commits)
    };
    bool ok = wait_all(bar(kQFull), 0);
    for (int j = 0; j < nt && ok; ++j) {
      if (j >= 2) {
        for (int x = 0; x < Cfg::kQT && ok; ++x)
          ok = wait_all(bar(kODone + 2 * x + (j & 1)), ((j - 2) >> 1) & 1);
        if (!ok) break;
      }
      if (!wait_all(bar(kKVFull + j % NS), (j / NS) & 1)) break;
      tc::fence_after_sync();
      if (lane == 0) issue_s(j);
      __syncwarp();
    }
  } else if (warp == 2 + 4 * Cfg::kQT) {
    // ------------------------------------------------------------ P V MMAs
    constexpr uint32_t kIdPV = tc::idesc_bf16_f32(128, 128, 1);  // B = V rows (MN-major)
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      const uint32_t vb = v_s(j % NS);
      for (int x = 0; x < Cfg::kQT && ok; ++x) {
        if (!wait_all(bar(kPFull + 2 * x + (j & 1)), (j >> 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (lane == 0) {
          // A = P from tensor memory (16 keys = 8 columns per k-step)
#pragma unroll
          for (int ks = 0; ks < KEYN / 16; ++ks)
            tc::mma_bf16_tmem_a(t_o(x), t_s(x, j & 1) + ks * 8,
                                tc::smem_desc_sw128(vb + ks * 2048, KVHALF, 1024), kIdPV,
                                j > 0 || ks > 0);
          tc::commit(bar(kODone + 2 * x + (j & 1)));
        }
      }
      if (ok && lane == 0) tc::commit(bar(kKVEmpty + j % NS));  // V of tile j read
      __syncwarp();
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int x = (warp - 2) >> 2;  // query tile of this warpgroup
    const int wq = warp & 3;        // this warp reaches tensor-memory lanes 32 wq .. 32 wq + 31
    const int r = wq * 32 + lane;
    const int tok = r / G, g = r - (r / G) * G;
    const int tx0 = tq0 + x * TOK;                  // first token of this query tile
    const int ntok = max(0, min(TOK, n - tx0));     // valid tokens of this query tile
    // position of its first token, and the last key visible to this row (every
    // row sees the whole key range in the shared-prefix mode)
    const int pos0 = PREFIX ? pos_last : min(L - n + tx0, pos_last);
    const int prow = PREFIX ? pos_last : (tok < ntok ? pos0 + tok : pos_last);
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float qs = p.q_scale;
    float m_use = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      if (!wait_all(bar(kSFull + 2 * x + (j & 1)), (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t sv[2][32];
      tc::ld32(t_s(x, j & 1) + lane_off, sv[0]);
      tc::ld32(t_s(x, j & 1) + lane_off + 32, sv[1]);
      tc::wait_ld();
      // the row maximum of the raw scores (scale > 0), masking only tiles that
      // reach past some row's position
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      const int key0 = key_lo + j * KEYN;
      if (key0 + KEYN - 1 <= pos0) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(sv[c][i]));
      } else {
        const int lim = prow - key0;  // keys 0 .. lim of this tile are visible
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float v = c * 32 + i <= lim ? __uint_as_float(sv[c][i]) : -INFINITY;
            sv[c][i] = __float_as_uint(v);
            mx4[i & 3] = fmaxf(mx4[i & 3], v);
          }
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * qs;
      // key 0 is visible to every row, so m_use is finite from the first tile on;
      // a row whose keys of this tile are all masked has mx = -inf and keeps m_use
      const bool move = mx > m_use + 8.0f;
      const float m_new = move ? mx : m_use;
      const float alpha = move ? ex2_approx(m_use - m_new) : 1.0f;  // 0 on the first tile
      // P = 2^(score * scale - m) as bf16 pairs, computed while the previous P V runs
      float rs0 = 0.0f, rs1 = 0.0f;
      uint32_t pw[KEYN / 2];
#pragma unroll
      for (int e = 0; e < KEYN / 2; ++e) {
        const int i0 = 2 * e;
        const float a = ex2_approx(fmaf(__uint_as_float(sv[i0 >> 5][i0 & 31]), qs, -m_new));
        const float b =
            ex2_approx(fmaf(__uint_as_float(sv[(i0 + 1) >> 5][(i0 + 1) & 31]), qs, -m_new));
        rs0 += a;
        rs1 += b;
        pw[e] = pack_bf16x2(a, b);
      }
      l_run = l_run * alpha + (rs0 + rs1);
      m_use = m_new;
      // The previous P V (tile j - 1) must be done before O is rescaled: wait
      // for it here only when some row of this warp moved its reference;
      // otherwise P is published first and the wait comes after, so this tile's
      // P V can follow the previous one at once. Either way every tile waits
      // once, before the next tile's P, which keeps this warp within one
      // phase of the barrier pair.
      const bool rescale = j > 0 && __any_sync(kFullMask, alpha != 1.0f);
      if (rescale) {
        if (!wait_all(bar(kODone + 2 * x + ((j - 1) & 1)), ((j - 1) >> 1) & 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tc::ld32(t_o(x) + lane_off + c * 32, ov);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tc::st32(t_o(x) + lane_off + c * 32, ov);
        }
      }
      // P (bf16 pairs, the lower key in the low half) over the first KEYN / 2
      // columns of this tile's S, which this thread has read: the A operand of
      // the P V MMA, from tensor memory
      tc::st32(t_s(x, j & 1) + lane_off, pw);
      tc::wait_st();
      if (x == 0 && j == nt - 1) {
        // keys past the context in the last tile: stale or unwritten V rows become
        // zeros (their P is 0, but 0 * NaN would not be); both P V of the tile
        // are issued after this warpgroup's P is published
        const int nkeys = L - key0;
        if (nkeys < KEYN) {
          const uint32_t vb = v_s(j % NS);
          for (int i = r; i < (KEYN - nkeys) * 16; i += 128) {
            const int row = nkeys + (i >> 4), c = i & 15;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                             vb + (c >> 3) * KVHALF + row * 128 + ((c & 7) << 4)),
                         "r"(0u)
                         : "memory");
          }
          // generic-proxy writes before the MMA's async-proxy reads
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
      }
      tc::fence_before_sync();
      mbar_arrive(bar(kPFull + 2 * x + (j & 1)));
      if (j > 0 && !rescale) {
        if (!wait_all(bar(kODone + 2 * x + ((j - 1) & 1)), ((j - 1) >> 1) & 1)) {
          ok = false;
          break;
        }
      }
    }
    if (PREFIX && ok && wait_all(bar(kODone + 2 * x + ((nt - 1) & 1)), ((nt - 1) >> 1) & 1)) {
      // the row's partial result over this key partition, for the decode merge
      tc::fence_after_sync();
      const int64_t row =
          (static_cast<int64_t>(tx0 + tok) * p.num_heads + h * G + g) * p.ws_slots + kpart;
      if (tok < ntok) {
        p.ws_m[row] = m_use;
        p.ws_l[row] = l_run;
      }
      float* dst = p.ws_acc + row * Cfg::kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tc::ld32(t_o(x) + lane_off + c * 32, ov);
        tc::wait_ld();
        if (tok < ntok) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *reinterpret_cast<uint4*>(dst + c * 32 + v * 4) =
                make_uint4(ov[4 * v], ov[4 * v + 1], ov[4 * v + 2], ov[4 * v + 3]);
        }
      }
    } else if (!PREFIX && ok &&
               wait_all(bar(kODone + 2 * x + ((nt - 1) & 1)), ((nt - 1) >> 1) & 1)) {
      tc::fence_after_sync();
      const float inv = 1.0f / l_run;
      __nv_bfloat16* dst = p.out + ((static_cast<int64_t>(q0) + tx0 + tok) * p.num_heads +
                                    h * G + g) * Cfg::kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tc::ld32(t_o(x) + lane_off + c * 32, ov);
        tc::wait_ld();
        if (tok < ntok) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[8 * v]) * inv, __uint_as_float(ov[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ov[8 * v + 2]) * inv, __uint_as_float(ov[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ov[8 * v + 4]) * inv, __uint_as_float(ov[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ov[8 * v + 6]) * inv, __uint_as_float(ov[8 * v + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + c * 32 + v * 8) = w;
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

template <int G, bool PREFIX>
cudaError_t launch_prefill_g(const PrefillParams& p, const void* q, const void* k_cache,
                             const void* v_cache, int64_t ctas, cudaStream_t stream) {
  using Cfg = PrefillConfig<G>;
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev % 64);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(pa_prefill_kernel<G, PREFIX>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared storage as shared memory (a per-kernel
    // preference, not a device setting)
    e = cudaFuncSetAttribute(pa_prefill_kernel<G, PREFIX>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  CUtensorMap qmap, kmap, vmap;
  const int rows = p.block_size < Cfg::kKeys ? p.block_size : Cfg::kKeys;
  if ((e = encode_q_map(&qmap, q, p.total_q, p.num_heads, G, Cfg::kTok)) != cudaSuccess) return e;
  if ((e = encode_kv_map(&kmap, k_cache, p.num_blocks, p.block_size, p.num_kv_heads, rows)) !=
      cudaSuccess)
    return e;
  if ((e = encode_kv_map(&vmap, v_cache, p.num_blocks, p.block_size, p.num_kv_heads, rows)) !=
      cudaSuccess)
    return e;
  if (ctas <= 0) return cudaSuccess;
  if (ctas > 0x7fffffff) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa_prefill_kernel<G, PREFIX>, qmap, kmap, vmap, p);
}

template <bool PREFIX>
cudaError_t dispatch_prefill(const PrefillParams& p, const void* q, const void* k_cache,
                             const void* v_cache, int64_t ctas, cudaStream_t stream) {
  switch (p.num_heads / p.num_kv_heads) {
    case 1: return launch_prefill_g<1, PREFIX>(p, q, k_cache, v_cache, ctas, stream);
    case 2: return launch_prefill_g<2, PREFIX>(p, q, k_cache, v_cache, ctas, stream);
    case 4: return launch_prefill_g<4, PREFIX>(p, q, k_cache, v_cache, ctas, stream);
    case 8: return launch_prefill_g<8, PREFIX>(p, q, k_cache, v_cache, ctas, stream);
    default: return cudaErrorNotSupported;
  }
}

PrefillParams common_params(int num_heads, int num_kv_heads, int block_size, int num_blocks,
                            int max_blocks_per_seq, float scale) {
  PrefillParams p{};
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  int lg = 0;
  while ((1 << lg) < block_size) ++lg;
  p.log2_block_size = lg;
  p.num_blocks = num_blocks;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.q_scale = scale * 1.4426950408889634f;  // log2(e)
  return p;
}

}  // namespace

cudaError_t launch_prefill(const PrefillShape& sh, void* out, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, const int32_t* query_start,
                           cudaStream_t stream) {
  if (sh.max_query_len <= 0 || sh.num_seqs <= 0) return cudaSuccess;
  PrefillParams p = common_params(sh.num_heads, sh.num_kv_heads, sh.block_size, sh.num_blocks,
                                  sh.max_blocks_per_seq, sh.scale);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start = query_start;
  cudaError_t e = device_error_word(&p.err);
  if (e != cudaSuccess) return e;
  p.num_seqs = sh.num_seqs;
  p.total_q = sh.total_q;
  p.max_query_len = sh.max_query_len;
  // work indices: every sequence could have max_query_len rows; those past
  // the last item exit at once (they are dispatched last). A planned call's
  // list has exactly the items that hold rows.
  const int tok = 2 * (128 / (sh.num_heads / sh.num_kv_heads));  // query tokens per CTA
  int64_t items = static_cast<int64_t>(sh.num_seqs) * ((sh.max_query_len + tok - 1) / tok);
  if (sh.work != nullptr) {
    p.work = sh.work;
    items = sh.num_items;
  }
  return dispatch_prefill<false>(p, q, k_cache, v_cache, items * sh.num_kv_heads, stream);
}

cudaError_t launch_prefix_attention(int num_seqs, int num_heads, int num_kv_heads, int block_size,
                                    int num_blocks, int max_blocks_per_seq, int prefix_len,
                                    int prefix_part, float scale, const void* q,
                                    const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, float* ws_m, float* ws_l,
                                    float* ws_acc, int ws_slots, cudaStream_t stream) {
  PrefillParams p = common_params(num_heads, num_kv_heads, block_size, num_blocks,
                                  max_blocks_per_seq, scale);
  p.block_tables = block_tables;
  cudaError_t e = device_error_word(&p.err);
  if (e != cudaSuccess) return e;
  p.num_seqs = num_seqs;
  p.total_q = num_seqs;
  p.max_query_len = num_seqs;
  p.prefix_keys = prefix_len;
  p.prefix_part = prefix_part;
  p.prefix_parts = (prefix_len + prefix_part - 1) / prefix_part;
  p.ws_slots = ws_slots;
  p.ws_m = ws_m;
  p.ws_l = ws_l;
  p.ws_acc = ws_acc;
  const int tok = 2 * (128 / (num_heads / num_kv_heads));
  const int64_t pairs = (static_cast<int64_t>(num_seqs) + tok - 1) / tok;
  return dispatch_prefill<true>(p, q, k_cache, v_cache,
                                static_cast<int64_t>(num_kv_heads) * p.prefix_parts * pairs,
                                stream);
}

}  // namespace pa
