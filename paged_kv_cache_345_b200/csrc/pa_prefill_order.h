// Work items of pa_prefill and the cost that orders them (host and device).
//
// A work item is one CTA's share of a sequence's chunk: `ctok` consecutive
// query rows (two query tiles), counted from the end of the chunk, so item
// z = 0 holds the chunk's last rows. Item z of a sequence with L cached
// tokens (its chunk's own included) and n query rows visits the key tiles
// 0 .. last(z) / keyn, where last(z) is the position of the last key its
// rows may see (causal attention). Its cost is that number of key tiles.
// The kernel hands items out longest first, which bounds the launch's tail:
// for a chunk on top of a long cached prefix every item of that sequence is
// expensive, and it must not be the last thing to start.
#pragma once

#include <cstdint>

#ifdef __CUDACC__
#define PA_ORDER_FN __host__ __device__ __forceinline__
#else
#define PA_ORDER_FN inline
#endif

namespace pa {
namespace prefill_order {

// Whether a sequence's arguments describe a chunk the kernel can run: rows
// [q0, q1) inside the batch, at most max_query_len of them (the grid was
// sized for that), no more rows than cached tokens, and a context that fits
// its block-table row.
PA_ORDER_FN bool chunk_ok(int q0, int q1, int L, int total_q, int max_query_len,
                          int64_t max_keys) {
  const int n = q1 - q0;
  return q0 >= 0 && q1 <= total_q && n >= 0 && n <= max_query_len && L >= n &&
         static_cast<int64_t>(L) <= max_keys;
}

PA_ORDER_FN int num_items(int n, int ctok) { return (n + ctok - 1) / ctok; }

// Position of the last key visible to item z's rows (z < num_items).
PA_ORDER_FN int64_t last_key(int L, int n, int z, int ctok) {
  const int items = num_items(n, ctok);
  const int64_t first_row = static_cast<int64_t>(items - 1 - z) * ctok;  // from the chunk start
  const int64_t rows = n - first_row < ctok ? n - first_row : ctok;
  return static_cast<int64_t>(L) - n + first_row + rows - 1;
}

// Key tiles item z visits.
PA_ORDER_FN int cost(int L, int n, int z, int ctok, int keyn) {
  return static_cast<int>(last_key(L, n, z, ctok) / keyn) + 1;
}

// Items of the chunk whose cost is at least c (c >= 1). Cost does not grow
// with z, so these are items 0 .. result-1. Item 0 sees key L - 1; item
// z >= 1 sees key L - r - 1 - (z - 1) * ctok, r = rows of item 0.
PA_ORDER_FN int items_at_least(int L, int n, int items, int c, int ctok, int keyn) {
  if (items <= 0) return 0;
  const int64_t t = static_cast<int64_t>(c - 1) * keyn;  // first key of tile c - 1
  if (static_cast<int64_t>(L) - 1 < t) return 0;
  const int64_t r = n - static_cast<int64_t>(items - 1) * ctok;
  const int64_t d = static_cast<int64_t>(L) - r - 1 - t;
  if (d < 0) return 1;
  const int64_t more = d / ctok + 1;
  return 1 + static_cast<int>(more < items - 1 ? more : items - 1);
}

// The same count from three numbers per sequence, taken once: the cost of
// item 0 (0 when the chunk has no rows), the last key visible to item 1, and
// the number of items. All in int32 (c never exceeds top here, so
// (c - 1) * keyn <= L - 1); ctok is a power of two, given as its log2.
struct ItemCosts {
  int top, key1, items;
};

PA_ORDER_FN ItemCosts item_costs(int L, int n, int ctok, int keyn) {
  ItemCosts q;
  q.items = num_items(n, ctok);
  q.top = q.items > 0 ? (L - 1) / keyn + 1 : 0;
  q.key1 = q.items > 0 ? L - (n - (q.items - 1) * ctok) - 1 : 0;
  return q;
}

PA_ORDER_FN int items_at_least(const ItemCosts& q, int c, int log2_ctok, int keyn) {
  if (c > q.top) return 0;
  const int d = q.key1 - (c - 1) * keyn;
  if (d < 0) return 1;
  const int more = (d >> log2_ctok) + 1;
  return 1 + (more < q.items - 1 ? more : q.items - 1);
}

}  // namespace prefill_order
}  // namespace pa
