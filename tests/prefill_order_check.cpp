// Host check of pa_prefill's work-item arithmetic (csrc/pa_prefill_order.h).
//
// 1. items_at_least(c) equals the brute-force count of items whose cost is at
//    least c, cost never grows with z, and last_key matches the causal bound
//    (item 0 sees the last cached key, the last item the chunk's first rows).
// 2. The compact per-sequence form (item_costs) gives the same counts.
// 3. The kernel's search (cost level by bisection over per-lane counts, then
//    the prefix over lanes 32k .. 32k + 31), replayed here lane by lane, maps
//    the work indices 0 .. items-1 one to one onto the items sorted by cost
//    downward, then sequence, then z; indices past the end find nothing.
// Prints "ok" and exits 0, else prints the first failure and exits 1.
#include <algorithm>
#include <cstdio>
#include <random>
#include <tuple>
#include <vector>

#include "pa_prefill_order.h"

namespace po = pa::prefill_order;

static int fail(const char* what, long a, long b, long c) {
  std::printf("FAIL %s %ld %ld %ld\n", what, a, b, c);
  return 1;
}

struct Seq { int L, n, items; };

static int lg(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

// The device search with the 32 lanes played one after another.
static bool search(const std::vector<Seq>& seqs, int j, int ctok, int keyn, int* s, int* z) {
  const int S = static_cast<int>(seqs.size());
  const int per = (S + 31) / 32;
  // as on the device: three numbers per sequence, held by its lane
  std::vector<po::ItemCosts> qc(32 * per, po::ItemCosts{0, 0, 0});
  for (int t = 0; t < S; ++t) qc[t] = po::item_costs(seqs[t].L, seqs[t].n, ctok, keyn);
  auto cnt = [&](int t, int c) { return po::items_at_least(qc[t], c, lg(ctok), keyn); };
  auto count = [&](int c) {
    long acc = 0;
    for (int t = 0; t < S; ++t) acc += cnt(t, c);
    return static_cast<int>(acc);
  };
  int cmax = 0;
  for (const po::ItemCosts& q : qc) cmax = std::max(cmax, q.top);
  if (cmax == 0 || j >= count(1)) return false;
  int lo = 1, hi = cmax + 1;
  while (hi - lo > 1) {
    const int mid = lo + ((hi - lo) >> 1);
    if (count(mid) > j) lo = mid;
    else hi = mid;
  }
  int o = j - count(lo + 1);
  for (int k = 0; k < per; ++k) {
    int incl[32], above[32], e[32];
    for (int lane = 0; lane < 32; ++lane) {
      above[lane] = cnt(32 * k + lane, lo + 1);
      e[lane] = cnt(32 * k + lane, lo) - above[lane];
      incl[lane] = e[lane] + (lane ? incl[lane - 1] : 0);
    }
    if (o < incl[31]) {
      int src = 0;
      while (!(incl[src] > o)) ++src;
      *z = above[src] + o - (incl[src] - e[src]);
      *s = 32 * k + src;
      return true;
    }
    o -= incl[31];
  }
  return false;
}

int main() {
  std::mt19937 rng(12345);
  const int keyn = 64;
  const int ctoks[] = {32, 64, 128, 256};  // query rows per item for groups 8, 4, 2, 1
  // 1. per-sequence counts against brute force
  for (int ctok : ctoks) {
    for (int trial = 0; trial < 4000; ++trial) {
      const int L = trial < 40 ? trial : static_cast<int>(rng() % 9000);
      const int n = L == 0 ? 0 : (trial % 3 == 0 ? L : static_cast<int>(rng() % (L + 1)));
      const int items = po::num_items(n, ctok);
      if (items > 0) {
        if (po::last_key(L, n, 0, ctok) != L - 1) return fail("last_key(0)", L, n, ctok);
        if (po::last_key(L, n, items - 1, ctok) != L - n + std::min(ctok, n) - 1)
          return fail("last_key(last)", L, n, ctok);
      }
      for (int z = 1; z < items; ++z)
        if (po::cost(L, n, z, ctok, keyn) > po::cost(L, n, z - 1, ctok, keyn))
          return fail("cost grows", L, n, z);
      const int top = items ? po::cost(L, n, 0, ctok, keyn) : 1;
      for (int c = 1; c <= top + 2; ++c) {
        int brute = 0;
        for (int z = 0; z < items; ++z) brute += po::cost(L, n, z, ctok, keyn) >= c;
        if (po::items_at_least(L, n, items, c, ctok, keyn) != brute)
          return fail("items_at_least", L, n, c);
        if (po::items_at_least(po::item_costs(L, n, ctok, keyn), c, lg(ctok), keyn) != brute)
          return fail("items_at_least (compact)", L, n, c);
      }
    }
  }
  // 2. the search is a bijection onto the longest-first order
  for (int ctok : ctoks) {
    for (int trial = 0; trial < 300; ++trial) {
      const int S = 1 + static_cast<int>(rng() % (trial < 200 ? 40 : 256));
      std::vector<Seq> seqs(S);
      std::vector<std::tuple<int, int, int>> order;  // (-cost, s, z)
      for (int t = 0; t < S; ++t) {
        const int L = static_cast<int>(rng() % (trial % 2 ? 5000 : 300));
        const int n = L == 0 || rng() % 5 == 0 ? 0 : static_cast<int>(rng() % (L + 1));
        seqs[t] = {L, n, po::num_items(n, ctok)};
        for (int z = 0; z < seqs[t].items; ++z)
          order.emplace_back(-po::cost(L, n, z, ctok, keyn), t, z);
      }
      std::sort(order.begin(), order.end());
      const int total = static_cast<int>(order.size());
      for (int j = 0; j < total + 3; ++j) {
        int s = -1, z = -1;
        const bool found = search(seqs, j, ctok, keyn, &s, &z);
        if (j >= total) {
          if (found) return fail("found past the end", j, total, ctok);
          continue;
        }
        if (!found) return fail("not found", j, total, ctok);
        if (s != std::get<1>(order[j]) || z != std::get<2>(order[j]))
          return fail("order", j, s, z);
      }
    }
  }
  std::printf("ok\n");
  return 0;
}
