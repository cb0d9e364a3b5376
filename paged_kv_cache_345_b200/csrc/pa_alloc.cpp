// Host block allocator and block manager behind the C ABI in pa.h.
//
// Pool: a LIFO stack of free physical block ids plus a reference count per
// block ("What is paged attention in vLLM, and why does it matter?", Step 3:
// the block manager keeps the block table beside a pool of free blocks and a
// reference count per block). Sequences: a block table (physical ids in token
// order) and a token count. A block is taken only when the tail block is full
// (Step 4); forked sequences share blocks by reference count and a shared tail
// block is copied before one sharer writes into it ("PagedAttention — AI
// Glossary", How it works, steps 4 and 5).

#include <algorithm>
#include <cstdint>
#include <new>
#include <string>
#include <utility>
#include <unordered_map>
#include <vector>

#include "pa.h"
#include "pa_internal.h"

struct pa_alloc {
  std::vector<int32_t> free_stack;  // top = back()
  std::vector<int32_t> refcount;
};

namespace {

struct Seq {
  bool live = false;
  int64_t length = 0;
  std::vector<int32_t> blocks;
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool valid_id(const pa_alloc* a, int32_t id) {
  return id >= 0 && static_cast<size_t>(id) < a->refcount.size();
}

}  // namespace

struct pa_bm {
  pa_alloc* pool = nullptr;
  int block_size = 0;
  std::vector<Seq> seqs;
  std::vector<int32_t> free_ids;  // reusable sequence ids

  Seq* get(int32_t id) {
    if (id < 0 || static_cast<size_t>(id) >= seqs.size() || !seqs[id].live) return nullptr;
    return &seqs[id];
  }
  const Seq* get(int32_t id) const {
    if (id < 0 || static_cast<size_t>(id) >= seqs.size() || !seqs[id].live) return nullptr;
    return &seqs[id];
  }
  int32_t new_id() {
    if (!free_ids.empty()) {
      int32_t id = free_ids.back();
      free_ids.pop_back();
      return id;
    }
    seqs.emplace_back();
    return static_cast<int32_t>(seqs.size() - 1);
  }
};

extern "C" {

// ------------------------------------------------------------------- allocator

pa_alloc* pa_alloc_create(int num_blocks) {
  if (num_blocks <= 0) {
    pa_set_error("pa_alloc_create: num_blocks must be > 0, got %d", num_blocks);
    return nullptr;
  }
  pa_alloc* a = new (std::nothrow) pa_alloc;
  if (!a) return nullptr;
  try {
    a->refcount.assign(num_blocks, 0);
    a->free_stack.resize(num_blocks);
    for (int i = 0; i < num_blocks; ++i) a->free_stack[i] = num_blocks - 1 - i;
  } catch (...) {
    delete a;
    pa_set_error("pa_alloc_create: out of host memory");
    return nullptr;
  }
  return a;
}

void pa_alloc_destroy(pa_alloc* a) { delete a; }

int pa_alloc_block(pa_alloc* a, int32_t* out_id) {
  if (!a || !out_id) return pa_fail(PA_ERR_INVALID, "pa_alloc_block: null argument");
  if (a->free_stack.empty()) return pa_fail(PA_ERR_NO_BLOCKS, "pa_alloc_block: pool exhausted");
  int32_t b = a->free_stack.back();
  a->free_stack.pop_back();
  a->refcount[b] = 1;
  *out_id = b;
  return PA_OK;
}

int pa_incref(pa_alloc* a, int32_t id) {
  if (!a || !valid_id(a, id)) return pa_fail(PA_ERR_INVALID, "pa_incref: bad block id %d", id);
  if (a->refcount[id] == 0) return pa_fail(PA_ERR_INVALID, "pa_incref: block %d is free", id);
  a->refcount[id] += 1;
  return PA_OK;
}

int pa_decref(pa_alloc* a, int32_t id) {
  if (!a || !valid_id(a, id)) return pa_fail(PA_ERR_INVALID, "pa_decref: bad block id %d", id);
  if (a->refcount[id] == 0)
    return pa_fail(PA_ERR_INVALID, "pa_decref: block %d is already free", id);
  if (--a->refcount[id] == 0) a->free_stack.push_back(id);
  return PA_OK;
}

int pa_refcount(const pa_alloc* a, int32_t id) {
  if (!a || !valid_id(a, id)) return -1;
  return a->refcount[id];
}

int pa_num_free(const pa_alloc* a) { return a ? static_cast<int>(a->free_stack.size()) : -1; }

int pa_num_blocks(const pa_alloc* a) { return a ? static_cast<int>(a->refcount.size()) : -1; }

int pa_alloc_set_free_order(pa_alloc* a, const int32_t* ids, int n) {
  if (!a || (n > 0 && !ids)) return pa_fail(PA_ERR_INVALID, "pa_alloc_set_free_order: null argument");
  if (static_cast<size_t>(n) != a->free_stack.size())
    return pa_fail(PA_ERR_INVALID, "pa_alloc_set_free_order: %d ids for %zu free blocks", n,
                   a->free_stack.size());
  std::vector<char> seen;
  try {
    seen.assign(a->refcount.size(), 0);
  } catch (...) {
    return pa_fail(PA_ERR_INVALID, "pa_alloc_set_free_order: out of host memory");
  }
  for (int i = 0; i < n; ++i) {
    int32_t b = ids[i];
    if (!valid_id(a, b) || a->refcount[b] != 0 || seen[b])
      return pa_fail(PA_ERR_INVALID, "pa_alloc_set_free_order: id %d is not a distinct free block", b);
    seen[b] = 1;
  }
  for (int i = 0; i < n; ++i) a->free_stack[i] = ids[n - 1 - i];
  return PA_OK;
}

// --------------------------------------------------------------- block manager

pa_bm* pa_bm_create(int num_blocks, int block_size) {
  if (block_size <= 0) {
    pa_set_error("pa_bm_create: block_size must be > 0, got %d", block_size);
    return nullptr;
  }
  pa_alloc* pool = pa_alloc_create(num_blocks);
  if (!pool) return nullptr;
  pa_bm* bm = new (std::nothrow) pa_bm;
  if (!bm) {
    pa_alloc_destroy(pool);
    return nullptr;
  }
  bm->pool = pool;
  bm->block_size = block_size;
  return bm;
}

void pa_bm_destroy(pa_bm* bm) {
  if (!bm) return;
  pa_alloc_destroy(bm->pool);
  delete bm;
}

pa_alloc* pa_bm_allocator(pa_bm* bm) { return bm ? bm->pool : nullptr; }

int pa_bm_block_size(const pa_bm* bm) { return bm ? bm->block_size : -1; }

int pa_bm_add_seq(pa_bm* bm, int32_t* seq_id) {
  if (!bm || !seq_id) return pa_fail(PA_ERR_INVALID, "pa_bm_add_seq: null argument");
  int32_t id;
  try {
    id = bm->new_id();
  } catch (...) {
    return pa_fail(PA_ERR_INVALID, "pa_bm_add_seq: out of host memory");
  }
  Seq& s = bm->seqs[id];
  s.live = true;
  s.length = 0;
  s.blocks.clear();
  *seq_id = id;
  return PA_OK;
}

int pa_bm_fork(pa_bm* bm, int32_t parent, int32_t* child) {
  if (!bm || !child) return pa_fail(PA_ERR_INVALID, "pa_bm_fork: null argument");
  if (!bm->get(parent)) return pa_fail(PA_ERR_INVALID, "pa_bm_fork: unknown sequence %d", parent);
  // Everything that can fail to allocate comes before the first change.
  std::vector<int32_t> blocks;
  int32_t id;
  try {
    blocks = bm->seqs[parent].blocks;
    id = bm->new_id();  // may grow seqs: index the parent again afterwards
  } catch (...) {
    return pa_fail(PA_ERR_INVALID, "pa_bm_fork: out of host memory");
  }
  const Seq& p = bm->seqs[parent];
  Seq& c = bm->seqs[id];
  for (int32_t b : blocks) bm->pool->refcount[b] += 1;
  c.live = true;
  c.length = p.length;
  c.blocks = std::move(blocks);
  *child = id;
  return PA_OK;
}

int pa_bm_free_seq(pa_bm* bm, int32_t seq_id) {
  if (!bm) return pa_fail(PA_ERR_INVALID, "pa_bm_free_seq: null manager");
  Seq* s = bm->get(seq_id);
  if (!s) return pa_fail(PA_ERR_INVALID, "pa_bm_free_seq: unknown sequence %d", seq_id);
  try {
    bm->free_ids.reserve(bm->free_ids.size() + 1);  // the push below cannot fail then
  } catch (...) {
    return pa_fail(PA_ERR_INVALID, "pa_bm_free_seq: out of host memory");
  }
  for (int32_t b : s->blocks) pa_decref(bm->pool, b);
  s->live = false;
  s->length = 0;
  s->blocks.clear();
  bm->free_ids.push_back(seq_id);
  return PA_OK;
}

int pa_bm_seq_len(const pa_bm* bm, int32_t seq_id) {
  const Seq* s = bm ? bm->get(seq_id) : nullptr;
  return s ? static_cast<int>(s->length) : -1;
}

int pa_bm_seq_num_blocks(const pa_bm* bm, int32_t seq_id) {
  const Seq* s = bm ? bm->get(seq_id) : nullptr;
  return s ? static_cast<int>(s->blocks.size()) : -1;
}

int pa_bm_append_slots(pa_bm* bm, const int32_t* seq_ids, const int32_t* counts, int n,
                       int64_t* slot_mapping, int64_t* cow_pairs, int cow_capacity,
                       int* num_cow) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !counts)) || !num_cow)
    return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: null or negative argument");
  // Validate everything and count what is needed before changing anything.
  int64_t need = 0, total = 0, cows = 0;
  std::vector<int32_t> sorted;
  try {
    sorted.assign(seq_ids, seq_ids + n);
  } catch (...) {
    return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: out of host memory");
  }
  std::sort(sorted.begin(), sorted.end());
  if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end())
    return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: a sequence id appears twice");
  const int bs = bm->block_size;
  // The apply loop below works sequence by sequence: once one sharer of a
  // partly filled tail has copied it, the tail has one holder fewer, and the
  // last holder writes in place. Count the same way: `dropped` holds, per
  // shared tail, the holders that earlier sequences of this batch took away.
  std::unordered_map<int32_t, int32_t> dropped;
  try {
    for (int i = 0; i < n; ++i) {
      const Seq* s = bm->get(seq_ids[i]);
      if (!s)
        return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: unknown sequence %d", seq_ids[i]);
      if (counts[i] < 0) return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: negative count");
      if (counts[i] == 0) continue;
      need += ceil_div(s->length + counts[i], bs) - ceil_div(s->length, bs);
      total += counts[i];
      if (s->length % bs != 0) {
        const int32_t tail = s->blocks[s->length / bs];
        int32_t& gone = dropped[tail];
        if (bm->pool->refcount[tail] - gone > 1) {  // still shared when this sequence writes
          cows += 1;
          need += 1;
          gone += 1;
        }
      }
    }
  } catch (...) {
    return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: out of host memory");
  }
  if (total > 0 && !slot_mapping)
    return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: slot_mapping is null");
  if (cows > cow_capacity || (cows > 0 && !cow_pairs))
    return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: %lld copy-on-write pairs, capacity %d",
                   static_cast<long long>(cows), cow_capacity);
  if (need > static_cast<int64_t>(bm->pool->free_stack.size()))
    return pa_fail(PA_ERR_NO_BLOCKS, "pa_bm_append_slots: need %lld blocks, %zu free",
                   static_cast<long long>(need), bm->pool->free_stack.size());
  // Room for every new table entry first, so that the loop below cannot fail
  // half-way (reserving changes no table).
  try {
    for (int i = 0; i < n; ++i) {
      Seq& s = *bm->get(seq_ids[i]);
      s.blocks.reserve(static_cast<size_t>(ceil_div(s.length + counts[i], bs)));
    }
  } catch (...) {
    return pa_fail(PA_ERR_INVALID, "pa_bm_append_slots: out of host memory");
  }

  int64_t k = 0;
  int ncow = 0;
  for (int i = 0; i < n; ++i) {
    Seq& s = *bm->get(seq_ids[i]);
    for (int32_t c = 0; c < counts[i]; ++c) {
      const int64_t lb = s.length / bs, off = s.length % bs;
      int32_t fresh;
      if (off == 0) {
        pa_alloc_block(bm->pool, &fresh);  // cannot fail: counted above
        s.blocks.push_back(fresh);
      } else if (bm->pool->refcount[s.blocks[lb]] > 1) {
        const int32_t shared = s.blocks[lb];
        pa_alloc_block(bm->pool, &fresh);
        pa_decref(bm->pool, shared);
        s.blocks[lb] = fresh;
        cow_pairs[2 * ncow] = shared;
        cow_pairs[2 * ncow + 1] = fresh;
        ++ncow;
      }
      slot_mapping[k++] = static_cast<int64_t>(s.blocks[lb]) * bs + off;
      s.length += 1;
    }
  }
  *num_cow = ncow;
  return PA_OK;
}

int pa_bm_block_tables(const pa_bm* bm, const int32_t* seq_ids, int n, int32_t* tables,
                       int max_blocks_per_seq, int32_t* context_lens) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !tables)) || max_blocks_per_seq <= 0)
    return pa_fail(PA_ERR_INVALID, "pa_bm_block_tables: null or bad argument");
  for (int i = 0; i < n; ++i) {
    const Seq* s = bm->get(seq_ids[i]);
    if (!s) return pa_fail(PA_ERR_INVALID, "pa_bm_block_tables: unknown sequence %d", seq_ids[i]);
    if (s->blocks.size() > static_cast<size_t>(max_blocks_per_seq))
      return pa_fail(PA_ERR_INVALID, "pa_bm_block_tables: sequence %d holds %zu blocks > %d",
                     seq_ids[i], s->blocks.size(), max_blocks_per_seq);
  }
  for (int i = 0; i < n; ++i) {
    const Seq* s = bm->get(seq_ids[i]);
    int32_t* row = tables + static_cast<int64_t>(i) * max_blocks_per_seq;
    std::copy(s->blocks.begin(), s->blocks.end(), row);
    std::fill(row + s->blocks.size(), row + max_blocks_per_seq, 0);
    if (context_lens) context_lens[i] = static_cast<int32_t>(s->length);
  }
  return PA_OK;
}

}  // extern "C"
