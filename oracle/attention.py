"""Cache writes, decode and prefill attention in float64 (oracle, test infrastructure).

What the method computes. Paging changes where the KV cache lives, not the
arithmetic: "PagedAttention — AI Glossary" (modelrefs.com), "Example: Where the
wasted memory actually was", says there is no change to the attention
mathematics, and "What is paged attention in vLLM, and why does it matter?",
"Common mistakes", says the same. "Paged Attention" (klaylearn.com glossary),
definition: the block table lets attention read a continuous context. So the
oracle is plain softmax attention over the logically contiguous context:

  1. gather: Kc[t] = k_cache[table[t // bs], t % bs] for t < L (same for V),
     upcast to float64;
  2. scores: x_t = scale * sum_i q[j, i] * Kc[t, h, i], with KV head h = j // G;
  3. softmax: w_t = exp(x_t - max x) / sum_u exp(x_u - max x);
  4. out[j] = sum_t w_t * Vc[t, h, :].

Readings where the pages are silent (they say nothing of grouped-query heads,
masks or dtypes): query head j reads KV head j // G with G = Hq / Hkv; no mask,
since the one decode query is the last position; a sequence with no cached
tokens yields zeros. Cache writes: the new token's K/V row goes to its flat
slot = physical block * bs + offset; a negative slot means "skip this row".
"""

from __future__ import annotations

import numpy as np

from . import blocks


def kv_head_of(j: int, group: int) -> int:
    """KV head read by query head j when `group` query heads share one KV head."""
    return j // group


def gather_context(cache: np.ndarray, block_table, length: int, block_size: int) -> np.ndarray:
    """[length, Hkv, d] float64: the tokens of one sequence in logical order.

    `cache` is [num_blocks, block_size, Hkv, d]; token t lives in physical block
    block_table[t // block_size] at offset t % block_size.
    """
    t = np.arange(length)
    logical_block, offset = blocks.logical_position(t, block_size)
    physical = np.asarray(block_table)[logical_block].astype(np.int64)
    return np.asarray(cache)[physical, offset].astype(np.float64)


def softmax_attention(q_vec: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float):
    """One query over contiguous keys/values ([L, d] each), float64, max-subtracted softmax."""
    q_vec = np.asarray(q_vec, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    x = scale * (keys @ q_vec)
    w = np.exp(x - x.max())
    w = w / w.sum()
    return w @ values


def decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, block_size: int):
    """Decode attention for a batch: out [S, Hq, d] float64.

    q: [S, Hq, d]; k_cache, v_cache: [num_blocks, block_size, Hkv, d];
    block_tables: [S, max_blocks] physical ids; context_lens: [S] tokens to attend.
    """
    q = np.asarray(q, dtype=np.float64)
    num_seqs, num_heads, head_dim = q.shape
    num_kv_heads = k_cache.shape[2]
    group = num_heads // num_kv_heads
    out = np.zeros((num_seqs, num_heads, head_dim), dtype=np.float64)
    for s in range(num_seqs):
        length = int(context_lens[s])
        if length == 0:
            continue
        keys = gather_context(k_cache, block_tables[s], length, block_size)
        values = gather_context(v_cache, block_tables[s], length, block_size)
        for j in range(num_heads):
            h = kv_head_of(j, group)
            out[s, j] = softmax_attention(q[s, j], keys[:, h, :], values[:, h, :], scale)
    return out


def kv_append(k_cache, v_cache, k_new, v_new, slot_mapping, block_size: int):
    """Copies of the caches with row i of k_new/v_new written at slot_mapping[i].

    Slot s is physical block s // block_size, offset s % block_size, i.e. row s
    of the cache viewed as [num_blocks * block_size, Hkv, d]. Rows with a
    negative slot are skipped; slots must be distinct.
    """
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    slots = np.asarray(slot_mapping, dtype=np.int64)
    keep = slots >= 0
    flat_k = k_out.reshape((-1,) + k_out.shape[2:])   # views: [num_blocks * bs, Hkv, d]
    flat_v = v_out.reshape((-1,) + v_out.shape[2:])
    flat_k[slots[keep]] = np.asarray(k_new)[keep]
    flat_v[slots[keep]] = np.asarray(v_new)[keep]
    return k_out, v_out


def copy_blocks(k_cache, v_cache, block_mapping):
    """Copies of the caches with block dst := block src for each (src, dst) pair.

    The copy-on-write step: only the block being written is copied
    ("PagedAttention — AI Glossary", How it works, step 5). Pairs are applied in
    order; callers keep source and destination sets disjoint.
    """
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    for src, dst in np.asarray(block_mapping).reshape(-1, 2).tolist():
        k_out[int(dst)] = k_out[int(src)]
        v_out[int(dst)] = v_out[int(src)]
    return k_out, v_out


def swap_blocks(dst_k, dst_v, src_k, src_v, block_mapping):
    """Copies of the destination pools with block dst := src-pool block src for
    each (src, dst) pair: moving whole blocks between a device pool and a host
    pool when a sequence is preempted and later resumed ("Paged Attention",
    klaylearn.com glossary, FAQ; "What is paged attention in vLLM...",
    Follow-up questions)."""
    k_out = np.array(dst_k, copy=True)
    v_out = np.array(dst_v, copy=True)
    for src, dst in np.asarray(block_mapping).reshape(-1, 2).tolist():
        k_out[int(dst)] = src_k[int(src)]
        v_out[int(dst)] = src_v[int(src)]
    return k_out, v_out


def chunk_positions(length: int, n: int) -> np.ndarray:
    """Absolute positions of a sequence's last n tokens (its query chunk)."""
    return length - n + np.arange(n)


def causal_visible(length: int, positions: np.ndarray) -> np.ndarray:
    """[n, length] mask: row i sees key t iff t <= positions[i]."""
    return np.arange(length)[None, :] <= np.asarray(positions)[:, None]


def prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale: float,
            block_size: int):
    """Causal attention of a chunk of new queries per sequence over its paged
    context (chunked prefill; a whole prompt is the chunk that starts at 0).

    "Paged Attention" (klaylearn.com glossary), definition: prefill fills blocks
    as the prompt's tokens produce K and V, and attention reads the context
    through the table; "What is paged attention in vLLM...", Steps 3-4 (the
    prompt's blocks, then decoding). Reading taken (the pages do not spell out
    prefill attention): the chunk's K/V are already in the cache; sequence s
    has L = context_lens[s] tokens, its n = query_start[s+1] - query_start[s]
    query rows are its last n positions, and row i (position p = L - n + i)
    attends the keys t <= p, each query head j through KV head j // G.

    q: [total_q, Hq, d] with sequence s's rows at query_start[s] .. query_start[s+1] - 1.
    Returns [total_q, Hq, d] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    total_q, num_heads, head_dim = q.shape
    num_kv_heads = k_cache.shape[2]
    group = num_heads // num_kv_heads
    out = np.zeros((total_q, num_heads, head_dim), dtype=np.float64)
    for s in range(len(context_lens)):
        r0, r1 = int(query_start[s]), int(query_start[s + 1])
        n, length = r1 - r0, int(context_lens[s])
        if n == 0:
            continue
        keys = gather_context(k_cache, block_tables[s], length, block_size)
        values = gather_context(v_cache, block_tables[s], length, block_size)
        pos = chunk_positions(length, n)
        visible = causal_visible(length, pos)
        for j in range(num_heads):
            h = kv_head_of(j, group)
            x = scale * (q[r0:r1, j, :] @ keys[:, h, :].T)    # [n, L] scores
            x = np.where(visible, x, -np.inf)
            w = np.exp(x - x.max(axis=1, keepdims=True))
            w = w / w.sum(axis=1, keepdims=True)
            out[r0:r1, j, :] = w @ values[:, h, :]
    return out
