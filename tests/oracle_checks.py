"""Pins for the CPU oracle: each check asserts something the pages or the
mathematics fix, independently of the oracle's own code.

The checks are plain functions so that `test_oracle_pins.py` runs them on the
oracle as written and `test_oracle_mutants.py` runs them on oracles with a
planted mistake, which at least one check must catch.
"""

from __future__ import annotations

import math

import numpy as np

import oracle
from oracle import attention as oatt
from oracle import blocks as oblk
from oracle import quant as oq


# ------------------------------------------------------------ block arithmetic

def check_seven_token_prompt(g):
    """Step 3 example: 7 tokens, 4 per block, logical 0 and 1 -> physical 7 and 1."""
    ex = g["seven_token_prompt"]
    bs = ex["block_size"]
    bm = oblk.BlockManager(num_blocks=8, block_size=bs)
    first = ex["physical_blocks_of_logical_0_1"]
    rest = [b for b in range(8) if b not in first]
    bm.set_free_order(first + rest)
    s = bm.new_sequence()
    slots, cows = bm.add_tokens(s, ex["prompt_tokens"])
    assert bm.tables[s] == first
    assert cows == []
    # tokens 0..3 in block 7 (slots 28..31), tokens 4..6 in block 1 (slots 4..6)
    assert slots == [7 * 4 + i for i in range(4)] + [1 * 4 + i for i in range(3)]
    # the last slot of block 1 waits for the next generated token: no new block
    nxt, cow = bm.append_slot(s)
    assert (nxt, cow) == (1 * 4 + 3, None)
    assert bm.tables[s] == first
    # the 9th token finds the tail full and takes the next free block
    ninth, _ = bm.append_slot(s)
    assert bm.tables[s] == first + [rest[0]]
    assert ninth == rest[0] * 4


def check_600_tokens(g):
    ex = g["reserve_4096_use_600"]
    assert oblk.blocks_for(ex["used_tokens"], ex["block_size"]) == ex["blocks"]
    used = 100.0 * ex["used_tokens"] / ex["reserved_tokens"]
    assert round(used) == ex["used_percent_about"]
    assert round(100.0 - used) == ex["idle_percent_about"]


def check_llama3_per_token(g):
    ex = g["llama3_8b_per_token"]
    per_token = oblk.kv_bytes_per_token(ex["layers"], ex["kv_heads"], ex["head_size"], 2)
    assert per_token == ex["bytes_per_token"] == 128 * 1024
    assert per_token * ex["max_positions"] == ex["bytes_per_full_reservation"] == 1 << 30
    used = 100.0 * ex["request_tokens"] / ex["max_positions"]
    assert round(used, 1) == ex["used_percent"]
    assert round(100.0 - used, 1) == ex["wasted_percent"]


def check_700_tokens(g):
    ex = g["request_700_in_blocks"]
    bs = ex["block_size"]
    assert oblk.blocks_for(ex["tokens"], bs) == ex["blocks"]
    slots = oblk.allocated_slots(ex["tokens"], bs)
    assert slots == ex["slots"]
    assert slots - ex["tokens"] == ex["idle_slots"]
    assert round(100.0 * (slots - ex["tokens"]) / slots, 2) == ex["idle_percent"]


def check_worked_example(g):
    ex = g["worked_example"]
    lens = ex["lengths"]
    bs = ex["block_size"]
    total = sum(lens)
    assert total == ex["total_tokens"]
    slab = len(lens) * g["llama3_8b_per_token"]["max_positions"]
    assert slab == ex["slab_slots"]
    assert round(100.0 * total / slab, 1) == ex["slab_used_percent"]
    paged = sum(oblk.allocated_slots(n, bs) for n in lens)
    assert paged == ex["paged_slots"]
    assert round(100.0 * total / paged, 1) == ex["paged_used_percent"]


def check_capacity(g):
    """Slabs fit 59 requests in 64e9 B; blocks fit about 367.

    The page's 367 follows from the batch's average ALLOCATED footprint,
    10,640 / 8 = 1,330 slots per request; its quoted average of about 1,322
    tokens is the filled count (10,578 / 8) and would give 369.
    """
    ex = g["worked_example"]
    per_token = oblk.kv_bytes_per_token(32, 8, 128, 2)
    budget = ex["cache_budget_bytes"]
    slab_bytes = g["llama3_8b_per_token"]["max_positions"] * per_token
    slabs = oblk.requests_that_fit(budget, slab_bytes)
    assert slabs == ex["slab_requests"]
    bs = ex["block_size"]
    lens = ex["lengths"]
    assert round(sum(lens) / len(lens)) == ex["average_length_about"]
    avg_alloc = sum(oblk.allocated_slots(n, bs) for n in lens) / len(lens)
    paged = oblk.requests_that_fit(budget, avg_alloc * per_token)
    assert paged == ex["paged_requests_about"]
    assert round(paged / slabs, 1) == ex["gain_times"]
    # the filled-token reading lands two requests higher
    assert oblk.requests_that_fit(budget, (sum(lens) / len(lens)) * per_token) == 369


def check_worked_example_block_manager(g):
    """The block manager holds the worked example in 665 blocks; one decode step
    appends a token to every request: only the 128-token request (tail exactly
    full) takes a new block, giving 666 blocks and 10,656 slots for 10,586 tokens."""
    ex = g["worked_example"]
    bs = ex["block_size"]
    lens = ex["lengths"]
    bm = oblk.BlockManager(num_blocks=700, block_size=bs)
    seqs = []
    for n in lens:
        s = bm.new_sequence()
        bm.add_tokens(s, n)
        seqs.append(s)
    held = sum(len(bm.tables[s]) for s in seqs)
    assert held * bs == ex["paged_slots"]
    assert bm.num_free() == 700 - held
    before = {s: len(bm.tables[s]) for s in seqs}
    for s in seqs:
        bm.append_slot(s)
    grew = [lens[i] for i, s in enumerate(seqs) if len(bm.tables[s]) > before[s]]
    assert grew == [128]
    assert sum(bm.lengths[s] for s in seqs) == ex["total_tokens"] + len(lens)
    assert sum(len(bm.tables[s]) for s in seqs) == held + 1
    assert (held + 1) * bs == 10_656
    for s in seqs:
        bm.free_sequence(s)
    assert bm.num_free() == 700


def check_sharing_and_copy_on_write():
    """Fork shares every block (count + 1); the first write into a shared,
    partly filled tail copies that one block only; counts return to zero."""
    bm = oblk.BlockManager(num_blocks=16, block_size=4)
    p = bm.new_sequence()
    bm.add_tokens(p, 6)                       # blocks [0, 1], block 1 half full
    c = bm.fork(p)
    assert bm.tables[c] == bm.tables[p] == [0, 1]
    assert bm.refcount[0] == bm.refcount[1] == 2
    slot, cow = bm.append_slot(c)             # child writes into the shared tail
    assert cow == (1, 2)                      # only the tail block is copied
    assert bm.tables[c] == [0, 2] and bm.tables[p] == [0, 1]
    assert slot == 2 * 4 + 2
    assert bm.refcount[0] == 2 and bm.refcount[1] == 1 and bm.refcount[2] == 1
    slot, cow = bm.append_slot(p)             # parent is now the only holder
    assert cow is None and slot == 1 * 4 + 2
    bm.free_sequence(c)
    bm.free_sequence(p)
    assert bm.num_free() == 16 and all(r == 0 for r in bm.refcount)


def check_exhaustion_leaves_state():
    bm = oblk.BlockManager(num_blocks=2, block_size=4)
    s = bm.new_sequence()
    bm.add_tokens(s, 8)
    free_before, table_before = bm.num_free(), list(bm.tables[s])
    try:
        bm.add_tokens(s, 1)
    except oblk.OutOfBlocks:
        pass
    else:
        raise AssertionError("expected OutOfBlocks")
    assert bm.num_free() == free_before and bm.tables[s] == table_before
    assert bm.lengths[s] == 8


# ------------------------------------------------------------------ attention

def _contiguous_case(seed, lengths, hq, hkv, d, bs, num_blocks):
    """Random contiguous K/V per sequence, stored through an explicit random placement."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_blocks)
    k_cache = rng.standard_normal((num_blocks, bs, hkv, d))
    v_cache = rng.standard_normal((num_blocks, bs, hkv, d))
    max_blocks = max(-(-n // bs) for n in lengths)
    tables = np.zeros((len(lengths), max_blocks), dtype=np.int64)
    used = 0
    for s, n in enumerate(lengths):
        nb = -(-n // bs)
        tables[s, :nb] = perm[used:used + nb]
        used += nb
    q = rng.standard_normal((len(lengths), hq, d))
    return q, k_cache, v_cache, tables


def _brute_force_decode(q, k_cache, v_cache, tables, lengths, scale, bs):
    """Python loops and math.exp: walk the block table block by block."""
    num_seqs, hq, d = q.shape
    hkv = k_cache.shape[2]
    out = np.zeros((num_seqs, hq, d))
    for s in range(num_seqs):
        n = int(lengths[s])
        for j in range(hq):
            h = j * hkv // hq
            keys, vals = [], []
            for lb in range(-(-n // bs)):
                phys = int(tables[s][lb])
                for off in range(bs):
                    if lb * bs + off < n:
                        keys.append(k_cache[phys][off][h])
                        vals.append(v_cache[phys][off][h])
            if not keys:
                continue
            xs = [scale * sum(float(q[s, j, i]) * float(k[i]) for i in range(d)) for k in keys]
            top = max(xs)
            es = [math.exp(x - top) for x in xs]
            z = sum(es)
            for i in range(d):
                out[s, j, i] = sum(e * float(v[i]) for e, v in zip(es, vals)) / z
    return out


def check_brute_force_tiny():
    lengths = [1, 4, 5, 9, 0]
    bs, hq, hkv, d = 4, 4, 2, 4
    q, kc, vc, tables = _contiguous_case(11, lengths, hq, hkv, d, bs, 12)
    ref = _brute_force_decode(q, kc, vc, tables, lengths, 0.5, bs)
    got = oatt.decode(q, kc, vc, tables, lengths, 0.5, bs)
    assert np.max(np.abs(got - ref)) < 1e-12


def check_sdpa_identity_table():
    """Identity table + contiguous cache equals torch's float64 SDPA with the
    KV heads repeated G times (query head j -> KV head j // G)."""
    import torch

    rng = np.random.default_rng(7)
    hq, hkv, d, bs, n = 8, 2, 16, 8, 37
    nb = -(-n // bs)
    kc = rng.standard_normal((nb, bs, hkv, d))
    vc = rng.standard_normal((nb, bs, hkv, d))
    q = rng.standard_normal((1, hq, d))
    scale = 0.3
    got = oatt.decode(q, kc, vc, np.arange(nb)[None, :], [n], scale, bs)
    keys = torch.from_numpy(kc.reshape(nb * bs, hkv, d)[:n]).permute(1, 0, 2)   # [hkv, n, d]
    vals = torch.from_numpy(vc.reshape(nb * bs, hkv, d)[:n]).permute(1, 0, 2)
    keys = keys.repeat_interleave(hq // hkv, dim=0)
    vals = vals.repeat_interleave(hq // hkv, dim=0)
    qt = torch.from_numpy(q[0]).unsqueeze(1)                                      # [hq, 1, d]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, keys, vals, scale=scale)
    assert np.max(np.abs(got[0] - ref[:, 0, :].numpy())) < 1e-12


def check_closed_forms():
    rng = np.random.default_rng(3)
    hq, hkv, d, bs = 4, 2, 8, 4
    # one cached token: the output is that token's value row, exactly
    kc = rng.standard_normal((3, bs, hkv, d))
    vc = rng.standard_normal((3, bs, hkv, d))
    q = rng.standard_normal((1, hq, d))
    out = oatt.decode(q, kc, vc, np.array([[2]]), [1], 0.7, bs)
    for j in range(hq):
        assert np.array_equal(out[0, j], vc[2, 0, j // 2])
    # q = 0: uniform weights, the output is the mean of the value rows
    table = np.array([[1, 0, 2]])
    n = 10
    out = oatt.decode(np.zeros((1, hq, d)), kc, vc, table, [n], 0.7, bs)
    rows = np.concatenate([vc[1], vc[0], vc[2]])[:n]
    for j in range(hq):
        assert np.allclose(out[0, j], rows[:, j // 2].mean(axis=0), rtol=0, atol=1e-14)
    # all keys equal: also uniform weights
    kc_eq = np.broadcast_to(rng.standard_normal((1, 1, hkv, d)), kc.shape).copy()
    out = oatt.decode(q, kc_eq, vc, table, [n], 0.7, bs)
    for j in range(hq):
        assert np.allclose(out[0, j], rows[:, j // 2].mean(axis=0), rtol=0, atol=1e-13)
    # one dominant score (q parallel to key t, large): output is that value row
    keys = np.concatenate([kc[1], kc[0], kc[2]])[:n]
    t = 6
    qd = np.zeros((1, hq, d))
    for j in range(hq):
        qd[0, j] = 40.0 * keys[t, j // 2] / np.linalg.norm(keys[t, j // 2])
    out = oatt.decode(qd, kc, vc, table, [n], 1.0, bs)
    for j in range(hq):
        assert np.allclose(out[0, j], rows[t, j // 2], rtol=0, atol=1e-6)


def check_placement_and_sharing_invariance():
    """Output depends only on the logical token sequence: a different physical
    placement, or prefix blocks shared instead of duplicated, gives the
    identical float64 result."""
    rng = np.random.default_rng(5)
    hq, hkv, d, bs = 4, 2, 8, 4
    n_prefix, n_a, n_b = 12, 3, 6          # prefix of 3 full blocks, then private tails
    prefix_k = rng.standard_normal((n_prefix, hkv, d))
    prefix_v = rng.standard_normal((n_prefix, hkv, d))
    tail = {s: (rng.standard_normal((m, hkv, d)), rng.standard_normal((m, hkv, d)))
            for s, m in ((0, n_a), (1, n_b))}
    q = rng.standard_normal((2, hq, d))

    def store(order, share):
        nb = 16
        kc = np.full((nb, bs, hkv, d), np.nan)
        vc = np.full((nb, bs, hkv, d), np.nan)
        free = list(order)
        tables = np.zeros((2, 5), dtype=np.int64)
        shared = [free.pop(0) for _ in range(3)] if share else None
        for s in (0, 1):
            kt = np.concatenate([prefix_k, tail[s][0]])
            vt = np.concatenate([prefix_v, tail[s][1]])
            nblk = -(-len(kt) // bs)
            ids = list(shared) + [free.pop(0) for _ in range(nblk - 3)] if share else \
                [free.pop(0) for _ in range(nblk)]
            for t in range(len(kt)):
                kc[ids[t // bs], t % bs] = kt[t]
                vc[ids[t // bs], t % bs] = vt[t]
            tables[s, :nblk] = ids
        return kc, vc, tables

    lens = [n_prefix + n_a, n_prefix + n_b]
    base = oatt.decode(q, *store(range(16), False), lens, 0.4, bs)
    for order in (rng.permutation(16), rng.permutation(16)):
        assert np.array_equal(base, oatt.decode(q, *store(order, False), lens, 0.4, bs))
        assert np.array_equal(base, oatt.decode(q, *store(order, True), lens, 0.4, bs))


def check_append_and_copy_roundtrip():
    rng = np.random.default_rng(9)
    nb, bs, hkv, d = 6, 4, 2, 3
    kc = rng.standard_normal((nb, bs, hkv, d))
    vc = rng.standard_normal((nb, bs, hkv, d))
    k_new = rng.standard_normal((4, hkv, d))
    v_new = rng.standard_normal((4, hkv, d))
    slots = np.array([5 * 4 + 1, -1, 0, 2 * 4 + 3])
    k2, v2 = oatt.kv_append(kc, vc, k_new, v_new, slots, bs)
    for i, slot in enumerate(slots):
        if slot >= 0:
            assert np.array_equal(k2[slot // bs, slot % bs], k_new[i])
            assert np.array_equal(v2[slot // bs, slot % bs], v_new[i])
    touched = {(int(x) // bs, int(x) % bs) for x in slots if x >= 0}
    for b in range(nb):
        for o in range(bs):
            if (b, o) not in touched:
                assert np.array_equal(k2[b, o], kc[b, o]) and np.array_equal(v2[b, o], vc[b, o])
    # gather through a table returns exactly what was appended
    table = np.array([5])
    got = oatt.gather_context(k2, table, 2, bs)
    assert np.array_equal(got[1], k_new[0])
    k3, v3 = oatt.copy_blocks(k2, v2, np.array([[5, 1], [0, 4]]))
    assert np.array_equal(k3[1], k2[5]) and np.array_equal(v3[4], v2[0])
    for b in (0, 2, 3, 5):
        assert np.array_equal(k3[b], k2[b]) and np.array_equal(v3[b], v2[b])


def check_swap_roundtrip():
    """Swapping blocks out to another pool and back restores them exactly and
    touches nothing else."""
    rng = np.random.default_rng(13)
    dev_k = rng.standard_normal((6, 4, 2, 3))
    dev_v = rng.standard_normal((6, 4, 2, 3))
    host_k = np.zeros((4, 4, 2, 3))
    host_v = np.zeros((4, 4, 2, 3))
    out_pairs = np.array([[5, 0], [1, 3], [2, 1]])
    hk, hv = oatt.swap_blocks(host_k, host_v, dev_k, dev_v, out_pairs)
    assert np.array_equal(hk[0], dev_k[5]) and np.array_equal(hv[3], dev_v[1])
    assert np.array_equal(hk[2], host_k[2])
    back_k, back_v = oatt.swap_blocks(np.zeros_like(dev_k), np.zeros_like(dev_v), hk, hv,
                                      out_pairs[:, ::-1])
    for src, _ in out_pairs:
        assert np.array_equal(back_k[src], dev_k[src]) and np.array_equal(back_v[src], dev_v[src])
    assert not back_k[0].any() and not back_v[4].any()



# ---------------------------------------------------------------- E4M3 codes

def check_e4m3_against_torch():
    """Inside the finite range the encoder agrees bit for bit with torch's
    float8_e4m3fn cast (round to nearest even), ties included."""
    import torch

    rng = np.random.default_rng(17)
    x = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 4,
        (rng.standard_normal(2000) * 2.0 ** -8).astype(np.float32),
        rng.uniform(-447, 447, 2000).astype(np.float32),
        # exact ties between neighbouring codes at several exponents
        np.array([(1 + (2 * k + 1) / 16) * 2.0 ** e for k in range(7) for e in range(-6, 8)],
                 dtype=np.float32),
        np.array([(2 * k + 1) * 2.0 ** -10 for k in range(8)], dtype=np.float32),
    ])
    x = x[np.abs(x) < 447.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oq.e4m3_encode(x), ref)


def check_e4m3_hand_values():
    cases = {1.0: 0x38, 448.0: 0x7E, 1000.0: 0x7E, -1000.0: 0xFE, 2.0 ** -9: 0x01,
             2.0 ** -10: 0x00, 3 * 2.0 ** -10: 0x02, 1.0625: 0x38, 1.1875: 0x3A,
             2.0 ** -6: 0x08, -3.0: 0xC4, 240.0: 0x77}
    got = oq.e4m3_encode(np.array(list(cases), dtype=np.float32))
    assert got.tolist() == list(cases.values())
    assert oq.e4m3_decode(np.array([0x7E, 0x01, 0x38, 0xC4])).tolist() == [448.0, 2.0 ** -9, 1.0,
                                                                             -3.0]


def check_e4m3_roundtrip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(oq.e4m3_encode(oq.e4m3_decode(codes).astype(np.float32)), codes)
    vals = oq.e4m3_decode(codes)
    assert np.nanmax(vals) == 448.0 and np.nanmin(vals) == -448.0


def check_e4m3_scale():
    """The per-head scale: the stored code is that of value / scale, the cache
    value is decode(code) * scale ("What is paged attention in vLLM, and why
    does it matter?", Trade-offs and edge cases, fourth point: narrower cache
    values; the scale convention is the E4M3 reading)."""
    # 3 / 0.5 = 6 = 1.5 * 2^2: exponent field 2 + 7 = 9, mantissa 4 -> 0x4C
    assert int(oq.quantize(np.float32(3.0), np.float32(0.5))) == 0x4C
    # and back: 6 * 0.5 = 3
    assert float(oq.dequantize(np.uint8(0x4C), 0.5)) == 3.0
    # decode(0x3A) = 1.25; times a scale that is not a power of two
    assert float(oq.dequantize(np.uint8(0x3A), np.float32(0.3))) == 1.25 * float(np.float32(0.3))
    # a power-of-two scale divides exactly: quantise(x, 1/32) is the code of 32 x
    rng = np.random.default_rng(23)
    x = (rng.standard_normal(512) * 4).astype(np.float32)
    assert np.array_equal(oq.quantize(x, np.float32(1 / 32)), oq.e4m3_encode(32 * x))
    # The division is float32 and its rounding can decide the code. With
    # x = 2.375 - 2^-22 (= 9961471 * 2^-22) and s = 2 - 2^-23 (= 16777215 * 2^-23)
    # the exact quotient is 19922942 / 16777215 = 1.1875 - 0.8125 / 16777215,
    # 4.84e-8 below 1.1875; the float32 spacing there is 2^-23 = 1.19e-7, so the
    # float32 quotient is 1.1875 exactly, the midpoint between the E4M3 values
    # 1.125 (0x39) and 1.25 (0x3A), and ties-to-even gives 0x3A (even mantissa
    # 2). Dividing in float64 instead would keep the quotient below the
    # midpoint and give 0x39.
    xs = np.float32(9961471 * 2.0 ** -22)
    ss = np.float32(16777215 * 2.0 ** -23)
    assert float(xs) == 2.375 - 2.0 ** -22 and float(ss) == 2.0 - 2.0 ** -23
    assert int(oq.quantize(xs, ss)) == 0x3A
    # scales broadcast per KV head: column h uses scale[h]
    rows = np.array([[3.0, 3.0], [-1.5, 0.75]], dtype=np.float32)
    sc = np.array([0.5, 0.25], dtype=np.float32)
    assert oq.quantize(rows, sc).tolist() == [[0x4C, 0x54], [0xC4, 0x44]]


# ------------------------------------------------------------------ prefill

def _prefill_case(rng, lens, chunks, hq=4, hkv=2, d=16, bs=4, shuffle=True):
    nb = sum(-(-n // bs) for n in lens) + 3
    kc = rng.standard_normal((nb, bs, hkv, d))
    vc = rng.standard_normal((nb, bs, hkv, d))
    ids = rng.permutation(nb) if shuffle else np.arange(nb)
    mb = max(-(-n // bs) for n in lens)
    tables = np.zeros((len(lens), mb), dtype=np.int64)
    k = 0
    for s, n in enumerate(lens):
        nbk = -(-n // bs)
        tables[s, :nbk] = ids[k:k + nbk]
        k += nbk
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int64)
    q = rng.standard_normal((int(qs[-1]), hq, d))
    return q, kc, vc, tables, qs


def check_prefill_single_query_is_decode():
    """A one-token chunk is the decode step: it sees the whole context."""
    rng = np.random.default_rng(31)
    lens = [1, 5, 13, 40]
    q, kc, vc, tables, qs = _prefill_case(rng, lens, [1, 1, 1, 1])
    got = oatt.prefill(q, kc, vc, tables, lens, qs, 0.3, 4)
    ref = oatt.decode(q, kc, vc, tables, lens, 0.3, 4)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


def check_prefill_full_matches_causal_sdpa():
    """A whole prompt (chunk = context) against torch's float64 causal attention."""
    import torch

    rng = np.random.default_rng(32)
    L, hq, hkv, d, bs = 37, 8, 2, 16, 4
    q, kc, vc, tables, qs = _prefill_case(rng, [L], [L], hq, hkv, d, bs, shuffle=False)
    got = oatt.prefill(q, kc, vc, tables, [L], qs, 0.25, bs)
    keys = kc.reshape(-1, hkv, d)[:L]
    vals = vc.reshape(-1, hkv, d)[:L]
    g = hq // hkv
    tq = torch.from_numpy(q).permute(1, 0, 2)                         # [Hq, L, d]
    tk = torch.from_numpy(keys).permute(1, 0, 2).repeat_interleave(g, 0)
    tv = torch.from_numpy(vals).permute(1, 0, 2).repeat_interleave(g, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                           scale=0.25)
    assert np.allclose(got, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def check_prefill_first_row_and_chunks():
    """Row 0 of a prompt sees only itself (its value row exactly); a chunk is
    the matching suffix of the whole prompt's rows, wherever the blocks sit."""
    rng = np.random.default_rng(33)
    L, n = 29, 6
    q, kc, vc, tables, qs = _prefill_case(rng, [L], [L])
    full = oatt.prefill(q, kc, vc, tables, [L], qs, 0.4, 4)
    v0 = oatt.gather_context(vc, tables[0], 1, 4)[0]
    for j in range(q.shape[1]):
        assert np.array_equal(full[0, j], v0[j // 2])
    chunk = oatt.prefill(q[L - n:], kc, vc, tables, [L], np.array([0, n]), 0.4, 4)
    assert np.allclose(chunk, full[L - n:], rtol=0, atol=1e-12)
    # identical logical contents in other physical blocks
    perm = rng.permutation(kc.shape[0])
    inv = np.argsort(perm)
    kc2, vc2 = kc[perm], vc[perm]
    tables2 = inv[tables]
    moved = oatt.prefill(q, kc2, vc2, tables2, [L], qs, 0.4, 4)
    assert np.array_equal(moved, full)


def check_prefill_brute_force():
    """Python loops and math.exp on a tiny chunked case."""
    import math

    rng = np.random.default_rng(34)
    lens, chunks = [6, 9], [2, 4]
    q, kc, vc, tables, qs = _prefill_case(rng, lens, chunks, hq=2, hkv=1, d=3, bs=2)
    got = oatt.prefill(q, kc, vc, tables, lens, qs, 0.7, 2)
    for s, (L, n) in enumerate(zip(lens, chunks)):
        for i in range(n):
            p = L - n + i
            for j in range(2):
                xs = []
                for t in range(p + 1):
                    blk, off = tables[s][t // 2], t % 2
                    xs.append(0.7 * sum(q[qs[s] + i, j, c] * kc[blk, off, 0, c] for c in range(3)))
                m = max(xs)
                w = [math.exp(x - m) for x in xs]
                tot = sum(w)
                for c in range(3):
                    ref = sum(w[t] * vc[tables[s][t // 2], t % 2, 0, c] for t in range(p + 1)) / tot
                    assert abs(got[qs[s] + i, j, c] - ref) < 1e-12


BLOCK_CHECKS = [
    check_seven_token_prompt, check_600_tokens, check_llama3_per_token, check_700_tokens,
    check_worked_example, check_capacity, check_worked_example_block_manager,
]
PLAIN_BLOCK_CHECKS = [check_sharing_and_copy_on_write, check_exhaustion_leaves_state]
ATTENTION_CHECKS = [
    check_brute_force_tiny, check_sdpa_identity_table, check_closed_forms,
    check_placement_and_sharing_invariance, check_append_and_copy_roundtrip,
    check_swap_roundtrip, check_e4m3_against_torch, check_e4m3_hand_values, check_e4m3_roundtrip,
    check_e4m3_scale,
    check_prefill_single_query_is_decode, check_prefill_full_matches_causal_sdpa,
    check_prefill_first_row_and_chunks, check_prefill_brute_force,
]

assert oracle is not None
