"""PagedKVCache's host logic on the CPU (no GPU).

The kernel calls it makes are replaced by recorders; what it hands them (slot
mappings, copy-on-write pairs, block tables, context lengths, query offsets,
the host bound on chunk length) must agree with the oracle's block manager
driven through the same operations. The native block manager does the
bookkeeping; the oracle only checks it."""

import numpy as np
import pytest
import torch

import paged_kv_cache_345_b200.cache as cm
from oracle import blocks as ob
from paged_kv_cache_345_b200.cache import PagedKVCache

NB, BS, HKV, HQ, D = 32, 4, 2, 4, 8
CALLS = ("pa_kv_append", "pa_kv_append_fp8", "pa_copy_blocks", "pa_decode", "pa_decode_fp8",
         "pa_decode_append", "pa_decode_append_fp8", "pa_decode_planned", "pa_prefill")


@pytest.fixture
def rec(monkeypatch):
    log = []

    def recorder(name):
        # positional arguments, then the keyword ones as one dict at the end
        def fn(*args, **kwargs):
            log.append((name, args + (kwargs,)))
        return fn

    for name in CALLS:
        monkeypatch.setattr(cm, name, recorder(name))
    monkeypatch.setattr(PagedKVCache, "_to_device",
                        lambda self, a: torch.from_numpy(np.ascontiguousarray(a)))
    return log


def _pair(dtype="bf16"):
    order = np.random.default_rng(7).permutation(NB)
    cache = PagedKVCache(NB, BS, HKV, D, dtype, "cpu", free_order=order)
    ref = ob.BlockManager(NB, BS)
    ref.set_free_order(order)
    return cache, ref


def _tables(ref, seqs):
    width = max(1, max(len(ref.tables[s]) for s in seqs))
    t = np.zeros((len(seqs), width), dtype=np.int32)
    for i, s in enumerate(seqs):
        t[i, :len(ref.tables[s])] = ref.tables[s]
    return t, np.array([ref.lengths[s] for s in seqs], dtype=np.int32)


def rows(n, h=HKV):
    return torch.zeros((n, h, D), dtype=torch.bfloat16)


def test_write_fork_decode_step_and_prefill_match_the_oracle(rec):
    cache, ref = _pair()
    s0, r0 = cache.add_sequence(), ref.new_sequence()
    cache.write([s0], [6], rows(6), rows(6))
    slots, cows = ref.add_tokens(r0, 6)
    (name, a), = rec
    assert name == "pa_kv_append" and a[2].tolist() == slots and not cows

    # fork: the child shares both blocks; the next token of the parent copies
    # the shared, partly filled tail first
    s1, r1 = cache.fork(s0), ref.fork(r0)
    rec.clear()
    kn, vn = rows(2), rows(2)
    out = cache.decode_step(torch.zeros((2, HQ, D), dtype=torch.bfloat16), kn, vn, [s0, s1])
    _, cow0 = ref.append_slot(r0)
    _, cow1 = ref.append_slot(r1)
    assert cow0 is not None and cow1 is None
    assert [n for n, _ in rec] == ["pa_copy_blocks", "pa_decode_planned"]
    assert rec[0][1][2].tolist() == [list(cow0)]
    # (out, q, k_cache, v_cache, tables, lens, work, max_len, scale, partition, ws, kwargs)
    a = rec[1][1]
    t, lens = _tables(ref, [r0, r1])
    assert np.array_equal(a[4].numpy(), t) and a[5].tolist() == lens.tolist() == [7, 7]
    ps = a[9]
    assert ps == cm.pa_decode_partition_size(2, HKV, 7)
    assert np.array_equal(a[6].numpy(), cm.pa_decode_plan(lens, ps))
    assert a[7] == 7 and a[8] == pytest.approx(1 / np.sqrt(D)) and out.shape == (2, HQ, D)
    assert a[-1]["k_new"] is kn and a[-1]["v_new"] is vn

    # decode: the same tables, no writes
    rec.clear()
    cache.decode(torch.zeros((2, HQ, D), dtype=torch.bfloat16), [s1, s0])
    (name, a), = rec
    t, lens = _tables(ref, [r1, r0])
    assert name == "pa_decode_planned" and np.array_equal(a[4].numpy(), t)
    assert a[5].tolist() == lens.tolist() and a[7] == 7
    assert a[-1]["k_new"] is None and a[-1]["v_new"] is None

    # the plain grid on request: pa_decode_append / pa_decode with the same tables
    rec.clear()
    cache.decode(torch.zeros((2, HQ, D), dtype=torch.bfloat16), [s1, s0], planned=False)
    (name, a), = rec
    assert name == "pa_decode" and np.array_equal(a[4].numpy(), t)
    assert a[5].tolist() == lens.tolist() and a[6] == 7

    # prefill: a 3-row chunk for s0, nothing for s1
    rec.clear()
    cache.prefill(torch.zeros((3, HQ, D), dtype=torch.bfloat16), rows(3), rows(3), [s0, s1],
                  [3, 0])
    slots, _ = ref.add_tokens(r0, 3)
    assert [n for n, _ in rec] == ["pa_kv_append", "pa_prefill"]
    assert rec[0][1][2].tolist() == slots
    a = rec[1][1]
    t, lens = _tables(ref, [r0, r1])
    assert np.array_equal(a[4].numpy(), t) and a[5].tolist() == lens.tolist() == [10, 7]
    assert a[6].tolist() == [0, 3, 3] and a[7] == 3

    # freeing the child returns only the blocks nobody else holds: its old
    # tail (the parent copied it), not the shared first block
    free_before, ref_before = cache.bm.allocator.num_free(), ref.num_free()
    cache.free(s1)
    ref.free_sequence(r1)
    assert cache.bm.allocator.num_free() - free_before == ref.num_free() - ref_before == 1
    assert cache.bm.allocator.num_free() == ref.num_free()


def test_fp8_cache_routes_to_the_e4m3_calls(rec):
    cache, ref = _pair("fp8_e4m3")
    assert cache.k_cache.dtype == torch.uint8 and cache.k_scale.shape == (HKV,)
    s0, r0 = cache.add_sequence(), ref.new_sequence()
    cache.write([s0], [5], rows(5), rows(5))
    slots, _ = ref.add_tokens(r0, 5)
    cache.decode_step(torch.zeros((1, HQ, D), dtype=torch.bfloat16), rows(1), rows(1), [s0])
    cache.decode(torch.zeros((1, HQ, D), dtype=torch.bfloat16), [s0])
    cache.decode_step(torch.zeros((1, HQ, D), dtype=torch.bfloat16), rows(1), rows(1), [s0],
                      planned=False)
    cache.decode(torch.zeros((1, HQ, D), dtype=torch.bfloat16), [s0], planned=False)
    assert [n for n, _ in rec] == ["pa_kv_append_fp8", "pa_decode_planned", "pa_decode_planned",
                                   "pa_decode_append_fp8", "pa_decode_fp8"]
    assert rec[0][1][2].tolist() == slots
    for _, a in rec[1:3]:   # the planned calls carry the per-head scales
        assert a[-1]["k_scale"] is cache.k_scale and a[-1]["v_scale"] is cache.v_scale
    with pytest.raises(NotImplementedError):
        cache.prefill(torch.zeros((1, HQ, D), dtype=torch.bfloat16), rows(1), rows(1), [s0], [1])


def test_unfused_step_writes_then_decodes(rec):
    cache, ref = _pair()
    s0, r0 = cache.add_sequence(), ref.new_sequence()
    cache.write([s0], [4], rows(4), rows(4))
    ref.add_tokens(r0, 4)
    rec.clear()
    cache.decode_step(torch.zeros((1, HQ, D), dtype=torch.bfloat16), rows(1), rows(1), [s0],
                      fused=False)
    slots, _ = ref.add_tokens(r0, 1)
    assert [n for n, _ in rec] == ["pa_kv_append", "pa_decode_planned"]
    assert rec[0][1][2].tolist() == slots and rec[1][1][5].tolist() == [5]
    rec.clear()
    cache.decode_step(torch.zeros((1, HQ, D), dtype=torch.bfloat16), rows(1), rows(1), [s0],
                      fused=False, planned=False)
    slots, _ = ref.add_tokens(r0, 1)
    assert [n for n, _ in rec] == ["pa_kv_append", "pa_decode"]
    assert rec[0][1][2].tolist() == slots and rec[1][1][5].tolist() == [6]


def test_block_manager_output_buffers():
    """append_slots / block_tables into caller buffers give what the allocating
    calls give, on two identical managers, including a copy-on-write step."""
    import numpy as np

    import paged_kv_cache_345_b200 as pa

    def make():
        bm = pa.BlockManager(200, 16)
        seqs = [bm.add_seq() for _ in range(5)]
        bm.append_slots(seqs, [3, 16, 17, 40, 1])
        seqs.append(bm.fork(seqs[2]))            # shares a partly filled tail
        return bm, seqs

    a, sa = make()
    b, sb = make()
    slot_buf = np.full(32, -7, np.int64)
    cow_buf = np.full((8, 2), -7, np.int64)
    tab_buf = np.full(64, -7, np.int32)
    len_buf = np.full(8, -7, np.int32)
    for step in range(3):
        s1, c1 = a.append_slots(sa, [1] * len(sa))
        t1, l1 = a.block_tables(sa, 5)
        s2, c2 = b.append_slots(sb, np.ones(len(sb), np.int32), slot_buf, cow_buf)
        t2, l2 = b.block_tables(sb, 5, tab_buf, len_buf)
        assert np.array_equal(s1, s2) and np.array_equal(c1, c2)
        assert np.array_equal(t1, t2) and np.array_equal(l1, l2)
        assert np.shares_memory(s2, slot_buf) and np.shares_memory(t2, tab_buf)
        if step == 0:
            assert len(c2) == 1                  # the fork's shared tail copied once
    with pytest.raises(ValueError):
        b.append_slots(sb, [1] * len(sb), np.empty(2, np.int64))
    with pytest.raises(ValueError):
        b.block_tables(sb, 5, np.empty(64, np.int64))
