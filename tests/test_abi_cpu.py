"""C-ABI library on the CPU: it loads, exports every declared symbol, rejects bad
arguments on the host before any launch, and its block manager matches the
oracle's bit for bit. No GPU and no kernel launch."""

import copy
import ctypes
import os
import re

import numpy as np
import pytest

import paged_kv_cache_345_b200 as pa
from oracle import blocks as oblk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    declared = _declared_functions()
    assert len(declared) >= 25
    lib = ctypes.CDLL(pa.lib_path)
    missing = [name for name in declared if not hasattr(lib, name)]
    assert missing == []
    assert sorted(pa.EXPORTED) == declared


def test_library_is_built_for_sm100a():
    # the build compiles every CUDA source for sm_100a and nothing else
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "pa_build", os.path.join(ROOT, "paged_kv_cache_345_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings():
    assert pa._lib.pa_status_string(pa.PA_ERR_NO_BLOCKS) == b"PA_ERR_NO_BLOCKS"
    assert pa._lib.pa_status_string(99) == b"PA_ERR_UNKNOWN"


# ------------------------------------------------------ host-side validation
# Fake, never-dereferenced pointers: each call must fail validation before any
# CUDA call is made.
FAKE = ctypes.c_void_p(0x10000)


def _decode(**over):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, cl=FAKE, S=2, Hq=32, Hkv=8, D=128, bs=16,
             nb=64, mbps=8, maxlen=100, scale=0.1, P=0, ws=None, wsb=0, dt=pa.PA_BF16)
    a.update(over)
    st = pa._lib.pa_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["S"], a["Hq"],
                           a["Hkv"], a["D"], a["bs"], a["nb"], a["mbps"], a["maxlen"], a["scale"],
                           a["P"], a["ws"], a["wsb"], a["dt"], None)
    return st, pa._lib.pa_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(Hq=30), pa.PA_ERR_INVALID),                  # heads not a multiple of kv heads
    (dict(Hq=24, Hkv=8), pa.PA_ERR_UNSUPPORTED),       # group 3
    (dict(Hq=128, Hkv=8), pa.PA_ERR_UNSUPPORTED),      # group 16
    (dict(D=96), pa.PA_ERR_UNSUPPORTED),
    (dict(bs=12), pa.PA_ERR_INVALID),
    (dict(bs=512), pa.PA_ERR_INVALID),
    (dict(maxlen=8 * 16 + 1), pa.PA_ERR_INVALID),      # beyond the table's capacity
    (dict(maxlen=-1), pa.PA_ERR_INVALID),
    (dict(P=100), pa.PA_ERR_INVALID),                  # not a multiple of 16
    (dict(scale=float("nan")), pa.PA_ERR_INVALID),
    (dict(dt=7), pa.PA_ERR_UNSUPPORTED),
    (dict(out=None), pa.PA_ERR_INVALID),
    (dict(q=ctypes.c_void_p(0x10008)), pa.PA_ERR_INVALID),   # misaligned
    (dict(maxlen=128, P=16), pa.PA_ERR_INVALID),       # needs a workspace, none given
    (dict(nb=0), pa.PA_ERR_INVALID),
])
def test_decode_rejects_on_host(over, status):
    st, msg = _decode(**over)
    assert st == status, msg
    assert msg


def test_decode_zero_sequences_is_a_no_op():
    assert _decode(S=0)[0] == pa.PA_OK


def _contig(**over):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, cl=FAKE, S=2, Hq=32, Hkv=8, D=128, slab=4112,
             maxlen=4101, scale=0.1, P=0, ws=FAKE, wsb=1 << 30, dt=pa.PA_BF16)
    a.update(over)
    st = pa._lib.pa_decode_contiguous(a["out"], a["q"], a["k"], a["v"], a["cl"], a["S"], a["Hq"],
                                      a["Hkv"], a["D"], a["slab"], a["maxlen"], a["scale"],
                                      a["P"], a["ws"], a["wsb"], a["dt"], None)
    return st, pa._lib.pa_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(dt=pa.PA_F32), pa.PA_ERR_UNSUPPORTED),        # bf16 only
    (dict(dt=pa.PA_FP8_E4M3), pa.PA_ERR_UNSUPPORTED),
    (dict(Hq=24), pa.PA_ERR_UNSUPPORTED),               # group 3
    (dict(Hq=30), pa.PA_ERR_INVALID),
    (dict(D=96), pa.PA_ERR_UNSUPPORTED),
    (dict(slab=8, maxlen=8), pa.PA_ERR_INVALID),        # slabs of at least 16 tokens
    (dict(maxlen=4113), pa.PA_ERR_INVALID),             # longer than a slab
    (dict(maxlen=-1), pa.PA_ERR_INVALID),
    (dict(P=24), pa.PA_ERR_INVALID),
    (dict(scale=float("inf")), pa.PA_ERR_INVALID),
    (dict(k=None), pa.PA_ERR_INVALID),
    (dict(v=ctypes.c_void_p(0x10004)), pa.PA_ERR_INVALID),   # misaligned
    (dict(ws=None, wsb=0), pa.PA_ERR_INVALID),          # split sequences need a workspace
    (dict(S=-1), pa.PA_ERR_INVALID),
])
def test_contiguous_decode_rejects_on_host(over, status):
    st, msg = _contig(**over)
    assert st == status, msg
    assert msg


def _shared(**over):
    a = dict(out=FAKE, q=FAKE, kn=None, vn=None, k=FAKE, v=FAKE, bt=FAKE, cl=FAKE, S=64, Hq=32,
             Hkv=8, D=128, bs=16, nb=8192, mbps=256, prefix=2048, maxlen=3054, scale=0.1, P=0,
             ws=FAKE, wsb=1 << 30, dt=pa.PA_BF16)
    a.update(over)
    st = pa._lib.pa_decode_shared_prefix(
        a["out"], a["q"], a["kn"], a["vn"], a["k"], a["v"], a["bt"], a["cl"], a["S"], a["Hq"],
        a["Hkv"], a["D"], a["bs"], a["nb"], a["mbps"], a["prefix"], a["maxlen"], a["scale"],
        a["P"], a["ws"], a["wsb"], a["dt"], None)
    return st, pa._lib.pa_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(dt=pa.PA_F32), pa.PA_ERR_UNSUPPORTED),
    (dict(D=64), pa.PA_ERR_UNSUPPORTED),
    (dict(bs=4, mbps=1024), pa.PA_ERR_UNSUPPORTED),      # the prefix kernel's boxes need >= 8
    (dict(Hq=24), pa.PA_ERR_UNSUPPORTED),                # group 3
    (dict(prefix=0), pa.PA_ERR_INVALID),
    (dict(prefix=2050), pa.PA_ERR_INVALID),              # not a multiple of the block size
    (dict(prefix=3072), pa.PA_ERR_INVALID),              # past max_context_len
    (dict(scale=-0.1), pa.PA_ERR_INVALID),
    (dict(kn=FAKE), pa.PA_ERR_INVALID),                  # k_new without v_new
    (dict(kn=ctypes.c_void_p(0x10008), vn=FAKE), pa.PA_ERR_INVALID),   # misaligned
    (dict(ws=None, wsb=0), pa.PA_ERR_INVALID),
    (dict(wsb=1024), pa.PA_ERR_INVALID),                 # workspace too small
    (dict(P=24), pa.PA_ERR_INVALID),
])
def test_shared_prefix_decode_rejects_on_host(over, status):
    st, msg = _shared(**over)
    assert st == status, msg
    assert msg


def test_shared_prefix_workspace_holds_both_parts():
    # the prefix's partitions and the suffix's, more than a plain decode of the suffix
    both = pa.pa_decode_shared_prefix_workspace_bytes(64, 32, 8, 128, 2048, 3054, 0)
    rest = pa.pa_decode_workspace_bytes(64, 32, 8, 128, 3054 - 2048, 0)
    assert both > rest > 0
    assert pa.pa_decode_shared_prefix_workspace_bytes(64, 32, 8, 128, 0, 3054, 0) == 0
    assert _shared(S=0)[0] == pa.PA_OK


def test_contiguous_decode_zero_sequences_is_a_no_op():
    assert _contig(S=0)[0] == pa.PA_OK


def test_append_and_copy_reject_on_host():
    lib = pa._lib
    assert lib.pa_kv_append(FAKE, FAKE, FAKE, -1, FAKE, FAKE, 4, 4, 2, 64, 0, None) == \
        pa.PA_ERR_INVALID
    assert lib.pa_kv_append(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 4, 2, 64, 0, None) == pa.PA_OK
    assert lib.pa_kv_append(FAKE, FAKE, FAKE, 3, FAKE, FAKE, 4, 4, 1, 2, 1, None) == \
        pa.PA_ERR_UNSUPPORTED                                         # 4-byte rows
    assert lib.pa_kv_append(None, FAKE, FAKE, 3, FAKE, FAKE, 4, 4, 2, 64, 0, None) == \
        pa.PA_ERR_INVALID
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 0, 4, 4, 2, 64, 0, None) == pa.PA_OK
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, -2, 4, 4, 2, 64, 0, None) == pa.PA_ERR_INVALID
    assert lib.pa_copy_blocks(FAKE, FAKE, ctypes.c_void_p(0x10004), 2, 4, 4, 2, 64, 0, None) == \
        pa.PA_ERR_INVALID


def test_e4m3_swap_and_fused_step_reject_on_host():
    lib, F, E = pa._lib, FAKE, pa.PA_FP8_E4M3
    err = lambda: lib.pa_last_error().decode()  # noqa: E731
    # E4M3 caches go through the _fp8 entry points
    assert lib.pa_kv_append(F, F, F, 3, F, F, 4, 4, 2, 128, E, None) == pa.PA_ERR_UNSUPPORTED
    assert "pa_kv_append_fp8" in err()
    assert _decode(dt=E)[0] == pa.PA_ERR_UNSUPPORTED
    # pa_kv_append_fp8: scales present and aligned, head_dim a multiple of 16
    assert lib.pa_kv_append_fp8(F, F, F, 3, F, F, None, F, 4, 4, 2, 128, None) == \
        pa.PA_ERR_INVALID
    assert lib.pa_kv_append_fp8(F, F, F, 3, F, F, F, F, 4, 4, 2, 40, None) == \
        pa.PA_ERR_UNSUPPORTED
    assert lib.pa_kv_append_fp8(F, F, F, 3, F, F, ctypes.c_void_p(0x10002), F, 4, 4, 2, 128,
                                None) == pa.PA_ERR_INVALID
    assert lib.pa_kv_append_fp8(F, F, F, 0, F, F, F, F, 4, 4, 2, 128, None) == pa.PA_OK
    # pa_decode_fp8: head_dim 128 only, scales required
    fp8 = lambda **o: lib.pa_decode_fp8(  # noqa: E731
        F, F, F, F, o.get("ks", F), F, F, F, 2, 32, 8, o.get("D", 128), 16, 64, 8, 100, 0.1, 0,
        None, 0, None)
    assert fp8(D=64) == pa.PA_ERR_UNSUPPORTED and "head_dim" in err()
    assert fp8(ks=None) == pa.PA_ERR_INVALID and "scale" in err()
    # fused steps need the new rows
    assert lib.pa_decode_append(F, F, None, F, F, F, F, F, 2, 32, 8, 128, 16, 64, 8, 100, 0.1, 0,
                                None, 0, pa.PA_BF16, None) == pa.PA_ERR_INVALID
    assert lib.pa_decode_append_fp8(F, F, F, ctypes.c_void_p(0x10008), F, F, F, F, F, F, 2, 32, 8,
                                    128, 16, 64, 8, 100, 0.1, 0, None, 0, None) == \
        pa.PA_ERR_INVALID
    # pa_swap_blocks: pointers, pair count, block bytes
    swap = lambda **o: lib.pa_swap_blocks(  # noqa: E731
        o.get("dk", F), F, 4, F, F, 4, o.get("m", F), o.get("n", 2), o.get("bs", 4), 2,
        o.get("D", 64), o.get("dt", pa.PA_BF16), None)
    assert swap(n=0) == pa.PA_OK
    assert swap(n=-1) == pa.PA_ERR_INVALID
    assert swap(dk=None) == pa.PA_ERR_INVALID
    assert swap(m=ctypes.c_void_p(0x10004)) == pa.PA_ERR_INVALID
    assert swap(bs=1, D=2, dt=E) == pa.PA_ERR_UNSUPPORTED            # 4-byte blocks
    assert swap(dt=9) == pa.PA_ERR_UNSUPPORTED


def _prefill(**over):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, cl=FAKE, qs=FAKE, S=2, tq=300, Hq=32,
             Hkv=8, D=128, bs=16, nb=64, mbps=8, maxq=200, scale=0.1, dt=pa.PA_BF16)
    a.update(over)
    st = pa._lib.pa_prefill(a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["qs"], a["S"],
                            a["tq"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["nb"], a["mbps"],
                            a["maxq"], a["scale"], a["dt"], None)
    return st, pa._lib.pa_last_error().decode()


@pytest.mark.parametrize("over,status,words", [
    (dict(dt=pa.PA_F32), pa.PA_ERR_UNSUPPORTED, "dtype"),
    (dict(D=64), pa.PA_ERR_UNSUPPORTED, "head_dim"),
    (dict(Hq=24), pa.PA_ERR_UNSUPPORTED, "group"),
    (dict(Hq=30), pa.PA_ERR_INVALID, "multiple"),
    (dict(bs=4), pa.PA_ERR_UNSUPPORTED, "block_size"),
    (dict(bs=24), pa.PA_ERR_UNSUPPORTED, "block_size"),
    (dict(maxq=301), pa.PA_ERR_INVALID, "max_query_len"),
    (dict(scale=0.0), pa.PA_ERR_INVALID, "scale"),
    (dict(scale=float("nan")), pa.PA_ERR_INVALID, "scale"),
    (dict(S=-1), pa.PA_ERR_INVALID, "negative"),
    (dict(k=None), pa.PA_ERR_INVALID, "null"),
    # one CTA per KV head and work item: 65,535 sequences of up to 2^20 rows
    # would need more than 2^31 - 1 CTAs
    (dict(S=65535, tq=1 << 20, maxq=1 << 20), pa.PA_ERR_UNSUPPORTED, "grid"),
    (dict(qs=ctypes.c_void_p(0x10002)), pa.PA_ERR_INVALID, "misaligned"),
])
def test_prefill_rejects_on_host(over, status, words):
    st, msg = _prefill(**over)
    assert st == status and words in msg, msg


def test_prefill_empty_batch_is_a_no_op():
    for over in (dict(S=0), dict(tq=0, maxq=0), dict(maxq=0)):
        assert _prefill(**over)[0] == pa.PA_OK


def test_partition_size_and_workspace():
    for s, h, n in [(8, 8, 4101), (256, 8, 4096), (1, 1, 7), (16, 8, 32768), (64, 8, 3054)]:
        p = pa.pa_decode_partition_size(s, h, n)
        assert p % 16 == 0 and 64 <= p <= 768
    # about five CTAs per SM for the Llama batch; the 256-sequence batch at the cap
    assert pa.pa_decode_partition_size(8, 8, 4101) == 96
    assert pa.pa_decode_partition_size(256, 8, 4096) == 768
    # one partition: no workspace
    assert pa.pa_decode_workspace_bytes(2, 4, 2, 64, 34, 64) == 0
    # 3 partitions of 16 tokens: m, l and acc regions, each 256-byte aligned
    rows = 2 * 4 * 3
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert pa.pa_decode_workspace_bytes(2, 4, 2, 64, 34, 16) == \
        up(rows * 4) * 2 + up(rows * 64 * 4)


# ----------------------------------------------- block manager vs the oracle

def _snapshot_native(bm, seqs):
    tables, lens = bm.block_tables(seqs, 4096)
    return ([list(tables[i, :bm.seq_num_blocks(s)]) for i, s in enumerate(seqs)], list(lens),
            bm.allocator.num_free())


def _snapshot_oracle(ob, seqs):
    return [list(ob.tables[s]) for s in seqs], [ob.lengths[s] for s in seqs], ob.num_free()


@pytest.mark.parametrize("seed,nb,bs", [(12, 300, 4), (13, 64, 1), (14, 500, 16), (15, 40, 3),
                                         (16, 120, 8)])
def test_block_manager_matches_oracle_on_random_operations(seed, nb, bs):
    """Random add / fork / free / multi-sequence appends, native against oracle
    after every operation; small pools run out often, block size 1 and a block
    size that is not a power of two included."""
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb).astype(np.int32)
    seen = {"cow": 0, "exhausted": 0}
    nat = pa.BlockManager(nb, bs)
    nat.allocator.set_free_order(order)
    ob = oblk.BlockManager(nb, bs)
    ob.set_free_order(order.tolist())
    live_n, live_o = [], []
    for step in range(400):
        op = rng.integers(0, 10)
        if op <= 1 or not live_n:
            live_n.append(nat.add_seq())
            live_o.append(ob.new_sequence())
        elif op == 2:
            i = rng.integers(len(live_n))
            live_n.append(nat.fork(live_n[i]))
            live_o.append(ob.fork(live_o[i]))
        elif op == 3 and len(live_n) > 1:
            i = rng.integers(len(live_n))
            nat.free_seq(live_n.pop(i))
            ob.free_sequence(live_o.pop(i))
        else:
            k = int(rng.integers(1, min(len(live_n), 6) + 1))
            idx = rng.choice(len(live_n), size=k, replace=False)
            counts = rng.integers(0, 9, size=k)
            # the batch is all or nothing, and succeeds exactly when appending its
            # sequences one after the other does (a shared tail copied by one
            # sharer is written in place by the last)
            trial = copy.deepcopy(ob)
            try:
                for i, c in zip(idx, counts):
                    trial.add_tokens(live_o[i], int(c))
                fits = True
            except oblk.OutOfBlocks:
                fits = False
            if not fits:
                with pytest.raises(pa.PagedAttentionError) as ei:
                    nat.append_slots([live_n[i] for i in idx], counts)
                assert ei.value.status == pa.PA_ERR_NO_BLOCKS
                seen["exhausted"] += 1
                assert _snapshot_native(nat, live_n) == _snapshot_oracle(ob, live_o)
                continue
            slots_n, cows_n = nat.append_slots([live_n[i] for i in idx], counts)
            slots_o, cows_o = [], []
            for i, c in zip(idx, counts):
                sl, cw = ob.add_tokens(live_o[i], int(c))
                slots_o += sl
                cows_o += cw
            assert slots_n.tolist() == slots_o
            assert [tuple(x) for x in cows_n.tolist()] == cows_o
            seen["cow"] += len(cows_o)
        assert _snapshot_native(nat, live_n) == _snapshot_oracle(ob, live_o)
        for b in range(0, nb, 7):
            assert nat.allocator.refcount(b) == ob.refcount[b]
    # one token per block: a shared tail is always full, so nothing is ever copied
    assert (seen["cow"] == 0) if bs == 1 else (seen["cow"] > 0)
    assert seen["exhausted"] > 0 or nb >= 300


def test_two_sharers_of_one_tail_need_one_copy():
    """Two sequences share a partly filled tail (reference count 2) and append
    in the same batch with one free block left: the first copies the tail into
    that block, the second is then its only holder and writes in place. One
    block and one copy pair suffice, as when they append one after the other."""
    bs = 4
    nat = pa.BlockManager(3, bs)
    ob = oblk.BlockManager(3, bs)
    parent_n, parent_o = nat.add_seq(), ob.new_sequence()
    nat.append_slots([parent_n], [6])          # blocks [b0, b1], b1 half full
    ob.add_tokens(parent_o, 6)
    child_n, child_o = nat.fork(parent_n), ob.fork(parent_o)
    assert nat.allocator.num_free() == 1
    # raw call with room for exactly one copy pair
    ids = np.array([child_n, parent_n], dtype=np.int32)
    cnt = np.array([1, 1], dtype=np.int32)
    slots = np.empty(2, dtype=np.int64)
    cows = np.empty((1, 2), dtype=np.int64)
    ncow = ctypes.c_int(-1)
    i32p = ctypes.POINTER(ctypes.c_int32)
    i64p = ctypes.POINTER(ctypes.c_int64)
    st = pa._lib.pa_bm_append_slots(nat._h, ids.ctypes.data_as(i32p), cnt.ctypes.data_as(i32p), 2,
                                    slots.ctypes.data_as(i64p), cows.ctypes.data_as(i64p), 1,
                                    ctypes.byref(ncow))
    assert st == pa.PA_OK, pa._lib.pa_last_error().decode()
    s1, c1 = ob.add_tokens(child_o, 1)
    s2, c2 = ob.add_tokens(parent_o, 1)
    assert ncow.value == 1 and [tuple(cows[0])] == c1 + c2
    assert slots.tolist() == s1 + s2
    assert nat.allocator.num_free() == 0 == ob.num_free()
    assert _snapshot_native(nat, [parent_n, child_n]) == _snapshot_oracle(ob, [parent_o, child_o])


def test_block_manager_worked_example_and_exhaustion(golden):
    ex = golden["worked_example"]
    bm = pa.BlockManager(700, ex["block_size"])
    seqs = [bm.add_seq() for _ in ex["lengths"]]
    slots, cows = bm.append_slots(seqs, ex["lengths"])
    assert len(slots) == ex["total_tokens"] and len(cows) == 0
    assert sum(bm.seq_num_blocks(s) for s in seqs) * ex["block_size"] == ex["paged_slots"]
    _, _ = bm.append_slots(seqs, [1] * len(seqs))
    assert sum(bm.seq_num_blocks(s) for s in seqs) == 666
    free_before = bm.allocator.num_free()
    with pytest.raises(pa.PagedAttentionError) as ei:
        bm.append_slots(seqs[:1], [100_000])
    assert ei.value.status == pa.PA_ERR_NO_BLOCKS
    assert bm.allocator.num_free() == free_before and bm.seq_len(seqs[0]) == 129


def test_allocator_rejects_bad_ids():
    a = pa.Allocator(4)
    b = a.alloc()
    a.decref(b)
    for bad in (lambda: a.decref(b), lambda: a.incref(b), lambda: a.decref(99),
                lambda: a.set_free_order([0, 1, 2])):
        with pytest.raises(pa.PagedAttentionError) as ei:
            bad()
        assert ei.value.status == pa.PA_ERR_INVALID
    assert a.refcount(99) == -1
    for _ in range(4):
        a.alloc()
    with pytest.raises(pa.PagedAttentionError) as ei:
        a.alloc()
    assert ei.value.status == pa.PA_ERR_NO_BLOCKS
