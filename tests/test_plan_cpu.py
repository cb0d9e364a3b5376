"""Host side of the planned calls: pa_decode_plan's and pa_prefill_plan's work
lists and the argument checks of pa_decode_planned and pa_prefill_planned (no
GPU: every rejected call fails before any CUDA call).

"Paged Attention" (klaylearn.com glossary), definition: decode reads each
sequence's blocks through its table; the split of a context into partitions
and the order in which the partitions run change no result, so the plan is
pinned here by what it must list (every partition that holds a token, once),
how it encodes it, and the order it promises.
"""

import ctypes

import numpy as np
import pytest

import paged_kv_cache_345_b200 as pa

FAKE = ctypes.c_void_p(0x10000)


def _items(work):
    seq = work[:, 0]
    part = work[:, 1] & 0xFFFF
    count = (work[:, 1].astype(np.int64) & 0xFFFFFFFF) >> 16
    return seq, part, count


def test_plan_worked_example():
    # lengths 0, 16, 40, 96 in partitions of 32 tokens:
    #   whole partitions: seq 2 part 0; seq 3 parts 0, 1, 2
    #   ragged last ones by size: seq 1 (16 tokens), seq 2 part 1 (8), seq 0 (empty)
    work = pa.pa_decode_plan(np.array([0, 16, 40, 96], dtype=np.int32), 32)
    seq, part, count = _items(work)
    assert seq.tolist() == [2, 3, 3, 3, 1, 2, 0]
    assert part.tolist() == [0, 0, 1, 2, 0, 1, 0]
    assert count.tolist() == [2, 3, 3, 3, 1, 2, 1]


@pytest.mark.parametrize("seed,ps", [(0, 16), (1, 96), (2, 768), (3, 64)])
def test_plan_lists_every_partition_once_in_order(seed, ps):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 3000, size=300).astype(np.int32)
    lens[rng.integers(0, 300, size=20)] = 0
    lens[rng.integers(0, 300, size=20)] = ps * rng.integers(1, 5, size=20)   # exact multiples
    work = pa.pa_decode_plan(lens, ps)
    seq, part, count = _items(work)
    need = np.maximum(1, -(-lens // ps))
    # every (sequence, partition) that holds a token, exactly once, with its count
    got = sorted(zip(seq.tolist(), part.tolist()))
    want = sorted((s, k) for s in range(lens.size) for k in range(need[s]))
    assert got == want
    assert np.array_equal(count, need[seq])
    # tokens per item: whole partitions first, then the rest longest first,
    # ties by sequence
    size = np.minimum(ps, np.maximum(0, lens[seq] - part * ps))
    whole = size == ps
    nw = int(whole.sum())
    assert whole[:nw].all() and not whole[nw:].any()
    assert np.array_equal(seq[:nw], np.sort(seq[:nw], kind="stable"))
    tail = list(zip((-size[nw:]).tolist(), seq[nw:].tolist()))
    assert tail == sorted(tail)
    # each tail item is its sequence's last partition
    assert np.array_equal(part[nw:], need[seq[nw:]] - 1)


def test_plan_writes_into_a_caller_buffer_and_reports_capacity():
    lens = np.array([100, 5, 0, 64], dtype=np.int32)
    buf = np.full((16, 2), -7, dtype=np.int32)
    work = pa.pa_decode_plan(lens, 32, out=buf)
    assert work.base is buf or np.shares_memory(work, buf)
    assert len(work) == 4 + 1 + 1 + 2
    assert (buf[len(work):] == -7).all()
    n = ctypes.c_int(0)
    small = np.zeros((3, 2), dtype=np.int32)
    st = pa._lib.pa_decode_plan(lens.ctypes.data_as(pa._i32p), 4, 32,
                                small.ctypes.data_as(pa._i32p), 3, ctypes.byref(n))
    assert st == pa.PA_ERR_INVALID and n.value == 8
    assert "capacity" in pa._lib.pa_last_error().decode()


@pytest.mark.parametrize("lens,ps,status", [
    ([10, -1], 32, pa.PA_ERR_INVALID),
    ([10], 0, pa.PA_ERR_INVALID),
    ([10], 24, pa.PA_ERR_INVALID),
    ([10], (1 << 20) + 16, pa.PA_ERR_INVALID),
    ([65536 * 16 + 1], 16, pa.PA_ERR_UNSUPPORTED),
])
def test_plan_rejects(lens, ps, status):
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_plan(np.array(lens, dtype=np.int32), ps,
                          out=np.zeros((70000, 2), dtype=np.int32))
    assert e.value.status == status


def test_plan_of_no_sequences_is_empty():
    assert len(pa.pa_decode_plan(np.zeros(0, dtype=np.int32), 64)) == 0


def _planned(**over):
    a = dict(out=FAKE, q=FAKE, kn=FAKE, vn=FAKE, k=FAKE, v=FAKE, ks=None, vs=None, bt=FAKE,
             cl=FAKE, work=FAKE, n=4, S=2, Hq=32, Hkv=8, D=128, bs=16, nb=64, mbps=8, maxlen=100,
             scale=0.1, P=32, ws=FAKE, wsb=1 << 30, dt=pa.PA_BF16)
    a.update(over)
    st = pa._lib.pa_decode_planned(a["out"], a["q"], a["kn"], a["vn"], a["k"], a["v"], a["ks"],
                                   a["vs"], a["bt"], a["cl"], a["work"], a["n"], a["S"], a["Hq"],
                                   a["Hkv"], a["D"], a["bs"], a["nb"], a["mbps"], a["maxlen"],
                                   a["scale"], a["P"], a["ws"], a["wsb"], a["dt"], None)
    return st, pa._lib.pa_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(dt=pa.PA_F32), pa.PA_ERR_UNSUPPORTED),        # bf16 and E4M3 caches only
    (dict(dt=9), pa.PA_ERR_UNSUPPORTED),
    (dict(vn=None), pa.PA_ERR_INVALID),                 # k_new without v_new
    (dict(kn=ctypes.c_void_p(0x10008)), pa.PA_ERR_INVALID),
    (dict(work=None), pa.PA_ERR_INVALID),
    (dict(work=ctypes.c_void_p(0x10004)), pa.PA_ERR_INVALID),   # not 8-byte aligned
    (dict(P=0), pa.PA_ERR_INVALID),                     # the plan's size, never automatic
    (dict(P=24), pa.PA_ERR_INVALID),
    (dict(n=1), pa.PA_ERR_INVALID),                     # fewer items than sequences
    (dict(n=2 * 4 + 1), pa.PA_ERR_INVALID),             # more than S * partitions
    (dict(ks=FAKE, vs=FAKE), pa.PA_ERR_INVALID),        # scales for a bf16 cache
    (dict(dt=pa.PA_FP8_E4M3), pa.PA_ERR_INVALID),       # E4M3 without scales
    (dict(ws=None, wsb=0), pa.PA_ERR_INVALID),          # split sequences need a workspace
    (dict(Hq=24), pa.PA_ERR_UNSUPPORTED),
    (dict(maxlen=8 * 16 + 1), pa.PA_ERR_INVALID),
])
def test_planned_decode_rejects_on_host(over, status):
    st, msg = _planned(**over)
    assert st == status, msg
    assert msg


def test_planned_decode_zero_sequences_is_a_no_op():
    assert _planned(S=0, n=0)[0] == pa.PA_OK


# ------------------------------------------------------------- prefill plan

def _prefill_items(qs, lens, group, keyn=64):
    """(-cost, sequence, item) of every item, from the definition: item z of a
    chunk of n rows holds rows [first, first + rows) counted from the chunk's
    start, first = (items - 1 - z) * ctok, and its last row sees key
    L - n + first + rows - 1; its cost is the key tiles up to that key."""
    ctok = 256 // group
    out = []
    for s in range(len(lens)):
        n, L = int(qs[s + 1] - qs[s]), int(lens[s])
        items = -(-n // ctok)
        for z in range(items):
            first = (items - 1 - z) * ctok
            rows = min(ctok, n - first)
            out.append((-((L - n + first + rows - 1) // keyn + 1), s, z))
    return sorted(out)


@pytest.mark.parametrize("seed,group,S", [(0, 4, 40), (1, 1, 40), (2, 8, 40), (3, 2, 40),
                                          (4, 4, 300)])
def test_prefill_plan_is_longest_first(seed, group, S):
    """(S = 300: past the 256 sequences the kernel's own search handles; the
    list has no such limit.)"""
    rng = np.random.default_rng(seed)
    n = rng.integers(0, 900, size=S)
    n[rng.integers(0, S, size=5)] = 0                       # sequences without rows
    lens = (n + rng.integers(0, 5000, size=S)).astype(np.int32)
    lens[rng.integers(0, S, size=5)] = 0                    # contexts of only the chunk
    lens = np.maximum(lens, n).astype(np.int32)
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    work = pa.pa_prefill_plan(qs, lens, 8 * group, 8)
    want = _prefill_items(qs, lens, group)
    assert work[:, 0].tolist() == [s for _, s, _ in want]
    assert work[:, 1].tolist() == [z for _, _, z in want]


def test_prefill_plan_rejects():
    qs = np.array([0, 10, 30], dtype=np.int32)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_prefill_plan(qs, np.array([10, 19], dtype=np.int32), 32, 8)   # 20 rows over 19
    assert e.value.status == pa.PA_ERR_INVALID
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_prefill_plan(qs, np.array([10, 30], dtype=np.int32), 24, 8)   # group 3
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_prefill_plan(qs, np.array([10, 30], dtype=np.int32), 32, 8,
                           out=np.zeros((1, 2), dtype=np.int32))               # capacity
    assert e.value.status == pa.PA_ERR_INVALID


def _prefill_planned(**over):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, cl=FAKE, qs=FAKE, work=FAKE, n=4, S=2,
             tq=100, Hq=32, Hkv=8, D=128, bs=16, nb=64, mbps=16, mq=64, scale=0.1,
             dt=pa.PA_BF16)
    a.update(over)
    st = pa._lib.pa_prefill_planned(a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["qs"],
                                    a["work"], a["n"], a["S"], a["tq"], a["Hq"], a["Hkv"],
                                    a["D"], a["bs"], a["nb"], a["mbps"], a["mq"], a["scale"],
                                    a["dt"], None)
    return st, pa._lib.pa_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(work=None), pa.PA_ERR_INVALID),
    (dict(work=ctypes.c_void_p(0x10004)), pa.PA_ERR_INVALID),
    (dict(n=-1), pa.PA_ERR_INVALID),
    (dict(n=3), pa.PA_ERR_INVALID),        # more than S * ceil(64 / 64) = 2 items
    (dict(dt=pa.PA_F32), pa.PA_ERR_UNSUPPORTED),
    (dict(Hq=24), pa.PA_ERR_UNSUPPORTED),
])
def test_planned_prefill_rejects_on_host(over, status):
    st, msg = _prefill_planned(**over)
    assert st == status, msg


def test_planned_prefill_without_items_is_a_no_op():
    assert _prefill_planned(n=0)[0] == pa.PA_OK
