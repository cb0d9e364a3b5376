"""pa_kv_append and pa_copy_blocks on the GPU: bit-exact against the oracle."""

import numpy as np
import pytest
import torch

import paged_kv_cache_345_b200 as pa
from oracle import attention as oatt

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _random_cache(rng, nb, bs, hkv, d, dtype):
    k = torch.from_numpy(rng.standard_normal((nb, bs, hkv, d), dtype=np.float32)).to(DT[dtype])
    v = torch.from_numpy(rng.standard_normal((nb, bs, hkv, d), dtype=np.float32)).to(DT[dtype])
    return k, v


def _bits(t):
    return t.cpu().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("nb,bs,hkv,d,n", [(64, 16, 8, 128, 37), (32, 4, 2, 64, 1),
                                           (16, 1, 1, 8, 9), (3000, 16, 8, 128, 20000)])
def test_kv_append_bit_exact(dtype, nb, bs, hkv, d, n):
    rng = np.random.default_rng(nb * 7 + n)
    k_cache, v_cache = _random_cache(rng, nb, bs, hkv, d, dtype)
    slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int64)
    slots[::5] = -1                       # padding rows are skipped
    k_new = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32)).to(DT[dtype])
    v_new = torch.from_numpy(rng.standard_normal((n, hkv, d), dtype=np.float32)).to(DT[dtype])
    ref_k, ref_v = oatt.kv_append(_bits(k_cache), _bits(v_cache), _bits(k_new), _bits(v_new),
                                  slots, bs)
    kc, vc = k_cache.cuda(), v_cache.cuda()
    pa.pa_kv_append(k_new.cuda(), v_new.cuda(), torch.from_numpy(slots).cuda(), kc, vc)
    assert pa.pa_device_errors() == 0
    assert np.array_equal(_bits(kc), ref_k)
    assert np.array_equal(_bits(vc), ref_v)


def test_kv_append_out_of_range_slot_is_flagged_and_skipped():
    rng = np.random.default_rng(1)
    k_cache, v_cache = _random_cache(rng, 8, 4, 2, 64, "bf16")
    kc, vc = k_cache.cuda(), v_cache.cuda()
    slots = torch.tensor([3, 8 * 4, 10**9, 5], dtype=torch.int64, device="cuda")
    k_new = torch.ones((4, 2, 64), dtype=torch.bfloat16, device="cuda")
    pa.pa_kv_append(k_new, k_new, slots, kc, vc)
    assert pa.pa_device_errors() & pa.PA_DEVERR_SLOT
    assert pa.pa_device_errors() == 0     # read clears the word
    ref_k, _ = oatt.kv_append(_bits(k_cache), _bits(v_cache), _bits(k_new.cpu()),
                              _bits(k_new.cpu()), np.array([3, -1, -1, 5]), 4)
    assert np.array_equal(_bits(kc), ref_k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("nb,bs,hkv,d,pairs", [(128, 16, 8, 128, 63), (16, 4, 2, 64, 3),
                                               (8, 1, 1, 8, 1)])
def test_copy_blocks_bit_exact(dtype, nb, bs, hkv, d, pairs):
    rng = np.random.default_rng(nb + pairs)
    k_cache, v_cache = _random_cache(rng, nb, bs, hkv, d, dtype)
    ids = rng.permutation(nb)
    mapping = np.stack([ids[:pairs], ids[pairs:2 * pairs]], axis=1).astype(np.int64)
    ref_k, ref_v = oatt.copy_blocks(_bits(k_cache), _bits(v_cache), mapping)
    kc, vc = k_cache.cuda(), v_cache.cuda()
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(mapping).cuda())
    assert pa.pa_device_errors() == 0
    assert np.array_equal(_bits(kc), ref_k)
    assert np.array_equal(_bits(vc), ref_v)


def test_copy_blocks_bad_pair_is_flagged_and_skipped():
    rng = np.random.default_rng(2)
    k_cache, v_cache = _random_cache(rng, 8, 4, 2, 64, "f32")
    kc, vc = k_cache.cuda(), v_cache.cuda()
    mapping = torch.tensor([[0, 1], [2, 99], [-1, 3], [4, 5]], dtype=torch.int64, device="cuda")
    pa.pa_copy_blocks(kc, vc, mapping)
    assert pa.pa_device_errors() & pa.PA_DEVERR_COPY_PAIR
    ref_k, ref_v = oatt.copy_blocks(_bits(k_cache), _bits(v_cache), np.array([[0, 1], [4, 5]]))
    assert np.array_equal(_bits(kc), ref_k) and np.array_equal(_bits(vc), ref_v)


def test_copy_then_diverge_keeps_sharers_apart():
    """Copy-on-write end to end: after the copy, writing the new block leaves the
    shared source block (still read by the other sharer) unchanged."""
    from paged_kv_cache_345_b200.cache import PagedKVCache

    c = PagedKVCache(16, 4, 2, 64, "bf16")
    p = c.add_sequence()
    rows = torch.randn((6, 2, 64), device="cuda").to(torch.bfloat16)
    c.write([p], [6], rows, rows)
    child = c.fork(p)
    before = c.k_cache.clone()
    new = torch.full((1, 2, 64), 7.0, device="cuda", dtype=torch.bfloat16)
    slots = c.write([child], [1], new, new)
    torch.cuda.synchronize()
    tab_p, _ = c.bm.block_tables([p], 4)
    tab_c, _ = c.bm.block_tables([child], 4)
    shared_tail, own_tail = int(tab_p[0, 1]), int(tab_c[0, 1])
    assert shared_tail != own_tail and int(tab_p[0, 0]) == int(tab_c[0, 0])
    assert torch.equal(c.k_cache[shared_tail], before[shared_tail])
    assert torch.equal(c.k_cache[own_tail, :2], before[shared_tail, :2])
    assert torch.equal(c.k_cache[own_tail, 2], new[0])
    assert int(slots[0]) == own_tail * 4 + 2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mapping_on_host", [False, True])
def test_swap_out_to_pinned_host_and_back_bit_exact(dtype, mapping_on_host):
    """Preemption by swapping: blocks go from the device pool to a page-locked
    host pool and come back to other device blocks, bit for bit."""
    rng = np.random.default_rng(21)
    nb, hb, bs, hkv, d = 64, 40, 16, 8, 128
    k_cache, v_cache = _random_cache(rng, nb, bs, hkv, d, dtype)
    kd, vd = k_cache.cuda(), v_cache.cuda()
    host_k = torch.zeros((hb, bs, hkv, d), dtype=DT[dtype]).pin_memory()
    host_v = torch.zeros((hb, bs, hkv, d), dtype=DT[dtype]).pin_memory()
    ids = rng.permutation(nb)[:30]
    out_pairs = np.stack([ids, rng.permutation(hb)[:30]], axis=1).astype(np.int64)
    mapping = torch.from_numpy(out_pairs)
    mapping = mapping.pin_memory() if mapping_on_host else mapping.cuda()
    pa.pa_swap_blocks(host_k, host_v, kd, vd, mapping)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    ref_k, ref_v = oatt.swap_blocks(_bits(torch.zeros_like(host_k)), _bits(torch.zeros_like(host_v)),
                                    _bits(k_cache), _bits(v_cache), out_pairs)
    assert np.array_equal(_bits(host_k), ref_k) and np.array_equal(_bits(host_v), ref_v)
    # swap back into a fresh device pool at other block ids
    kd2 = torch.zeros_like(kd)
    vd2 = torch.zeros_like(vd)
    in_pairs = np.stack([out_pairs[:, 1], rng.permutation(nb)[:30]], axis=1).astype(np.int64)
    pa.pa_swap_blocks(kd2, vd2, host_k, host_v, torch.from_numpy(in_pairs).cuda())
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    for (src_dev, _), (_, dst_dev) in zip(out_pairs, in_pairs):
        assert torch.equal(kd2[dst_dev].cpu(), k_cache[src_dev])
        assert torch.equal(vd2[dst_dev].cpu(), v_cache[src_dev])


def test_swap_bad_pair_is_flagged_and_skipped():
    kd = torch.ones((4, 4, 2, 64), dtype=torch.bfloat16, device="cuda")
    host = torch.zeros((4, 4, 2, 64), dtype=torch.bfloat16).pin_memory()
    host_v = torch.zeros_like(host).pin_memory()
    pairs = torch.tensor([[0, 1], [9, 2], [1, -1]], dtype=torch.int64, device="cuda")
    pa.pa_swap_blocks(host, host_v, kd, kd, pairs)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() & pa.PA_DEVERR_COPY_PAIR
    assert bool((host[1] == 1).all()) and not bool(host[2].any()) and not bool(host[0].any())
