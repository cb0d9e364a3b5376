"""E4M3 (8-bit) KV caches on the GPU, through the C ABI, against the oracle.

Quantising writes are bit-exact against oracle.quant (float32 division by the
KV head's scale, round to nearest even, saturation at +-448). Decode over the
codes is compared with the float64 oracle run on the dequantised values of the
oracle's own codes for the same bfloat16 rows; the results are bit-identical
across block sizes and placements, as for bfloat16 caches.
"""

import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from oracle import attention as oatt
from oracle import quant as oquant
from workloads import configs, synth

pytestmark = pytest.mark.gpu

FP8 = gh.FP8


def _fp8(wl, **kw):
    return dataclasses.replace(wl, kv_dtype=FP8, **kw)


def _edge_rows(rng, n, hkv, d, k_scale):
    """bfloat16 rows ~N(0, 3) with, per head, values that land on the format's
    edges once divided by the head's scale: zeros of both signs, the largest
    code, saturation, the subnormal range and exact ties between codes."""
    x = rng.standard_normal((n, hkv, d)).astype(np.float32) * 3
    for h in range(hkv):
        s = float(k_scale[h])
        special = np.array([0.0, -0.0, 448 * s, -448 * s, 1e4 * s, -3e4 * s, 2.0 ** -9 * s,
                            3 * 2.0 ** -10 * s, 1.0625 * s, -1.1875 * s, 2.0 ** -6 * s,
                            240 * s, 0.5 * 2.0 ** -9 * s], dtype=np.float32)
        flat = x[:, h].reshape(-1)
        flat[:special.size] = special
        x[:, h] = flat.reshape(n, d)
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("nb,bs,hkv,d,n", [(64, 16, 8, 128, 37), (32, 4, 2, 64, 5),
                                           (16, 1, 1, 16, 9), (3000, 16, 8, 128, 20000)])
def test_kv_append_fp8_bit_exact(nb, bs, hkv, d, n):
    rng = np.random.default_rng(nb + 3 * n)
    ks = rng.uniform(0.005, 0.08, hkv).astype(np.float32)
    ks[0] = 1.0                       # a unit scale keeps the bfloat16 ties exact ties
    vs = rng.uniform(0.005, 0.08, hkv).astype(np.float32)
    k_new, v_new = _edge_rows(rng, n, hkv, d, ks), _edge_rows(rng, n, hkv, d, vs)
    slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int64)
    slots[1::7] = -1                  # padding rows are skipped
    kc = torch.from_numpy(rng.integers(0, 256, (nb, bs, hkv, d), dtype=np.uint8))
    vc = torch.from_numpy(rng.integers(0, 256, (nb, bs, hkv, d), dtype=np.uint8))
    ref_k, ref_v = oatt.kv_append(kc.numpy(), vc.numpy(),
                                  gh.e4m3_codes(k_new.float().numpy(), ks),
                                  gh.e4m3_codes(v_new.float().numpy(), vs), slots, bs)
    kd, vd = kc.cuda(), vc.cuda()
    pa.pa_kv_append_fp8(k_new.cuda(), v_new.cuda(), torch.from_numpy(slots).cuda(), kd, vd,
                        torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda())
    assert pa.pa_device_errors() == 0
    assert np.array_equal(kd.cpu().numpy(), ref_k)
    assert np.array_equal(vd.cpu().numpy(), ref_v)


def test_kv_append_fp8_bad_slot_is_flagged_and_skipped():
    kd = torch.zeros((8, 4, 2, 128), dtype=torch.uint8, device="cuda")
    vd = torch.zeros_like(kd)
    rows = torch.ones((3, 2, 128), dtype=torch.bfloat16, device="cuda")
    sc = torch.full((2,), 0.25, device="cuda")
    pa.pa_kv_append_fp8(rows, rows, torch.tensor([5, 32, 7], device="cuda"), kd, vd, sc, sc)
    assert pa.pa_device_errors() & pa.PA_DEVERR_SLOT
    flat = kd.view(32, 2, 128).cpu()
    assert bool((flat[5] == 0x48).all()) and bool((flat[7] == 0x48).all())   # 4.0 = 0x48
    assert int(flat.sum()) == 2 * 2 * 128 * 0x48


def test_llama_layer_fp8_matches_oracle_and_codes_are_exact():
    wl = _fp8(configs.llama3_8b_layer())
    case = gh.build_case(wl, poisoned=True)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", "fp8 llama layer")
    # the cache holds exactly the oracle's codes of every row, read through the tables
    tables, _ = case.cache.bm.block_tables(case.seqs, case.cache.max_blocks_per_seq)
    kc = case.cache.k_cache.cpu().numpy()
    for i in (0, 3, 7):
        L = wl.context_lens[i] + 1
        t = np.arange(L)
        got = kc[tables[i][t // wl.block_size], t % wl.block_size]
        k, _ = synth.kv_rows(wl.value_seed, i, L, wl.num_kv_heads, wl.head_dim)
        assert np.array_equal(got, gh.e4m3_codes(gh.stored(k, "bf16"), case.k_scale))


@pytest.mark.parametrize("partition", [0, 16, 64, 512, 4112])
def test_fp8_partitions(partition):
    case = gh.build_case(_fp8(configs.llama3_8b_layer()), partition_size=partition)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", f"fp8 P={partition}")


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (8, 1), (16, 2), (6, 3), (64, 8)])
def test_fp8_groups(hq, hkv):
    lens = (0, 1, 15, 16, 17, 300, 1000)
    wl = _fp8(configs.llama3_8b_layer(), num_heads=hq, num_kv_heads=hkv, context_lens=lens,
              num_blocks=256)
    case = gh.build_case(wl, partition_size=64, poisoned=True)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", f"fp8 {hq}/{hkv}")


def test_fp8_block_sizes_and_placement_are_bitwise_invariant():
    base = _fp8(configs.llama3_8b_layer())
    ref = gh.build_case(base, partition_size=128)
    gh.assert_close(gh.gpu_out(ref), gh.expected_all(ref), "bf16", "fp8 bs=16")
    want = ref.out.view(torch.int16).cpu()
    for bs in (1, 2, 4, 8, 32, 64, 256):
        need = sum(-(-(n + 1) // bs) for n in base.context_lens)
        wl = dataclasses.replace(base, block_size=bs, num_blocks=need + 16)
        got = gh.build_case(wl, partition_size=128, keep=set())
        assert torch.equal(got.out.view(torch.int16).cpu(), want), f"block_size {bs}"
    ident = gh.build_case(base, partition_size=128, free_order=np.arange(base.num_blocks),
                          keep=set())
    assert torch.equal(ident.out.view(torch.int16).cpu(), want), "identity placement"


def test_fp8_fused_and_unfused_steps_agree_bitwise():
    wl = _fp8(configs.llama3_8b_layer())
    fused = gh.build_case(wl, partition_size=64, keep=set())
    split = gh.build_case(wl, partition_size=64, keep=set(), fused=False)
    assert torch.equal(fused.out.view(torch.int16), split.out.view(torch.int16))
    assert torch.equal(fused.cache.k_cache, split.cache.k_cache)
    assert torch.equal(fused.cache.v_cache, split.cache.v_cache)


def test_fp8_shared_prefix_with_copy_on_write():
    wl = _fp8(configs.shared_prefix())
    keep = {0, 1, 31, 63}
    case = gh.build_case(wl, keep=keep)
    got = gh.gpu_out(case)
    for s in keep:
        for j in (0, 5, 31):
            gh.assert_close(got[s, j], gh.expected_one(case, s, j), "bf16", f"fp8 prefix s={s}")


def test_fp8_long_context_sampled():
    wl = _fp8(configs.long_context(16))
    keep = {0, 9, 15}
    case = gh.build_case(wl, keep=keep)
    got = gh.gpu_out(case)
    for s in keep:
        for j in (0, 13, 31):
            gh.assert_close(got[s, j], gh.expected_one(case, s, j), "bf16", f"fp8 long s={s}")


def test_fp8_copy_and_swap_blocks_move_codes_bit_for_bit():
    rng = np.random.default_rng(5)
    k = torch.from_numpy(rng.integers(0, 256, (64, 16, 8, 128), dtype=np.uint8))
    v = torch.from_numpy(rng.integers(0, 256, (64, 16, 8, 128), dtype=np.uint8))
    pairs = np.stack([np.arange(0, 20), np.arange(30, 50)], axis=1).astype(np.int64)
    ref_k, ref_v = oatt.copy_blocks(k.numpy(), v.numpy(), pairs)
    kd, vd = k.cuda(), v.cuda()
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(pairs).cuda())
    assert pa.pa_device_errors() == 0
    assert np.array_equal(kd.cpu().numpy(), ref_k) and np.array_equal(vd.cpu().numpy(), ref_v)
    hk = torch.zeros((24, 16, 8, 128), dtype=torch.uint8).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    out_pairs = np.stack([np.arange(40, 64), np.arange(24)], axis=1).astype(np.int64)
    pa.pa_swap_blocks(hk, hv, kd, vd, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert torch.equal(hk, kd[40:].cpu()) and torch.equal(hv, vd[40:].cpu())


def test_fp8_refusals():
    kd = torch.zeros((4, 16, 2, 64), dtype=torch.uint8, device="cuda")
    q = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    lens = torch.ones((1,), dtype=torch.int32, device="cuda")
    sc = torch.ones((2,), device="cuda")
    with pytest.raises(pa.PagedAttentionError, match="PA_ERR_UNSUPPORTED.*head_dim 64"):
        pa.pa_decode_fp8(torch.empty_like(q), q, kd, kd, sc, sc, tables, lens, 1, 0.125)
    # the 16-bit entry point refuses E4M3 caches before launching anything
    out = torch.full_like(q, 3.0)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = pa._lib.pa_decode(p(out), p(q), p(kd), p(kd), p(tables), p(lens), 1, 4, 2, 64, 16, 4, 1,
                           1, 0.125, 0, None, 0, pa.PA_FP8_E4M3,
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pa.PA_ERR_UNSUPPORTED and "pa_decode_fp8" in pa._lib.pa_last_error().decode()
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    rows = torch.zeros((1, 2, 64), dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PagedAttentionError, match="PA_ERR_UNSUPPORTED.*pa_kv_append_fp8"):
        pa.pa_kv_append(rows, rows, torch.zeros(1, dtype=torch.int64, device="cuda"), kd, kd)
    assert pa.pa_device_errors() == 0


def test_fp8_oracle_values_span_the_format():
    """The decode cases above exercise saturation-free codes of every exponent:
    the scales put |x| / scale of N(0, 1) rows up to ~150 (codes up to 0x70s)."""
    ks, _ = synth.e4m3_scales(8)
    k, _ = synth.kv_rows(1002, 0, 2000, 8, 128)
    codes = gh.e4m3_codes(gh.stored(k, "bf16"), ks)
    mags = np.unique(codes & 0x7F)
    assert mags.max() >= 0x68 and mags.min() == 0 and len(mags) > 100
    assert np.abs(oquant.e4m3_decode(codes)).max() < 448
