"""pa_decode on the GPU against the float64 oracle, plus the invariances the
pages fix (placement, sharing, block size) and the edge cases."""

import dataclasses

import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from oracle import attention as oatt
from oracle import blocks as oblk
from workloads import configs, synth

pytestmark = pytest.mark.gpu


def test_tiny_fp32_full_oracle_path():
    """Tiny workload: the oracle runs its own block manager (same free order), its
    own cache writes and its own gather; tables must match bit for bit and the
    outputs within 1e-5."""
    wl = configs.tiny()
    case = gh.build_case(wl)
    order = synth.block_permutation(wl.num_blocks, wl.placement_seed)
    ob = oblk.BlockManager(wl.num_blocks, wl.block_size)
    ob.set_free_order(order.tolist())
    kc = np.zeros((wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim))
    vc = np.zeros_like(kc)
    seqs = [ob.new_sequence() for _ in range(wl.num_seqs)]
    for s, n in enumerate(wl.context_lens):
        slots, _ = ob.add_tokens(seqs[s], n + 1)
        kc, vc = oatt.kv_append(kc, vc, case.rows_k[s], case.rows_v[s], slots, wl.block_size)
    max_blocks = max(len(ob.tables[s]) for s in seqs)
    tables = np.zeros((wl.num_seqs, max_blocks), dtype=np.int64)
    for i, s in enumerate(seqs):
        tables[i, :len(ob.tables[s])] = ob.tables[s]
    lens = [ob.lengths[s] for s in seqs]
    ref = oatt.decode(case.q, kc, vc, tables, lens, wl.scale, wl.block_size)
    nat_tables, nat_lens = case.cache.bm.block_tables(case.seqs, max_blocks)
    assert nat_tables.tolist() == tables.tolist() and nat_lens.tolist() == lens
    err = gh.assert_close(gh.gpu_out(case), ref, "f32", "tiny")
    assert err < 1e-5
    assert pa.pa_device_errors() == 0


@pytest.mark.parametrize("partition_size", [0, 16, 64, 512, 4112])
def test_llama3_8b_layer_bf16(partition_size):
    wl = configs.llama3_8b_layer()
    case = gh.build_case(wl, partition_size=partition_size)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", f"P={partition_size}")
    assert pa.pa_device_errors() == 0


def _custom(hq, hkv, d, dtype, bs, lens, pool=None, seed=7):
    need = sum(-(-(n + 1) // bs) for n in lens)
    return configs.Workload(f"custom_{hq}_{hkv}_{d}_{dtype}_{bs}", hq, hkv, d, dtype, bs,
                            pool or need + 8, tuple(lens), 5000 + seed, 6000 + seed)


RAGGED = (0, 1, 14, 15, 16, 17, 31, 47, 100, 257)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_group_and_head_dim(dtype, d, group):
    wl = _custom(2 * group, 2, d, dtype, 16, RAGGED)
    for ps in (16, 48, 0):
        case = gh.build_case(wl, partition_size=ps)
        gh.assert_close(gh.gpu_out(case), gh.expected_all(case), dtype, f"P={ps}")
    assert pa.pa_device_errors() == 0


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 32, 64, 128, 256])
def test_block_sizes_match_oracle_and_each_other(bs):
    """Same tokens under every block size: within tolerance of the oracle and
    bit-identical to block size 16 (chunks hold the same 16 logical tokens)."""
    wl = _custom(8, 2, 128, "bf16", 16, RAGGED + (600,))
    base = gh.gpu_out(gh.build_case(wl, partition_size=64))
    case = gh.build_case(dataclasses.replace(wl, block_size=bs,
                                             num_blocks=sum(-(-(n + 1) // bs)
                                                            for n in wl.context_lens) + 3),
                         partition_size=64)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", f"bs={bs}")
    assert np.array_equal(gh.gpu_out(case), base)


def test_placement_invariance_is_bitwise():
    wl = configs.llama3_8b_layer()
    a = gh.build_case(wl)
    b = gh.build_case(wl, free_order=synth.block_permutation(wl.num_blocks, 99))
    c = gh.build_case(wl, free_order=np.arange(wl.num_blocks, dtype=np.int32))  # contiguous
    assert not np.array_equal(a.cache.bm.block_tables(a.seqs, 300)[0],
                              b.cache.bm.block_tables(b.seqs, 300)[0])
    assert torch.equal(a.out, b.out) and torch.equal(a.out, c.out)


def test_shared_prefix_copy_on_write():
    """64 sequences fork a 2053-token parent (128 full + 1 partial shared block).
    Matches the oracle; equals the same tokens stored unshared bit for bit."""
    wl = configs.shared_prefix()
    case = gh.build_case(wl)
    a = case.cache.bm.allocator
    tables, _ = case.cache.bm.block_tables(case.seqs, 200)
    shared = tables[:, :128]
    assert (shared == shared[0]).all()                       # full prefix blocks shared
    assert all(a.refcount(int(b)) == 64 for b in shared[0])
    assert len(set(tables[:, 128].tolist())) == 64            # the partial tail was copied
    ref = np.stack([gh.expected_one(case, s, j) for s in range(0, 64, 9) for j in range(32)])
    got = gh.gpu_out(case)[0:64:9].reshape(-1, 128)
    gh.assert_close(got, ref, "bf16", "shared prefix")
    unshared = gh.build_case(wl, share_prefix=False)
    assert torch.equal(case.out, unshared.out)
    assert pa.pa_device_errors() == 0


def test_identical_suffixes_give_identical_outputs():
    wl = dataclasses.replace(configs.shared_prefix(), context_lens=(2053 + 40,) * 4)
    case = gh.build_case(wl)
    # sequences differ only by their own suffix tokens; make two of them equal
    torch.cuda.synchronize()
    out = gh.gpu_out(case)
    gh.assert_close(out, gh.expected_all(case), "bf16", "4 seqs")
    # same q row for all sequences and same suffix tokens -> same output
    from paged_kv_cache_345_b200.cache import PagedKVCache
    c = PagedKVCache(400, 16, 8, 128, "bf16", max_blocks_per_seq=200)
    p = c.add_sequence()
    rows = torch.randn((2053 + 40, 8, 128), device="cuda").to(torch.bfloat16)
    c.write([p], [2053], rows[:2053], rows[:2053])
    kids = [c.fork(p) for _ in range(3)]
    for s in [p] + kids:
        c.write([s], [40], rows[2053:], rows[2053:])
    q = torch.randn((1, 32, 128), device="cuda").to(torch.bfloat16).expand(4, 32, 128).contiguous()
    o = c.decode(q, [p] + kids)
    torch.cuda.synchronize()
    for i in range(1, 4):
        assert torch.equal(o[0], o[i])


def test_large_batch_ten_steps():
    """256 lognormal sequences on a fragmented 80,000-block pool; 10 decode steps,
    each appending one token per sequence (new blocks when a tail fills)."""
    wl = configs.large_batch()
    case = gh.build_case(wl)
    cache, seqs = case.cache, case.seqs
    for step in range(1, wl.decode_steps):
        k_new, v_new = synth.new_token_kv(wl.value_seed, step, wl.num_seqs, wl.num_kv_heads,
                                          wl.head_dim)
        k_new, v_new = gh.stored(k_new, "bf16"), gh.stored(v_new, "bf16")
        q = gh.stored(synth.queries(wl.value_seed, step, wl.num_seqs, wl.num_heads, wl.head_dim),
                      "bf16")
        for s in range(wl.num_seqs):
            case.rows_k[s] = np.concatenate([case.rows_k[s], k_new[s:s + 1]])
            case.rows_v[s] = np.concatenate([case.rows_v[s], v_new[s:s + 1]])
        dev = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
        case.out = cache.decode_step(dev(q), dev(k_new), dev(v_new), seqs, wl.scale)
        case.q = q
        if step in (1, 5):
            sample = [(s, j) for s in range(0, 256, 37) for j in (0, 13, 31)]
            got = gh.gpu_out(case)
            gh.assert_close(np.stack([got[s, j] for s, j in sample]),
                            np.stack([gh.expected_one(case, s, j) for s, j in sample]), "bf16",
                            f"step {step}")
    lens = [cache.context_len(s) for s in seqs]
    assert lens == [n + wl.decode_steps for n in wl.context_lens]
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", "last step")
    assert pa.pa_device_errors() == 0


def test_long_context_split_k_and_block_size_sweep():
    """16 x 32,768 cached tokens, partitions of 512 (65 per sequence), block sizes
    8..128 over the same token values: sampled outputs against the oracle, all
    block sizes bit-identical."""
    sample = [(0, 0), (3, 17), (9, 31), (15, 8)]
    staged = gh.stage_rows(configs.long_context(16), keep={s for s, _ in sample})
    outs = {}
    for bs in (8, 16, 32, 64, 128):
        case = gh.build_case(configs.long_context(bs), staged=staged)
        outs[bs] = case.out.clone()
        if bs == 16:
            got = gh.gpu_out(case)
            gh.assert_close(np.stack([got[s, j] for s, j in sample]),
                            np.stack([gh.expected_one(case, s, j) for s, j in sample]), "bf16",
                            "long context")
        del case
        torch.cuda.empty_cache()
    for bs in (8, 32, 64, 128):
        assert torch.equal(outs[bs], outs[16]), f"block size {bs} differs from 16"
    assert pa.pa_device_errors() == 0


def test_empty_and_bad_contexts_and_bad_block_ids():
    from paged_kv_cache_345_b200.cache import PagedKVCache

    c = PagedKVCache(8, 4, 2, 64, "f32", max_blocks_per_seq=4)
    s = c.add_sequence()
    rows = torch.randn((5, 2, 64), device="cuda")
    c.write([s], [5], rows, rows)
    q = torch.randn((3, 4, 64), device="cuda")
    out = torch.full_like(q, 5.0)
    tables = torch.tensor([[0, 1, 0, 0], [0, 0, 0, 0], [0, 7, 0, 0]], dtype=torch.int32,
                          device="cuda")
    real = c.bm.block_tables([s], 4)[0][0]
    tables[0] = torch.from_numpy(real).cuda()
    tables[2, 0] = int(real[0])
    tables[2, 1] = 1000                                     # outside the 8-block pool
    lens = torch.tensor([5, 0, 5], dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, c.k_cache, c.v_cache, tables, lens, 16, 0.125, 0, None)
    flags = pa.pa_device_errors()
    assert flags & pa.PA_DEVERR_BLOCK_ID
    o = out.cpu().numpy()
    assert np.array_equal(o[1], np.zeros((4, 64)))          # empty context -> zeros
    kc, vc = c.k_cache.cpu().double().numpy(), c.v_cache.cpu().double().numpy()
    ref = oatt.decode(q.cpu().double().numpy()[:1], kc, vc, real[None, :], [5], 0.125, 4)
    assert np.max(np.abs(o[0] - ref[0])) < 1e-5
    assert np.isfinite(o[2]).all()                          # bad id read as zeros, no fault
    # a context longer than max_context_len is flagged and zero-filled
    lens2 = torch.tensor([5, 9, 5], dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, c.k_cache, c.v_cache, tables, lens2, 8, 0.125, 0, None)
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT
    assert np.array_equal(out[1].cpu().numpy(), np.zeros((4, 64)))


def test_short_contexts_under_a_large_grid():
    """max_context_len far above the real lengths: the extra partitions exit."""
    wl = _custom(8, 2, 128, "bf16", 16, (3, 20, 70), pool=1200)
    case = gh.build_case(wl, partition_size=16)
    S, Hq, D = case.q.shape
    bt, cl, _ = case.cache.tables(case.seqs, max_blocks_per_seq=1024)
    out = torch.empty_like(case.out)
    ws = torch.zeros(pa.pa_decode_workspace_bytes(S, Hq, 2, D, 16000, 16), dtype=torch.uint8,
                     device="cuda")
    pa.pa_decode(out, case.out.new_tensor(case.q).to(torch.bfloat16), case.cache.k_cache,
                 case.cache.v_cache, bt, cl, 16000, case.scale, 16, ws)
    gh.assert_close(out.float().cpu().numpy(), gh.expected_all(case), "bf16", "large grid")
    assert pa.pa_device_errors() == 0


@pytest.mark.parametrize("bs", [1, 4, 16, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fused_step_equals_append_then_decode(bs, dtype):
    """pa_decode_append (one launch) == pa_kv_append + pa_decode, bit for bit,
    in the output and in the caches it wrote."""
    wl = _custom(8, 2, 128, dtype, bs, RAGGED + (600,))
    a = gh.build_case(wl, partition_size=48, fused=True)
    b = gh.build_case(wl, partition_size=48, fused=False)
    assert torch.equal(a.out, b.out)
    assert torch.equal(a.cache.k_cache, b.cache.k_cache)
    assert torch.equal(a.cache.v_cache, b.cache.v_cache)
    gh.assert_close(gh.gpu_out(a), gh.expected_all(a), dtype, f"fused bs={bs}")
    assert pa.pa_device_errors() == 0


def test_a_thousand_short_sequences():
    """1,100 and 1,000 short sequences (empty and exact-multiple lengths
    included) at partitions of 16 tokens: a wide grid of mostly single-chunk
    CTAs, against the oracle."""
    rng = np.random.default_rng(77)
    lens = [int(x) for x in rng.integers(0, 60, size=1100)]
    lens[:4] = [0, 15, 47, 48]
    wl = _custom(8, 2, 128, "bf16", 16, lens, seed=11)
    case = gh.build_case(wl, partition_size=16)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", "S=1100")
    small = _custom(8, 2, 128, "bf16", 16, lens[:1000], seed=11)
    case2 = gh.build_case(small, partition_size=16)
    gh.assert_close(gh.gpu_out(case2), gh.expected_all(case2), "bf16", "S=1000")
    assert pa.pa_device_errors() == 0
