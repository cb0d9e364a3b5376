"""pa_prefill (causal chunked prefill over the paged cache, tcgen05) against the oracle.

The GPU side goes through PagedKVCache.prefill: the chunk's K/V rows are
appended through the native block manager and pa_kv_append, then pa_prefill
attends. The oracle side is oracle.attention.prefill (or, for sampled rows of
large cases, the plain softmax over the generator's rows), fed from the same
seeded generator rows and never from the GPU.
"""

import ctypes

import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from oracle import attention as oatt
from paged_kv_cache_345_b200.cache import PagedKVCache
from workloads import synth

pytestmark = pytest.mark.gpu

D = 128
SEED = 1006


def _rows(s, n, hkv):
    k, v = synth.kv_rows(SEED, s, n, hkv, D)
    return gh.stored(k, "bf16"), gh.stored(v, "bf16")


def _queries(s, n, hq):
    return gh.stored(synth.queries(SEED, 1 + s, n, hq, D), "bf16")


def _run(before, chunks, hq=32, hkv=8, bs=16, free_order=None, poisoned=False, spare=8):
    """Prefill `before[s]` tokens (cache writes only), then one chunk of
    `chunks[s]` tokens per sequence through PagedKVCache.prefill."""
    lens = [b + c for b, c in zip(before, chunks)]
    nb = sum(-(-L // bs) for L in lens) + spare
    if free_order is None:
        free_order = synth.block_permutation(nb, 2006 + bs)
    cache = PagedKVCache(nb, bs, hkv, D, "bf16", "cuda", max_blocks_per_seq=max(
        1, max(-(-L // bs) for L in lens)), free_order=free_order)
    if poisoned:
        gh.poison(cache.k_cache)
        gh.poison(cache.v_cache)
    seqs = [cache.add_sequence() for _ in lens]
    rows = [_rows(s, L, hkv) for s, L in enumerate(lens)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.bfloat16)  # noqa
    if sum(before):
        cache.write(seqs, list(before), dev(np.concatenate([r[0][:b] for r, b in zip(rows, before)])),
                    dev(np.concatenate([r[1][:b] for r, b in zip(rows, before)])))
    q = np.concatenate([_queries(s, c, hq) for s, c in enumerate(chunks)])
    kc = dev(np.concatenate([r[0][b:] for r, b in zip(rows, before)]))
    vc = dev(np.concatenate([r[1][b:] for r, b in zip(rows, before)]))
    qd = dev(q)
    out = torch.full_like(qd, float("nan"))     # a row the kernel skips stays NaN
    out = cache.prefill(qd, kc, vc, seqs, list(chunks), 1 / np.sqrt(D), out=out)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out.float().cpu().numpy(), q, rows, lens


def _expected(q, rows, lens, chunks, hq):
    """Oracle prefill over the generator's rows in an identity-placed block-size-1 cache."""
    kc = np.concatenate([r[0] for r in rows])[:, None]
    vc = np.concatenate([r[1] for r in rows])[:, None]
    offs = np.concatenate([[0], np.cumsum(lens)])
    tables = np.zeros((len(lens), max(lens)), dtype=np.int64)
    for s, L in enumerate(lens):
        tables[s, :L] = np.arange(offs[s], offs[s] + L)
    qs = np.concatenate([[0], np.cumsum(chunks)])
    return oatt.prefill(q, kc, vc, tables, lens, qs, 1 / np.sqrt(D), 1)


def _expected_row(q_row, rows_s, L, n, i, hq, hkv):
    """One query row (all heads) by the plain softmax over its visible keys."""
    p = L - n + i
    g = hq // hkv
    return np.stack([oatt.softmax_attention(q_row[j], rows_s[0][:p + 1, j // g],
                                            rows_s[1][:p + 1, j // g], 1 / np.sqrt(D))
                     for j in range(hq)])


def test_prefill_whole_and_chunked_prompts_match_oracle():
    before, chunks = [0, 0, 100, 250, 7], [1, 37, 60, 300, 129]
    got, q, rows, lens = _run(before, chunks)
    gh.assert_close(got, _expected(q, rows, lens, chunks, 32), "bf16", "prefill")


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (16, 2), (64, 8), (8, 1)])
def test_prefill_group_sizes(hq, hkv):
    before, chunks = [0, 200, 3], [300, 129, 1]
    got, q, rows, lens = _run(before, chunks, hq=hq, hkv=hkv)
    gh.assert_close(got, _expected(q, rows, lens, chunks, hq), "bf16", f"prefill {hq}/{hkv}")


@pytest.mark.parametrize("S,hq,hkv,seed", [(5, 2, 2, 1), (33, 16, 2, 2), (70, 8, 2, 3),
                                         (200, 4, 2, 4), (300, 8, 2, 5)])
def test_prefill_work_order_covers_every_row(S, hq, hkv, seed):
    """Batches of 5 to 300 sequences with mixed lengths and empty chunks: CTAs
    take their work items longest first (up to 256 sequences, the per-lane
    layouts of 1, 2, 4 and 8 sequences per lane) or pair by pair past that;
    every row must be computed exactly once."""
    rng = np.random.default_rng(seed)
    total = rng.integers(0, 300 if S <= 70 else 40, S)
    chunks = [0 if rng.random() < 0.2 else int(rng.integers(0, L + 1)) for L in total]
    before = [int(L) - c for L, c in zip(total, chunks)]
    got, q, rows, lens = _run(before, chunks, hq=hq, hkv=hkv)
    keep = [s for s, c in enumerate(chunks) if c]
    ref = _expected(q, [rows[s] for s in keep], [lens[s] for s in keep],
                    [chunks[s] for s in keep], hq)
    gh.assert_close(got, ref, "bf16", f"prefill order S={S}")


def test_prefill_is_bitwise_invariant_to_block_size_and_placement():
    before, chunks = [0, 130, 400], [250, 97, 128]
    ref, q, rows, lens = _run(before, chunks, bs=16)
    gh.assert_close(ref, _expected(q, rows, lens, chunks, 32), "bf16", "prefill bs=16")
    for bs in (8, 32, 64, 128, 256):
        got, *_ = _run(before, chunks, bs=bs)
        assert np.array_equal(got, ref), f"block_size {bs}"
    nb = sum(-(-L // 16) for L in lens) + 8
    got, *_ = _run(before, chunks, bs=16, free_order=np.arange(nb))
    assert np.array_equal(got, ref), "identity placement"


def test_prefill_poisoned_pool_and_ragged_tails():
    """Every slot never written holds NaN bits: keys past the context must never
    reach the output, whatever the block tail or the last key tile holds."""
    before, chunks = [0, 5, 129, 0], [3, 11, 126, 255]
    got, q, rows, lens = _run(before, chunks, poisoned=True)
    gh.assert_close(got, _expected(q, rows, lens, chunks, 32), "bf16", "prefill poisoned")


def test_prefill_worked_example_prompts_sampled():
    """The worked example's eight prompts, whole (10,578 query rows): sampled rows,
    including every sequence's first and last rows and rows at tile edges."""
    lens = list(synth.LLAMA3_8B_BATCH_LENGTHS)
    got, q, rows, _ = _run([0] * len(lens), lens)
    qs = np.concatenate([[0], np.cumsum(lens)])
    rng = np.random.default_rng(5)
    for s, L in enumerate(lens):
        picks = {0, L - 1, min(L - 1, 31), min(L - 1, 32), min(L - 1, 127), min(L - 1, 128)}
        picks |= set(rng.integers(0, L, 4).tolist())
        for i in sorted(picks):
            ref = _expected_row(q[qs[s] + i], rows[s], L, L, i, 32, 8)
            gh.assert_close(got[qs[s] + i], ref, "bf16", f"prefill s={s} row {i}")


def test_prefill_one_token_chunks_are_decode_steps():
    before = [5, 300, 1000]
    got, q, rows, lens = _run(before, [1, 1, 1])
    ref = _expected(q, rows, lens, [1, 1, 1], 32)
    gh.assert_close(got, ref, "bf16", "prefill of one-token chunks")
    # the decode oracle on the same rows (context = the whole sequence)
    dec = np.stack([np.stack([oatt.softmax_attention(q[s, j], rows[s][0][:, j // 4],
                                                     rows[s][1][:, j // 4], 1 / np.sqrt(D))
                              for j in range(32)]) for s in range(3)])
    assert np.allclose(ref, dec, atol=1e-12, rtol=0)


def _raw_prefill(out, q, k, v, tables, lens, qs, S, total_q, hq, hkv, bs, nb, mbps, maxq, dtype):
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return pa._lib.pa_prefill(p(out), p(q), p(k), p(v), p(tables), p(lens), p(qs), S, total_q, hq,
                              hkv, D, bs, nb, mbps, maxq, 0.1, dtype,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_prefill_bad_chunk_is_flagged_and_skipped():
    k = torch.zeros((4, 16, 2, D), dtype=torch.bfloat16, device="cuda")
    q = torch.ones((8, 4, D), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 5.0)
    tables = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([3, 20], dtype=torch.int32, device="cuda")   # seq 0: 4 rows > 3 tokens
    qs = torch.tensor([0, 4, 8], dtype=torch.int32, device="cuda")
    st = _raw_prefill(out, q, k, k, tables, lens, qs, 2, 8, 4, 2, 16, 4, 2, 4, pa.PA_BF16)
    assert st == pa.PA_OK
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT
    assert bool((out[:4] == 5.0).all())          # skipped
    assert bool((out[4:] == 0.0).all())          # V = 0 everywhere -> zeros


def test_prefill_refusals():
    k = torch.zeros((4, 4, 2, D), dtype=torch.bfloat16, device="cuda")
    q = torch.ones((4, 4, D), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 5.0)
    tables = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    lens = torch.tensor([4], dtype=torch.int32, device="cuda")
    qs = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    st = _raw_prefill(out, q, k, k, tables, lens, qs, 1, 4, 4, 2, 4, 4, 4, 4, pa.PA_BF16)
    assert st == pa.PA_ERR_UNSUPPORTED and "block_size" in pa._lib.pa_last_error().decode()
    st = _raw_prefill(out, q, k, k, tables, lens, qs, 1, 4, 4, 2, 16, 1, 4, 4, pa.PA_F32)
    assert st == pa.PA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((out == 5.0).all())


def test_prefill_empty_chunks_and_empty_sequences():
    """Sequences with no query rows in the batch (a zero-row chunk, or nothing
    cached at all) produce nothing and disturb nothing."""
    before, chunks = [5, 0, 40, 0], [3, 0, 0, 70]
    got, q, rows, lens = _run(before, chunks)
    keep = [s for s, c in enumerate(chunks) if c]
    ref = _expected(q, [rows[s] for s in keep], [lens[s] for s in keep],
                    [chunks[s] for s in keep], 32)
    gh.assert_close(got, ref, "bf16", "prefill with empty chunks")


def test_prefill_chunk_above_host_bound_is_flagged_and_skipped():
    """A chunk longer than max_query_len would have rows outside the grid: the
    sequence is flagged and skipped, the others are computed as usual."""
    k = torch.zeros((4, 16, 2, D), dtype=torch.bfloat16, device="cuda")
    q = torch.ones((9, 4, D), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 5.0)
    tables = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([20, 20], dtype=torch.int32, device="cuda")
    qs = torch.tensor([0, 5, 9], dtype=torch.int32, device="cuda")   # seq 0: 5 rows > bound 4
    st = _raw_prefill(out, q, k, k, tables, lens, qs, 2, 9, 4, 2, 16, 4, 2, 4, pa.PA_BF16)
    assert st == pa.PA_OK
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT
    assert bool((out[:5] == 5.0).all())          # skipped
    assert bool((out[5:] == 0.0).all())          # V = 0 everywhere -> zeros


def _planned_case(hq, hkv, before, chunks, bs=16):
    lens = [b + c for b, c in zip(before, chunks)]
    nb = sum(-(-L // bs) for L in lens) + 8
    cache = PagedKVCache(nb, bs, hkv, D, "bf16", "cuda",
                         max_blocks_per_seq=max(1, max(-(-L // bs) for L in lens)),
                         free_order=synth.block_permutation(nb, 3006 + bs))
    seqs = [cache.add_sequence() for _ in lens]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.bfloat16)  # noqa
    rows = [_rows(s, L, hkv) for s, L in enumerate(lens)]
    cache.write(seqs, lens, dev(np.concatenate([r[0] for r in rows])),
                dev(np.concatenate([r[1] for r in rows])))
    q = dev(np.concatenate([_queries(s, c, hq) for s, c in enumerate(chunks)]))
    tables, ctx, _ = cache.tables(seqs)
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    return cache, q, tables, ctx, qs, np.asarray(lens, dtype=np.int32)


@pytest.mark.parametrize("hq,hkv,before,chunks", [
    (32, 8, [0, 0, 0, 0, 0], [129, 700, 1500, 300, 2900]),      # whole prompts, G = 4
    (32, 8, [128, 700, 1500, 300], [512, 512, 512, 512]),       # chunks on cached contexts
    (8, 8, [0, 50, 0, 3], [300, 7, 1000, 0]),                   # G = 1, an empty chunk
    (32, 4, [10, 0], [600, 900]),                               # G = 8
])
def test_planned_prefill_equals_the_searching_kernel(hq, hkv, before, chunks):
    """pa_prefill_planned on pa_prefill_plan's list: every row computed, bit for
    bit what pa_prefill (each CTA finding its own item) computes."""
    cache, q, tables, ctx, qs, lens = _planned_case(hq, hkv, before, chunks)
    qs_d = torch.from_numpy(qs).cuda()
    work = torch.from_numpy(np.ascontiguousarray(pa.pa_prefill_plan(qs, lens, hq, hkv))).cuda()
    a, b = torch.full_like(q, float("nan")), torch.full_like(q, float("nan"))
    pa.pa_prefill(a, q, cache.k_cache, cache.v_cache, tables, ctx, qs_d, max(chunks),
                  1 / np.sqrt(D))
    pa.pa_prefill(b, q, cache.k_cache, cache.v_cache, tables, ctx, qs_d, max(chunks),
                  1 / np.sqrt(D), work=work)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert not torch.isnan(b).any()
    assert torch.equal(a, b)


def test_planned_prefill_flags_an_item_outside_the_batch():
    cache, q, tables, ctx, qs, lens = _planned_case(32, 8, [0, 0], [200, 300])
    work = np.ascontiguousarray(pa.pa_prefill_plan(qs, lens, 32, 8)).copy()
    work[0, 0] = 2                                   # no sequence 2
    out = torch.full_like(q, float("nan"))
    pa.pa_prefill(out, q, cache.k_cache, cache.v_cache, tables, ctx, torch.from_numpy(qs).cuda(),
                  300, 1 / np.sqrt(D), work=torch.from_numpy(work).cuda())
    torch.cuda.synchronize()
    assert pa.pa_device_errors() & pa.PA_DEVERR_PLAN
