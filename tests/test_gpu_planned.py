"""pa_decode_planned on the GPU: the decode on a pa_decode_plan work list.

The plan changes which CTAs run and in what order, never what a CTA computes,
so the planned call must match the plain (partition, sequence) grid bit for
bit (outputs and the caches after the fused append) for every group size,
block size, partition size and mix of lengths, bf16 and E4M3 alike; and it is
checked against the float64 oracle on a batch of mixed lengths. A work list
that disagrees with the device lengths, or names a sequence outside the
batch, sets PA_DEVERR_PLAN (no out-of-range access: the kernel checks every
item before using it). The library reads the list only when its items take
more than one wave of resident CTAs (a few hundred on a B200), so the cases
here list 600 to 3,000 items; one small case checks that a list that fits
one wave is not read. "Paged Attention" (klaylearn.com glossary),
definition: decode reads each sequence's blocks through its table.
"""


import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from workloads import configs, synth

pytestmark = pytest.mark.gpu

RAGGED = (0, 1, 14, 15, 16, 17, 31, 47, 100, 257, 600)
LONG = RAGGED + tuple(range(400, 6400, 400))   # ~51k tokens: 3,200 items of 16 tokens


def _custom(hq, hkv, d, bs, lens, kv="", seed=11):
    need = sum(-(-(n + 1) // bs) for n in lens)
    return configs.Workload(f"planned_{hq}_{hkv}_{d}_{bs}", hq, hkv, d, "bf16", bs, need + 8,
                            tuple(lens), 7000 + seed, 8000 + seed, kv_dtype=kv)


def _pair(wl, ps, fused=True):
    """The same step planned and on the plain grid, from one staging of the rows."""
    staged = gh.stage_rows(wl, keep=set())
    a = gh.build_case(wl, partition_size=ps, planned=True, staged=staged, fused=fused)
    b = gh.build_case(wl, partition_size=ps, planned=False, staged=staged, fused=fused)
    return a, b


def _same(a, b, what):
    assert torch.equal(a.out, b.out), f"{what}: outputs differ"
    assert torch.equal(a.cache.k_cache, b.cache.k_cache), f"{what}: K caches differ"
    assert torch.equal(a.cache.v_cache, b.cache.v_cache), f"{what}: V caches differ"


@pytest.mark.parametrize("kv", ["", gh.FP8])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_planned_equals_plain_grid(kv, group):
    wl = _custom(2 * group, 2, 128, 16, LONG, kv)
    for ps in (16, 64):
        a, b = _pair(wl, ps)
        _same(a, b, f"kv={kv or 'bf16'} G={group} P={ps}")
    assert pa.pa_device_errors() == 0


@pytest.mark.parametrize("kv", ["", gh.FP8])
@pytest.mark.parametrize("bs", [1, 4, 32, 256])
def test_planned_block_sizes(kv, bs):
    wl = _custom(8, 2, 128, bs, LONG, kv)
    a, b = _pair(wl, 16)
    _same(a, b, f"bs={bs}")
    assert pa.pa_device_errors() == 0


def test_planned_head_dim_64_and_unfused():
    wl = _custom(16, 4, 64, 16, LONG)
    for fused in (True, False):
        a, b = _pair(wl, 32, fused)
        _same(a, b, f"d=64 fused={fused}")
    assert pa.pa_device_errors() == 0


@pytest.mark.parametrize("kv", ["", gh.FP8])
def test_planned_mixed_batch_against_oracle(kv):
    """60 lognormal lengths (many short, a few of several partitions) plus empty
    and exact-multiple contexts: every row against the float64 oracle."""
    lens = synth.lognormal_lengths(60, 300, 0.9, 1, 2000, 4242).tolist() + [0, 127, 255, 1023]
    wl = _custom(32, 8, 128, 16, lens, kv, seed=3)
    case = gh.build_case(wl, partition_size=64, planned=True)
    # (E4M3: the oracle runs on the dequantised codes; the bf16 tolerance)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", f"planned {kv or 'bf16'}")
    assert pa.pa_device_errors() == 0


def _direct(case, work, max_len, ps, ws):
    tables, lens, _ = case.cache.tables(case.seqs)
    out = torch.empty_like(case.out)
    q = torch.from_numpy(case.q).to("cuda", torch.bfloat16)
    pa.pa_decode_planned(out, q, case.cache.k_cache, case.cache.v_cache, tables, lens,
                         torch.from_numpy(np.ascontiguousarray(work)).cuda(), max_len,
                         case.scale, ps, ws)
    torch.cuda.synchronize()
    return out


def test_plan_mismatch_and_bad_items_are_flagged():
    wl = _custom(8, 2, 128, 16, (40, 3000, 7000, 5))      # 630 items of 16 tokens
    case = gh.build_case(wl, partition_size=16, planned=False)
    lens = np.asarray([case.cache.context_len(s) for s in case.seqs], dtype=np.int32)
    ps, max_len = 16, int(lens.max())
    ws = torch.empty(pa.pa_decode_workspace_bytes(4, 8, 2, 128, max_len, ps), dtype=torch.uint8,
                     device="cuda")
    assert pa.pa_device_errors() == 0
    # the right plan: the plain grid's output, no flag
    good = pa.pa_decode_plan(lens, ps)
    ref = _direct(case, good, max_len, ps, ws)
    assert torch.equal(ref, case.out)
    assert pa.pa_device_errors() == 0
    # a plan made for shorter contexts: too few partitions for sequence 2
    short = lens.copy()
    short[2] -= 2000
    _direct(case, pa.pa_decode_plan(short, ps), max_len, ps, ws)
    assert pa.pa_device_errors() & pa.PA_DEVERR_PLAN
    # an item naming a sequence outside the batch, and one past every partition
    bad = good.copy()
    bad[0, 0] = 4
    bad[1, 1] = (bad[1, 1] & ~0xFFFF) | 0x7FFF
    _direct(case, bad, max_len, ps, ws)
    assert pa.pa_device_errors() & pa.PA_DEVERR_PLAN
    # the device is still fine: the right plan again
    assert torch.equal(_direct(case, good, max_len, ps, ws), case.out)
    assert pa.pa_device_errors() == 0


def test_a_list_within_one_wave_is_not_read():
    """Four short sequences: every item fits one wave, the plain grid runs and a
    list with a bad item changes nothing (not read, not flagged)."""
    wl = _custom(8, 2, 128, 16, (40, 300, 700, 5))
    case = gh.build_case(wl, partition_size=64, planned=False)
    lens = np.asarray([case.cache.context_len(s) for s in case.seqs], dtype=np.int32)
    max_len = int(lens.max())
    ws = torch.empty(pa.pa_decode_workspace_bytes(4, 8, 2, 128, max_len, 64), dtype=torch.uint8,
                     device="cuda")
    bad = pa.pa_decode_plan(lens, 64).copy()
    bad[0, 0] = 4
    assert torch.equal(_direct(case, bad, max_len, 64, ws), case.out)
    assert pa.pa_device_errors() == 0


def test_planned_steps_in_a_serving_loop_and_a_graph():
    """Several cache-level decode steps (contexts grow, partitions appear),
    planned vs plain on two identical caches; then the planned call captured
    in a CUDA graph and replayed gives the same output."""
    lens0 = (3, 60, 95, 96, 97, 250, 511) + tuple(range(1000, 9000, 1000))   # ~1,160 items
    wl = _custom(32, 8, 128, 16, lens0)
    n = len(lens0)
    a, b = _pair(wl, 32)
    _same(a, b, "first step")
    rng = np.random.default_rng(5)
    for step in range(6):
        q = torch.from_numpy(rng.standard_normal((n, 32, 128)).astype(np.float32)).cuda()
        kn = torch.from_numpy(rng.standard_normal((n, 8, 128)).astype(np.float32)).cuda()
        q, kn = q.to(torch.bfloat16), kn.to(torch.bfloat16)
        vn = (kn * 0.5).contiguous()
        oa = a.cache.decode_step(q, kn, vn, a.seqs, wl.scale, 32, planned=True)
        ob = b.cache.decode_step(q, kn, vn, b.seqs, wl.scale, 32, planned=False)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob), f"step {step}"
    assert torch.equal(a.cache.k_cache, b.cache.k_cache)
    assert pa.pa_device_errors() == 0

    tables, lens_d, max_len = a.cache.tables(a.seqs)
    lens = lens_d.cpu().numpy()
    work = torch.from_numpy(np.ascontiguousarray(pa.pa_decode_plan(lens, 32))).cuda()
    ws = a.cache.workspace(n, 32, max_len, 32)
    q = torch.from_numpy(rng.standard_normal((n, 32, 128)).astype(np.float32)).cuda()
    q = q.to(torch.bfloat16)
    eager = torch.empty_like(q)
    pa.pa_decode_planned(eager, q, a.cache.k_cache, a.cache.v_cache, tables, lens_d, work,
                         max_len, wl.scale, 32, ws)
    out = torch.zeros_like(q)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        pa.pa_decode_planned(out, q, a.cache.k_cache, a.cache.v_cache, tables, lens_d, work,
                             max_len, wl.scale, 32, ws, stream=stream)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    del graph
    assert pa.pa_device_errors() == 0


LLAMA_LENS = (128, 700, 1500, 300, 2900, 50, 4100, 900)


@pytest.mark.parametrize("kv", ["", gh.FP8])
@pytest.mark.parametrize("hq,hkv,ps", [(32, 8, 96), (32, 8, 512), (8, 8, 128), (32, 4, 160)])
def test_one_wave_planned_calls_match_the_unplanned_ones(kv, hq, hkv, ps):
    """Batches whose items fit one wave (the Llama-3-8B layer's lengths): the
    planned call runs the plain grid; it equals the unplanned call bit for bit,
    call after call, and in a CUDA graph replayed three times."""
    wl = _custom(hq, hkv, 128, 16, LLAMA_LENS, kv, seed=21)
    a, b = _pair(wl, ps)
    _same(a, b, f"{kv or 'bf16'} {hq}/{hkv} P={ps}")
    tables, lens_d, max_len = a.cache.tables(a.seqs)
    lens = lens_d.cpu().numpy()
    work = torch.from_numpy(np.ascontiguousarray(pa.pa_decode_plan(lens, ps))).cuda()
    n = len(LLAMA_LENS)
    ws = a.cache.workspace(n, hq, max_len, ps)
    sc = dict(k_scale=a.cache.k_scale, v_scale=a.cache.v_scale) if kv else {}
    rng = np.random.default_rng(ps + hq)
    for i in range(3):
        q = torch.from_numpy(rng.standard_normal((n, hq, 128)).astype(np.float32))
        q = q.to("cuda", torch.bfloat16)
        got, want = torch.empty_like(q), torch.empty_like(q)
        pa.pa_decode_planned(got, q, a.cache.k_cache, a.cache.v_cache, tables, lens_d, work,
                             max_len, wl.scale, ps, ws, **sc)
        if kv:
            pa.pa_decode_fp8(want, q, b.cache.k_cache, b.cache.v_cache, b.cache.k_scale,
                             b.cache.v_scale, tables, lens_d, max_len, wl.scale, ps,
                             b.cache.workspace(n, hq, max_len, ps))
        else:
            pa.pa_decode(want, q, b.cache.k_cache, b.cache.v_cache, tables, lens_d, max_len,
                         wl.scale, ps, b.cache.workspace(n, hq, max_len, ps))
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"call {i}"
    q = torch.from_numpy(rng.standard_normal((n, hq, 128)).astype(np.float32))
    q = q.to("cuda", torch.bfloat16)
    eager, out = torch.empty_like(q), torch.zeros_like(q)
    pa.pa_decode_planned(eager, q, a.cache.k_cache, a.cache.v_cache, tables, lens_d, work,
                         max_len, wl.scale, ps, ws, **sc)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        pa.pa_decode_planned(out, q, a.cache.k_cache, a.cache.v_cache, tables, lens_d, work,
                             max_len, wl.scale, ps, ws, stream=stream, **sc)
    for _ in range(3):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    del graph
    assert pa.pa_device_errors() == 0
