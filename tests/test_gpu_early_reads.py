"""PA_DECODE_EARLY_CACHE_READS on the GPU.

With the option, a decode kernel reads context lengths, block tables and the
cached K/V before its dependent-launch wait, and reads q / k_new / v_new and
writes anything only after it. These tests chain calls so that the kernel
before a decode is one of the library's own kernels that lets its successor
start early, and that kernel produces the decode's q (or its k_new / v_new)
and reads the workspace the decode writes; every result must equal the same
chain run without the option, bit for bit.
"""

import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from workloads import configs

pytestmark = pytest.mark.gpu


def _chain(case, ps, ws, early, rounds=4):
    """out_0 = decode(q); out_{k+1} = decode(out_k): each call's q is the
    previous call's output, written by its merge kernel."""
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    outs = []
    with pa.decode_options(pa.PA_DECODE_EARLY_CACHE_READS if early else 0):
        for _ in range(rounds):
            out = torch.empty_like(q)
            pa.pa_decode(out, q, case.cache.k_cache, case.cache.v_cache, tables, lens, max_len,
                         case.scale, ps, ws)
            outs.append(out)
            q = out
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("ps", [0, 32])
def test_chained_decodes_equal_normal_mode(ps):
    case = gh.build_case(configs.llama3_8b_layer(), partition_size=ps)
    tables, lens, max_len = case.cache.tables(case.seqs)
    s, hq, d = case.q.shape
    need = pa.pa_decode_workspace_bytes(s, hq, case.cache.num_kv_heads, d, max_len, ps)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    normal = _chain(case, ps, ws, early=False)
    early = _chain(case, ps, ws, early=True)
    assert pa.pa_device_errors() == 0
    for a, b in zip(normal, early):
        assert torch.equal(a, b)
    # the first link against the oracle
    gh.assert_close(early[0].float().cpu().numpy(), gh.expected_all(case), "bf16", "early")


def test_fused_append_reads_new_rows_after_the_wait():
    """A decode step whose new K/V rows are the previous call's output (G = 1,
    so the output has the rows' shape): the rows appended to the cache and the
    step's output must equal those of the normal mode."""
    wl = configs.Workload("early_g1", 8, 8, 128, "bf16", 16, 1400, (128, 700, 1500, 300, 2900, 50),
                          5201, 6201)
    results = []
    for early in (False, True):
        case = gh.build_case(wl, partition_size=64)
        tables, lens, max_len = case.cache.tables(case.seqs)
        s, hq, d = case.q.shape
        q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
        need = pa.pa_decode_workspace_bytes(s, hq, wl.num_kv_heads, d, max_len + 1, 64)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        # the step appends one more token per sequence: slots from the block manager
        slots, cows = case.cache.bm.append_slots(case.seqs, [1] * s)
        assert len(cows) == 0
        tables2, lens2, max_len2 = case.cache.tables(case.seqs)
        with pa.decode_options(pa.PA_DECODE_EARLY_CACHE_READS if early else 0):
            rows = torch.empty_like(q)          # [S, 8, 128]: the new rows' shape (G = 1)
            pa.pa_decode(rows, q, case.cache.k_cache, case.cache.v_cache, tables, lens, max_len,
                         wl.scale, 64, ws)       # produced by a merge kernel
            out = torch.empty_like(q)
            pa.pa_decode_append(out, q, rows, rows, case.cache.k_cache, case.cache.v_cache,
                                tables2, lens2, max_len2, wl.scale, 64, ws)
        torch.cuda.synchronize()
        slot = torch.from_numpy(slots).cuda()
        flat_k = case.cache.k_cache.view(-1, wl.num_kv_heads, wl.head_dim)
        assert torch.equal(flat_k.index_select(0, slot), rows)
        results.append((rows, out))
    assert pa.pa_device_errors() == 0
    assert torch.equal(results[0][0], results[1][0])
    assert torch.equal(results[0][1], results[1][1])


def test_graph_of_layers_equals_eager_normal_mode():
    """Four 'layers' (cache replicas) captured in one CUDA graph with the option,
    the way a model's layer loop runs: each output equals the eager call
    without the option."""
    case = gh.build_case(configs.llama3_8b_layer(), partition_size=0)
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    s, hq, d = q.shape
    ps = pa.pa_decode_partition_size(s, case.cache.num_kv_heads, max_len)
    need = pa.pa_decode_workspace_bytes(s, hq, case.cache.num_kv_heads, d, max_len, ps)
    layers = []
    for i in range(4):
        k = case.cache.k_cache.clone()
        v = case.cache.v_cache.clone()
        k.mul_(1.0 + 0.25 * i)                   # every layer different
        layers.append((k, v, torch.empty_like(q), torch.empty(need, dtype=torch.uint8,
                                                                device="cuda")))
    ref = []
    for k, v, _, ws in layers:
        o = torch.empty_like(q)
        pa.pa_decode(o, q, k, v, tables, lens, max_len, case.scale, ps, ws)
        ref.append(o)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream), pa.decode_options(pa.PA_DECODE_EARLY_CACHE_READS):
        for k, v, o, ws in layers:               # warm-up outside the capture
            pa.pa_decode(o, q, k, v, tables, lens, max_len, case.scale, ps, ws)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for k, v, o, ws in layers:
                pa.pa_decode(o, q, k, v, tables, lens, max_len, case.scale, ps, ws)
    torch.cuda.synchronize()
    for _ in range(3):
        for _, _, o, _ in layers:
            o.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for (_, _, o, _), r in zip(layers, ref):
            assert torch.equal(o, r)
    assert pa.pa_device_errors() == 0
    del graph


def test_option_is_per_thread_and_restored():
    import threading

    assert pa.pa_set_decode_options(0) == 0
    with pa.decode_options(pa.PA_DECODE_EARLY_CACHE_READS):
        seen = []
        t = threading.Thread(target=lambda: seen.append(pa.pa_set_decode_options(0)))
        t.start()
        t.join()
        assert seen == [0]                       # another thread keeps its own options
        assert pa.pa_set_decode_options(pa.PA_DECODE_EARLY_CACHE_READS) == \
            pa.PA_DECODE_EARLY_CACHE_READS
    assert pa.pa_set_decode_options(0) == 0


@pytest.mark.parametrize("kv", ["", "fp8_e4m3"])
def test_chained_planned_decodes_equal_normal_mode(kv):
    """The same chain through pa_decode_planned with a work list of more items
    than one wave (partitions of 16 tokens: 665 items), so the list is read
    before the dependent-launch wait under the option: bit-identical to the
    chain without it, and to the unplanned chain."""
    import dataclasses

    import numpy as np

    wl = configs.llama3_8b_layer()
    if kv:
        wl = dataclasses.replace(wl, kv_dtype=kv)
    ps = 16
    case = gh.build_case(wl, partition_size=ps)
    tables, lens, max_len = case.cache.tables(case.seqs)
    work = torch.from_numpy(np.ascontiguousarray(pa.pa_decode_plan(lens.cpu().numpy(), ps)))
    work = work.cuda()
    assert work.shape[0] * 2 > 444
    s, hq, d = case.q.shape
    need = pa.pa_decode_workspace_bytes(s, hq, case.cache.num_kv_heads, d, max_len, ps)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    sc = dict(k_scale=case.cache.k_scale, v_scale=case.cache.v_scale) if kv else {}

    def chain(early, planned):
        q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
        outs = []
        with pa.decode_options(pa.PA_DECODE_EARLY_CACHE_READS if early else 0):
            for _ in range(4):
                out = torch.empty_like(q)
                if planned:
                    pa.pa_decode_planned(out, q, case.cache.k_cache, case.cache.v_cache, tables,
                                         lens, work, max_len, case.scale, ps, ws, **sc)
                elif kv:
                    pa.pa_decode_fp8(out, q, case.cache.k_cache, case.cache.v_cache,
                                     case.cache.k_scale, case.cache.v_scale, tables, lens,
                                     max_len, case.scale, ps, ws)
                else:
                    pa.pa_decode(out, q, case.cache.k_cache, case.cache.v_cache, tables, lens,
                                 max_len, case.scale, ps, ws)
                outs.append(out)
                q = out
        torch.cuda.synchronize()
        return outs

    ref = chain(False, False)
    for early in (False, True):
        for a, b in zip(ref, chain(early, True)):
            assert torch.equal(a, b)
    assert pa.pa_device_errors() == 0
