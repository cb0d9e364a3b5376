"""The split-K workspace of pa_decode, on the GPU.

A sequence longer than one partition is split: each partition's partial
results (running maximum, sum, unnormalised output) go to the caller's
workspace, and a merge kernel combines them. The workspace needs no clearing,
before the first call or between calls of any shape, because every value the
merge reads is written by the same call first; these tests hold the library
to that: garbage-filled, reused and graph-replayed workspaces give
bit-identical outputs, which also agree with the float64 oracle.
"""

import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from workloads import configs

pytestmark = pytest.mark.gpu


def _decode(case, ps, ws, q=None, lens_override=None):
    tables, lens, max_len = case.cache.tables(case.seqs)
    if lens_override is not None:
        lens = lens_override
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16) if q is None else q
    out = torch.full_like(q, float("nan"))
    pa.pa_decode(out, q, case.cache.k_cache, case.cache.v_cache, tables, lens, max_len,
                 case.scale, ps, ws)
    return out


def _workspace_bytes(case, ps):
    tables, lens, max_len = case.cache.tables(case.seqs)
    s, hq, d = case.q.shape
    return pa.pa_decode_workspace_bytes(s, hq, case.cache.num_kv_heads, d, max_len, ps)


@pytest.mark.parametrize("ps", [16, 64])
def test_workspace_contents_are_ignored(ps):
    """Zeros, all-ones bytes, random bytes and a workspace left behind by a call
    with another partition size all give the same bits."""
    case = gh.build_case(configs.llama3_8b_layer(), partition_size=ps)
    need = _workspace_bytes(case, ps)
    outs = []
    for fill in ("zeros", "ones", "random"):
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        if fill == "ones":
            ws.fill_(0xFF)
        elif fill == "random":
            ws.random_(0, 256, generator=torch.Generator("cuda").manual_seed(5))
        outs.append(_decode(case, ps, ws))
    # a larger workspace first used with partitions of 48 tokens (records and
    # counters in other places), then reused
    other = _workspace_bytes(case, 48)
    ws = torch.zeros(max(need, other) + 4096, dtype=torch.uint8, device="cuda")
    _decode(case, 48, ws)
    outs.append(_decode(case, ps, ws))
    outs.append(_decode(case, ps, ws))
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    gh.assert_close(outs[0].float().cpu().numpy(), gh.expected_all(case), "bf16", f"P={ps}")


def test_graph_replays_match_eager():
    """One workspace, the decode captured in a CUDA graph and replayed: every
    replay gives the eager call's bits."""
    ps = 32
    case = gh.build_case(configs.llama3_8b_layer(), partition_size=ps)
    need = _workspace_bytes(case, ps)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    eager = _decode(case, ps, ws, q=q)
    torch.cuda.synchronize()
    out = torch.zeros_like(q)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        pa.pa_decode(out, q, case.cache.k_cache, case.cache.v_cache, tables, lens, max_len,
                     case.scale, ps, ws)   # warm-up outside the capture
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            pa.pa_decode(out, q, case.cache.k_cache, case.cache.v_cache, tables, lens, max_len,
                         case.scale, ps, ws)
    torch.cuda.synchronize()
    for _ in range(3):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    assert pa.pa_device_errors() == 0
    del graph


def test_back_to_back_calls_sharing_a_workspace():
    """Two different batches decoded one after the other with the same
    workspace (other lengths, so other units split into other numbers of
    partitions): each equals its own call on a fresh workspace."""
    ps = 48
    case = gh.build_case(configs.llama3_8b_layer(), partition_size=ps)
    tables, lens, max_len = case.cache.tables(case.seqs)
    short = (lens.cpu() // 3).to(torch.int32).cuda()      # every context a third as long
    need = _workspace_bytes(case, ps)
    shared = torch.empty(need, dtype=torch.uint8, device="cuda")
    a1 = _decode(case, ps, shared)
    b1 = _decode(case, ps, shared, lens_override=short)
    a2 = _decode(case, ps, shared)
    b2 = _decode(case, ps, shared, lens_override=short)
    a_ref = _decode(case, ps, torch.zeros(need, dtype=torch.uint8, device="cuda"))
    b_ref = _decode(case, ps, torch.zeros(need, dtype=torch.uint8, device="cuda"),
                    lens_override=short)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert torch.equal(a1, a_ref) and torch.equal(a2, a_ref)
    assert torch.equal(b1, b_ref) and torch.equal(b2, b_ref)
    assert not torch.equal(a_ref, b_ref)
    # the shortened batch against the oracle (first third of each context)
    n = short.cpu().numpy()
    for s in range(len(n)):
        case.rows_k[s] = case.rows_k[s][:n[s]]
        case.rows_v[s] = case.rows_v[s][:n[s]]
    gh.assert_close(b_ref.float().cpu().numpy(), gh.expected_all(case), "bf16", "short batch")


@pytest.mark.parametrize("group", [1, 8])
def test_many_pieces_merge(group):
    """A 3000-token context at partitions of 16 tokens: 188 partitions merged
    for one sequence (more than the merge loads in one batch)."""
    wl = configs.Workload(f"pieces_g{group}", 2 * group, 2, 128, "bf16", 16, 200, (2999, 40),
                          5101, 6101)
    case = gh.build_case(wl, partition_size=16)
    gh.assert_close(gh.gpu_out(case), gh.expected_all(case), "bf16", f"G={group}")
    assert pa.pa_device_errors() == 0
    assert np.isfinite(gh.gpu_out(case)).all()
