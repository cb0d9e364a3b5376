"""pa_decode_shared_prefix on the GPU: decode for sequences that share their
first blocks ("PagedAttention — AI Glossary", How it works, step 4), the shared
prefix attended once for the whole batch on the tensor cores, each sequence's
own tokens by the decode kernel, the two merged per row.

The result is attention over each sequence's whole context: it must match the
float64 oracle (bf16 tolerance) and the plain paged decode of the same tokens;
with the step's append, the cache rows it writes must equal pa_decode_append's
bit for bit.
"""

import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from workloads import configs

pytestmark = pytest.mark.gpu


def _shared_decode(case, prefix_len, k_new=None, v_new=None, ps=0):
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    s, hq, d = q.shape
    need = pa.pa_decode_shared_prefix_workspace_bytes(s, hq, case.cache.num_kv_heads, d,
                                                      prefix_len, max_len, ps)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)  # contents on entry are ignored
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_shared_prefix(out, q, k_new, v_new, case.cache.k_cache, case.cache.v_cache,
                               tables, lens, prefix_len, max_len, case.scale, ps, ws)
    torch.cuda.synchronize()
    return out


def test_shared_prefix_workload_matches_oracle_and_paged_decode():
    """64 sequences forked from a 2,053-token parent (the 128 whole blocks stay
    shared, the partly filled 129th was copied on write) plus their own
    suffixes: attended after the step's append."""
    wl = configs.shared_prefix()
    case = gh.build_case(wl)
    prefix = (wl.shared_prefix // wl.block_size) * wl.block_size
    out = _shared_decode(case, prefix)
    assert pa.pa_device_errors() == 0
    got = out.float().cpu().numpy()
    gh.assert_close(got, gh.expected_all(case), "bf16", "shared prefix vs oracle")
    gh.assert_close(got, gh.gpu_out(case), "bf16", "shared prefix vs pa_decode_append")


def _custom(hq, hkv, bs, prefix, suffixes, seed):
    lens = tuple(prefix + x for x in suffixes)
    nb = -(-prefix // bs) + sum(-(-(x + 2) // bs) for x in suffixes) + 16
    return configs.Workload(f"shared_{hq}_{hkv}_{bs}_{prefix}", hq, hkv, 128, "bf16", bs, nb, lens,
                            5400 + seed, 6400 + seed, shared_prefix=prefix)


@pytest.mark.parametrize("hq,hkv,bs,prefix,nseq", [
    (8, 8, 16, 144, 5),      # group 1; a prefix that is not a multiple of 64 keys
    (16, 8, 32, 320, 12),    # group 2, block 32
    (32, 8, 8, 512, 70),     # group 4, block 8, two pairs of query tiles (64 rows each)
    (16, 2, 64, 1024, 9),    # group 8, block 64
])
def test_ragged_shapes(hq, hkv, bs, prefix, nseq):
    rng = np.random.default_rng(nseq)
    suffixes = [0] + [int(x) for x in rng.integers(0, 300, size=nseq - 1)]
    wl = _custom(hq, hkv, bs, prefix, suffixes, nseq)
    case = gh.build_case(wl)
    out = _shared_decode(case, prefix, ps=64)
    assert pa.pa_device_errors() == 0
    got = out.float().cpu().numpy()
    gh.assert_close(got, gh.expected_all(case), "bf16", f"G={hq // hkv} bs={bs}")
    gh.assert_close(got, gh.gpu_out(case), "bf16", "vs pa_decode_append")


def test_fused_append_writes_what_decode_append_writes():
    """A second decode step, once through pa_decode_append and once through
    pa_decode_shared_prefix on a copy of the cache: identical cache contents,
    outputs within tolerance of each other."""
    wl = _custom(32, 8, 16, 256, [3, 40, 17, 200], 1)
    case = gh.build_case(wl)
    s = len(case.seqs)
    slots, cows = case.cache.bm.append_slots(case.seqs, [1] * s)
    assert len(cows) == 0
    tables, lens, max_len = case.cache.tables(case.seqs)
    gen = torch.Generator(device="cuda").manual_seed(3)
    k_new = torch.randn((s, 8, 128), device="cuda", generator=gen).to(torch.bfloat16)
    v_new = torch.randn((s, 8, 128), device="cuda", generator=gen).to(torch.bfloat16)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    k_a, v_a = case.cache.k_cache.clone(), case.cache.v_cache.clone()
    ws_a = torch.empty(pa.pa_decode_workspace_bytes(s, 32, 8, 128, max_len, 64) + 16,
                       dtype=torch.uint8, device="cuda")
    out_a = torch.empty_like(q)
    pa.pa_decode_append(out_a, q, k_new, v_new, k_a, v_a, tables, lens, max_len, wl.scale, 64,
                        ws_a)
    ws_b = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(s, 32, 8, 128, 256, max_len, 64),
                       dtype=torch.uint8, device="cuda")
    out_b = torch.empty_like(q)
    pa.pa_decode_shared_prefix(out_b, q, k_new, v_new, case.cache.k_cache, case.cache.v_cache,
                               tables, lens, 256, max_len, wl.scale, 64, ws_b)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert torch.equal(case.cache.k_cache, k_a) and torch.equal(case.cache.v_cache, v_a)
    gh.assert_close(out_b.float().cpu().numpy(), out_a.float().cpu().numpy(), "bf16", "append")


def test_context_shorter_than_the_prefix_is_flagged():
    wl = _custom(32, 8, 16, 256, [10, 20], 2)
    case = gh.build_case(wl)
    tables, lens, max_len = case.cache.tables(case.seqs)
    short = lens.clone()
    short[1] = 100                     # shorter than the 256-token prefix
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(2, 32, 8, 128, 256, max_len, 0),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    pa.pa_decode_shared_prefix(out, q, None, None, case.cache.k_cache, case.cache.v_cache, tables,
                               short, 256, max_len, wl.scale, 0, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() & pa.PA_DEVERR_CONTEXT
    # the sequence with a valid context is still right
    ref = gh.expected_all(case)
    gh.assert_close(out[0].float().cpu().numpy(), ref[0], "bf16", "valid row")


def test_every_context_is_the_prefix():
    """No sequence has tokens of its own (contexts of exactly the prefix, no
    newest token to append): every CTA of the suffix decode leaves at once, and
    the merge still waits for the prefix pass; each row is the attention over
    the prefix alone."""
    from oracle import attention as oatt

    wl = _custom(32, 8, 16, 512, [0, 5, 9], 3)
    case = gh.build_case(wl)
    tables, lens, _ = case.cache.tables(case.seqs)
    lens = torch.full_like(lens, 512)           # the same blocks, attended up to the prefix
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_bytes(3, 32, 8, 128, 512, 512, 0),
                     dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_shared_prefix(out, q, None, None, case.cache.k_cache, case.cache.v_cache, tables,
                               lens, 512, 512, wl.scale, 0, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    got = out.float().cpu().numpy()
    for s in range(3):
        for j in range(32):
            h = oatt.kv_head_of(j, 4)
            ref = oatt.softmax_attention(case.q[s, j], case.rows_k[s][:512, h],
                                         case.rows_v[s][:512, h], wl.scale)
            gh.assert_close(got[s, j], ref, "bf16", f"seq {s} head {j}")


def test_under_the_early_read_option():
    """The cascade ignores PA_DECODE_EARLY_CACHE_READS: same result with it set."""
    wl = _custom(32, 8, 16, 256, [3, 40, 17, 200], 4)
    case = gh.build_case(wl)
    plain = _shared_decode(case, 256, ps=64)
    with pa.decode_options(pa.PA_DECODE_EARLY_CACHE_READS):
        early = _shared_decode(case, 256, ps=64)
    assert pa.pa_device_errors() == 0
    assert torch.equal(plain, early)


def test_graph_of_cascades_equals_eager():
    """Three cascade calls (one per cache copy, as a model's layers) captured in
    one CUDA graph: every replay equals the eager calls bit for bit."""
    wl = configs.shared_prefix()
    case = gh.build_case(wl)
    prefix = (wl.shared_prefix // wl.block_size) * wl.block_size
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    s, hq, d = q.shape
    need = pa.pa_decode_shared_prefix_workspace_bytes(s, hq, wl.num_kv_heads, d, prefix, max_len, 0)
    layers = []
    for i in range(3):
        k = case.cache.k_cache.clone()
        k.mul_(1.0 + 0.5 * i)                    # every layer different
        layers.append((k, case.cache.v_cache.clone(), torch.empty_like(q),
                       torch.empty(need, dtype=torch.uint8, device="cuda")))
    ref = []
    for k, v, _, ws in layers:
        o = torch.empty_like(q)
        pa.pa_decode_shared_prefix(o, q, None, None, k, v, tables, lens, prefix, max_len,
                                   wl.scale, 0, ws)
        ref.append(o)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for k, v, o, ws in layers:
            pa.pa_decode_shared_prefix(o, q, None, None, k, v, tables, lens, prefix, max_len,
                                       wl.scale, 0, ws)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for k, v, o, ws in layers:
                pa.pa_decode_shared_prefix(o, q, None, None, k, v, tables, lens, prefix,
                                           max_len, wl.scale, 0, ws)
    torch.cuda.synchronize()
    for _ in range(3):
        for _, _, o, _ in layers:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for (_, _, o, _), r in zip(layers, ref):
            assert torch.equal(o, r)
    assert pa.pa_device_errors() == 0
    del graph


def _forked_cache(seed):
    from paged_kv_cache_345_b200.cache import PagedKVCache
    from workloads import synth

    cache = PagedKVCache(96, 16, 8, 128, "bf16", "cuda", max_blocks_per_seq=32,
                         free_order=synth.block_permutation(96, seed))
    root = cache.add_sequence()
    k, v = synth.kv_rows(seed, 0, 64, 8, 128)
    to = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
    cache.write([root], [64], to(k), to(v))
    seqs = [root] + [cache.fork(root) for _ in range(3)]
    for i, (sq, n) in enumerate(zip(seqs, [7, 30, 0, 91])):
        if n:
            k, v = synth.kv_rows(seed, 1 + i, n, 8, 128)
            cache.write([sq], [n], to(k), to(v))
    return cache, seqs


def test_cache_decode_step_with_shared_prefix():
    """PagedKVCache.decode_step(shared_prefix=64) against the plain fused step
    on an identical cache: same cache contents after the step, outputs within
    the bf16 tolerance of each other."""
    from workloads import synth

    a, sa = _forked_cache(77)
    b, sb = _forked_cache(77)
    q = torch.from_numpy(synth.queries(77, 9, 4, 32, 128)).cuda().to(torch.bfloat16)
    kn, vn = [torch.from_numpy(x).cuda().to(torch.bfloat16)
              for x in synth.new_token_kv(77, 9, 4, 8, 128)]
    out_a = a.decode_step(q, kn, vn, sa, shared_prefix=64)
    out_b = b.decode_step(q, kn, vn, sb)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.v_cache, b.v_cache)
    gh.assert_close(out_a.float().cpu().numpy(), out_b.float().cpu().numpy(), "bf16", "step")
