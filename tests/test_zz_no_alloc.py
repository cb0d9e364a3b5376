"""pa_decode_noalloc on the GPU, through the C ABI.

pa_decode_noalloc is for callers that cannot allocate device memory where they
decode (their framework owns the device pool, their loop must not synchronise
on an allocation, or they are C hosts handed pointers only): it keeps the
split-K partials in a scratch array built into the library instead of a
caller-provided workspace. Both run the same kernels on the same inputs, so
their outputs must agree bit for bit. These checks first fill the scratch with
another batch's partial results (other queries, shorter contexts, more
partitions), then call pa_decode_noalloc twice in a row on a batch that needs
the scratch and compare each result with pa_decode's; they also check that an
oversized call is refused before any launch and that a bad argument is
reported as such. The file sorts last so a run that stops at the first failure
has already run every other test; it also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from workloads import configs

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc(out, q, cache, tables, lens, max_len, scale, partition_size):
    nb, bs, hkv, d = cache.k_cache.shape
    s, hq, _ = q.shape
    return pa._lib.pa_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(cache.k_cache), _ptr(cache.v_cache), _ptr(tables), _ptr(lens),
        s, hq, hkv, d, bs, nb, tables.shape[1], max_len, scale, partition_size, pa.PA_BF16,
        _stream())


def test_noalloc_matches_pa_decode_on_two_calls_in_a_row():
    wl = configs.llama3_8b_layer()
    partition = 64
    case = gh.build_case(wl, partition_size=partition)
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    s, hq, d = q.shape
    need = pa.pa_decode_workspace_bytes(s, hq, wl.num_kv_heads, d, max_len, partition)
    assert 0 < need <= pa._lib.pa_decode_noalloc_scratch_bytes()   # the scratch is used

    ref = torch.empty_like(q)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    pa.pa_decode(ref, q, case.cache.k_cache, case.cache.v_cache, tables, lens, max_len,
                 wl.scale, partition, ws)
    torch.cuda.synchronize()

    # another batch first: other queries, contexts a third as long, partitions
    # of 48 tokens (86 for the longest bound instead of 65), so the scratch
    # holds other partial results and counters
    other_q = (q.float() * -0.5 + 0.25).to(torch.bfloat16)
    other_lens = (lens.cpu() // 3).to(torch.int32).cuda()
    other = torch.full_like(q, float("nan"))
    st = _noalloc(other, other_q, case.cache, tables, other_lens, max_len, wl.scale, 48)
    assert st == pa.PA_OK, pa._lib.pa_last_error().decode()
    other_ref = torch.empty_like(q)
    pa.pa_decode(other_ref, other_q, case.cache.k_cache, case.cache.v_cache, tables, other_lens,
                 max_len, wl.scale, 48,
                 torch.empty(pa.pa_decode_workspace_bytes(s, hq, wl.num_kv_heads, d, max_len, 48),
                             dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(other, other_ref)

    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        status = _noalloc(out, q, case.cache, tables, lens, max_len, wl.scale, partition)
        assert status == pa.PA_OK, pa._lib.pa_last_error().decode()
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        assert torch.equal(out, ref), "pa_decode_noalloc differs from pa_decode"
    # and pa_decode agrees with the float64 oracle
    gh.assert_close(ref.float().cpu().numpy(), gh.expected_all(case), "bf16", "pa_decode vs oracle")


def test_noalloc_refuses_a_call_beyond_its_scratch():
    wl = configs.llama3_8b_layer()
    case = gh.build_case(wl, partition_size=16)
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    s, hq, d = q.shape
    huge = pa.pa_decode_workspace_bytes(s, hq, wl.num_kv_heads, d, max_len, 16)
    assert huge > pa._lib.pa_decode_noalloc_scratch_bytes()
    out = torch.full_like(q, 7.0)
    status = _noalloc(out, q, case.cache, tables, lens, max_len, wl.scale, 16)
    assert status == pa.PA_ERR_INVALID
    assert "scratch" in pa._lib.pa_last_error().decode()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())   # nothing was launched
    # a bad argument is reported as that, not as a scratch shortfall
    status = _noalloc(out, q, case.cache, tables, lens, max_len, wl.scale, 24)
    assert status == pa.PA_ERR_INVALID
    assert "partition_size" in pa._lib.pa_last_error().decode()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    assert np.isfinite(out.float().cpu().numpy()).all()
