"""pa_decode_contiguous on the GPU: the table-free decode over one slab per
sequence, the baseline paging is measured against ("What is paged attention
in vLLM, and why does it matter?", Trade-offs and edge cases, first point).

On the same tokens it must equal the paged decode bit for bit (same chunks,
same reduction order; only the addressing differs) and the float64 oracle
within the bf16 tolerance. The oracle reads a slab as a paged cache whose one
block per sequence is the whole slab (identity table).
"""

import numpy as np
import pytest
import torch

import gpu_harness as gh
import paged_kv_cache_345_b200 as pa
from oracle import attention as oatt
from workloads import configs

pytestmark = pytest.mark.gpu


def _slabs(case, slab_len):
    s = len(case.seqs)
    hkv, d = case.cache.num_kv_heads, case.cache.head_dim
    k = torch.zeros((s, slab_len, hkv, d), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    for i in range(s):
        n = case.rows_k[i].shape[0]
        k[i, :n] = torch.from_numpy(case.rows_k[i]).to("cuda", torch.bfloat16)
        v[i, :n] = torch.from_numpy(case.rows_v[i]).to("cuda", torch.bfloat16)
    return k, v


def _contiguous(case, k, v, ps):
    tables, lens, max_len = case.cache.tables(case.seqs)
    q = torch.from_numpy(case.q).cuda().to(torch.bfloat16)
    s, hq, d = q.shape
    ps_eff = ps or pa.pa_decode_partition_size(s, k.shape[2], max_len)
    need = pa.pa_decode_workspace_bytes(s, hq, k.shape[2], d, max_len, ps_eff)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_contiguous(out, q, k, v, lens, max_len, case.scale, ps, ws)
    torch.cuda.synchronize()
    return out, lens


@pytest.mark.parametrize("ps", [0, 64])
def test_equals_paged_decode_bit_for_bit(ps):
    case = gh.build_case(configs.llama3_8b_layer(), partition_size=ps)
    k, v = _slabs(case, 4112)
    out, _ = _contiguous(case, k, v, ps)
    assert pa.pa_device_errors() == 0
    assert torch.equal(out, case.out)
    gh.assert_close(out.float().cpu().numpy(), gh.expected_all(case), "bf16", f"P={ps}")


@pytest.mark.parametrize("group,d", [(1, 128), (4, 64), (8, 128)])
def test_ragged_lengths_against_the_oracle(group, d):
    lens = (0, 1, 15, 16, 17, 100, 257, 600)
    wl = configs.Workload(f"contig_g{group}_d{d}", 2 * group, 2, d, "bf16", 16, 200, lens,
                          5301, 6301)
    case = gh.build_case(wl, partition_size=48)
    slab = 608
    k, v = _slabs(case, slab)
    out, lens_dev = _contiguous(case, k, v, 48)
    assert pa.pa_device_errors() == 0
    assert torch.equal(out, case.out)
    # the oracle over the slabs themselves (one block per sequence, identity table)
    kc = k.float().cpu().numpy().astype(np.float64)
    vc = v.float().cpu().numpy().astype(np.float64)
    tables = np.arange(len(lens))[:, None]
    ref = oatt.decode(case.q, kc, vc, tables, lens_dev.cpu().numpy(), wl.scale, slab)
    gh.assert_close(out.float().cpu().numpy(), ref, "bf16", f"G={group} d={d}")
