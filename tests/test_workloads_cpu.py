"""The synthetic input recipe (workloads/) on the CPU.

These inputs feed both the kernels and the oracle, so their stated
properties are checked here: per-sequence K/V streams whose first rows do
not depend on the sequence's length, exact bfloat16 rounding, length
distributions with the stated mean and bounds, placements that are
permutations, E4M3 scales that keep N(0, 1) rows inside the format, and
workloads whose pools hold what they must."""

import numpy as np
import pytest
import torch

from workloads import configs, synth


def test_kv_rows_are_prefix_stable_and_independent():
    k7, v7 = synth.kv_rows(11, 3, 7, 2, 16)
    k20, v20 = synth.kv_rows(11, 3, 20, 2, 16)
    assert np.array_equal(k7, k20[:7]) and np.array_equal(v7, v20[:7])
    assert not np.array_equal(k20, v20)                       # K and V: separate streams
    assert not np.array_equal(k20, synth.kv_rows(11, 4, 20, 2, 16)[0])   # per sequence
    assert np.array_equal(k20, synth.kv_rows(11, 3, 20, 2, 16)[0])       # seeded
    q = synth.queries(11, 0, 4, 8, 16)
    assert q.shape == (4, 8, 16) and q.dtype == np.float32
    assert not np.array_equal(q, synth.queries(11, 1, 4, 8, 16))


def test_draws_are_standard_normal():
    x = synth.normal_f32(5, (200_000,)).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01


def test_round_to_bf16_is_exact_and_nearest():
    x = synth.normal_f32(6, (4096,)) * np.float32(37.0)
    r = synth.round_to_bf16(x)
    t = torch.from_numpy(r)
    assert torch.equal(t.to(torch.bfloat16).to(torch.float32), t)    # representable
    # nearest: within half a bfloat16 step (2^-8 of the binade) of the input
    step = np.exp2(np.floor(np.log2(np.abs(x))) - 7)
    assert np.all(np.abs(r.astype(np.float64) - x) <= step / 2)


def test_lognormal_mean_and_bounds():
    # the unclipped draw has arithmetic mean `mean` (mu = ln(mean) - sigma^2 / 2)
    x = synth.lognormal_lengths(400_000, 600.0, 0.75, 0, 10**9, seed=1)
    assert abs(x.mean() / 600.0 - 1.0) < 0.01
    y = synth.lognormal_lengths(10_000, 600.0, 0.75, 16, 4096, seed=2)
    assert y.min() >= 16 and y.max() <= 4096 and y.dtype == np.int64


def test_uniform_lengths_cover_the_closed_range():
    u = synth.uniform_lengths(5_000, 3, 6, seed=4)
    assert set(u.tolist()) == {3, 4, 5, 6}


def test_block_permutation():
    p = synth.block_permutation(1000, 9)
    assert sorted(p.tolist()) == list(range(1000)) and p.dtype == np.int32
    assert not np.array_equal(p, synth.block_permutation(1000, 10))
    assert not np.array_equal(p, np.arange(1000))


def test_e4m3_scales_keep_normal_rows_inside_the_format():
    k, v = synth.e4m3_scales(8)
    for s in (k, v):
        assert s.dtype == np.float32 and np.all(s > 0)
        # a row drawn from N(0, 1) at |x| <= 8 (never reached in 10^9 draws) stays below 448
        assert np.all(8.0 / s < 448.0)
    # K head 0 divides exactly (1/32); every other scale makes the division round
    power_of_two = np.frexp(np.concatenate([k, v]).astype(np.float64))[0] == 0.5
    assert power_of_two.tolist() == [True] + [False] * 15


@pytest.mark.parametrize("make", [configs.tiny, configs.llama3_8b_layer, configs.shared_prefix,
                                  lambda: configs.large_batch(1), configs.long_context])
def test_workload_pools_hold_their_sequences(make):
    wl = make()
    bs = wl.block_size
    need = sum(-(-(n + wl.decode_steps) // bs) for n in wl.context_lens)
    if wl.shared_prefix:
        shared = wl.shared_prefix // bs
        need -= shared * (wl.num_seqs - 1)           # full prefix blocks are stored once
    live_ghosts = sum(-(-n // bs) for i, n in enumerate(wl.ghost_lens) if i % 2)
    assert need + live_ghosts <= wl.num_blocks
    assert wl.num_heads % wl.num_kv_heads == 0


def test_worked_example_batch():
    wl = configs.llama3_8b_layer()
    assert sum(wl.context_lens) == 10_578
    assert sum(-(-n // 16) * 16 for n in wl.context_lens) == 10_640
    assert (wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.dtype) == (32, 8, 128, "bf16")
