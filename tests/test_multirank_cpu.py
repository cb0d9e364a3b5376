"""The N > 1 path of bench.py on the CPU with two gloo ranks (no GPU).

Decode is data parallel with no exchange step: every rank runs its own
replica, so the only multi-rank logic is the max-over-ranks timing, the
whole-job rate and which rank prints. These run with the gloo backend over
127.0.0.1 in spawned processes."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank            # rank 1 is the slow one
        slowest = bench.max_over_ranks(mine, world)
        rate = bench.whole_job_rate(1000.0, 4, world, slowest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["slowest"] == 15.0                       # every rank sees the max
        assert g["rate"] == pytest.approx(1000.0 * 4 * 2 / 15e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(10.0, 2, 1, 4.0) == pytest.approx(5000.0)


def test_reference_arm_under_two_ranks_prints_once():
    """--impl reference under torchrun: rank 0 runs the oracle and prints one
    line; rank 1 exits 0 without work (tiny sample so it stays fast)."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e",
                "cpu_baseline"):
        assert key in line, key
    assert line["n_gpus"] == 2 and line["steps"] == 1 and line["value"] > 0
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"]["value"] == line["value"] and line["config"]["workload"]


def test_prefill_flop_count_is_the_causal_pair_count():
    """bench.py's prefill flops: 4 * head_dim * heads per (query row, visible key)
    pair, the pairs counted here one by one."""
    bench = _bench()
    for before, chunks in (([0], [5]), ([3], [4]), ([0, 7], [7, 2]), ([128], [1])):
        pairs = sum(b + i + 1 for b, c in zip(before, chunks) for i in range(c))
        assert bench.prefill_flops(before, chunks, 2, 8) == 4 * 8 * 2 * pairs
    before, chunks = bench.prefill_shape("prefill")
    assert before == [0] * 8 and sum(chunks) == 10_578
    assert bench.prefill_flops(before, chunks) == 4 * 128 * 32 * sum(L * (L + 1) // 2 for L in chunks)


def _bench():
    sys.path.insert(0, ROOT)
    import bench

    return bench


def test_reference_arm_sample_is_bounded_and_valid():
    """The CPU reference arm runs the worked-example batch whole and the larger
    workloads on their first sequences in a compact, unshared pool."""
    bench = _bench()
    from workloads import configs

    wl, note = bench.reference_workload(configs.llama3_8b_layer())
    assert wl.context_lens == configs.llama3_8b_layer().context_lens and "whole" in note
    for big in (configs.large_batch(steps=1), configs.shared_prefix(), configs.long_context(16)):
        small, note = bench.reference_workload(big)
        assert 1 <= small.num_seqs <= big.num_seqs
        assert sum(n + 1 for n in small.context_lens) <= 40_000 or small.num_seqs == 1
        assert small.context_lens == big.context_lens[:small.num_seqs]
        assert small.shared_prefix == 0 and small.ghost_lens == ()
        assert small.num_blocks >= sum(-(-(n + 1) // small.block_size) for n in small.context_lens)
        assert str(small.num_seqs) in note


def test_decode_step_bytes_are_the_oracles_per_token_bytes():
    """bench.py's algorithmic bytes per decode step (the roofline's numerator):
    every attended token (context plus the appended one) costs one layer's K
    and V rows, the oracle's per-token figure pinned to the pages' 128 KiB for
    32 layers."""
    from oracle import blocks as oblk
    from workloads import configs

    bench = _bench()
    wl = configs.llama3_8b_layer()
    tokens = sum(n + 1 for n in wl.context_lens)
    assert tokens == 10_586
    assert bench.kv_bytes(wl) == tokens * oblk.kv_bytes_per_token(1, 8, 128, 2) == 43_360_256
    fp8 = configs.Workload(**{**wl.__dict__, "kv_dtype": "fp8_e4m3"})
    assert bench.kv_bytes(fp8) * 2 == bench.kv_bytes(wl)
    tiny = configs.tiny()
    assert bench.kv_bytes(tiny) == sum(n + 1 for n in tiny.context_lens) * \
        oblk.kv_bytes_per_token(1, 2, 64, 4)


def test_host_metrics_reproduce_the_worked_example():
    """bench.py's host figures: the worked example's cache utilisation through
    the native block manager is the page's 99.4 % (10,578 tokens in 10,640
    slots), the slab figure its 16.1 %; the allocator step covers 256 sequences."""
    sys.path.insert(0, ROOT)
    import bench

    m = bench.host_allocator_metrics(steps=4)
    cu = m["cache_utilisation"]
    assert (cu["tokens_before_step"], cu["slots_before_step"]) == (10_578, 10_640)
    assert round(100 * cu["paged_before_step"], 1) == 99.4
    assert round(100 * cu["slab"], 1) == 16.1
    assert cu["paged_after_step"] == 10_586 / 10_656
    a = m["allocator_step"]
    assert a["sequences"] == 256 and a["us_per_step_p50"] > 0 and a["us_per_step_c_abi_p50"] > 0
    assert 0.9 < a["utilisation_after"] <= 1.0
    dp = m["decode_plan"]
    assert dp["sequences"] == 256 and dp["items"] >= 256 and dp["us_p50_c_abi"] > 0
