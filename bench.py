#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

One step = one decode step of a batch: pa_kv_append of each sequence's new
token, then pa_decode over every sequence's whole cached context (split-K
partitions merged by a second kernel when a sequence spans more than one).
Default workload: one Llama-3-8B-shaped layer (32/8 heads, head_dim 128, bf16,
block 16) holding the eight requests of the pages' worked example
(128, 700, 1500, 300, 2900, 50, 4100, 900 cached tokens), physical blocks a
seeded random permutation of a 2048-block pool.

Timing: W warm-up steps, then K steps, each bracketed by CUDA events on the
launching stream; the L2 is flushed (a 2 x L2 write) between steps, outside
the events. Under torchrun each rank runs its own replica (replicas only:
sequences never exchange data) and the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference   # the float64 CPU oracle as the reference arm
"""

from __future__ import annotations

import argparse
import ctypes
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read GB/s (fraction of HBM peak) and attended tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default="llama3_8b_layer",
                    choices=["llama3_8b_layer", "large_batch", "shared_prefix", "long_context",
                             "swap", "prefill", "chunked_prefill"])
    ap.add_argument("--placement", choices=["random", "identity"], default="random",
                    help="physical block order: a seeded permutation (default) or identity "
                         "(each sequence's blocks contiguous in memory)")
    ap.add_argument("--block-size", type=int, default=16, help="long_context only")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8_e4m3"], default="bf16",
                    help="cache element type (fp8_e4m3: 8-bit codes, per-KV-head scales)")
    ap.add_argument("--partition-size", type=int, default=-1,
                    help="tokens per split-K partition (-1: tuned default, 0: library choice)")
    ap.add_argument("--unfused", action="store_true",
                    help="time pa_kv_append + pa_decode instead of the fused pa_decode_append")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-back-to-back", action="store_true")
    ap.add_argument("--layers", type=int, default=32,
                    help="cache replicas of the back-to-back figure (one per model layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def make_workload(name: str, block_size: int):
    from workloads import configs

    if name == "long_context":
        return configs.long_context(block_size)
    if name == "large_batch":
        return configs.large_batch(steps=1)
    return configs.ALL[name]()


# Partition sizes measured best per workload (tokens); -1 on the command line picks these.
TUNED_PARTITION = {"llama3_8b_layer": 0, "large_batch": 0, "shared_prefix": 0,
                   "long_context": 512}


def kv_bytes(wl) -> int:
    """K and V bytes the decode step reads: every attended token, every KV head."""
    return (sum(n + 1 for n in wl.context_lens) * wl.num_kv_heads * 2 * wl.head_dim *
            wl.cache_elem_bytes)


# ------------------------------------------------------------- rank plumbing

def max_over_ranks(value_ms: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank contributes its own measured time and
    all get the max (NCCL on GPUs, gloo on CPU). One rank: the value itself."""
    if world <= 1:
        return float(value_ms)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value_ms)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step: float, steps: int, world: int, time_ms: float) -> float:
    """Units per second of the whole job: every rank runs its own replica of the
    step, so the job does world x steps x units in the slowest rank's time."""
    return units_per_step * steps * world / (time_ms * 1e-3)


# ------------------------------------------------------------------ GPU setup

def build_on_gpu(wl, device, placement="random"):
    """Prefill every sequence through the library, then prepare one decode step."""
    import torch

    from paged_kv_cache_345_b200.cache import PagedKVCache
    from workloads import synth

    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    bs = wl.block_size
    max_blocks = max(-(-(n + 1) // bs) for n in wl.context_lens)
    order = synth.block_permutation(wl.num_blocks, wl.placement_seed) if placement == "random" \
        else np.arange(wl.num_blocks, dtype=np.int32)
    fp8 = wl.cache_dtype == "fp8_e4m3"
    ks, vs = synth.e4m3_scales(wl.num_kv_heads) if fp8 else (None, None)
    cache = PagedKVCache(wl.num_blocks, bs, wl.num_kv_heads, wl.head_dim, wl.cache_dtype, device,
                         max_blocks_per_seq=max_blocks, free_order=order,
                         k_scale=None if ks is None else torch.from_numpy(ks),
                         v_scale=None if vs is None else torch.from_numpy(vs))
    ghosts = [cache.add_sequence() for _ in wl.ghost_lens]
    if ghosts:
        cache.bm.append_slots(ghosts, list(wl.ghost_lens))
        for i in range(0, len(ghosts), 2):
            cache.free(ghosts[i])

    def rows(seq_index, n):
        k, v = synth.kv_rows(wl.value_seed, seq_index, n, wl.num_kv_heads, wl.head_dim)
        return (torch.from_numpy(k).to(device=device, dtype=tdt),
                torch.from_numpy(v).to(device=device, dtype=tdt))

    start = 0
    if wl.shared_prefix:
        parent = cache.add_sequence()
        pk, pv = rows(100_000, wl.shared_prefix)
        cache.write([parent], [wl.shared_prefix], pk, pv)
        seqs = [parent] + [cache.fork(parent) for _ in range(wl.num_seqs - 1)]
        start = wl.shared_prefix
    else:
        seqs = [cache.add_sequence() for _ in range(wl.num_seqs)]
    cow_pairs = 0
    for s, n in enumerate(wl.context_lens):     # one sequence at a time bounds host memory
        if n - start > 0:
            k, v = rows(s, n - start)
            slots, cows = cache.bm.append_slots([seqs[s]], [n - start])
            cow_pairs += len(cows)
            if len(cows):
                from paged_kv_cache_345_b200 import pa_copy_blocks
                pa_copy_blocks(cache.k_cache, cache.v_cache, torch.from_numpy(cows).to(device))
            from paged_kv_cache_345_b200 import pa_kv_append, pa_kv_append_fp8
            sd = torch.from_numpy(slots).to(device)
            if fp8:
                pa_kv_append_fp8(k, v, sd, cache.k_cache, cache.v_cache, cache.k_scale,
                                 cache.v_scale)
            else:
                pa_kv_append(k, v, sd, cache.k_cache, cache.v_cache)
    torch.cuda.synchronize(device)

    # the decode step: one new token per sequence, appended then attended
    new_k, new_v = synth.new_token_kv(wl.value_seed, 0, wl.num_seqs, wl.num_kv_heads, wl.head_dim)
    q = synth.queries(wl.value_seed, 0, wl.num_seqs, wl.num_heads, wl.head_dim)
    slots, cows = cache.bm.append_slots(seqs, [1] * len(seqs))
    assert len(cows) == 0
    tables, lens = cache.bm.block_tables(seqs, max_blocks)
    host, dev = pack_step_inputs({
        "q": torch.from_numpy(q).to(tdt),
        "k_new": torch.from_numpy(new_k).to(tdt),
        "v_new": torch.from_numpy(new_v).to(tdt),
        "slots": torch.from_numpy(slots),
        "tables": torch.from_numpy(tables),
        "lens": torch.from_numpy(lens),
    }, device)
    return cache, seqs, host, dev, int(lens.max()), cow_pairs


def pack_step_inputs(arrays, device):
    """One page-locked host buffer and one device buffer holding every per-step
    input at 256-byte-aligned offsets, with typed views into both: a step's
    inputs then travel host -> device in a single copy. The views are returned
    by name; "_pack" is the whole buffer."""
    import torch

    offs, total = {}, 0
    for name, t in arrays.items():
        offs[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host_pack = torch.zeros(total, dtype=torch.uint8).pin_memory()
    dev_pack = torch.zeros(total, dtype=torch.uint8, device=device)
    host, dev = {"_pack": host_pack}, {"_pack": dev_pack}
    for name, t in arrays.items():
        nbytes = t.numel() * t.element_size()
        host[name] = host_pack[offs[name]:offs[name] + nbytes].view(t.dtype).view(t.shape)
        host[name].copy_(t)
        dev[name] = dev_pack[offs[name]:offs[name] + nbytes].view(t.dtype).view(t.shape)
    dev_pack.copy_(host_pack)
    return host, dev


class StepCalls:
    """The C-ABI calls of one decode step with their arguments marshalled once.

    fused: the step is one pa_decode_append call (append each newest token, then
    attend); otherwise pa_kv_append followed by pa_decode (same result)."""

    def __init__(self, cache, dev, max_len, scale, partition_size, stream, fused=True):
        import torch

        import paged_kv_cache_345_b200 as pa

        self.lib = pa._lib
        s, hq, d = dev["q"].shape
        nb, bs, hkv, _ = cache.k_cache.shape
        self.fp8 = cache.k_cache.dtype == torch.uint8
        dt = pa.PA_BF16 if cache.k_cache.dtype == torch.bfloat16 else pa.PA_F32
        self.partition_size = partition_size or pa.pa_decode_partition_size(s, hkv, max_len)
        ws_bytes = pa.pa_decode_workspace_bytes(s, hq, hkv, d, max_len, self.partition_size)
        self.workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev["q"].device)
        self.out = torch.empty_like(dev["q"])
        self.num_partitions = -(-max_len // self.partition_size)
        st = ctypes.c_void_p(stream.cuda_stream)
        p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        ws = (p(self.workspace), self.workspace.numel())
        mbps = dev["tables"].shape[1]
        if self.fp8:
            sc = (p(cache.k_scale), p(cache.v_scale))
            self.append_args = (p(dev["k_new"]), p(dev["v_new"]), p(dev["slots"]), s,
                                p(cache.k_cache), p(cache.v_cache), *sc, nb, bs, hkv, d, st)
            self.decode_args = (p(self.out), p(dev["q"]), p(cache.k_cache), p(cache.v_cache),
                                *sc, p(dev["tables"]), p(dev["lens"]), s, hq, hkv, d, bs, nb,
                                mbps, max_len, scale, self.partition_size, *ws, st)
            self.step_args = (p(self.out), p(dev["q"]), p(dev["k_new"]), p(dev["v_new"]),
                              p(cache.k_cache), p(cache.v_cache), *sc, p(dev["tables"]),
                              p(dev["lens"]), s, hq, hkv, d, bs, nb, mbps, max_len, scale,
                              self.partition_size, *ws, st)
            self.fns = (self.lib.pa_kv_append_fp8, self.lib.pa_decode_fp8,
                        self.lib.pa_decode_append_fp8)
        else:
            self.append_args = (p(dev["k_new"]), p(dev["v_new"]), p(dev["slots"]), s,
                                p(cache.k_cache), p(cache.v_cache), nb, bs, hkv, d, dt, st)
            self.decode_args = (p(self.out), p(dev["q"]), p(cache.k_cache), p(cache.v_cache),
                                p(dev["tables"]), p(dev["lens"]), s, hq, hkv, d, bs, nb,
                                mbps, max_len, scale, self.partition_size, *ws, dt, st)
            self.step_args = (p(self.out), p(dev["q"]), p(dev["k_new"]), p(dev["v_new"]),
                              p(cache.k_cache), p(cache.v_cache), p(dev["tables"]),
                              p(dev["lens"]), s, hq, hkv, d, bs, nb, mbps, max_len, scale,
                              self.partition_size, *ws, dt, st)
            self.fns = (self.lib.pa_kv_append, self.lib.pa_decode, self.lib.pa_decode_append)
        self.fused = fused
        self.launches_per_step = (1 if fused else 2) + (1 if self.num_partitions > 1 else 0)

    def _call(self, fn, args):
        st = fn(*args)
        if st:
            raise RuntimeError(f"{fn.__name__}: {self.lib.pa_last_error().decode()}")

    def append(self):
        self._call(self.fns[0], self.append_args)

    def decode(self):
        self._call(self.fns[1], self.decode_args)

    def step(self):
        if not self.fused:
            self.append()
            self.decode()
            return
        self._call(self.fns[2], self.step_args)


# --------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# -------------------------------------------------------------- CPU baseline

def oracle_inputs(wl):
    """The oracle's own cache (float64) built by its own block manager from the
    same seeded rows and free order; never read back from the GPU."""
    from oracle import attention as oatt
    from oracle import blocks as oblk
    from workloads import synth

    def stored(x):
        return synth.round_to_bf16(x) if wl.dtype == "bf16" else x

    fp8 = wl.cache_dtype == "fp8_e4m3"
    if fp8:
        from oracle import quant as oquant
        ks, vs = synth.e4m3_scales(wl.num_kv_heads)

        def cache_values(rows, scales):   # the oracle's codes of the rows, dequantised
            return np.stack([oquant.dequantize(oquant.quantize(rows[:, h], scales[h]), scales[h])
                             for h in range(rows.shape[1])], axis=1)

    ob = oblk.BlockManager(wl.num_blocks, wl.block_size)
    ob.set_free_order(synth.block_permutation(wl.num_blocks, wl.placement_seed).tolist())
    kc = np.zeros((wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_dim))
    vc = np.zeros_like(kc)
    new_k, new_v = synth.new_token_kv(wl.value_seed, 0, wl.num_seqs, wl.num_kv_heads, wl.head_dim)
    seqs = []
    for s, n in enumerate(wl.context_lens):
        sid = ob.new_sequence()
        seqs.append(sid)
        k, v = synth.kv_rows(wl.value_seed, s, n, wl.num_kv_heads, wl.head_dim)
        k = np.concatenate([stored(k), stored(new_k[s:s + 1])])
        v = np.concatenate([stored(v), stored(new_v[s:s + 1])])
        if fp8:
            k, v = cache_values(k, ks), cache_values(v, vs)
        slots, _ = ob.add_tokens(sid, n + 1)
        kc, vc = oatt.kv_append(kc, vc, k, v, slots, wl.block_size)
    mb = max(len(ob.tables[s]) for s in seqs)
    tables = np.zeros((len(seqs), mb), dtype=np.int64)
    for i, s in enumerate(seqs):
        tables[i, :len(ob.tables[s])] = ob.tables[s]
    q = stored(synth.queries(wl.value_seed, 0, wl.num_seqs, wl.num_heads, wl.head_dim))
    return q, kc, vc, tables, [ob.lengths[s] for s in seqs]


def cpu_oracle_run(wl, budget_s: float, min_steps: int = 1, max_steps: int | None = None):
    """Time the oracle's decode step on the host cores: whole steps, repeated
    until `budget_s` is spent (at least min_steps, at most max_steps)."""
    from oracle import attention as oatt

    if wl.shared_prefix or wl.ghost_lens or sum(wl.context_lens) > 200_000:
        raise ValueError("the CPU oracle leg runs the single-layer worked-example workload")
    q, kc, vc, tables, lens = oracle_inputs(wl)
    times = []
    t_end = time.perf_counter() + budget_s
    while len(times) < min_steps or (time.perf_counter() < t_end and
                                     (max_steps is None or len(times) < max_steps)):
        t0 = time.perf_counter()
        oatt.decode(q, kc, vc, tables, lens, wl.scale, wl.block_size)
        times.append(time.perf_counter() - t0)
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        blas = 1
    return times, max(1, min(cores, blas))


# --------------------------------------------------------------------- arms

REFERENCE_BUDGET_S = 180.0  # wall time the reference arm's timed steps may take


def reference_workload(wl):
    """The workload the CPU oracle runs: the workload itself when its float64
    cache is small (the worked-example layer), else its first sequences in a
    compact pool (bounded sample)."""
    import dataclasses

    if not (wl.shared_prefix or wl.ghost_lens or sum(wl.context_lens) > 200_000):
        return wl, f"the whole {wl.num_seqs}-sequence batch"
    lens, total = [], 0
    for n in wl.context_lens:
        if lens and total + n + 1 > 40_000:
            break
        lens.append(n)
        total += n + 1
    need = sum(-(-(n + 1) // wl.block_size) for n in lens) + 16
    small = dataclasses.replace(wl, context_lens=tuple(lens), num_blocks=need, ghost_lens=(),
                                shared_prefix=0)
    return small, (f"the first {len(lens)} of the {wl.num_seqs} sequences, unshared, in a "
                   f"{need}-block pool")


def run_reference(args, wl, rank):
    """The reference arm: the float64 CPU oracle, as it stands, on the same
    workload (or a bounded sample of it), each timed step one oracle decode."""
    if rank != 0:
        return
    from oracle import attention as oatt

    rwl, sample = reference_workload(wl)
    q, kc, vc, tables, lens = oracle_inputs(rwl)
    row_bytes = rwl.num_kv_heads * 2 * rwl.head_dim * rwl.cache_elem_bytes
    t0 = time.perf_counter()
    oatt.decode(q, kc, vc, tables, lens, rwl.scale, rwl.block_size)
    one = time.perf_counter() - t0
    # a step attends the whole sample, or one sequence of it (rotating) when
    # whole steps would not fit the time budget
    rotate = args.steps * one > REFERENCE_BUDGET_S
    S = len(lens)

    def step(i):
        if rotate:
            s = i % S
            oatt.decode(q[s:s + 1], kc, vc, tables[s:s + 1], lens[s:s + 1], rwl.scale,
                        rwl.block_size)
            return lens[s] * row_bytes
        oatt.decode(q, kc, vc, tables, lens, rwl.scale, rwl.block_size)
        return sum(lens) * row_bytes

    for i in range(max(1, args.warmup)):
        step(i)
    moved, t0 = 0, time.perf_counter()
    for i in range(args.steps):
        moved += step(i)
    total = time.perf_counter() - t0
    value = moved / total / 1e9
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        cores = max(1, min(cores, max((i.get("num_threads", 1) for i in threadpool_info()),
                                      default=1)))
    except Exception:  # noqa: BLE001
        pass
    sample = (f"{args.steps} oracle decode steps over {sample}"
              + (", one sequence per step in turn (whole steps exceed the time budget)"
                 if rotate else ""))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs": wl.num_seqs, "block_size": wl.block_size,
                   "kv_cache": wl.cache_dtype},
        "attended_tokens_per_s": moved / row_bytes / total,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


DECODE_SOURCES = ("pa_decode.cuh", "pa_decode_mma.cuh", "pa_device.cuh", "pa_kernels.cu")
PREFILL_SOURCES = ("pa_prefill.cu", "pa_prefill_order.h", "pa_tc.cuh", "pa_device.cuh")


def kernel_source_digest(files=DECODE_SOURCES) -> str:
    """sha256 (first 16 hex digits) over the sources of a kernel."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_345_b200", "csrc")
    for name in files:
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


def load_traffic(kernel_key: str, files=DECODE_SOURCES):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (matching source hash), else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel_key}.traffic.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    digest = kernel_source_digest(files)
    if vals.get("source_sha256_16") != digest:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def run_b200(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import paged_kv_cache_345_b200 as pa

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", device_id=device)
    # a stream of our own (CUDA graphs cannot be captured on the default stream)
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)

    cache, seqs, host, dev, max_len, cow_pairs = build_on_gpu(wl, device, args.placement)
    ps = TUNED_PARTITION[wl.name.split("_bs")[0]] if args.partition_size < 0 else args.partition_size
    calls = StepCalls(cache, dev, max_len, wl.scale, ps, stream, fused=not args.unfused)
    bytes_step = kv_bytes(wl)
    tokens_step = sum(n + 1 for n in wl.context_lens)

    # L2 flush between steps: write a buffer larger than L2, then read another
    # one, so the timed step starts with L2 holding clean, unrelated lines (a
    # write alone would leave the step paying for the write-back of its dirty
    # lines).
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush_w = torch.empty(2 * l2 + (64 << 20), dtype=torch.uint8, device=device)
    flush_r = torch.ones((2 * l2 + (64 << 20)) // 4, dtype=torch.float32, device=device)

    class _Flush:
        def zero_(self):
            flush_w.zero_()
            flush_r.sum()

        def numel(self):
            return flush_w.numel() + flush_r.numel() * 4

    flush = _Flush()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize(device)

    # ---- device-resident steps
    for _ in range(args.warmup):
        flush.zero_()
        calls.step()
    torch.cuda.synchronize(device)
    if pa.pa_device_errors() != 0:
        raise RuntimeError("device error word set during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        calls.step()
        ev[i][1].record(stream)
    barrier()
    wall = time.perf_counter() - t_wall
    clk = clocks.stop()
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    decode_ms = step_ms  # the step's kernels: (append +) decode + split-K merge
    total_ms = max_over_ranks(sum(step_ms), world, device)
    if pa.pa_device_errors() != 0:
        raise RuntimeError("device error word set during the timed steps")

    # ---- end to end: pinned host inputs -> device -> kernels -> host output
    e2e = None
    if not args.no_e2e:
        out_host = torch.empty(calls.out.shape, dtype=calls.out.dtype).pin_memory()
        # q, new K/V rows, slot mapping, tables and lengths: one packed copy
        h2d = host["_pack"].numel()
        d2h = out_host.numel() * out_host.element_size()

        def e2e_step():
            dev["_pack"].copy_(host["_pack"], non_blocking=True)
            calls.step()
            out_host.copy_(calls.out, non_blocking=True)

        for _ in range(args.warmup):
            flush.zero_()
            e2e_step()
        ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            flush.zero_()
            ee[i][0].record(stream)
            e2e_step()
            ee[i][1].record(stream)
        barrier()
        e2e_ms = max_over_ranks(sum(ee[i][0].elapsed_time(ee[i][1]) for i in range(args.steps)),
                                world, device)
        e2e = {"value": whole_job_rate(bytes_step, args.steps, world, e2e_ms) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / args.steps}

    # ---- back to back: the same step over `layers` different cache replicas
    # (one per model layer, together far larger than L2, so no flush), all
    # layers captured in one CUDA graph and replayed. Consecutive layers
    # overlap launch and start-up through programmatic dependent launch.
    b2b = None
    if not args.no_back_to_back and world == 1:
        reps = []
        for _ in range(args.layers):
            kc = cache.k_cache.clone()
            vc = cache.v_cache.clone()
            reps.append((kc, vc))
        del kc, vc
        layer_calls = []
        for kc, vc in reps:
            view = type("CacheView", (), {})()
            view.k_cache, view.v_cache = kc, vc
            if calls.fp8:
                view.k_scale, view.v_scale = cache.k_scale, cache.v_scale
            layer_calls.append(StepCalls(view, dev, max_len, wl.scale, calls.partition_size,
                                         stream, fused=calls.fused))
        for c in layer_calls:   # warm-up, eager
            c.step()
        torch.cuda.synchronize(device)
        graph = torch.cuda.CUDAGraph()
        early = 0 if os.environ.get("PA_BENCH_NO_EARLY") else pa.PA_DECODE_EARLY_CACHE_READS
        with torch.cuda.graph(graph, stream=stream), pa.decode_options(early):
            for c in layer_calls:
                c.step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize(device)
        reps_n = max(5, min(50, args.steps // args.layers))
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps_n)]
        for i in range(reps_n):
            gev[i][0].record(stream)
            graph.replay()
            gev[i][1].record(stream)
        torch.cuda.synchronize(device)
        per_layer_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in gev) / args.layers
        if pa.pa_device_errors() != 0:
            raise RuntimeError("device error word set during the back-to-back replay")
        b2b = {"layers": args.layers, "us_per_layer": 1e3 * per_layer_ms,
               "kv_GB_per_s": bytes_step / (per_layer_ms * 1e-3) / 1e9,
               "how": "one CUDA graph of the step over per-layer cache replicas, no L2 flush"}
        del graph, layer_calls, reps
        torch.cuda.empty_cache()

    # ---- roofline of pa_decode (decode kernel + split-K merge kernel)
    peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(peaks_path):
        peak, peak_src = float(json.load(open(peaks_path))["hbm_gbs"]), "measured"
    else:
        peak, peak_src = FALLBACK_HBM_GBS, "fallback"
    if b2b is not None:
        b2b["frac_of_peak"] = b2b["kv_GB_per_s"] / peak
    dec_s = statistics.mean(decode_ms) * 1e-3
    achieved = bytes_step / dec_s / 1e9
    traffic = load_traffic(f"pa_decode_{wl.name}" + ("_fp8" if calls.fp8 else ""))

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            times, cores = cpu_oracle_run(wl, args.cpu_budget_s)
            cpu = {"value": bytes_step * len(times) / sum(times) / 1e9, "unit": "GB/s",
                   "cores": cores, "kind": "oracle",
                   "sample": f"{len(times)} whole decode steps of the {wl.num_seqs}-sequence "
                             f"batch in {sum(times):.1f} s (float64 NumPy)"}
        except ValueError as exc:
            cpu = {"value": None, "unit": "GB/s", "cores": 0, "kind": "oracle",
                   "sample": f"not run: {exc}"}

    value = whole_job_rate(bytes_step, args.steps, world, total_ms) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.cache_dtype, "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs": wl.num_seqs, "num_heads": wl.num_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                   "block_size": wl.block_size, "num_blocks": wl.num_blocks,
                   "attended_tokens": tokens_step, "kv_bytes_per_step": bytes_step,
                   "partition_size": calls.partition_size,
                   "num_partitions": calls.num_partitions, "copy_on_write_pairs": cow_pairs,
                   "placement": args.placement, "kv_cache": wl.cache_dtype,
                   "l2": f"flushed between steps ({flush_w.numel() >> 20} MiB written, then "
                         f"{(flush_r.numel() * 4) >> 20} MiB of another buffer read; outside the "
                         "timed events)",
                   "parallelism": f"replicas x{world}"},
        "attended_tokens_per_s": whole_job_rate(tokens_step, args.steps, world, total_ms),
        "us_per_step": 1e3 * total_ms / args.steps,
        "step_us_p10_p50_p90": [1e3 * float(np.percentile(decode_ms, p)) for p in (10, 50, 90)],
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": ("pa_decode_append (fused append + decode kernel, split-K "
                                "merge kernel)" if calls.fused else
                                "pa_kv_append + pa_decode (decode + split-K merge kernels)"),
                     "peak_source": f"{peak_src} hbm_gbs"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "back_to_back": b2b,
        "gpu_launches": calls.launches_per_step * args.steps,
        "clocks": clk,
        "wall_s_timed_region": wall,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()


def run_swap(args, rank, world, local_rank):
    """pa_swap_blocks throughput: every block of the Llama-3-8B layer batch swapped
    out to a page-locked host pool, then back into the device pool."""
    import torch

    import paged_kv_cache_345_b200 as pa

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    wl = make_workload("llama3_8b_layer", 16)
    cache, seqs, host, dev, max_len, _ = build_on_gpu(wl, device)
    tables = host["tables"].numpy()
    ids = sorted({int(b) for i, s in enumerate(seqs)
                  for b in tables[i, :cache.bm.seq_num_blocks(s)]})
    n = len(ids)
    shape = (n,) + tuple(cache.k_cache.shape[1:])
    host_k = torch.empty(shape, dtype=cache.k_cache.dtype).pin_memory()
    host_v = torch.empty(shape, dtype=cache.k_cache.dtype).pin_memory()
    out_map = torch.tensor([[b, i] for i, b in enumerate(ids)], dtype=torch.int64, device=device)
    in_map = out_map.flip(1).contiguous()
    block_bytes = cache.k_cache[0].numel() * cache.k_cache.element_size()
    moved = 2 * n * block_bytes
    res = {}
    for name, fn in (("device_to_host", lambda: pa.pa_swap_blocks(host_k, host_v, cache.k_cache,
                                                                  cache.v_cache, out_map)),
                     ("host_to_device", lambda: pa.pa_swap_blocks(cache.k_cache, cache.v_cache,
                                                                  host_k, host_v, in_map))):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(device)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        torch.cuda.synchronize(device)
        ms = a.elapsed_time(b) / args.steps
        res[name] = {"GB_per_s": moved / (ms * 1e-3) / 1e9, "us_per_call": 1e3 * ms}
    if pa.pa_device_errors() != 0:
        raise RuntimeError("device error word set during the swap benchmark")
    if rank == 0:
        print(json.dumps({
            "metric": "pa_swap_blocks bytes moved per second (device <-> page-locked host)",
            "value": min(r["GB_per_s"] for r in res.values()), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "swap: every block of the Llama-3-8B layer batch",
                       "blocks": n, "bytes_per_call": moved},
            "directions": res, "gpu_launches": 2 * args.steps}), flush=True)


# ------------------------------------------------------------------ prefill

PREFILL_METRIC = "paged causal prefill attention TFLOP/s (fraction of bf16 tensor peak)"


def prefill_shape(name: str):
    """(cached tokens before the chunk, chunk tokens) per sequence: the worked
    example's eight prompts prefilled whole, or a 512-token chunk on top of
    each of those contexts."""
    from workloads import synth

    lens = list(synth.LLAMA3_8B_BATCH_LENGTHS)
    if name == "prefill":
        return [0] * len(lens), lens
    return lens, [512] * len(lens)


def prefill_flops(before, chunks, num_heads=32, head_dim=128) -> float:
    """q.k and p.v multiply-adds over every (query row, visible key) pair, all heads."""
    pairs = sum(c * (b + 1) + c * (c - 1) // 2 for b, c in zip(before, chunks))
    return 4.0 * head_dim * num_heads * pairs


def run_prefill(args, rank, world, local_rank):
    import torch

    import paged_kv_cache_345_b200 as pa
    from paged_kv_cache_345_b200.cache import PagedKVCache
    from workloads import synth

    hq, hkv, d, bs, seed = 32, 8, 128, args.block_size, 1007
    before, chunks = prefill_shape(args.workload)
    lens = [b + c for b, c in zip(before, chunks)]
    flops = prefill_flops(before, chunks, hq, d)
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    total_q = int(qs[-1])

    if args.impl == "reference":
        if rank != 0:
            return
        from oracle import attention as oatt
        # bounded sample: the 700-token sequence alone, float64 NumPy, whole steps
        s = 1
        k, v = synth.kv_rows(seed, s, lens[s], hkv, d)
        q1 = synth.queries(seed, 1 + s, chunks[s], hq, d)
        kc, vc = k[:, None], v[:, None]
        tables = np.arange(lens[s])[None]
        f1 = prefill_flops([before[s]], [chunks[s]], hq, d)
        for _ in range(max(1, args.warmup)):
            oatt.prefill(q1, kc, vc, tables, [lens[s]], [0, chunks[s]], 1 / np.sqrt(d), 1)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oatt.prefill(q1, kc, vc, tables, [lens[s]], [0, chunks[s]], 1 / np.sqrt(d), 1)
        dt = time.perf_counter() - t0
        value = f1 * args.steps / dt / 1e12
        print(json.dumps({
            "impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample": f"sequence {s} only"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
                             "kind": "oracle", "sample": f"sequence {s} ({chunks[s]} rows)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)
    nb = sum(-(-L // bs) for L in lens) + 16
    cache = PagedKVCache(nb, bs, hkv, d, "bf16", device, max_blocks_per_seq=max(-(-L // bs) for L in lens),
                         free_order=synth.block_permutation(nb, 2007))
    seqs = [cache.add_sequence() for _ in lens]
    for s, L in enumerate(lens):   # every token's K/V, chunk included, written through the library
        k, v = synth.kv_rows(seed, s, L, hkv, d)
        cache.write([seqs[s]], [L], torch.from_numpy(k).to(device, torch.bfloat16),
                    torch.from_numpy(v).to(device, torch.bfloat16))
    q_host = torch.from_numpy(np.concatenate(
        [synth.queries(seed, 1 + s, c, hq, d) for s, c in enumerate(chunks)])).to(torch.bfloat16)
    q_host = q_host.pin_memory()
    q = q_host.to(device)
    out = torch.empty_like(q)
    out_host = torch.empty_like(q_host).pin_memory()
    tables, ctx, _ = cache.tables(seqs)
    qs_dev = torch.from_numpy(qs).to(device)
    torch.cuda.synchronize(device)
    lib = pa._lib
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = ctypes.c_void_p(stream.cuda_stream)
    call_args = (ptr(out), ptr(q), ptr(cache.k_cache), ptr(cache.v_cache), ptr(tables), ptr(ctx),
                 ptr(qs_dev), len(lens), total_q, hq, hkv, d, bs, nb, tables.shape[1],
                 int(max(chunks)), 1 / float(np.sqrt(d)), pa.PA_BF16, st)

    def step():
        if lib.pa_prefill(*call_args):
            raise RuntimeError(f"pa_prefill: {lib.pa_last_error().decode()}")

    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush_w = torch.empty(2 * l2 + (64 << 20), dtype=torch.uint8, device=device)
    flush_r = torch.ones((2 * l2 + (64 << 20)) // 4, dtype=torch.float32, device=device)

    def flush():
        flush_w.zero_()
        flush_r.sum()

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize(device)
    if pa.pa_device_errors() != 0:
        raise RuntimeError("device error word set during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    torch.cuda.synchronize(device)
    for i in range(args.steps):
        flush()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(ms), world, device)
    e2e = None
    if not args.no_e2e:
        ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush()
            ee[i][0].record(stream)
            q.copy_(q_host, non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)
            ee[i][1].record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ee), world, device)
        nbytes = q_host.numel() * 2
        e2e = {"value": whole_job_rate(flops, args.steps, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "ms_per_step": e2e_ms / args.steps}
    if pa.pa_device_errors() != 0:
        raise RuntimeError("device error word set during the timed steps")
    peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(peaks_path):
        peak, src = float(json.load(open(peaks_path))["bf16_tflops"]), "measured bf16_tflops (burst)"
    else:
        peak, src = 1590.0, "fallback"
    achieved = flops / (statistics.mean(ms) * 1e-3) / 1e12
    value = whole_job_rate(flops, args.steps, world, total_ms) / 1e12
    if rank == 0:
        print(json.dumps({
            "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": args.workload, "num_seqs": len(lens), "cached_before": before,
                       "chunk_tokens": chunks, "num_heads": hq, "num_kv_heads": hkv,
                       "head_dim": d, "block_size": bs, "causal_flops_per_step": flops,
                       "l2": "flushed between steps (outside the timed events)"},
            "step_us_p10_p50_p90": [1e3 * float(np.percentile(ms, p)) for p in (10, 50, 90)],
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "traffic": load_traffic(f"pa_prefill_{args.workload}", PREFILL_SOURCES),
                         "kernel": "pa_prefill_kernel",
                         "peak_source": src},
            "e2e": e2e, "gpu_launches": args.steps, "clocks": clk}), flush=True)


def main():
    args = parse_args()
    if args.warmup < 3 and args.impl == "b200":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    rank, world, local_rank = dist_env()
    if args.workload in ("prefill", "chunked_prefill"):
        run_prefill(args, rank, world, local_rank)
        return
    if args.workload == "swap":
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable":
                                  "the oracle has no device/host memory to swap between"}))
            return
        run_swap(args, rank, world, local_rank)
        return
    wl = make_workload(args.workload, args.block_size)
    if args.kv_dtype != "bf16":
        wl = dataclasses.replace(wl, kv_dtype=args.kv_dtype)
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return
    run_b200(args, wl, rank, world, local_rank)


if __name__ == "__main__":
    main()
