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
                             "swap", "prefill", "chunked_prefill", "layout_sweep"])
    ap.add_argument("--placement", choices=["random", "identity"], default="random",
                    help="physical block order: a seeded permutation (default) or identity "
                         "(each sequence's blocks contiguous in memory)")
    ap.add_argument("--block-size", type=int, default=16, help="long_context only")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8_e4m3"], default="bf16",
                    help="cache element type (fp8_e4m3: 8-bit codes, per-KV-head scales)")
    ap.add_argument("--partition-size", type=int, default=-1,
                    help="tokens per split-K partition (-1: tuned default, 0: library choice)")
    ap.add_argument("--unplanned", action="store_true",
                    help="decode on the (partition, sequence) grid up to the longest context "
                         "instead of a pa_decode_plan work list")
    ap.add_argument("--unfused", action="store_true",
                    help="time pa_kv_append + pa_decode instead of the fused pa_decode_append")
    ap.add_argument("--cascade", action="store_true",
                    help="shared_prefix only: time pa_decode_shared_prefix (the prefix once "
                         "for the batch) instead of pa_decode_append")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-back-to-back", action="store_true")
    ap.add_argument("--compact-pool", action="store_true",
                    help="a pool just large enough for the batch, no ghost sequences (a small "
                         "case of the same step for profilers)")
    ap.add_argument("--no-side-workloads", action="store_true",
                    help="skip the large-batch, long-context and shared-prefix lines")
    ap.add_argument("--no-early-reads", action="store_true",
                    help="decode without PA_DECODE_EARLY_CACHE_READS")
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
                   "long_context": 512,
                   # E4M3 codes halve a partition's bytes; on the planned grid 640
                   # tokens measured 62.4 us cold against 64.5 at the library's 768
                   # (57.2 / 56.5 us back to back)
                   "large_batch_fp8": 640}


def tuned_partition(wl) -> int:
    """The partition size measured best for a workload (0: the library's choice);
    an E4M3 form may have its own."""
    base = wl.name.split("_bs")[0].replace("_compact", "")
    if wl.cache_dtype == "fp8_e4m3" and base + "_fp8" in TUNED_PARTITION:
        return TUNED_PARTITION[base + "_fp8"]
    return TUNED_PARTITION[base]


def kv_bytes(wl) -> int:
    """K and V bytes the decode step reads: every attended token, every KV head."""
    return (sum(n + 1 for n in wl.context_lens) * wl.num_kv_heads * 2 * wl.head_dim *
            wl.cache_elem_bytes)


def kv_bytes_unique(wl) -> int:
    """K and V bytes of the distinct physical rows the step reads: a prefix held
    in shared blocks is stored once however many sequences attend it ("PagedAttention
    — AI Glossary", How it works, step 4: sharers point at the same blocks). Only the
    whole blocks of the prefix stay shared; a partly filled shared tail is copied
    before the first divergent write, so every sequence reads its own copy of it."""
    shared = (wl.shared_prefix // wl.block_size) * wl.block_size
    tokens = shared + sum(n + 1 - shared for n in wl.context_lens)
    return tokens * wl.num_kv_heads * 2 * wl.head_dim * wl.cache_elem_bytes


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

def build_on_gpu(wl, device, placement="random", extra_tokens=0):
    """Prefill every sequence through the library, then prepare one decode step.
    extra_tokens: room in the block tables for that many more decode steps."""
    import torch

    from paged_kv_cache_345_b200.cache import PagedKVCache
    from workloads import synth

    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    bs = wl.block_size
    max_blocks = max(-(-(n + 1 + extra_tokens) // bs) for n in wl.context_lens)
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


def plan_inputs(host, dev, partition_size, capacity_len=0):
    """The packed step inputs with the decode work list added: pa_decode_plan of
    the host lengths for this partition size, in room for every item a context
    of up to capacity_len tokens (default: the longest now) could need. Returns
    (host, dev, num_items); the device pack then carries the list with the
    other inputs, in the same one copy."""
    import torch

    import paged_kv_cache_345_b200 as pa

    lens = host["lens"].numpy()
    cap_len = max(int(capacity_len), int(lens.max(initial=0)))
    cap = max(1, lens.size * max(1, -(-cap_len // partition_size)))
    work = np.zeros((cap, 2), dtype=np.int32)
    n = len(pa.pa_decode_plan(lens, partition_size, out=work))
    arrays = {k: v for k, v in host.items() if k != "_pack"}
    arrays["work"] = torch.from_numpy(work)
    host2, dev2 = pack_step_inputs(arrays, dev["_pack"].device)
    return host2, dev2, n


class StepCalls:
    """The C-ABI calls of one decode step with their arguments marshalled once.

    fused: the step is one pa_decode_append call (append each newest token, then
    attend); otherwise pa_kv_append followed by pa_decode (same result).
    num_items > 0 (with dev["work"], a plan_inputs pack; bf16 and E4M3 caches):
    the decode runs on the work list's grid through pa_decode_planned (same
    result, no CTAs for partitions past a sequence's end).
    prefix_len > 0: the step is one pa_decode_shared_prefix call with the append
    (every sequence's first prefix_len tokens in the same blocks)."""

    def __init__(self, cache, dev, max_len, scale, partition_size, stream, fused=True,
                 prefix_len=0, num_items=0):
        import torch

        import paged_kv_cache_345_b200 as pa

        self.lib = pa._lib
        # the calls below hold raw pointers only: keep every tensor they point
        # into alive for as long as this object (a cache copy made for one
        # layer would otherwise be freed while a captured graph still uses it)
        self._keep = (cache.k_cache, cache.v_cache, getattr(cache, "k_scale", None),
                      getattr(cache, "v_scale", None), dict(dev))
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
        self.planned = bool(num_items) and "work" in dev and not prefix_len and \
            cache.k_cache.dtype in (torch.bfloat16, torch.uint8)
        if self.planned:
            sc = (p(cache.k_scale), p(cache.v_scale)) if self.fp8 else (None, None)
            dcode = pa.PA_FP8_E4M3 if self.fp8 else pa.PA_BF16
            head = (p(self.out), p(dev["q"]))
            tail = (p(cache.k_cache), p(cache.v_cache), *sc, p(dev["tables"]), p(dev["lens"]),
                    p(dev["work"]))
            rest = (s, hq, hkv, d, bs, nb, mbps, max_len, scale, self.partition_size, *ws,
                    dcode, st)
            self._items_at = len(head) + 2 + len(tail)   # where num_items sits in the args
            self.decode_args = (*head, None, None, *tail, int(num_items), *rest)
            self.step_args = (*head, p(dev["k_new"]), p(dev["v_new"]), *tail, int(num_items),
                              *rest)
            self.fns = (self.fns[0], self.lib.pa_decode_planned, self.lib.pa_decode_planned)
        self.num_items = int(num_items) if self.planned else 0
        self.fused = fused
        self.launches_per_step = (1 if fused else 2) + (1 if self.num_partitions > 1 else 0)
        self.prefix_len = prefix_len
        if prefix_len:
            # the cascade step: shared prefix on the tensor cores, each sequence's
            # own tokens (with the append) by the decode kernel, then the merge
            if self.fp8 or dt != pa.PA_BF16:
                raise ValueError("the shared-prefix step runs on a bf16 cache")
            need = pa.pa_decode_shared_prefix_workspace_bytes(s, hq, hkv, d, prefix_len, max_len,
                                                              partition_size)
            self.prefix_workspace = torch.empty(need, dtype=torch.uint8, device=dev["q"].device)
            self.step_args = (p(self.out), p(dev["q"]), p(dev["k_new"]), p(dev["v_new"]),
                              p(cache.k_cache), p(cache.v_cache), p(dev["tables"]),
                              p(dev["lens"]), s, hq, hkv, d, bs, nb, mbps, prefix_len, max_len,
                              scale, partition_size, p(self.prefix_workspace), need, dt, st)
            self.fns = (self.fns[0], self.fns[1], self.lib.pa_decode_shared_prefix)
            self.fused = True
            self.launches_per_step = 3
            self.partition_size = partition_size   # 0: the library's choice for the suffixes

    def set_items(self, num_items):
        """A new plan of another length in the same work-list buffer."""
        i = self._items_at
        self.decode_args = (*self.decode_args[:i], int(num_items), *self.decode_args[i + 1:])
        self.step_args = (*self.step_args[:i], int(num_items), *self.step_args[i + 1:])
        self.num_items = int(num_items)

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


def load_peak(key="hbm_gbs", fallback=FALLBACK_HBM_GBS):
    """(peak, source): the measured figure from MEASURED_PEAKS.json, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))[key]), "measured"
    return fallback, "fallback"


class L2Flush:
    """Between timed steps: write a buffer larger than L2, then read another one,
    so a step starts with L2 holding clean, unrelated lines (a write alone would
    leave the step paying for the write-back of dirty lines)."""

    def __init__(self, device):
        import torch

        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        self.w = torch.empty(2 * l2 + (64 << 20), dtype=torch.uint8, device=device)
        self.r = torch.ones((2 * l2 + (64 << 20)) // 4, dtype=torch.float32, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.sum()

    def describe(self):
        return (f"flushed between steps ({self.w.numel() >> 20} MiB written, then "
                f"{(self.r.numel() * 4) >> 20} MiB of another buffer read; outside the timed "
                "events)")


def cold_steps(step, flush, steps, warmup, stream, barrier=None):
    """Per-step device times (ms): each step bracketed by CUDA events on the
    launching stream, L2 flushed before it, outside the events."""
    import torch

    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    if barrier:
        barrier()
    for i in range(steps):
        flush()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def host_allocator_metrics(steps: int = 10):
    """The host block manager's decode step on the large batch (256 lognormal
    sequences in a fragmented 80,000-block pool): append_slots (next slot, a new
    block when a tail is full, copy-on-write when it is shared) + block_tables,
    through the Python binding, for `steps` steps; and cache utilisation
    (tokens / allocated slots) of the worked example's batch, before and after
    one decode step, beside the slab figure of the same batch ("What is paged
    attention in vLLM...", Worked example: 99.4 % vs 16.1 %)."""
    import paged_kv_cache_345_b200 as pa
    from workloads import configs, synth

    wl = configs.large_batch(steps=steps)
    bm = pa.BlockManager(wl.num_blocks, wl.block_size)
    bm.allocator.set_free_order(synth.block_permutation(wl.num_blocks, wl.placement_seed))
    ghosts = [bm.add_seq() for _ in wl.ghost_lens]
    bm.append_slots(ghosts, list(wl.ghost_lens))
    for i in range(0, len(ghosts), 2):
        bm.free_seq(ghosts[i])
    seqs = [bm.add_seq() for _ in wl.context_lens]
    bm.append_slots(seqs, list(wl.context_lens))
    mb = -(-(max(wl.context_lens) + steps) // wl.block_size)
    free0 = bm.allocator.num_free()
    times = []
    ones = [1] * len(seqs)
    for _ in range(steps):
        t0 = time.perf_counter()
        slots, cows = bm.append_slots(seqs, ones)
        tables, lens = bm.block_tables(seqs, mb)
        times.append(time.perf_counter() - t0)
    # through the binding with the caller's buffers (no allocation per step)
    ids = np.asarray(seqs, dtype=np.int32)
    cnt = np.ones(len(seqs), dtype=np.int32)
    mb2 = mb + 2 * steps // wl.block_size + 2
    b_slots = np.empty(len(seqs), dtype=np.int64)
    b_cows = np.empty((len(seqs), 2), dtype=np.int64)
    b_tabs = np.empty(len(seqs) * mb2, dtype=np.int32)
    b_lens = np.empty(len(seqs), dtype=np.int32)
    b_times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        bm.append_slots(ids, cnt, b_slots, b_cows)
        bm.block_tables(ids, mb2, b_tabs, b_lens)
        b_times.append(time.perf_counter() - t0)
    # the same step called through the C ABI with preallocated buffers (what a
    # native caller pays): 10 more steps
    slot_buf = np.empty(len(seqs), dtype=np.int64)
    cow_buf = np.empty((len(seqs), 2), dtype=np.int64)
    tab_buf = np.empty((len(seqs), mb2), dtype=np.int32)
    len_buf = np.empty(len(seqs), dtype=np.int32)
    ncow = ctypes.c_int(0)
    i32p, i64p = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
    args_a = (bm._h, ids.ctypes.data_as(i32p), cnt.ctypes.data_as(i32p), len(seqs),
              slot_buf.ctypes.data_as(i64p), cow_buf.ctypes.data_as(i64p), len(seqs),
              ctypes.byref(ncow))
    args_t = (bm._h, ids.ctypes.data_as(i32p), len(seqs), tab_buf.ctypes.data_as(i32p), mb2,
              len_buf.ctypes.data_as(i32p))
    c_times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        if pa._lib.pa_bm_append_slots(*args_a) or pa._lib.pa_bm_block_tables(*args_t):
            raise RuntimeError(pa._lib.pa_last_error().decode())
        c_times.append(time.perf_counter() - t0)
    # the decode's work list for the lengths the last step left (pa_decode_plan,
    # host only): through the binding into a caller buffer, then through the C ABI
    plan_lens = len_buf.copy()
    ps = pa.pa_decode_partition_size(len(seqs), wl.num_kv_heads, int(plan_lens.max()))
    cap = len(seqs) * max(1, -(-int(plan_lens.max()) // ps))
    work_buf = np.empty((cap, 2), dtype=np.int32)
    nitems = ctypes.c_int(0)
    args_p = (plan_lens.ctypes.data_as(i32p), len(seqs), ps, work_buf.ctypes.data_as(i32p), cap,
              ctypes.byref(nitems))
    p_times, pc_times = [], []
    for _ in range(steps):
        t0 = time.perf_counter()
        pa.pa_decode_plan(plan_lens, ps, out=work_buf)
        p_times.append(time.perf_counter() - t0)
    for _ in range(steps):
        t0 = time.perf_counter()
        if pa._lib.pa_decode_plan(*args_p):
            raise RuntimeError(pa._lib.pa_last_error().decode())
        pc_times.append(time.perf_counter() - t0)
    new_blocks = free0 - bm.allocator.num_free()
    held = sum(bm.seq_num_blocks(s) for s in seqs)
    tokens = sum(bm.seq_len(s) for s in seqs)

    ex = configs.llama3_8b_layer()
    wb = pa.BlockManager(ex.num_blocks, ex.block_size)
    wseqs = [wb.add_seq() for _ in ex.context_lens]
    wb.append_slots(wseqs, list(ex.context_lens))

    def util(b, ss):
        t = sum(b.seq_len(x) for x in ss)
        slots_ = sum(b.seq_num_blocks(x) for x in ss) * b.block_size
        return t, slots_

    t_pre, s_pre = util(wb, wseqs)
    wb.append_slots(wseqs, [1] * len(wseqs))
    t_post, s_post = util(wb, wseqs)
    max_positions = 8192   # Llama-3-8B context length: the slab a contiguous cache reserves
    return {
        "allocator_step": {
            "us_per_step_mean": 1e6 * statistics.mean(times),
            "us_per_step_p50": 1e6 * statistics.median(times),
            "us_per_step_buffers_p50": 1e6 * statistics.median(b_times),
            "us_per_step_c_abi_p50": 1e6 * statistics.median(c_times),
            "sequences": len(seqs), "steps": 3 * steps, "new_blocks": int(new_blocks),
            "what": "pa_bm_append_slots (slot, new block when the tail is full, copy-on-write "
                    "check) + pa_bm_block_tables: the first figures through the Python binding "
                    "with Python lists (10 steps), the buffers one through the binding with "
                    "the caller's arrays (10 more), the c_abi one through ctypes with "
                    "preallocated buffers (10 more)",
            "utilisation_after": tokens / (held * wl.block_size)},
        "decode_plan": {
            "us_p50_binding": 1e6 * statistics.median(p_times),
            "us_p50_c_abi": 1e6 * statistics.median(pc_times),
            "items": int(nitems.value), "partition_size": ps, "sequences": len(seqs),
            "what": "pa_decode_plan of the 256 lengths (the planned decode's work list), "
                    "into a caller buffer: through the binding, then through ctypes"},
        "cache_utilisation": {
            "workload": "worked example (8 requests, block 16)",
            "paged_before_step": t_pre / s_pre, "paged_after_step": t_post / s_post,
            "tokens_before_step": t_pre, "slots_before_step": s_pre,
            "slab": t_pre / (len(wseqs) * max_positions),
            "slab_slots": len(wseqs) * max_positions},
    }


def cpu_baseline_line(wl, bytes_step, budget_s):
    """The oracle on the host cores (all of them, then one), bounded samples."""
    try:
        times, cores = cpu_oracle_run(wl, budget_s)
    except ValueError as exc:
        return {"value": None, "unit": "GB/s", "cores": 0, "kind": "oracle",
                "sample": f"not run: {exc}"}
    line = {"value": bytes_step * len(times) / sum(times) / 1e9, "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{len(times)} whole decode steps of the {wl.num_seqs}-sequence batch in "
                      f"{sum(times):.1f} s (float64 NumPy)"}
    try:
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=1):
            t1, _ = cpu_oracle_run(wl, budget_s / 2)
        line["one_core"] = {"value": bytes_step * len(t1) / sum(t1) / 1e9, "unit": "GB/s",
                            "cores": 1,
                            "sample": f"{len(t1)} whole decode steps in {sum(t1):.1f} s, BLAS "
                                      "limited to one thread"}
    except Exception as exc:  # noqa: BLE001
        line["one_core"] = {"value": None, "sample": f"not run: {exc}"}
    return line


def measure_workload(name, args, device, stream, flush, peak, steps, warmup=3):
    """One more workload in the same process: the fused decode step, cold (L2
    flushed), its rate against the HBM peak, with its own clock record. A name
    ending in _fp8 is the same workload over an E4M3 cache."""
    import torch

    fp8 = name.endswith("_fp8")
    wl2 = make_workload(name[:-4] if fp8 else name, 16)
    if fp8:
        wl2 = dataclasses.replace(wl2, kv_dtype="fp8_e4m3")
    steps_after = 10 if name == "large_batch" else 0
    cache, seqs, host, dev, max_len, cow_pairs = build_on_gpu(wl2, device,
                                                              extra_tokens=steps_after)
    import paged_kv_cache_345_b200 as pa

    ps = tuned_partition(wl2) or \
        pa.pa_decode_partition_size(wl2.num_seqs, wl2.num_kv_heads, max_len)
    items = 0
    if not args.unplanned:
        host, dev, items = plan_inputs(host, dev, ps, max_len + steps_after)
    calls = StepCalls(cache, dev, max_len, wl2.scale, ps, stream, num_items=items)
    clocks = ClockSampler(device.index or 0)
    clocks.start()
    ms = cold_steps(calls.step, flush, steps, warmup, stream)
    clk = clocks.stop()
    mean_s = statistics.mean(ms) * 1e-3
    logical, unique = kv_bytes(wl2), kv_bytes_unique(wl2)
    res = {"us_per_step": 1e3 * statistics.mean(ms),
           "step_us_p10_p50_p90": [1e3 * float(np.percentile(ms, p)) for p in (10, 50, 90)],
           "kv_bytes_per_step": unique, "GB_per_s": unique / mean_s / 1e9,
           "frac": unique / mean_s / 1e9 / peak,
           "attended_tokens_per_s": sum(n + 1 for n in wl2.context_lens) / mean_s,
           "num_seqs": wl2.num_seqs, "block_size": wl2.block_size, "kv_cache": wl2.cache_dtype,
           "partition_size": calls.partition_size, "planned_grid": calls.planned,
           "steps": steps, "clocks": clk}
    if unique != logical:
        res["kv_bytes_logical"] = logical
        res["GB_per_s_logical"] = logical / mean_s / 1e9
        res["copy_on_write_pairs"] = cow_pairs
    if steps_after:
        res["ten_steps"] = serving_steps(cache, seqs, host, dev, max_len, wl2, stream,
                                         steps_after, ps)
    if wl2.shared_prefix:
        # the same step through the cascade entry point: the shared blocks read
        # once for the whole batch
        prefix = (wl2.shared_prefix // wl2.block_size) * wl2.block_size
        cascade = StepCalls(cache, dev, max_len, wl2.scale, 0, stream, prefix_len=prefix)
        clocks = ClockSampler(device.index or 0)
        clocks.start()
        cms = cold_steps(cascade.step, flush, steps, warmup, stream)
        cclk = clocks.stop()
        cmean = statistics.mean(cms) * 1e-3
        res["shared_prefix_step"] = {
            "entry": "pa_decode_shared_prefix", "prefix_len": prefix,
            "us_per_step": 1e3 * statistics.mean(cms),
            "step_us_p10_p50_p90": [1e3 * float(np.percentile(cms, p)) for p in (10, 50, 90)],
            "GB_per_s": unique / cmean / 1e9, "frac": unique / cmean / 1e9 / peak,
            "attended_tokens_per_s": sum(n + 1 for n in wl2.context_lens) / cmean,
            "launches_per_step": cascade.launches_per_step, "clocks": cclk}
        del cascade
    pa_device_errors_or_raise()
    del calls, cache, dev, host
    torch.cuda.empty_cache()
    return res


def serving_steps(cache, seqs, host, dev, max_len, wl, stream, steps, partition_size):
    """`steps` decode steps of a serving loop after the timed step above: per
    step, the host block manager's step through the C ABI (the next slot of
    every sequence, a new block where the tail is full, the copy-on-write
    check, the new tables), its output (slots, tables, lengths) host -> device
    in one copy, and the fused append + decode. q and the new K/V rows are the
    previous layer's output in a model, so they are staged on the device
    beforehand (one set per step, each step's call reading its own). Contexts grow by one token a step. With a
    work list in the pack (plan_inputs), each step also plans its decode grid
    from the new lengths (pa_decode_plan, host) into the pack. Host time by
    perf_counter, device time (the copy + the kernels) by CUDA events."""
    import torch

    import paged_kv_cache_345_b200 as pa
    from workloads import synth

    s = len(seqs)
    mbps = dev["tables"].shape[1]
    tdt = dev["q"].dtype
    staged = [(torch.from_numpy(synth.queries(wl.value_seed, 100 + i, s, wl.num_heads,
                                              wl.head_dim)).to(dev["q"].device, tdt),
               *[torch.from_numpy(a).to(dev["q"].device, tdt) for a in
                 synth.new_token_kv(wl.value_seed, 100 + i, s, wl.num_kv_heads, wl.head_dim)])
              for i in range(steps)]
    # one marshalled call per step, reading that step's staged q and rows
    planned = "work" in dev
    calls = [StepCalls(cache, dict(dev, q=q, k_new=k, v_new=v), max_len + steps, wl.scale,
                       partition_size, stream, num_items=1 if planned else 0)
             for q, k, v in staged]
    # the host-made part of the packed inputs: slots, tables, lengths (and the
    # work list), contiguous
    last = dev["work"] if planned else dev["lens"]
    lo = dev["slots"].data_ptr() - dev["_pack"].data_ptr()
    hi = last.data_ptr() + last.numel() * 4 - dev["_pack"].data_ptr()
    work_buf = host["work"].numpy() if planned else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    host_us, bytes_step, new_blocks = [], [], 0
    # the block manager writes straight into the pinned pack (no allocation per step)
    ids, ones = np.asarray(seqs, dtype=np.int32), np.ones(s, dtype=np.int32)
    slot_buf, tab_buf, len_buf = (host["slots"].numpy(), host["tables"].numpy(),
                                  host["lens"].numpy())
    cow_buf = np.empty((s, 2), dtype=np.int64)
    torch.cuda.synchronize()
    for i in range(steps):
        free_before = cache.bm.allocator.num_free()
        t0 = time.perf_counter()
        slots, cows = cache.bm.append_slots(ids, ones, slot_buf, cow_buf)
        tables, lens = cache.bm.block_tables(ids, mbps, tab_buf, len_buf)
        if planned:
            n_items = len(pa.pa_decode_plan(lens, partition_size, out=work_buf))
        host_us.append(1e6 * (time.perf_counter() - t0))
        if planned:
            calls[i].set_items(n_items)
        new_blocks += free_before - cache.bm.allocator.num_free()
        if len(cows):
            pa.pa_copy_blocks(cache.k_cache, cache.v_cache, torch.from_numpy(cows).to(dev["q"].device))
        bytes_step.append(int(lens.astype(np.int64).sum()) * wl.num_kv_heads * 2 * wl.head_dim *
                          wl.cache_elem_bytes)
        ev[i][0].record(stream)
        dev["_pack"][lo:hi].copy_(host["_pack"][lo:hi], non_blocking=True)
        calls[i].step()
        ev[i][1].record(stream)
        stream.synchronize()
    dev_us = [1e3 * a.elapsed_time(b) for a, b in ev]
    pa_device_errors_or_raise()
    return {"steps": steps, "host_block_manager_us": [round(x, 1) for x in host_us],
            "device_us": [round(x, 2) for x in dev_us], "h2d_bytes_per_step": hi - lo,
            "mean_host_us": statistics.mean(host_us), "mean_device_us": statistics.mean(dev_us),
            "median_host_us": statistics.median(host_us),
            "median_device_us": statistics.median(dev_us),
            "mean_kv_GB_per_s": statistics.mean(b / (u * 1e-6) / 1e9
                                                for b, u in zip(bytes_step, dev_us)),
            "new_blocks": new_blocks,
            "how": "per step: pa_bm_append_slots + pa_bm_block_tables" +
                   (" + pa_decode_plan" if planned else "") +
                   " (host, through the binding, written straight into the pinned input "
                   "pack); slots, tables, lengths" + (" and work list" if planned else "") +
                   " host -> device in one copy; " +
                   ("pa_decode_planned" if planned else "pa_decode_append") +
                   " (append + decode) on q and new rows staged on the device (a model's "
                   "previous layer makes them); no L2 flush (the cache is 0.63 GB)"}


def pa_device_errors_or_raise():
    import paged_kv_cache_345_b200 as pa

    if pa.pa_device_errors() != 0:
        raise RuntimeError("device error word set")


def replica_calls(cache, dev, max_len, scale, ps, stream, layers, fused=True, fp8=False,
                  prefix_len=0, num_items=0):
    """StepCalls over `layers` copies of the cache (one per model layer)."""
    import paged_kv_cache_345_b200 as pa  # noqa: F401

    out = []
    for _ in range(layers):
        view = type("CacheView", (), {})()
        view.k_cache, view.v_cache = cache.k_cache.clone(), cache.v_cache.clone()
        if fp8:
            view.k_scale, view.v_scale = cache.k_scale, cache.v_scale
        out.append(StepCalls(view, dev, max_len, scale, ps, stream, fused=fused,
                             prefix_len=prefix_len, num_items=num_items))
    return out


def back_to_back(layer_calls, stream, reps, early):
    """One CUDA graph of the step over every layer's cache (together far larger
    than L2, so no flush), replayed: mean time per layer (ms)."""
    import torch

    import paged_kv_cache_345_b200 as pa

    for c in layer_calls:   # warm-up, eager
        c.step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream), pa.decode_options(early):
        for c in layer_calls:
            c.step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for i in range(reps):
        gev[i][0].record(stream)
        graph.replay()
        gev[i][1].record(stream)
    torch.cuda.synchronize()
    per_layer = statistics.mean(e[0].elapsed_time(e[1]) for e in gev) / len(layer_calls)
    del graph
    return per_layer


def e2e_overlapped(cache, host, max_len, scale, ps, stream, layers, reps, early, fp8=False,
                   prefix_len=0, num_items=0):
    """End to end through the C ABI with the host copies pipelined: two pinned
    host packs and two device packs; for step i the inputs go host -> device on
    an upload stream (pack i % 2, once step i - 2 has finished reading it), the
    step runs on the compute stream, its output goes device -> host on a
    download stream, so step i + 1's input copy and step i - 1's output copy
    overlap step i's kernels. Steps rotate over per-layer cache copies (no flush);
    the whole pipeline of `layers` steps is one CUDA graph. Returns ms per step."""
    import torch

    import paged_kv_cache_345_b200 as pa

    device = cache.k_cache.device
    packs = [pack_step_inputs({k: v for k, v in host.items() if k != "_pack"}, device)
             for _ in range(2)]
    calls = []
    for i in range(layers):
        view = type("CacheView", (), {})()
        view.k_cache, view.v_cache = cache.k_cache.clone(), cache.v_cache.clone()
        if fp8:
            view.k_scale, view.v_scale = cache.k_scale, cache.v_scale
        calls.append(StepCalls(view, packs[i % 2][1], max_len, scale, ps, stream,
                               prefix_len=prefix_len, num_items=num_items))
    outs_host = [torch.empty(calls[0].out.shape, dtype=calls[0].out.dtype).pin_memory()
                 for _ in range(2)]
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    for c in calls:
        c.step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    done = [None, None]
    with torch.cuda.graph(graph, stream=stream), pa.decode_options(early):
        up.wait_stream(stream)
        down.wait_stream(stream)
        for i, c in enumerate(calls):
            b = i % 2
            if done[b] is not None:
                up.wait_event(done[b])
            with torch.cuda.stream(up):
                packs[b][1]["_pack"].copy_(packs[b][0]["_pack"], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(up)
            stream.wait_event(ready)
            c.step()
            fin = torch.cuda.Event()
            fin.record(stream)
            done[b] = fin
            down.wait_event(fin)
            with torch.cuda.stream(down):
                outs_host[b].copy_(c.out, non_blocking=True)
        stream.wait_stream(up)
        stream.wait_stream(down)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for i in range(reps):
        gev[i][0].record(stream)
        graph.replay()
        gev[i][1].record(stream)
    torch.cuda.synchronize()
    per_step = statistics.mean(e[0].elapsed_time(e[1]) for e in gev) / layers
    h2d = packs[0][0]["_pack"].numel()
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    del graph, calls
    torch.cuda.empty_cache()
    return per_step, h2d, d2h


# workloads measured beside the headline one, in the same process
SIDE_WORKLOADS = ("large_batch", "large_batch_fp8", "long_context", "shared_prefix")


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
    peak, peak_src = load_peak()
    early = 0 if args.no_early_reads else pa.PA_DECODE_EARLY_CACHE_READS

    cache, seqs, host, dev, max_len, cow_pairs = build_on_gpu(wl, device, args.placement)
    ps = tuned_partition(wl) if args.partition_size < 0 else args.partition_size
    prefix_len = 0
    if args.cascade:
        if not wl.shared_prefix:
            raise SystemExit("--cascade needs a workload with a shared prefix")
        prefix_len = (wl.shared_prefix // wl.block_size) * wl.block_size
        ps = 0 if args.partition_size < 0 else args.partition_size
    items = 0
    if not prefix_len and not args.unplanned and wl.cache_dtype in ("bf16", "fp8_e4m3"):
        # the decode grid from the host lengths: no CTAs past a sequence's end
        ps = ps or pa.pa_decode_partition_size(wl.num_seqs, wl.num_kv_heads, max_len)
        host, dev, items = plan_inputs(host, dev, ps)
    calls = StepCalls(cache, dev, max_len, wl.scale, ps, stream, fused=not args.unfused,
                      prefix_len=prefix_len, num_items=items)
    launches_per_step, part_size = calls.launches_per_step, calls.partition_size
    planned = calls.planned
    num_partitions = calls.num_partitions
    bytes_step = kv_bytes_unique(wl)
    bytes_logical = kv_bytes(wl)
    tokens_step = sum(n + 1 for n in wl.context_lens)
    flush = L2Flush(device)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize(device)

    # ---- device-resident steps (the headline): cold, L2 flushed before each
    clocks = ClockSampler(local_rank)
    clocks.start()
    t_wall = time.perf_counter()
    with pa.decode_options(early):
        step_ms = cold_steps(calls.step, flush, args.steps, args.warmup, stream, barrier)
    wall = time.perf_counter() - t_wall
    clk = clocks.stop()
    pa_device_errors_or_raise()
    total_ms = max_over_ranks(sum(step_ms), world, device)

    # ---- end to end: pinned host inputs -> device -> kernels -> host output
    e2e = None
    if not args.no_e2e:
        out_host = torch.empty(calls.out.shape, dtype=calls.out.dtype).pin_memory()
        h2d = host["_pack"].numel()     # q, new K/V rows, slot mapping, tables, lengths, work list
        d2h = out_host.numel() * out_host.element_size()

        def e2e_step():
            dev["_pack"].copy_(host["_pack"], non_blocking=True)
            calls.step()
            out_host.copy_(calls.out, non_blocking=True)

        with pa.decode_options(early):
            e_ms = cold_steps(e2e_step, flush, args.steps, args.warmup, stream, barrier)
        e2e_ms = max_over_ranks(sum(e_ms), world, device)
        e2e = {"value": whole_job_rate(bytes_step, args.steps, world, e2e_ms) / 1e9,
               "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / args.steps,
               "how": "serial: one packed host->device copy, the step, the output copy back, "
                      "per step, L2 flushed between steps"}
        if world == 1 and not args.no_back_to_back:
            ov_ms, oh2d, od2h = e2e_overlapped(cache, host, max_len, wl.scale,
                                               calls.partition_size, stream, args.layers,
                                               max(5, min(50, args.steps // args.layers)), early,
                                               calls.fp8, prefix_len, items)
            pa_device_errors_or_raise()
            e2e["overlapped"] = {
                "value": bytes_step / (ov_ms * 1e-3) / 1e9, "unit": "GB/s",
                "ms_per_step": ov_ms, "h2d_bytes_per_step": oh2d, "d2h_bytes_per_step": od2h,
                "how": f"two host/device packs, uploads and downloads on two more streams "
                       f"overlapping the neighbouring steps, {args.layers} steps over per-layer cache copies in "
                       "one CUDA graph (no flush)"}

    # ---- back to back: the same step over `layers` cache copies in one graph
    b2b = None
    if not args.no_back_to_back and world == 1:
        layer_calls = replica_calls(cache, dev, max_len, wl.scale, calls.partition_size, stream,
                                    args.layers, fused=calls.fused, fp8=calls.fp8,
                                    prefix_len=prefix_len, num_items=items)
        reps = max(5, min(50, args.steps // args.layers))
        per_layer_ms = back_to_back(layer_calls, stream, reps, early)
        pa_device_errors_or_raise()
        b2b = {"layers": args.layers, "us_per_layer": 1e3 * per_layer_ms,
               "kv_GB_per_s": bytes_step / (per_layer_ms * 1e-3) / 1e9,
               "frac_of_peak": bytes_step / (per_layer_ms * 1e-3) / 1e9 / peak,
               "early_cache_reads": bool(early),
               "how": "one CUDA graph of the step over per-layer cache copies (together larger "
                      "than L2), no flush; consecutive layers overlap through programmatic "
                      "dependent launch"}
        del layer_calls
        torch.cuda.empty_cache()

    # ---- the other workloads, same process (one GPU, default workload only)
    side = None
    if world == 1 and wl.name == "llama3_8b_layer" and not args.no_side_workloads:
        del calls
        torch.cuda.empty_cache()
        side = {}
        with pa.decode_options(early):
            for name in SIDE_WORKLOADS:
                side[name] = measure_workload(name, args, device, stream, flush, peak,
                                              steps=max(10, min(args.steps, 100)))
        calls = None

    # ---- roofline of the headline step
    dec_s = statistics.mean(step_ms) * 1e-3
    achieved = bytes_step / dec_s / 1e9
    traffic = load_traffic(f"pa_decode_{wl.name}" + ("_fp8" if wl.cache_dtype != "bf16" else "")
                           + ("_cascade" if prefix_len else ""))

    # ---- host side and CPU baseline (rank 0, one GPU only)
    host_side = host_allocator_metrics() if rank == 0 else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_line(wl, bytes_logical, args.cpu_budget_s)

    value = whole_job_rate(bytes_step, args.steps, world, total_ms) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.cache_dtype, "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs": wl.num_seqs, "num_heads": wl.num_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                   "block_size": wl.block_size, "num_blocks": wl.num_blocks,
                   "attended_tokens": tokens_step, "kv_bytes_per_step": bytes_step,
                   "kv_bytes_logical_per_step": bytes_logical,
                   "partition_size": part_size, "num_partitions": num_partitions,
                   "planned_grid": planned, "work_items": items,
                   "copy_on_write_pairs": cow_pairs,
                   "placement": args.placement, "kv_cache": wl.cache_dtype,
                   "early_cache_reads": bool(early), "shared_prefix_len": prefix_len,
                   "l2": flush.describe(), "parallelism": f"replicas x{world}"},
        "attended_tokens_per_s": whole_job_rate(tokens_step, args.steps, world, total_ms),
        "us_per_step": 1e3 * total_ms / args.steps,
        "step_us_p10_p50_p90": [1e3 * float(np.percentile(step_ms, p)) for p in (10, 50, 90)],
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": ("pa_decode_shared_prefix (prefix attention kernel, fused "
                                "append + suffix decode kernel, merge kernel)" if prefix_len else
                                ("pa_decode_planned" if planned else "pa_decode_append") +
                                " (fused append + decode kernel, split-K merge kernel)"
                                if not args.unfused else
                                "pa_kv_append + " +
                                ("pa_decode_planned" if planned else "pa_decode") +
                                " (decode + split-K merge kernels)"),
                     "peak_source": f"{peak_src} hbm_gbs"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "back_to_back": b2b,
        "workloads": side,
        "host": host_side,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "wall_s_timed_region": wall,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()


LAYOUT_METRIC = "decode attention over paged vs contiguous caches: us per call and KV-read GB/s"


def run_layout_sweep(args, rank, world, local_rank):
    """The cost of paging on this GPU ("What is paged attention in vLLM, and why
    does it matter?", Trade-offs and edge cases, first point: table reads,
    extra branches and irregular accesses made the 2023 paged kernel 20-26 %
    slower than a kernel over contiguous caches; "Paged Attention" glossary,
    FAQ: small blocks mean more lookups). The same tokens are decoded
    (pa_decode, no append) from paged caches at block sizes 8..128 with a
    random and an in-order (identity) physical placement, and from one
    contiguous slab per sequence (pa_decode_contiguous: no table at all), on the
    Llama-3-8B-shaped batch and on the long-context batch. Each call is timed
    cold (L2 flushed before it); every paged output is checked bit for bit
    against the contiguous one."""
    import torch

    import paged_kv_cache_345_b200 as pa
    from workloads import configs, synth

    if rank != 0:
        return
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)
    peak, peak_src = load_peak()
    flush = L2Flush(device)
    clocks = ClockSampler(local_rank)
    clocks.start()
    table = {}
    for name, steps in (("llama3_8b_layer", min(args.steps, 200)),
                        ("long_context", min(args.steps, 40))):
        wl = make_workload(name, 16)
        lens = [n + 1 for n in wl.context_lens]          # the step's attended tokens
        S, hkv, d = wl.num_seqs, wl.num_kv_heads, wl.head_dim
        slab_len = -(-max(lens) // 16) * 16
        ks = torch.zeros((S, slab_len, hkv, d), dtype=torch.bfloat16, device=device)
        vs = torch.zeros_like(ks)
        for s, n in enumerate(lens):
            k, v = synth.kv_rows(wl.value_seed, s, n, hkv, d)
            ks[s, :n] = torch.from_numpy(k).to(device).to(torch.bfloat16)
            vs[s, :n] = torch.from_numpy(v).to(device).to(torch.bfloat16)
        q = torch.from_numpy(synth.queries(wl.value_seed, 0, S, wl.num_heads, d)).to(
            device).to(torch.bfloat16)
        lens_d = torch.tensor(lens, dtype=torch.int32, device=device)
        max_len = max(lens)
        ps = wl.partition_size or pa.pa_decode_partition_size(S, hkv, max_len)
        ws = torch.empty(max(16, pa.pa_decode_workspace_bytes(S, wl.num_heads, hkv, d, max_len,
                                                               ps)),
                         dtype=torch.uint8, device=device)
        bytes_call = sum(lens) * hkv * 2 * d * 2
        out_c = torch.empty_like(q)

        def contig():
            pa.pa_decode_contiguous(out_c, q, ks, vs, lens_d, max_len, wl.scale, ps, ws)

        ms = cold_steps(contig, flush, steps, 3, stream)
        rows = {"contiguous": {"us_per_call": 1e3 * statistics.median(ms),
                               "GB_per_s": bytes_call / (statistics.median(ms) * 1e-3) / 1e9}}
        for bs in (8, 16, 32, 64, 128):
            for placement in ("random", "identity"):
                nb = sum(-(-n // bs) for n in lens) + 16
                bm = pa.BlockManager(nb, bs)
                order = synth.block_permutation(nb, wl.placement_seed + bs) \
                    if placement == "random" else np.arange(nb, dtype=np.int32)
                bm.allocator.set_free_order(order)
                seqs = [bm.add_seq() for _ in lens]
                kc = torch.empty((nb, bs, hkv, d), dtype=torch.bfloat16, device=device)
                vc = torch.empty_like(kc)
                for s, n in enumerate(lens):
                    slots, _ = bm.append_slots([seqs[s]], [n])
                    pa.pa_kv_append(ks[s, :n], vs[s, :n], torch.from_numpy(slots).to(device),
                                    kc, vc)
                mb = -(-max_len // bs)
                tables, lens_bm = bm.block_tables(seqs, mb)
                tables = torch.from_numpy(tables).to(device)
                out_p = torch.empty_like(q)

                def paged():
                    pa.pa_decode(out_p, q, kc, vc, tables, lens_d, max_len, wl.scale, ps, ws)

                ms = cold_steps(paged, flush, steps, 3, stream)
                pa_device_errors_or_raise()
                med = statistics.median(ms)
                rows[f"bs{bs}_{placement}"] = {
                    "us_per_call": 1e3 * med, "GB_per_s": bytes_call / (med * 1e-3) / 1e9,
                    "vs_contiguous": med / (rows["contiguous"]["us_per_call"] * 1e-3),
                    "bit_identical_to_contiguous": bool(torch.equal(out_p, out_c))}
                del kc, vc, tables, bm
                torch.cuda.empty_cache()
        table[name] = {"num_seqs": S, "attended_tokens": sum(lens), "kv_bytes_per_call":
                       bytes_call, "partition_size": ps, "slab_len": slab_len, "steps": steps,
                       "results": rows}
        del ks, vs, ws
        torch.cuda.empty_cache()
    clk = clocks.stop()
    ref = table["llama3_8b_layer"]["results"]["contiguous"]
    print(json.dumps({
        "metric": LAYOUT_METRIC, "value": ref["GB_per_s"], "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": 3, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "layout_sweep: llama3_8b_layer and long_context, block sizes "
                               "8-128, random / identity placement, contiguous slabs",
                   "l2": flush.describe()},
        "peak": peak, "peak_source": f"{peak_src} hbm_gbs", "layouts": table, "clocks": clk,
        "gpu_launches": None}), flush=True)


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
    head = (ptr(out), ptr(q), ptr(cache.k_cache), ptr(cache.v_cache), ptr(tables), ptr(ctx),
            ptr(qs_dev))
    rest = (len(lens), total_q, hq, hkv, d, bs, nb, tables.shape[1], int(max(chunks)),
            1 / float(np.sqrt(d)), pa.PA_BF16, st)
    planned = not args.unplanned
    if planned:
        # the work items listed on the host in the kernel's own order
        # (pa_prefill_plan): each CTA reads its item instead of searching
        work_h = pa.pa_prefill_plan(qs, np.asarray(lens, dtype=np.int32), hq, hkv)
        work_d = torch.from_numpy(np.ascontiguousarray(work_h)).to(device)
        call_args = (*head, ptr(work_d), len(work_h), *rest)
        fn, name = lib.pa_prefill_planned, "pa_prefill_planned"
    else:
        call_args = (*head, *rest)
        fn, name = lib.pa_prefill, "pa_prefill"

    def step():
        if fn(*call_args):
            raise RuntimeError(f"{name}: {lib.pa_last_error().decode()}")

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
                       "planned_grid": planned,
                       "l2": "flushed between steps (outside the timed events)"},
            "step_us_p10_p50_p90": [1e3 * float(np.percentile(ms, p)) for p in (10, 50, 90)],
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "traffic": load_traffic(f"pa_prefill_{args.workload}", PREFILL_SOURCES),
                         "kernel": "pa_prefill_kernel (" + name + ")",
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
    if args.workload == "layout_sweep":
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable":
                                  "the oracle has no kernels whose memory layout could be compared"}))
            return
        run_layout_sweep(args, rank, world, local_rank)
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
    if args.compact_pool:
        need = sum(-(-(n + 2) // wl.block_size) for n in wl.context_lens) + 64
        wl = dataclasses.replace(wl, num_blocks=need, ghost_lens=(),
                                 name=wl.name + "_compact")
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return
    run_b200(args, wl, rank, world, local_rank)


if __name__ == "__main__":
    main()
