"""Shapes, sizes and seeds of the five paged decode workloads.

Each workload is a decode batch: one query token per sequence, one appended
token per sequence, then attention over the whole cached context. These are
plain descriptions; nothing here computes blocks or slots.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    num_heads: int            # query heads
    num_kv_heads: int
    head_dim: int
    dtype: str                # "f32" or "bf16": cache, query and output dtype
    block_size: int
    num_blocks: int           # physical pool size
    context_lens: tuple       # tokens cached BEFORE the decode step's append
    value_seed: int
    placement_seed: int
    # Shared-prefix workloads: tokens every sequence shares, written once by a
    # parent sequence and then forked to all others.
    shared_prefix: int = 0
    # Fragmented pools: lengths of ghost sequences allocated first; every other
    # ghost (even indices) is then freed, the rest stay live.
    ghost_lens: tuple = field(default_factory=tuple)
    partition_size: int = 0   # 0 = let the library choose
    decode_steps: int = 1
    # Cache element type when it differs from `dtype`: "fp8_e4m3" stores E4M3
    # codes with per-KV-head scales (queries, new rows and output stay bf16).
    kv_dtype: str = ""

    @property
    def num_seqs(self) -> int:
        return len(self.context_lens)

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.head_dim))

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def cache_dtype(self) -> str:
        return self.kv_dtype or self.dtype

    @property
    def cache_elem_bytes(self) -> int:
        return 1 if self.cache_dtype == "fp8_e4m3" else self.elem_bytes


def tiny() -> Workload:
    """2 sequences (7 and 33 cached tokens), block 4, 4/2 heads, head_dim 64, fp32, pool 32."""
    return Workload("tiny", 4, 2, 64, "f32", 4, 32, (7, 33), 1001, 2001)


def llama3_8b_layer() -> Workload:
    """One Llama-3-8B-shaped layer: the worked example's 8 requests, 32/8 heads, d 128, bf16."""
    return Workload("llama3_8b_layer", 32, 8, 128, "bf16", 16, 2048,
                    synth.LLAMA3_8B_BATCH_LENGTHS, 1002, 2002)


def large_batch(steps: int = 10) -> Workload:
    """256 lognormal lengths (mean 600, sigma 0.75, clip [16, 4096]); 80,000-block fragmented pool."""
    lens = synth.lognormal_lengths(256, 600.0, 0.75, 16, 4096, seed=3003)
    ghosts = synth.lognormal_lengths(512, 600.0, 0.75, 16, 4096, seed=4003)
    return Workload("large_batch", 32, 8, 128, "bf16", 16, 80_000, tuple(int(x) for x in lens),
                    1003, 2003, ghost_lens=tuple(int(x) for x in ghosts), decode_steps=steps)


def shared_prefix() -> Workload:
    """64 sequences sharing 2048 + 5 prompt tokens, then a private suffix uniform in [50, 1000]."""
    suffix = synth.uniform_lengths(64, 50, 1000, seed=3004)
    prefix = 2048 + 5
    lens = tuple(int(prefix + x) for x in suffix)
    return Workload("shared_prefix", 32, 8, 128, "bf16", 16, 8192, lens, 1004, 2004,
                    shared_prefix=prefix)


def long_context(block_size: int = 16) -> Workload:
    """16 sequences of 32,768 cached tokens, split-K partitions of 512 tokens."""
    lens = (32_768,) * 16
    need = 16 * (32_768 + block_size) // block_size
    pool = need + need // 100
    return Workload(f"long_context_bs{block_size}", 32, 8, 128, "bf16", block_size, pool, lens,
                    1005, 2005 + block_size, partition_size=512)


ALL = {
    "tiny": tiny,
    "llama3_8b_layer": llama3_8b_layer,
    "large_batch": large_batch,
    "shared_prefix": shared_prefix,
    "long_context": long_context,
}
