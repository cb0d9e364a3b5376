"""Seeded random draws for the paged-attention workloads.

Every array here is a function of an integer seed and a shape. Keys and values
are drawn per (seed, sequence, K-or-V) stream, one token row after another, so
token t of a sequence has the same values whatever the sequence's final length
and whatever block size or placement later stores it.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "LLAMA3_8B_BATCH_LENGTHS",
    "normal_f32",
    "kv_rows",
    "queries",
    "new_token_kv",
    "round_to_bf16",
    "lognormal_lengths",
    "uniform_lengths",
    "block_permutation",
]

# The eight request lengths of the worked example on "What is paged attention in
# vLLM, and why does it matter?" (section "Worked example").
LLAMA3_8B_BATCH_LENGTHS = (128, 700, 1500, 300, 2900, 50, 4100, 900)


def normal_f32(seed, shape) -> np.ndarray:
    """Standard normal float32 draws from numpy's PCG64 stream for `seed`.

    `seed` may be an int or a tuple of ints (numpy SeedSequence entropy).
    """
    rng = np.random.default_rng(seed if isinstance(seed, int) else list(seed))
    return rng.standard_normal(size=shape, dtype=np.float32)


def kv_rows(seed: int, seq_index: int, num_tokens: int, num_kv_heads: int, head_dim: int):
    """K and V rows [num_tokens, num_kv_heads, head_dim] (float32) of one sequence.

    K and V come from separate streams, so the first t rows do not depend on
    num_tokens.
    """
    shape = (num_tokens, num_kv_heads, head_dim)
    return normal_f32((seed, seq_index, 0), shape), normal_f32((seed, seq_index, 1), shape)


def queries(seed: int, step: int, num_seqs: int, num_heads: int, head_dim: int) -> np.ndarray:
    """One decode query per sequence: [num_seqs, num_heads, head_dim] float32."""
    return normal_f32((seed, 1_000_000 + step, 2), (num_seqs, num_heads, head_dim))


def new_token_kv(seed: int, step: int, num_seqs: int, num_kv_heads: int, head_dim: int):
    """K and V of the one token each sequence appends at decode step `step`."""
    shape = (num_seqs, num_kv_heads, head_dim)
    return (normal_f32((seed, 2_000_000 + step, 0), shape),
            normal_f32((seed, 2_000_000 + step, 1), shape))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 array whose every value is exactly representable in bfloat16.

    Rounds to nearest even through torch's own float32 -> bfloat16 cast, so a
    later `torch.from_numpy(r).to(torch.bfloat16)` is exact and the float64
    upcast of `r` is exactly the stored cache value.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def lognormal_lengths(n: int, mean: float, sigma: float, lo: int, hi: int, seed: int) -> np.ndarray:
    """n lengths from a lognormal whose arithmetic mean before clipping is `mean`.

    mu = ln(mean) - sigma^2 / 2 makes E[exp(N(mu, sigma^2))] = mean. Values are
    rounded to integers and clipped to [lo, hi].
    """
    rng = np.random.default_rng(seed)
    mu = np.log(mean) - 0.5 * sigma * sigma
    x = rng.lognormal(mean=mu, sigma=sigma, size=n)
    return np.clip(np.rint(x), lo, hi).astype(np.int64)


def uniform_lengths(n: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """n integer lengths uniform on the closed range [lo, hi]."""
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=n).astype(np.int64)


def block_permutation(num_blocks: int, seed: int) -> np.ndarray:
    """A seeded permutation of the physical block ids 0..num_blocks-1 (int32).

    Used as the order in which a fresh pool hands out free blocks, which makes
    the physical placement of every sequence random.
    """
    rng = np.random.default_rng(seed)
    return rng.permutation(num_blocks).astype(np.int32)


def e4m3_scales(num_kv_heads: int):
    """Per-KV-head scales of an E4M3 cache for rows drawn from N(0, 1): around
    1/32, so |x| / scale reaches ~150 of the format's 448. K head 0 is exactly
    1/32 (the quantising division is exact there); every other scale is not a
    power of two, so the division rounds. Returns float32 (k_scale, v_scale)."""
    h = np.arange(num_kv_heads, dtype=np.float64)
    return ((1.0 + 0.37 * h) / 32.0).astype(np.float32), ((1.3 + 0.29 * h) / 32.0).astype(np.float32)
