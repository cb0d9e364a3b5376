"""Build paged decode workloads on the GPU through the library's public API and
compute the oracle's expected outputs from the same seeded rows.

The GPU side: PagedKVCache (native block manager + pa_copy_blocks +
pa_kv_append + pa_decode). The oracle side: float64 softmax attention over
each sequence's logically contiguous rows, straight from the generator; the
two share only the generator's arrays.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from oracle import attention as oatt
from oracle import quant as oquant
from workloads import synth

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}
PREFIX_STREAM = 100_000  # generator stream index of a shared prefix


def stored(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values exactly as the cache stores them."""
    return synth.round_to_bf16(x) if dtype == "bf16" else np.asarray(x, np.float32)


def tolerance(dtype: str):
    """(abs, rel): |gpu - ref| <= abs + rel * |ref| elementwise."""
    return (2e-2, 1e-2) if dtype == "bf16" else (1e-5, 0.0)


def assert_close(got, ref, dtype: str, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    atol, rtol = tolerance(dtype)
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert not np.isnan(got).any(), f"{what}: NaN in GPU output"
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"max abs err {err.max():.3e}")
    return float(err.max())


FP8 = "fp8_e4m3"
NAN_BITS = {torch.float32: (torch.int32, 0x7FC00000), torch.bfloat16: (torch.int16, 0x7FC0),
            torch.uint8: (torch.uint8, 0x7F)}


def e4m3_codes(rows: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Oracle E4M3 codes of rows [n, Hkv, d] with one scale per KV head."""
    return np.stack([oquant.quantize(rows[:, h], scales[h]) for h in range(rows.shape[1])], axis=1)


def e4m3_values(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Oracle cache values (float64) of codes [n, Hkv, d]."""
    return np.stack([oquant.dequantize(codes[:, h], scales[h]) for h in range(codes.shape[1])],
                    axis=1)


def poison(t: torch.Tensor) -> None:
    """Fill a cache with NaN bit patterns: any read of a row that was never
    written (or of a slot past a sequence's end) shows up as NaN."""
    view, bits = NAN_BITS[t.dtype]
    t.view(view).fill_(bits)


@dataclass
class Case:
    cache: object          # PagedKVCache
    seqs: list             # sequence ids in batch order
    rows_k: dict           # kept sequences: float32 [L_s + 1, Hkv, d] (stored values)
    rows_v: dict
    q: np.ndarray          # float32 [S, Hq, d] (stored values)
    out: torch.Tensor      # GPU output of the decode step
    scale: float
    dtype: str
    k_scale: np.ndarray = None   # E4M3 caches: per-KV-head scales
    v_scale: np.ndarray = None


def sequence_rows(wl, s, n, prefix_rows=None):
    """Rows of sequence s: the shared prefix (if any) then its own tokens, n in total."""
    if prefix_rows is None:
        k, v = synth.kv_rows(wl.value_seed, s, n, wl.num_kv_heads, wl.head_dim)
        return stored(k, wl.dtype), stored(v, wl.dtype)
    pk, pv = prefix_rows
    own = n - len(pk)
    k, v = synth.kv_rows(wl.value_seed, s, own, wl.num_kv_heads, wl.head_dim)
    return (np.concatenate([pk, stored(k, wl.dtype)]), np.concatenate([pv, stored(v, wl.dtype)]))


def stage_rows(wl, device="cuda", keep=None):
    """Every sequence's rows (context + the decode step's token) on the device,
    sequence-major [sum(L_s + 1), Hkv, d] in the cache dtype, plus host float32
    copies of the sequences in `keep` (all when None)."""
    tdt = TORCH_DTYPES[wl.dtype]
    n = [L + 1 for L in wl.context_lens]
    offs = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    shape = (int(offs[-1]), wl.num_kv_heads, wl.head_dim)
    sk = torch.empty(shape, dtype=tdt, device=device)
    sv = torch.empty(shape, dtype=tdt, device=device)
    prefix = None
    if wl.shared_prefix:
        pk, pv = synth.kv_rows(wl.value_seed, PREFIX_STREAM, wl.shared_prefix, wl.num_kv_heads,
                               wl.head_dim)
        prefix = (stored(pk, wl.dtype), stored(pv, wl.dtype))
    keep_k, keep_v = {}, {}
    for s in range(wl.num_seqs):
        k, v = sequence_rows(wl, s, n[s], prefix)
        sk[offs[s]:offs[s + 1]] = torch.from_numpy(k).to(device=device, dtype=tdt)
        sv[offs[s]:offs[s + 1]] = torch.from_numpy(v).to(device=device, dtype=tdt)
        if keep is None or s in keep:
            keep_k[s], keep_v[s] = k, v
    return sk, sv, offs, keep_k, keep_v


def build_case(wl, device="cuda", free_order=None, partition_size=None, share_prefix=True,
               staged=None, keep=None, fused=True, poisoned=False, planned=True):
    """Prefill every sequence, then one decode step (append one token each + attend).
    E4M3 caches (wl.kv_dtype): rows are quantised on the device; the kept rows
    are replaced by the oracle's cache values of the same rows. planned: the
    step's decode on the work-list grid (bf16 and E4M3 caches; the cache's
    default), else on the plain (partition, sequence) grid."""
    from paged_kv_cache_345_b200.cache import PagedKVCache

    bs = wl.block_size
    if wl.shared_prefix and not share_prefix:
        # the same tokens stored unshared need a block per sequence per 16 tokens
        import dataclasses
        wl = dataclasses.replace(wl, num_blocks=sum(-(-(n + 1) // bs) for n in wl.context_lens) + 64)
    if free_order is None:
        free_order = synth.block_permutation(wl.num_blocks, wl.placement_seed)
    max_blocks = max(-(-(n + 1) // bs) for n in wl.context_lens)
    fp8 = wl.cache_dtype == FP8
    ks, vs = synth.e4m3_scales(wl.num_kv_heads) if fp8 else (None, None)
    cache = PagedKVCache(wl.num_blocks, bs, wl.num_kv_heads, wl.head_dim, wl.cache_dtype, device,
                         max_blocks_per_seq=max_blocks, free_order=free_order,
                         k_scale=None if ks is None else torch.from_numpy(ks),
                         v_scale=None if vs is None else torch.from_numpy(vs))
    if poisoned:
        poison(cache.k_cache)
        poison(cache.v_cache)
    tdt = TORCH_DTYPES[wl.dtype]
    sk, sv, offs, rows_k, rows_v = staged if staged is not None else stage_rows(wl, device, keep)

    # fragment the pool: ghosts take blocks, every other ghost returns them
    ghosts = [cache.add_sequence() for _ in wl.ghost_lens]
    if ghosts:
        cache.bm.append_slots(ghosts, list(wl.ghost_lens))
        for i in range(0, len(ghosts), 2):
            cache.free(ghosts[i])

    shared = bool(wl.shared_prefix) and share_prefix
    if shared:
        parent = cache.add_sequence()
        cache.write([parent], [wl.shared_prefix], sk[:wl.shared_prefix], sv[:wl.shared_prefix])
        seqs = [parent] + [cache.fork(parent) for _ in range(wl.num_seqs - 1)]
    else:
        seqs = [cache.add_sequence() for _ in range(wl.num_seqs)]
    start = wl.shared_prefix if shared else 0
    lens = wl.context_lens
    counts = [n - start for n in lens]
    if sum(counts):
        idx = torch.from_numpy(np.concatenate(
            [np.arange(offs[s] + start, offs[s] + n) for s, n in enumerate(lens)])).to(device)
        cache.write(seqs, counts, sk.index_select(0, idx), sv.index_select(0, idx))
    q = stored(synth.queries(wl.value_seed, 0, wl.num_seqs, wl.num_heads, wl.head_dim), wl.dtype)
    last = torch.from_numpy(np.asarray([offs[s] + n for s, n in enumerate(lens)])).to(device)
    k_new, v_new = sk.index_select(0, last), sv.index_select(0, last)
    ps = wl.partition_size if partition_size is None else partition_size
    qd = torch.from_numpy(q).to(device=device, dtype=tdt)
    out = cache.decode_step(qd, k_new, v_new, seqs, wl.scale, ps, fused=fused, planned=planned)
    torch.cuda.synchronize()
    if fp8:
        rows_k = {s: e4m3_values(e4m3_codes(r, ks), ks) for s, r in rows_k.items()}
        rows_v = {s: e4m3_values(e4m3_codes(r, vs), vs) for s, r in rows_v.items()}
    return Case(cache, seqs, rows_k, rows_v, q, out, wl.scale, wl.dtype, ks, vs)


def expected_one(case: Case, s: int, j: int) -> np.ndarray:
    group = case.q.shape[1] // case.rows_k[s].shape[1]
    h = oatt.kv_head_of(j, group)
    return oatt.softmax_attention(case.q[s, j], case.rows_k[s][:, h, :], case.rows_v[s][:, h, :],
                                  case.scale)


def expected_all(case: Case) -> np.ndarray:
    S, Hq, D = case.q.shape
    assert len(case.rows_k) == S, "expected_all needs every sequence's rows"
    ref = np.zeros((S, Hq, D))
    for s in range(S):
        for j in range(Hq):
            ref[s, j] = expected_one(case, s, j)
    return ref


def gpu_out(case: Case) -> np.ndarray:
    return case.out.float().cpu().numpy()
