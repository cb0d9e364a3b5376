"""PagedKVCache: one layer's paged K/V cache driven through the C ABI.

Holds the device caches [num_blocks, block_size, Hkv, d], the native block
manager (free list, reference counts, tables) and a reusable decode
workspace. Each method marshals arguments and calls libpa.so:

  write(seq_ids, counts, k_rows, v_rows)  reserve slots (native), copy shared
      tail blocks first when needed (pa_copy_blocks), then scatter the rows
      (pa_kv_append). Serves both prefill (many tokens) and decode (one token).
  prefill(q, k_rows, v_rows, seq_ids, counts)  append each sequence's chunk
      of counts[i] tokens (write), then causal attention of the chunk's query
      rows over the whole context (pa_prefill_planned on the work items
      pa_prefill_plan lists from the host lengths; planned=False: pa_prefill,
      same result); bf16 caches.
  decode(q, seq_ids)  block tables to the device, then pa_decode (bf16 and
      E4M3 caches: pa_decode_planned on the grid pa_decode_plan lists from the
      host lengths, which the block manager knows; planned=False: the plain
      grid, same result).
  decode_step(q, k_new, v_new, seq_ids)  one decode step: reserve each sequence's
      next slot (native; shared tail blocks copied first), then pa_decode_append
      writes the new K/V rows and attends in one launch (fused=False: separate
      pa_kv_append and pa_decode calls, same result); planned grid as decode. shared_prefix=n: the
      sequences' first n tokens (a multiple of the block size) sit in the same
      blocks (forked from one parent): pa_decode_shared_prefix attends them once
      for the batch, beside the decode of each sequence's own tokens; bf16.

dtype "fp8_e4m3": the caches hold uint8 E4M3 codes with one float32 scale per
KV head (k_scale, v_scale); rows come in as bfloat16 and are quantised on the
device (pa_kv_append_fp8 / pa_decode_append_fp8), decode reads the codes
(pa_decode_fp8).

"Paged Attention" (klaylearn.com glossary), definition: prefill allocates and
fills blocks, decode appends into the tail block or triggers an allocation,
finished requests return their blocks to the free list.
"""

from __future__ import annotations

import functools

import numpy as np
import torch

from . import (BlockManager, pa_copy_blocks, pa_decode, pa_decode_append, pa_decode_append_fp8,
               pa_decode_fp8, pa_decode_partition_size, pa_decode_plan, pa_decode_planned,
               pa_decode_shared_prefix,
               pa_decode_shared_prefix_workspace_bytes, pa_decode_workspace_bytes, pa_kv_append,
               pa_kv_append_fp8, pa_prefill, pa_prefill_plan)

_TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8_e4m3": torch.uint8}


def _on_stream(method):
    """Run the method with the cache's stream current (when it has one), so the
    tables' host-to-device copies and the buffers it allocates are ordered with
    the kernels it launches on that stream."""
    @functools.wraps(method)
    def run(self, *args, **kwargs):
        with torch.cuda.stream(self.stream):
            return method(self, *args, **kwargs)
    return run


class PagedKVCache:
    def __init__(self, num_blocks: int, block_size: int, num_kv_heads: int, head_dim: int,
                 dtype="bf16", device="cuda", max_blocks_per_seq: int | None = None,
                 free_order=None, stream=None, k_scale=None, v_scale=None):
        self.dtype = _TORCH_DTYPES.get(dtype, dtype)
        self.fp8 = self.dtype == torch.uint8
        if self.fp8:
            def per_head(x):
                x = torch.ones(num_kv_heads) if x is None else torch.as_tensor(x)
                return x.to(dtype=torch.float32).expand(num_kv_heads).contiguous().to(device)
            self.k_scale, self.v_scale = per_head(k_scale), per_head(v_scale)
        self.device = torch.device(device)
        self.block_size = block_size
        self.num_blocks = num_blocks
        self.num_kv_heads = num_kv_heads
        self.head_dim = head_dim
        self.max_blocks_per_seq = max_blocks_per_seq or num_blocks
        shape = (num_blocks, block_size, num_kv_heads, head_dim)
        self.k_cache = torch.zeros(shape, dtype=self.dtype, device=self.device)
        self.v_cache = torch.zeros(shape, dtype=self.dtype, device=self.device)
        self.bm = BlockManager(num_blocks, block_size)
        if free_order is not None:
            self.bm.allocator.set_free_order(free_order)
        self.stream = stream
        self._workspace = torch.zeros(0, dtype=torch.uint8, device=self.device)

    # ------------------------------------------------------------ sequences
    def add_sequence(self) -> int:
        return self.bm.add_seq()

    def fork(self, seq: int) -> int:
        return self.bm.fork(seq)

    def free(self, seq: int) -> None:
        self.bm.free_seq(seq)

    def context_len(self, seq: int) -> int:
        return self.bm.seq_len(seq)

    # --------------------------------------------------------------- writes
    def _to_device(self, a: np.ndarray):
        return torch.from_numpy(np.ascontiguousarray(a)).pin_memory().to(self.device,
                                                                          non_blocking=True)

    @_on_stream
    def write(self, seq_ids, counts, k_rows, v_rows):
        """Append counts[i] tokens to seq_ids[i]; k_rows/v_rows are [sum(counts), Hkv, d]
        device tensors in sequence order. Returns the host slot mapping."""
        slots, cows = self.bm.append_slots(seq_ids, counts)
        if len(cows):
            pa_copy_blocks(self.k_cache, self.v_cache, self._to_device(cows), stream=self.stream)
        if len(slots):
            if self.fp8:
                pa_kv_append_fp8(k_rows, v_rows, self._to_device(slots), self.k_cache,
                                 self.v_cache, self.k_scale, self.v_scale, stream=self.stream)
            else:
                pa_kv_append(k_rows, v_rows, self._to_device(slots), self.k_cache, self.v_cache,
                             stream=self.stream)
        return slots

    # -------------------------------------------------------------- prefill
    @_on_stream
    def prefill(self, q, k_rows, v_rows, seq_ids, counts, scale: float | None = None, out=None,
                planned: bool = True):
        """Append counts[i] tokens to seq_ids[i] and attend them causally: q, k_rows,
        v_rows are [sum(counts), H, d] device tensors in sequence order. planned:
        the work items listed on the host (pa_prefill_plan, pa_prefill_planned);
        else each CTA finds its own (pa_prefill). Same result."""
        if self.fp8:
            raise NotImplementedError("pa_prefill reads bf16 caches")
        self.write(seq_ids, counts, k_rows, v_rows)
        mbps = max(1, max(self.bm.seq_num_blocks(s) for s in seq_ids))
        tables, lens = self.bm.block_tables(seq_ids, mbps)
        block_tables, context_lens = self._to_device(tables), self._to_device(lens)
        qs = np.concatenate([[0], np.cumsum(np.asarray(counts, dtype=np.int64))]).astype(np.int32)
        out = torch.empty_like(q) if out is None else out
        scale = 1.0 / float(np.sqrt(self.head_dim)) if scale is None else scale
        work = None
        if planned and len(seq_ids) and int(qs[-1]) > 0:
            work = self._to_device(pa_prefill_plan(qs, lens, q.shape[1], self.num_kv_heads))
        pa_prefill(out, q, self.k_cache, self.v_cache, block_tables, context_lens,
                   self._to_device(qs), int(max(counts, default=0)), scale, stream=self.stream,
                   work=work)
        return out

    # --------------------------------------------------------------- decode
    @_on_stream
    def tables(self, seq_ids, max_blocks_per_seq: int | None = None):
        """(block_tables, context_lens, max_context_len) of the sequences: device
        int32 tensors and the host maximum."""
        mbps = max_blocks_per_seq or max(1, max(self.bm.seq_num_blocks(s) for s in seq_ids))
        tables, lens = self.bm.block_tables(seq_ids, mbps)
        return self._to_device(tables), self._to_device(lens), int(lens.max(initial=0))

    def _planned_decode(self, out, q, k_new, v_new, seq_ids, scale, partition_size):
        """Tables, lengths and the work list of the host lengths to the device,
        then pa_decode_planned (with the append when k_new is given)."""
        num_seqs, num_heads, _ = q.shape
        mbps = max(1, max(self.bm.seq_num_blocks(s) for s in seq_ids))
        tables, lens = self.bm.block_tables(seq_ids, mbps)
        max_len = int(lens.max(initial=0))
        if partition_size == 0:
            partition_size = pa_decode_partition_size(num_seqs, self.num_kv_heads, max_len)
        work = pa_decode_plan(lens, partition_size)
        ws = self.workspace(num_seqs, num_heads, max_len, partition_size)
        sc = dict(k_scale=self.k_scale, v_scale=self.v_scale) if self.fp8 else {}
        pa_decode_planned(out, q, self.k_cache, self.v_cache, self._to_device(tables),
                          self._to_device(lens), self._to_device(work), max_len, scale,
                          partition_size, ws, k_new=k_new, v_new=v_new, stream=self.stream, **sc)
        return out

    @_on_stream
    def _decode_step_shared(self, q, k_new, v_new, seq_ids, scale, partition_size, out,
                            prefix_len):
        _, cows = self.bm.append_slots(seq_ids, [1] * len(seq_ids))
        if len(cows):
            pa_copy_blocks(self.k_cache, self.v_cache, self._to_device(cows), stream=self.stream)
        num_seqs, num_heads, _ = q.shape
        block_tables, context_lens, max_len = self.tables(seq_ids)
        out = torch.empty_like(q) if out is None else out
        scale = 1.0 / float(np.sqrt(self.head_dim)) if scale is None else scale
        need = pa_decode_shared_prefix_workspace_bytes(num_seqs, num_heads, self.num_kv_heads,
                                                       self.head_dim, prefix_len, max_len,
                                                       partition_size)
        if need > self._workspace.numel():
            self._workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
        pa_decode_shared_prefix(out, q, k_new, v_new, self.k_cache, self.v_cache, block_tables,
                                context_lens, prefix_len, max_len, scale, partition_size,
                                self._workspace, stream=self.stream)
        return out

    def workspace(self, num_seqs, num_heads, max_context_len, partition_size=0):
        need = pa_decode_workspace_bytes(num_seqs, num_heads, self.num_kv_heads, self.head_dim,
                                         max_context_len, partition_size)
        if need > self._workspace.numel():
            self._workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._workspace if need > 0 else None

    @_on_stream
    def decode(self, q, seq_ids, scale: float | None = None, partition_size: int = 0, out=None,
               planned: bool = True):
        if planned and self.k_cache.dtype != torch.float32 and len(seq_ids):
            out = torch.empty_like(q) if out is None else out
            scale = 1.0 / float(np.sqrt(self.head_dim)) if scale is None else scale
            return self._planned_decode(out, q, None, None, seq_ids, scale, partition_size)
        num_seqs, num_heads, _ = q.shape
        block_tables, context_lens, max_len = self.tables(seq_ids)
        if partition_size == 0:
            partition_size = pa_decode_partition_size(num_seqs, self.num_kv_heads, max_len)
        out = torch.empty_like(q) if out is None else out
        scale = 1.0 / float(np.sqrt(self.head_dim)) if scale is None else scale
        ws = self.workspace(num_seqs, num_heads, max_len, partition_size)
        if self.fp8:
            pa_decode_fp8(out, q, self.k_cache, self.v_cache, self.k_scale, self.v_scale,
                          block_tables, context_lens, max_len, scale, partition_size, ws,
                          stream=self.stream)
        else:
            pa_decode(out, q, self.k_cache, self.v_cache, block_tables, context_lens, max_len,
                      scale, partition_size, ws, stream=self.stream)
        return out

    @_on_stream
    def decode_step(self, q, k_new, v_new, seq_ids, scale=None, partition_size: int = 0,
                    out=None, fused: bool = True, shared_prefix: int = 0, planned: bool = True):
        if shared_prefix:
            if self.fp8 or not fused:
                raise ValueError("shared_prefix: a bf16 cache and the fused step")
            return self._decode_step_shared(q, k_new, v_new, seq_ids, scale, partition_size, out,
                                            shared_prefix)
        if not fused:
            self.write(seq_ids, [1] * len(seq_ids), k_new, v_new)
            return self.decode(q, seq_ids, scale, partition_size, out, planned)
        _, cows = self.bm.append_slots(seq_ids, [1] * len(seq_ids))
        if len(cows):
            pa_copy_blocks(self.k_cache, self.v_cache, self._to_device(cows), stream=self.stream)
        if planned and self.k_cache.dtype != torch.float32 and len(seq_ids):
            out = torch.empty_like(q) if out is None else out
            scale = 1.0 / float(np.sqrt(self.head_dim)) if scale is None else scale
            return self._planned_decode(out, q, k_new, v_new, seq_ids, scale, partition_size)
        num_seqs, num_heads, _ = q.shape
        block_tables, context_lens, max_len = self.tables(seq_ids)
        if partition_size == 0:
            partition_size = pa_decode_partition_size(num_seqs, self.num_kv_heads, max_len)
        out = torch.empty_like(q) if out is None else out
        scale = 1.0 / float(np.sqrt(self.head_dim)) if scale is None else scale
        ws = self.workspace(num_seqs, num_heads, max_len, partition_size)
        if self.fp8:
            pa_decode_append_fp8(out, q, k_new, v_new, self.k_cache, self.v_cache, self.k_scale,
                                 self.v_scale, block_tables, context_lens, max_len, scale,
                                 partition_size, ws, stream=self.stream)
        else:
            pa_decode_append(out, q, k_new, v_new, self.k_cache, self.v_cache, block_tables,
                             context_lens, max_len, scale, partition_size, ws,
                             stream=self.stream)
        return out
