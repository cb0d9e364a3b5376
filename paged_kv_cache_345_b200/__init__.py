"""Paged KV cache decode path for B200 (sm_100a): Python binding of libpa.so.

This module only marshals arguments: it turns torch tensors and numpy arrays
into pointers and sizes and calls the C ABI declared in include/pa.h. Every
step of the hot path runs in the library's CUDA kernels or its C++ block
manager. There is no CPU fallback: importing this package fails if libpa.so
has not been built (python paged_kv_cache_345_b200/build.py).

Entry points (same names as the C ABI):
  pa_kv_append     write new tokens' K/V rows into their slots
  pa_copy_blocks   copy-on-write of shared blocks
  pa_swap_blocks   copy blocks between device and (pinned) host pools
  pa_decode        paged decode attention (split-K over partitions)
  pa_decode_append one decode step: append each newest token, then attend
  pa_prefill       causal (chunked) prefill attention over the paged context
  pa_kv_append_fp8, pa_decode_fp8, pa_decode_append_fp8
                   the same over 8-bit E4M3 caches with per-KV-head scales
  pa_decode_plan, pa_decode_planned
                   host work list of the (sequence, partition) pairs that hold
                   tokens, and the decode (bf16 or E4M3) on that grid
  pa_prefill_plan, pa_prefill_planned
                   host work list of the prefill's items in the kernel's
                   longest-first order, and the prefill on it
  BlockManager     host free list + reference counts + block tables
"""

from __future__ import annotations

import contextlib
import ctypes
import os

import numpy as np

__all__ = [
    "PagedAttentionError", "PA_OK", "PA_ERR_INVALID", "PA_ERR_UNSUPPORTED", "PA_ERR_CUDA",
    "PA_ERR_NO_BLOCKS", "PA_ERR_DEVICE_CHECK", "PA_DEVERR_SLOT", "PA_DEVERR_BLOCK_ID",
    "PA_DEVERR_CONTEXT", "PA_DEVERR_COPY_PAIR", "PA_DEVERR_TIMEOUT", "PA_DEVERR_PLAN",
    "lib_path", "pa_kv_append", "pa_copy_blocks", "pa_swap_blocks", "pa_decode",
    "pa_decode_append", "pa_kv_append_fp8", "pa_decode_fp8", "pa_decode_append_fp8", "PA_FP8_E4M3",
    "pa_prefill",
    "pa_decode_workspace_bytes",
    "pa_decode_partition_size", "pa_device_errors", "Allocator", "BlockManager",
    "pa_set_decode_options", "PA_DECODE_EARLY_CACHE_READS", "decode_options",
    "pa_decode_contiguous", "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_bytes",
    "pa_decode_plan", "pa_decode_planned", "pa_prefill_plan", "pa_prefill_planned",
]

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_NO_BLOCKS, PA_ERR_DEVICE_CHECK = \
    range(6)
PA_F32, PA_BF16, PA_FP8_E4M3 = 0, 1, 2
PA_DEVERR_SLOT, PA_DEVERR_BLOCK_ID, PA_DEVERR_CONTEXT, PA_DEVERR_COPY_PAIR, PA_DEVERR_TIMEOUT = \
    0x1, 0x2, 0x4, 0x8, 0x10
PA_DEVERR_PLAN = 0x20

lib_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")
if not os.path.exists(lib_path):
    raise ImportError(
        f"{lib_path} is missing: build the CUDA library first "
        "(python paged_kv_cache_345_b200/build.py). There is no CPU fallback.")
_lib = ctypes.CDLL(lib_path)

_vp, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, \
    ctypes.c_size_t
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def _sig(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


_sig("pa_kv_append", _i32, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp)
_sig("pa_kv_append_fp8", _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp)
_sig("pa_copy_blocks", _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp)
_sig("pa_swap_blocks", _i32, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _vp)
_sig("pa_decode_partition_size", _i32, _i32, _i32, _i32)
_sig("pa_set_decode_options", ctypes.c_uint, ctypes.c_uint)
_sig("pa_decode_shared_prefix_workspace_bytes", _sz, _i32, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("pa_decode_shared_prefix", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
     _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _i32, _vp)
_sig("pa_decode_contiguous", _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
     _f32, _i32, _vp, _sz, _i32, _vp)
_sig("pa_decode_workspace_bytes", _sz, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("pa_decode", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
     _i32, _f32, _i32, _vp, _sz, _i32, _vp)
_sig("pa_decode_append", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _i32, _f32, _i32, _vp, _sz, _i32, _vp)
_sig("pa_decode_fp8", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp)
_sig("pa_decode_append_fp8", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
     _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp)
_sig("pa_decode_plan", _i32, _i32p, _i32, _i32, _i32p, _i32, ctypes.POINTER(ctypes.c_int))
_sig("pa_decode_planned", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
     _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _i32, _vp)
_sig("pa_prefill_plan", _i32, _i32p, _i32p, _i32, _i32, _i32, _i32p, _i32,
     ctypes.POINTER(ctypes.c_int))
_sig("pa_prefill_planned", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
     _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp)
_sig("pa_prefill", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _f32, _i32, _vp)
_sig("pa_decode_noalloc", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _f32, _i32, _i32, _vp)
_sig("pa_decode_noalloc_scratch_bytes", _sz)
_sig("pa_device_errors", _i32, _vp, ctypes.POINTER(ctypes.c_uint))
_sig("pa_last_error", ctypes.c_char_p)
_sig("pa_status_string", ctypes.c_char_p, _i32)
_sig("pa_alloc_create", _vp, _i32)
_sig("pa_alloc_destroy", None, _vp)
_sig("pa_alloc_block", _i32, _vp, _i32p)
_sig("pa_incref", _i32, _vp, ctypes.c_int32)
_sig("pa_decref", _i32, _vp, ctypes.c_int32)
_sig("pa_refcount", _i32, _vp, ctypes.c_int32)
_sig("pa_num_free", _i32, _vp)
_sig("pa_num_blocks", _i32, _vp)
_sig("pa_alloc_set_free_order", _i32, _vp, _i32p, _i32)
_sig("pa_bm_create", _vp, _i32, _i32)
_sig("pa_bm_destroy", None, _vp)
_sig("pa_bm_allocator", _vp, _vp)
_sig("pa_bm_block_size", _i32, _vp)
_sig("pa_bm_add_seq", _i32, _vp, _i32p)
_sig("pa_bm_fork", _i32, _vp, ctypes.c_int32, _i32p)
_sig("pa_bm_free_seq", _i32, _vp, ctypes.c_int32)
_sig("pa_bm_seq_len", _i32, _vp, ctypes.c_int32)
_sig("pa_bm_seq_num_blocks", _i32, _vp, ctypes.c_int32)
_sig("pa_bm_append_slots", _i32, _vp, _i32p, _i32p, _i32, _i64p, _i64p, _i32,
     ctypes.POINTER(ctypes.c_int))
_sig("pa_bm_block_tables", _i32, _vp, _i32p, _i32, _i32p, _i32, _i32p)

EXPORTED = (
    "pa_kv_append", "pa_kv_append_fp8", "pa_copy_blocks", "pa_swap_blocks",
    "pa_decode_partition_size", "pa_set_decode_options", "pa_decode_workspace_bytes",
    "pa_decode", "pa_decode_append", "pa_decode_contiguous", "pa_decode_shared_prefix",
    "pa_decode_shared_prefix_workspace_bytes",
    "pa_decode_fp8", "pa_decode_append_fp8", "pa_decode_plan", "pa_decode_planned",
    "pa_prefill_plan", "pa_prefill_planned",
    "pa_prefill", "pa_decode_noalloc", "pa_decode_noalloc_scratch_bytes", "pa_device_errors",
    "pa_last_error", "pa_status_string", "pa_alloc_create",
    "pa_alloc_destroy", "pa_alloc_block", "pa_incref", "pa_decref", "pa_refcount", "pa_num_free",
    "pa_num_blocks", "pa_alloc_set_free_order", "pa_bm_create", "pa_bm_destroy",
    "pa_bm_allocator", "pa_bm_block_size", "pa_bm_add_seq", "pa_bm_fork", "pa_bm_free_seq",
    "pa_bm_seq_len", "pa_bm_seq_num_blocks", "pa_bm_append_slots", "pa_bm_block_tables",
)


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        name = _lib.pa_status_string(status).decode()
        super().__init__(f"{name}: {message}")


def _check(status: int) -> None:
    if status != PA_OK:
        raise PagedAttentionError(status, _lib.pa_last_error().decode())


# ------------------------------------------------------------ tensor helpers

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return PA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype} (float32, bfloat16, or uint8 E4M3 codes)")


def _is_fp8(t) -> bool:
    torch = _torch()
    return t.dtype in (torch.uint8, torch.float8_e4m3fn)


def _dev_ptr(t, name, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _on_device(tensors, stream):
    """(device guard, stream pointer) for one call. Its CUDA tensors must all be
    on one device (a kernel given another GPU's pointer would read outside its
    own memory), an explicit stream must belong to that device, and the call
    runs with that device current. CPU tensors (pinned host pools) are skipped."""
    torch = _torch()
    devs = {t.device for t in tensors if t is not None and t.is_cuda}
    if len(devs) > 1:
        raise ValueError("tensors of one call are on several devices: " +
                         ", ".join(sorted(str(d) for d in devs)))
    dev = devs.pop() if devs else None
    if dev is not None and stream is not None and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, the tensors on {dev}")
    guard = torch.cuda.device(dev) if dev is not None else contextlib.nullcontext()
    return guard, _stream(stream, dev)


# ---------------------------------------------------------------- kernels

def pa_kv_append(k_new, v_new, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """Write row i of k_new/v_new [N, Hkv, d] at flat slot slot_mapping[i] (int64) of the caches."""
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    if tuple(k_new.shape[1:]) != (hkv, d) or k_new.shape != v_new.shape:
        raise ValueError("k_new/v_new must be [N, num_kv_heads, head_dim] matching the cache")
    if v_cache.shape != k_cache.shape or slot_mapping.shape != (k_new.shape[0],):
        raise ValueError("cache or slot_mapping shape mismatch")
    dt = k_cache.dtype
    guard, st = _on_device((k_new, v_new, slot_mapping, k_cache, v_cache), stream)
    with guard:
        _check(_lib.pa_kv_append(
            _dev_ptr(k_new, "k_new", dt), _dev_ptr(v_new, "v_new", dt),
            _dev_ptr(slot_mapping, "slot_mapping", torch.int64), k_new.shape[0],
            _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache", dt), nb, bs, hkv, d,
            _dtype_code(k_cache), st))


def pa_kv_append_fp8(k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale,
                     stream=None) -> None:
    """Quantising append into E4M3 caches (uint8 codes [nb, bs, Hkv, d]): row i of
    k_new/v_new (bfloat16 [N, Hkv, d]) goes to flat slot slot_mapping[i] as the codes
    of value / scale[head]; k_scale/v_scale are float32 [Hkv] device tensors."""
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    if tuple(k_new.shape[1:]) != (hkv, d) or k_new.shape != v_new.shape:
        raise ValueError("k_new/v_new must be [N, num_kv_heads, head_dim] matching the cache")
    if v_cache.shape != k_cache.shape or slot_mapping.shape != (k_new.shape[0],):
        raise ValueError("cache or slot_mapping shape mismatch")
    if not (_is_fp8(k_cache) and _is_fp8(v_cache)):
        raise TypeError("caches must hold E4M3 codes (uint8 or float8_e4m3fn)")
    if k_scale.shape != (hkv,) or v_scale.shape != (hkv,):
        raise ValueError("k_scale/v_scale must be [num_kv_heads]")
    guard, st = _on_device((k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale),
                           stream)
    with guard:
        _check(_lib.pa_kv_append_fp8(
            _dev_ptr(k_new, "k_new", torch.bfloat16), _dev_ptr(v_new, "v_new", torch.bfloat16),
            _dev_ptr(slot_mapping, "slot_mapping", torch.int64), k_new.shape[0],
            _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
            _dev_ptr(k_scale, "k_scale", torch.float32),
            _dev_ptr(v_scale, "v_scale", torch.float32), nb, bs, hkv, d, st))


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None) -> None:
    """block dst := block src for each row (src, dst) of block_mapping [n, 2] (int64, device)."""
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    if block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be [num_pairs, 2]")
    guard, st = _on_device((k_cache, v_cache, block_mapping), stream)
    with guard:
        _check(_lib.pa_copy_blocks(
            _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache", k_cache.dtype),
            _dev_ptr(block_mapping, "block_mapping", torch.int64), block_mapping.shape[0], nb,
            bs, hkv, d, _dtype_code(k_cache), st))


def _mapped_ptr(t, name, dtype=None):
    """Pointer of a CUDA tensor, or of a page-locked CPU tensor (used by the
    device through unified addressing)."""
    if not t.is_cuda and not t.is_pinned():
        raise ValueError(f"{name} must be a CUDA tensor or page-locked (pinned) host memory")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, block_mapping, stream=None) -> None:
    """dst block := src block for each (src, dst) row of block_mapping [n, 2] (int64).
    Pools are [num_blocks, bs, Hkv, d], each on the device or in pinned host memory."""
    torch = _torch()
    snb, bs, hkv, d = src_k.shape
    dnb = dst_k.shape[0]
    if tuple(dst_k.shape[1:]) != (bs, hkv, d) or dst_v.shape != dst_k.shape or \
            src_v.shape != src_k.shape or dst_k.dtype != src_k.dtype:
        raise ValueError("pool shape / dtype mismatch")
    if block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be [num_pairs, 2]")
    dt = src_k.dtype
    guard, st = _on_device((dst_k, dst_v, src_k, src_v, block_mapping), stream)
    with guard:
        _check(_lib.pa_swap_blocks(
            _mapped_ptr(dst_k, "dst_k", dt), _mapped_ptr(dst_v, "dst_v", dt), dnb,
            _mapped_ptr(src_k, "src_k", dt), _mapped_ptr(src_v, "src_v", dt), snb,
            _mapped_ptr(block_mapping, "block_mapping", torch.int64), block_mapping.shape[0],
            bs, hkv, d, _dtype_code(src_k), st))


def pa_decode_partition_size(num_seqs: int, num_kv_heads: int, max_context_len: int) -> int:
    return int(_lib.pa_decode_partition_size(num_seqs, num_kv_heads, max_context_len))


PA_DECODE_EARLY_CACHE_READS = 0x1


def pa_set_decode_options(options: int) -> int:
    """Options of this host thread's later decode calls (PA_DECODE_EARLY_CACHE_READS);
    returns the previous options. See include/pa.h for when the option is safe."""
    return int(_lib.pa_set_decode_options(options))


class decode_options:
    """Context manager: `with decode_options(PA_DECODE_EARLY_CACHE_READS): ...`
    sets this thread's decode options and restores the previous ones on exit."""

    def __init__(self, options: int):
        self.options = options

    def __enter__(self):
        self.previous = pa_set_decode_options(self.options)
        return self

    def __exit__(self, *exc):
        pa_set_decode_options(self.previous)
        return False


def pa_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                              partition_size=0) -> int:
    return int(_lib.pa_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                              max_context_len, partition_size))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
              scale: float, partition_size: int = 0, workspace=None, stream=None) -> None:
    """Paged decode attention; see pa_decode in include/pa.h.

    out, q: [S, Hq, d]; caches: [num_blocks, bs, Hkv, d]; block_tables: int32
    [S, max_blocks_per_seq]; context_lens: int32 [S]; workspace: a uint8 CUDA
    tensor of at least pa_decode_workspace_bytes(...) bytes, or None when that is 0.
    """
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    s, hq, dq = q.shape
    if dq != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("q/out/cache shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    dt = k_cache.dtype
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev_ptr(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    guard, st = _on_device((out, q, k_cache, v_cache, block_tables, context_lens, workspace),
                           stream)
    with guard:
        _check(_lib.pa_decode(
            _dev_ptr(out, "out", dt), _dev_ptr(q, "q", dt), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache", dt), _dev_ptr(block_tables, "block_tables", torch.int32),
            _dev_ptr(context_lens, "context_lens", torch.int32), s, hq, hkv, d, bs, nb,
            block_tables.shape[1], int(max_context_len), float(scale), int(partition_size),
            ws_ptr, ws_bytes, _dtype_code(k_cache), st))


def pa_decode_shared_prefix_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                            prefix_len, max_context_len,
                                            partition_size=0) -> int:
    return int(_lib.pa_decode_shared_prefix_workspace_bytes(
        num_seqs, num_heads, num_kv_heads, head_dim, prefix_len, max_context_len, partition_size))


def pa_decode_shared_prefix(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens,
                            prefix_len: int, max_context_len: int, scale: float,
                            partition_size: int = 0, workspace=None, stream=None) -> None:
    """Decode (with the step's append when k_new / v_new are given) for sequences
    that all begin with the same prefix_len tokens in the same blocks; see
    pa_decode_shared_prefix in include/pa.h."""
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    s, hq, dq = q.shape
    if dq != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("q/out/cache shape mismatch")
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None and (k_new.shape != (s, hkv, d) or v_new.shape != k_new.shape):
        raise ValueError("k_new/v_new must be [S, num_kv_heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    if workspace is None:
        raise ValueError("pa_decode_shared_prefix needs a workspace")
    dt = k_cache.dtype
    guard, st = _on_device((out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens,
                            workspace), stream)
    with guard:
        _check(_lib.pa_decode_shared_prefix(
            _dev_ptr(out, "out", dt), _dev_ptr(q, "q", dt),
            None if k_new is None else _dev_ptr(k_new, "k_new", dt),
            None if v_new is None else _dev_ptr(v_new, "v_new", dt),
            _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache", dt),
            _dev_ptr(block_tables, "block_tables", torch.int32),
            _dev_ptr(context_lens, "context_lens", torch.int32), s, hq, hkv, d, bs, nb,
            block_tables.shape[1], int(prefix_len), int(max_context_len), float(scale),
            int(partition_size), _dev_ptr(workspace, "workspace"),
            workspace.numel() * workspace.element_size(), _dtype_code(k_cache), st))


def pa_decode_contiguous(out, q, k, v, context_lens, max_context_len: int, scale: float,
                         partition_size: int = 0, workspace=None, stream=None) -> None:
    """Decode attention over a contiguous cache (no block table); see
    pa_decode_contiguous in include/pa.h. k, v: [S, slab_len, Hkv, d] bf16."""
    torch = _torch()
    s, slab, hkv, d = k.shape
    _, hq, dq = q.shape
    if q.shape[0] != s or dq != d or out.shape != q.shape or v.shape != k.shape:
        raise ValueError("q/out/cache shape mismatch")
    if context_lens.shape != (s,):
        raise ValueError("context_lens must be [S]")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev_ptr(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    guard, st = _on_device((out, q, k, v, context_lens, workspace), stream)
    with guard:
        _check(_lib.pa_decode_contiguous(
            _dev_ptr(out, "out", k.dtype), _dev_ptr(q, "q", k.dtype), _dev_ptr(k, "k"),
            _dev_ptr(v, "v", k.dtype), _dev_ptr(context_lens, "context_lens", torch.int32), s, hq,
            hkv, d, slab, int(max_context_len), float(scale), int(partition_size), ws_ptr,
            ws_bytes, _dtype_code(k), st))


def pa_decode_append(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens,
                     max_context_len: int, scale: float, partition_size: int = 0, workspace=None,
                     stream=None) -> None:
    """Append each sequence's newest token (k_new / v_new [S, Hkv, d], at position
    context_lens[s] - 1 through the block table), then attend; see include/pa.h."""
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    s, hq, dq = q.shape
    if dq != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("q/out/cache shape mismatch")
    if k_new.shape != (s, hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("k_new/v_new must be [S, num_kv_heads, head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    dt = k_cache.dtype
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev_ptr(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    guard, st = _on_device((out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens,
                            workspace), stream)
    with guard:
        _check(_lib.pa_decode_append(
            _dev_ptr(out, "out", dt), _dev_ptr(q, "q", dt), _dev_ptr(k_new, "k_new", dt),
            _dev_ptr(v_new, "v_new", dt), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache", dt), _dev_ptr(block_tables, "block_tables", torch.int32),
            _dev_ptr(context_lens, "context_lens", torch.int32), s, hq, hkv, d, bs, nb,
            block_tables.shape[1], int(max_context_len), float(scale), int(partition_size),
            ws_ptr, ws_bytes, _dtype_code(k_cache), st))


def _fp8_decode_args(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                     workspace):
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    s, hq, dq = q.shape
    if dq != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("q/out/cache shape mismatch")
    if not (_is_fp8(k_cache) and _is_fp8(v_cache)):
        raise TypeError("caches must hold E4M3 codes (uint8 or float8_e4m3fn)")
    if k_scale.shape != (hkv,) or v_scale.shape != (hkv,):
        raise ValueError("k_scale/v_scale must be [num_kv_heads]")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev_ptr(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    return dict(
        k_cache=_dev_ptr(k_cache, "k_cache"), v_cache=_dev_ptr(v_cache, "v_cache"),
        k_scale=_dev_ptr(k_scale, "k_scale", torch.float32),
        v_scale=_dev_ptr(v_scale, "v_scale", torch.float32),
        tables=_dev_ptr(block_tables, "block_tables", torch.int32),
        lens=_dev_ptr(context_lens, "context_lens", torch.int32),
        sizes=(s, hq, hkv, d, bs, nb, block_tables.shape[1]), ws=(ws_ptr, ws_bytes))


def pa_decode_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                  max_context_len: int, scale: float, partition_size: int = 0, workspace=None,
                  stream=None) -> None:
    """pa_decode over E4M3 caches (uint8 codes, per-KV-head float32 scales);
    q and out are bfloat16 [S, Hq, d]. See pa_decode_fp8 in include/pa.h."""
    torch = _torch()
    a = _fp8_decode_args(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                         workspace)
    guard, st = _on_device((out, q, k_cache, v_cache, k_scale, v_scale, block_tables,
                            context_lens, workspace), stream)
    with guard:
        _check(_lib.pa_decode_fp8(
            _dev_ptr(out, "out", torch.bfloat16), _dev_ptr(q, "q", torch.bfloat16), a["k_cache"],
            a["v_cache"], a["k_scale"], a["v_scale"], a["tables"], a["lens"], *a["sizes"],
            int(max_context_len), float(scale), int(partition_size), *a["ws"], st))


def pa_decode_append_fp8(out, q, k_new, v_new, k_cache, v_cache, k_scale, v_scale, block_tables,
                         context_lens, max_context_len: int, scale: float,
                         partition_size: int = 0, workspace=None, stream=None) -> None:
    """pa_decode_append over E4M3 caches: quantise and write each sequence's newest
    token (k_new / v_new bfloat16 [S, Hkv, d]), then attend."""
    torch = _torch()
    a = _fp8_decode_args(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                         workspace)
    s, _, hkv, d = a["sizes"][:4]
    if k_new.shape != (s, hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("k_new/v_new must be [S, num_kv_heads, head_dim]")
    guard, st = _on_device((out, q, k_new, v_new, k_cache, v_cache, k_scale, v_scale,
                            block_tables, context_lens, workspace), stream)
    with guard:
        _check(_lib.pa_decode_append_fp8(
            _dev_ptr(out, "out", torch.bfloat16), _dev_ptr(q, "q", torch.bfloat16),
            _dev_ptr(k_new, "k_new", torch.bfloat16), _dev_ptr(v_new, "v_new", torch.bfloat16),
            a["k_cache"], a["v_cache"], a["k_scale"], a["v_scale"], a["tables"], a["lens"],
            *a["sizes"], int(max_context_len), float(scale), int(partition_size), *a["ws"], st))


def pa_decode_plan(context_lens, partition_size: int, out=None):
    """Work list of a planned decode from HOST context lengths (int32 [S]; the
    lengths the step's device context_lens will hold): int32 [num_items, 2],
    item = (sequence, partition | partitions of the sequence << 16), whole
    partitions first, then the ragged last ones, longest first. out: an int32
    [capacity, 2] array to write into (a view of its first rows is returned).
    See pa_decode_plan in include/pa.h."""
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    if lens.ndim != 1:
        raise ValueError("context_lens must be 1-D")
    ps = int(partition_size)
    if out is None:
        per = 1 if lens.size == 0 or ps <= 0 else max(1, -(-int(lens.max()) // ps))
        out = np.empty((max(1, lens.size * per), 2), dtype=np.int32)
    elif out.dtype != np.int32 or out.ndim != 2 or out.shape[1] != 2 or \
            not out.flags.c_contiguous:
        raise ValueError("out must be a C-contiguous int32 [capacity, 2] array")
    n = ctypes.c_int(0)
    _check(_lib.pa_decode_plan(lens.ctypes.data_as(_i32p), lens.size, ps,
                               out.ctypes.data_as(_i32p), out.shape[0], ctypes.byref(n)))
    return out[:n.value]


def pa_decode_planned(out, q, k_cache, v_cache, block_tables, context_lens, work,
                      max_context_len: int, scale: float, partition_size: int, workspace=None,
                      k_new=None, v_new=None, k_scale=None, v_scale=None, stream=None) -> None:
    """pa_decode (k_new / v_new None) or pa_decode_append on the grid of a work
    list (device int32 [num_items, 2] from pa_decode_plan with this
    partition_size), for bf16 caches or E4M3 caches (with k_scale / v_scale).
    See pa_decode_planned in include/pa.h."""
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    s, hq, dq = q.shape
    if dq != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("q/out/cache shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, max_blocks], context_lens [S]")
    if work.dim() != 2 or work.shape[1] != 2:
        raise ValueError("work must be [num_items, 2]")
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None and (k_new.shape != (s, hkv, d) or v_new.shape != k_new.shape):
        raise ValueError("k_new/v_new must be [S, num_kv_heads, head_dim]")
    fp8 = _is_fp8(k_cache)
    if fp8 != (k_scale is not None) or (k_scale is None) != (v_scale is None):
        raise ValueError("k_scale and v_scale go with (and only with) E4M3 caches")
    dt = torch.bfloat16
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev_ptr(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    opt = lambda t, n, ty=None: None if t is None else _dev_ptr(t, n, ty)  # noqa: E731
    guard, st = _on_device((out, q, k_new, v_new, k_cache, v_cache, k_scale, v_scale,
                            block_tables, context_lens, work, workspace), stream)
    with guard:
        _check(_lib.pa_decode_planned(
            _dev_ptr(out, "out", dt), _dev_ptr(q, "q", dt), opt(k_new, "k_new", dt),
            opt(v_new, "v_new", dt), _dev_ptr(k_cache, "k_cache"),
            _dev_ptr(v_cache, "v_cache", None if fp8 else dt),
            opt(k_scale, "k_scale", torch.float32), opt(v_scale, "v_scale", torch.float32),
            _dev_ptr(block_tables, "block_tables", torch.int32),
            _dev_ptr(context_lens, "context_lens", torch.int32),
            _dev_ptr(work, "work", torch.int32), work.shape[0], s, hq, hkv, d, bs, nb,
            block_tables.shape[1], int(max_context_len), float(scale), int(partition_size),
            ws_ptr, ws_bytes, _dtype_code(k_cache), st))


def pa_prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
               max_query_len: int, scale: float, stream=None, work=None) -> None:
    """Causal attention of each sequence's newest query rows over its paged context.

    q, out: bf16 [total_q, Hq, 128]; sequence s's rows are query_start[s] ..
    query_start[s+1] - 1 (int32 [S + 1], device) and are its last positions; the
    chunk's K/V must already be in the caches. See pa_prefill in include/pa.h.
    """
    torch = _torch()
    nb, bs, hkv, d = k_cache.shape
    total_q, hq, dq = q.shape
    s = context_lens.shape[0]
    if dq != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("q/out/cache shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or query_start.shape != (s + 1,):
        raise ValueError("block_tables must be [S, max_blocks], query_start [S + 1]")
    if work is not None and (work.dim() != 2 or work.shape[1] != 2):
        raise ValueError("work must be [num_items, 2]")
    bf = torch.bfloat16
    guard, st = _on_device((out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                            work), stream)
    head = (_dev_ptr(out, "out", bf), _dev_ptr(q, "q", bf), _dev_ptr(k_cache, "k_cache", bf),
            _dev_ptr(v_cache, "v_cache", bf), _dev_ptr(block_tables, "block_tables", torch.int32),
            _dev_ptr(context_lens, "context_lens", torch.int32),
            _dev_ptr(query_start, "query_start", torch.int32))
    rest = (s, total_q, hq, hkv, d, bs, nb, block_tables.shape[1], int(max_query_len),
            float(scale), PA_BF16, st)
    with guard:
        if work is None:
            _check(_lib.pa_prefill(*head, *rest))
        else:   # pa_prefill_planned: the kernel reads its item from the list
            _check(_lib.pa_prefill_planned(*head, _dev_ptr(work, "work", torch.int32),
                                           work.shape[0], *rest))


def pa_prefill_plan(query_start, context_lens, num_heads: int, num_kv_heads: int, out=None):
    """Work list of a planned prefill from HOST query_start (int32 [S + 1]) and
    context_lens (int32 [S]): int32 [num_items, 2] of {sequence, item}, in the
    order pa_prefill's CTAs would find. See pa_prefill_plan in include/pa.h."""
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    if qs.ndim != 1 or lens.ndim != 1 or qs.size != lens.size + 1:
        raise ValueError("query_start must be [S + 1] and context_lens [S]")
    if out is None:
        group = max(1, num_heads // max(1, num_kv_heads))
        tok = max(1, 256 // group)
        rows = np.diff(qs).astype(np.int64)
        out = np.empty((max(1, int(np.sum(np.maximum(0, -(-rows // tok))))), 2), dtype=np.int32)
    elif out.dtype != np.int32 or out.ndim != 2 or out.shape[1] != 2 or \
            not out.flags.c_contiguous:
        raise ValueError("out must be a C-contiguous int32 [capacity, 2] array")
    n = ctypes.c_int(0)
    _check(_lib.pa_prefill_plan(qs.ctypes.data_as(_i32p), lens.ctypes.data_as(_i32p), lens.size,
                                int(num_heads), int(num_kv_heads), out.ctypes.data_as(_i32p),
                                out.shape[0], ctypes.byref(n)))
    return out[:n.value]


def pa_device_errors(stream=None) -> int:
    """Synchronise, read and clear the device error word; returns its PA_DEVERR_* bits."""
    torch = _torch()
    flags = ctypes.c_uint(0)
    st = _lib.pa_device_errors(_stream(stream, torch.cuda.current_device()), ctypes.byref(flags))
    if st not in (PA_OK, PA_ERR_DEVICE_CHECK):
        _check(st)
    return int(flags.value)


# ------------------------------------------------------------- host allocator

def _i32_array(x):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int32))
    return a, a.ctypes.data_as(_i32p)


def _out_array(a, dtype, need, name):
    """A caller's output buffer, checked: a C-contiguous numpy array of `dtype`
    with at least `need` elements; returned flattened (a view, no copy)."""
    if not isinstance(a, np.ndarray) or a.dtype != dtype or not a.flags.c_contiguous:
        raise ValueError(f"{name} must be a C-contiguous numpy {np.dtype(dtype).name} array")
    if a.size < need:
        raise ValueError(f"{name} holds {a.size} elements, {need} needed")
    return a.reshape(-1)


class Allocator:
    """Free list + reference counts of a block pool (pa_alloc_*).

    Allocator(n) owns a new pool; BlockManager.allocator returns a view of the
    manager's pool that keeps the manager alive.
    """

    def __init__(self, num_blocks: int = 0, _handle=None, _owner=None):
        self._owner = _owner
        if _handle is not None:
            self._h = _handle
            self._own = False
        else:
            self._h = _lib.pa_alloc_create(num_blocks)
            if not self._h:
                raise PagedAttentionError(PA_ERR_INVALID, _lib.pa_last_error().decode())
            self._own = True

    def __del__(self):
        if getattr(self, "_own", False) and self._h:
            _lib.pa_alloc_destroy(self._h)
            self._h = None

    def alloc(self) -> int:
        out = ctypes.c_int32()
        _check(_lib.pa_alloc_block(self._h, ctypes.byref(out)))
        return out.value

    def incref(self, block: int) -> None:
        _check(_lib.pa_incref(self._h, block))

    def decref(self, block: int) -> None:
        _check(_lib.pa_decref(self._h, block))

    def refcount(self, block: int) -> int:
        return int(_lib.pa_refcount(self._h, block))

    def num_free(self) -> int:
        return int(_lib.pa_num_free(self._h))

    def num_blocks(self) -> int:
        return int(_lib.pa_num_blocks(self._h))

    def set_free_order(self, ids) -> None:
        a, p = _i32_array(ids)
        _check(_lib.pa_alloc_set_free_order(self._h, p, a.size))


class BlockManager:
    """Sequences over a block pool (pa_bm_*): tables, on-demand blocks, fork, copy-on-write."""

    def __init__(self, num_blocks: int, block_size: int):
        self._h = _lib.pa_bm_create(num_blocks, block_size)
        if not self._h:
            raise PagedAttentionError(PA_ERR_INVALID, _lib.pa_last_error().decode())
        self.block_size = block_size

    @property
    def allocator(self) -> Allocator:
        return Allocator(_handle=_lib.pa_bm_allocator(self._h), _owner=self)

    def __del__(self):
        if getattr(self, "_h", None):
            _lib.pa_bm_destroy(self._h)
            self._h = None

    def add_seq(self) -> int:
        out = ctypes.c_int32()
        _check(_lib.pa_bm_add_seq(self._h, ctypes.byref(out)))
        return out.value

    def fork(self, parent: int) -> int:
        out = ctypes.c_int32()
        _check(_lib.pa_bm_fork(self._h, parent, ctypes.byref(out)))
        return out.value

    def free_seq(self, seq: int) -> None:
        _check(_lib.pa_bm_free_seq(self._h, seq))

    def seq_len(self, seq: int) -> int:
        return int(_lib.pa_bm_seq_len(self._h, seq))

    def seq_num_blocks(self, seq: int) -> int:
        return int(_lib.pa_bm_seq_num_blocks(self._h, seq))

    def append_slots(self, seq_ids, counts, slots_out=None, cows_out=None):
        """Reserve slots; returns (slot_mapping int64 [sum(counts)], cow_pairs int64 [k, 2]).

        slots_out (int64, >= sum(counts) elements) and cows_out (int64 [>= n, 2],
        n = len(seq_ids)), both C-contiguous, are written in place and views of
        them returned: a serving loop then allocates nothing per step."""
        ids, pids = _i32_array(seq_ids)
        cnt, pcnt = _i32_array(counts)
        if ids.shape != cnt.shape:
            raise ValueError("seq_ids and counts differ in length")
        total = int(cnt.sum())
        slots = np.empty(total, dtype=np.int64) if slots_out is None else \
            _out_array(slots_out, np.int64, total, "slots_out")
        cows = np.empty((max(ids.size, 1), 2), dtype=np.int64) if cows_out is None else \
            _out_array(cows_out, np.int64, 2 * max(ids.size, 1), "cows_out").reshape(-1, 2)
        ncow = ctypes.c_int(0)
        _check(_lib.pa_bm_append_slots(self._h, pids, pcnt, ids.size,
                                       slots.ctypes.data_as(_i64p), cows.ctypes.data_as(_i64p),
                                       cows.shape[0], ctypes.byref(ncow)))
        if slots_out is not None:
            return slots[:total], cows[:ncow.value]
        return slots, cows[:ncow.value].copy()

    def block_tables(self, seq_ids, max_blocks_per_seq: int, tables_out=None, lens_out=None):
        """(tables int32 [n, max_blocks_per_seq], context_lens int32 [n]) for the sequences.

        tables_out / lens_out (int32, C-contiguous, n * max_blocks_per_seq and n
        elements at least) are written in place and views of them returned."""
        ids, pids = _i32_array(seq_ids)
        n = ids.size
        tables = np.empty((n, max_blocks_per_seq), dtype=np.int32) if tables_out is None else \
            _out_array(tables_out, np.int32, n * max_blocks_per_seq,
                       "tables_out")[:n * max_blocks_per_seq].reshape(n, max_blocks_per_seq)
        lens = np.empty(n, dtype=np.int32) if lens_out is None else \
            _out_array(lens_out, np.int32, n, "lens_out")[:n]
        _check(_lib.pa_bm_block_tables(self._h, pids, n, tables.ctypes.data_as(_i32p),
                                       max_blocks_per_seq, lens.ctypes.data_as(_i32p)))
        return tables, lens
