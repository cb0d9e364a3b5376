"""The Python binding's argument marshalling, on the CPU (no GPU).

Every kernel wrapper runs against a stand-in for libpa.so that records the
call; the argument count must equal the C signature registered for that
entry point, and the sizes must come from the tensors' shapes in the order
include/pa.h declares. Pointers are replaced by the argument's name, so the
order of the buffers is checked as well. The one-device rule of the
wrappers is checked with stand-in tensors on two GPUs."""

import types

import pytest
import torch

import paged_kv_cache_345_b200 as pa

BF, U8, I32, I64, F32 = torch.bfloat16, torch.uint8, torch.int32, torch.int64, torch.float32


@pytest.fixture
def calls(monkeypatch):
    real = pa._lib
    log = []

    class Lib:
        def __getattr__(self, name):
            arity = len(getattr(real, name).argtypes)

            def fn(*args):
                assert len(args) == arity, f"{name}: {len(args)} arguments, C takes {arity}"
                log.append((name, args))
                return pa.PA_OK
            return fn

    def ptr(t, name, dtype=None):
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        return name

    monkeypatch.setattr(pa, "_lib", Lib())
    monkeypatch.setattr(pa, "_dev_ptr", ptr)
    monkeypatch.setattr(pa, "_mapped_ptr", ptr)
    monkeypatch.setattr(pa, "_stream", lambda stream, device: "stream")
    return log


def z(*shape, dtype=BF):
    return torch.zeros(shape, dtype=dtype)


def test_cache_writes_and_block_copies(calls):
    kc, vc = z(6, 8, 2, 16), z(6, 8, 2, 16)
    pa.pa_kv_append(z(3, 2, 16), z(3, 2, 16), z(3, dtype=I64), kc, vc)
    assert calls[-1] == ("pa_kv_append", ("k_new", "v_new", "slot_mapping", 3, "k_cache",
                                          "v_cache", 6, 8, 2, 16, pa.PA_BF16, "stream"))
    k8, v8 = z(6, 8, 2, 128, dtype=U8), z(6, 8, 2, 128, dtype=U8)
    pa.pa_kv_append_fp8(z(3, 2, 128), z(3, 2, 128), z(3, dtype=I64), k8, v8, z(2, dtype=F32),
                        z(2, dtype=F32))
    assert calls[-1] == ("pa_kv_append_fp8", ("k_new", "v_new", "slot_mapping", 3, "k_cache",
                                              "v_cache", "k_scale", "v_scale", 6, 8, 2, 128,
                                              "stream"))
    pa.pa_copy_blocks(kc, vc, z(5, 2, dtype=I64))
    assert calls[-1] == ("pa_copy_blocks", ("k_cache", "v_cache", "block_mapping", 5, 6, 8, 2,
                                            16, pa.PA_BF16, "stream"))
    pa.pa_swap_blocks(z(4, 8, 2, 16), z(4, 8, 2, 16), kc, vc, z(3, 2, dtype=I64))
    assert calls[-1] == ("pa_swap_blocks", ("dst_k", "dst_v", 4, "src_k", "src_v", 6,
                                            "block_mapping", 3, 8, 2, 16, pa.PA_BF16, "stream"))


def test_shared_prefix_decode_call(calls):
    s, hq, hkv, d, nb, bs, mb = 3, 8, 2, 128, 10, 16, 4
    kc, vc = z(nb, bs, hkv, d), z(nb, bs, hkv, d)
    q, out = z(s, hq, d), z(s, hq, d)
    tables, lens, ws = z(s, mb, dtype=I32), z(s, dtype=I32), z(1024, dtype=U8)
    pa.pa_decode_shared_prefix(out, q, z(s, hkv, d), z(s, hkv, d), kc, vc, tables, lens, 32, 50,
                               0.125, 16, ws)
    name, a = calls[-1]
    assert name == "pa_decode_shared_prefix"
    assert a[:8] == ("out", "q", "k_new", "v_new", "k_cache", "v_cache", "block_tables",
                     "context_lens")
    assert a[8:20] == (s, hq, hkv, d, bs, nb, mb, 32, 50, pytest.approx(0.125), 16, "workspace")
    assert a[20:] == (1024, pa.PA_BF16, "stream")
    pa.pa_decode_shared_prefix(out, q, None, None, kc, vc, tables, lens, 32, 50, 0.125, 0, ws)
    assert calls[-1][1][2:4] == (None, None)


def test_contiguous_decode_call(calls):
    s, hq, hkv, d, slab = 3, 8, 2, 128, 64
    k, v = z(s, slab, hkv, d), z(s, slab, hkv, d)
    q, out, lens, ws = z(s, hq, d), z(s, hq, d), z(s, dtype=I32), z(1024, dtype=U8)
    pa.pa_decode_contiguous(out, q, k, v, lens, 50, 0.125, 32, ws)
    name, a = calls[-1]
    assert name == "pa_decode_contiguous"
    assert a[:5] == ("out", "q", "k", "v", "context_lens")
    assert a[5:13] == (s, hq, hkv, d, slab, 50, pytest.approx(0.125), 32)
    assert a[13:] == ("workspace", 1024, pa.PA_BF16, "stream")


def test_decode_calls(calls):
    s, hq, hkv, d, nb, bs, mb = 3, 8, 2, 128, 10, 16, 4
    kc, vc = z(nb, bs, hkv, d), z(nb, bs, hkv, d)
    q, out = z(s, hq, d), z(s, hq, d)
    tables, lens, ws = z(s, mb, dtype=I32), z(s, dtype=I32), z(1024, dtype=U8)
    sizes = (s, hq, hkv, d, bs, nb, mb, 50, pytest.approx(0.125), 64)
    pa.pa_decode(out, q, kc, vc, tables, lens, 50, 0.125, 64, ws)
    name, a = calls[-1]
    assert name == "pa_decode"
    assert a[:6] == ("out", "q", "k_cache", "v_cache", "block_tables", "context_lens")
    assert a[6:16] == sizes and a[16:] == ("workspace", 1024, pa.PA_BF16, "stream")
    pa.pa_decode_append(out, q, z(s, hkv, d), z(s, hkv, d), kc, vc, tables, lens, 50, 0.125, 64,
                        ws)
    name, a = calls[-1]
    assert a[:8] == ("out", "q", "k_new", "v_new", "k_cache", "v_cache", "block_tables",
                     "context_lens")
    assert a[8:18] == sizes and a[18:] == ("workspace", 1024, pa.PA_BF16, "stream")
    k8, v8, sc = z(nb, bs, hkv, d, dtype=U8), z(nb, bs, hkv, d, dtype=U8), z(hkv, dtype=F32)
    pa.pa_decode_fp8(out, q, k8, v8, sc, sc, tables, lens, 50, 0.125, 64, ws)
    name, a = calls[-1]
    assert a[:8] == ("out", "q", "k_cache", "v_cache", "k_scale", "v_scale", "block_tables",
                     "context_lens")
    assert a[8:18] == sizes and a[18:] == ("workspace", 1024, "stream")
    pa.pa_decode_append_fp8(out, q, z(s, hkv, d), z(s, hkv, d), k8, v8, sc, sc, tables, lens, 50,
                            0.125, 64, None)
    name, a = calls[-1]
    assert a[:10] == ("out", "q", "k_new", "v_new", "k_cache", "v_cache", "k_scale", "v_scale",
                      "block_tables", "context_lens")
    assert a[10:20] == sizes and a[20:] == (None, 0, "stream")


def test_prefill_call(calls):
    kc, vc = z(10, 16, 2, 128), z(10, 16, 2, 128)
    q = z(7, 8, 128)
    pa.pa_prefill(z(7, 8, 128), q, kc, vc, z(2, 5, dtype=I32), z(2, dtype=I32), z(3, dtype=I32),
                  4, 0.5)
    name, a = calls[-1]
    assert name == "pa_prefill"
    assert a[:7] == ("out", "q", "k_cache", "v_cache", "block_tables", "context_lens",
                     "query_start")
    assert a[7:] == (2, 7, 8, 2, 128, 16, 10, 5, 4, 0.5, pa.PA_BF16, "stream")


def test_wrappers_check_shapes_and_dtypes(calls):
    kc, vc = z(6, 8, 2, 16), z(6, 8, 2, 16)
    with pytest.raises(ValueError):
        pa.pa_kv_append(z(3, 2, 8), z(3, 2, 8), z(3, dtype=I64), kc, vc)
    with pytest.raises(TypeError):
        pa.pa_kv_append(z(3, 2, 16), z(3, 2, 16), z(3, dtype=I32), kc, vc)
    with pytest.raises(TypeError):
        pa.pa_kv_append_fp8(z(3, 2, 16), z(3, 2, 16), z(3, dtype=I64), kc, vc, z(2, dtype=F32),
                            z(2, dtype=F32))
    with pytest.raises(ValueError):
        pa.pa_prefill(z(7, 8, 128), z(7, 8, 128), z(10, 16, 2, 128), z(10, 16, 2, 128),
                      z(2, 5, dtype=I32), z(2, dtype=I32), z(2, dtype=I32), 4, 0.5)
    assert not calls


def _on(dev):
    return types.SimpleNamespace(device=torch.device(dev), is_cuda=dev.startswith("cuda"))


def test_one_device_per_call(monkeypatch):
    monkeypatch.setattr(pa, "_stream", lambda stream, device: ("stream", device))
    with pytest.raises(ValueError, match="several devices"):
        pa._on_device((_on("cuda:0"), _on("cuda:1")), None)
    with pytest.raises(ValueError, match="stream is on"):
        pa._on_device((_on("cuda:0"), None), types.SimpleNamespace(device=torch.device("cuda:1")))
    guard, st = pa._on_device((_on("cuda:1"), _on("cpu"), None), None)
    assert st == ("stream", torch.device("cuda:1"))
    assert isinstance(guard, torch.cuda.device) and guard.idx == 1
    guard, st = pa._on_device((_on("cpu"),), None)
    assert st == ("stream", None)
    with guard:  # no CUDA device involved: nothing to switch
        pass
