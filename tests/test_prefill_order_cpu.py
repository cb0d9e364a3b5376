"""pa_prefill's work-item arithmetic on the host (no GPU): the per-sequence
cost counts against brute force, and the kernel's longest-first search,
replayed lane by lane, as a one-to-one map onto the sorted items. The C++
check compiles the library's own header (csrc/pa_prefill_order.h)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_prefill_work_order(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    exe = tmp_path / "prefill_order_check"
    subprocess.run([cxx, "-O2", "-std=c++17", "-I",
                    os.path.join(ROOT, "paged_kv_cache_345_b200", "csrc"),
                    os.path.join(ROOT, "tests", "prefill_order_check.cpp"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr
