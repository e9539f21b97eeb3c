"""The cache of encoded TMA tensor maps, checked on the host: the native check program
(tests/native/map_cache_check.cpp) compiles the library's cache header with a fake encoder and
exercises hits, misses on every differing argument, eviction under collisions, the on/off
switch, failed encodes and concurrent callers; the library's switch and counters answer
through the C ABI without a GPU."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_include() -> str | None:
    nvcc = shutil.which("nvcc")
    if nvcc is None:
        return None
    inc = os.path.join(os.path.dirname(os.path.dirname(nvcc)), "include")
    return inc if os.path.exists(os.path.join(inc, "cuda.h")) else None


def test_native_cache_check(tmp_path):
    inc = _cuda_include()
    if inc is None or shutil.which("g++") is None:
        pytest.skip("needs g++ and the CUDA headers")
    exe = tmp_path / "map_cache_check"
    src = os.path.join(ROOT, "tests", "native", "map_cache_check.cpp")
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", f"-I{inc}",
                    f"-I{os.path.join(ROOT, 'fp8_block_scaled_tma_b200', 'csrc')}", src, "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "all checks passed" in r.stdout


@pytest.fixture(scope="module")
def dg():
    import __graft_entry__
    __graft_entry__._library_builder().build()
    import fp8_block_scaled_tma_b200 as mod
    return mod


def test_cache_switch_and_counters(dg):
    L = dg.lib
    assert L.dg_set_tensor_map_cache(2) == dg.DG_ERR_INVALID_ARG
    prev = dg.set_tensor_map_cache(False)
    assert prev is True                      # on by default
    assert dg.set_tensor_map_cache(True) is False
    hits, misses = dg.tensor_map_cache_stats()
    assert hits >= 0 and misses >= 0
    assert L.dg_get_tensor_map_cache_stats(None, None) == 0
