"""The per-context cache behind the library's context-bound values (the status
word's and the no-allocation scratch's device addresses, raised kernel
attributes, the host path's copy streams), compiled with g++ and run on the
CPU: a value made in one CUDA context is never handed to another, failed
lookups are retried, and full caches replace their oldest entry."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
def test_ctx_cache(tmp_path):
    exe = tmp_path / "ctx_cache_test"
    src = os.path.join(ROOT, "tests", "ctx_cache_test.cc")
    inc = os.path.join(ROOT, "video_dit_block_vsa_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-I", inc, src, "-o", str(exe), "-pthread"],
                   check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.strip() == "ok"
