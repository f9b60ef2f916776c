"""The C ABI used from plain C: tests/c/pool_from_c.c is compiled with gcc against include/paged_attn.h and
linked with libpaged_attn.so, then run (host block pool calls and host-side argument checks; no GPU)."""

from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "paged_kv_cache_330_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_pool_from_c(tmp_path):
    exe = tmp_path / "pool_from_c"
    build = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "c", "pool_from_c.c"), "-L", PKG, "-lpaged_attn",
                            f"-Wl,-rpath,{PKG}", "-o", str(exe)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stderr


@pytest.mark.skipif(shutil.which("g++") is None, reason="no C++ compiler")
def test_pool_batches_survive_host_allocation_failure(tmp_path):
    """tests/c/pool_alloc_fail.cpp replaces operator new to fail the k-th allocation of each batched pool call;
    every failed call must leave the pool unchanged (no live sequence dropped, no reference count moved)."""
    exe = tmp_path / "pool_alloc_fail"
    build = subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "c", "pool_alloc_fail.cpp"), "-L", PKG, "-lpaged_attn",
                            f"-Wl,-rpath,{PKG}", "-o", str(exe)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
