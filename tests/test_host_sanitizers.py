"""The native host code (block manager, scheduler) under AddressSanitizer and
UndefinedBehaviorSanitizer.

The host sources are compiled again with -fsanitize=address,undefined into a
temporary library, and the host test files -- golden traces, lockstep runs
against the oracle's models with evictions, swaps, forks and preemptions,
argument errors -- run in a child process whose pa_bm_* / pa_sched_* calls go
to that library.  Any out-of-bounds access, use after free or undefined
behaviour aborts the child.
"""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HOST = os.path.join(ROOT, "paged_kv_cache_381_b200", "csrc", "host")
FILES = ["tests/test_sched_prefix.py", "tests/test_prefix_cache.py", "tests/test_swap.py",
         "tests/test_prefix_swap.py", "tests/test_native_host.py"]


def _runtime(name):
    p = subprocess.run(["g++", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    return pa


def test_host_code_is_clean_under_sanitizers(pa, tmp_path):
    if shutil.which("g++") is None:
        pytest.skip("no g++")
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("sanitizer runtimes not installed")
    lib = str(tmp_path / "libpa_host_sanitized.so")
    subprocess.run(["g++", "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined", "-fno-omit-frame-pointer",
                    "-fno-sanitize-recover=undefined", "-shared", "-fPIC", "-I", os.path.join(ROOT, "include"),
                    "-I", HOST, os.path.join(HOST, "block_manager.cpp"), os.path.join(HOST, "scheduler.cpp"),
                    "-o", lib], check=True, cwd=ROOT)
    env = dict(os.environ)
    log = str(tmp_path / "sanitizer")
    env.update(LD_PRELOAD=f"{asan}:{ubsan}", ASAN_OPTIONS=f"detect_leaks=0:halt_on_error=1:log_path={log}",
               UBSAN_OPTIONS=f"halt_on_error=1:print_stacktrace=1:log_path={log}", PA_SANITIZED_HOST_LIB=lib,
               PYTHONPATH=os.pathsep.join([os.path.join(ROOT, "tests"), ROOT, env.get("PYTHONPATH", "")]))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "not gpu", "-p", "sanitized_host",
                        "-p", "no:cacheprovider", *FILES], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=1200)
    reports = "".join(open(tmp_path / f).read() for f in sorted(os.listdir(tmp_path)) if f.startswith("sanitizer"))
    tail = reports[:4000] + (r.stdout + r.stderr)[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
