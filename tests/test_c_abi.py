"""The C ABI from plain C: include/pa.h compiles as strict C11, and a C
program linked against libpa.so runs the host calls (block manager with
copy-on-write, a scheduler step through the prefix cache with a C token
function) with hand-worked expected values.  No device call is made."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "paged_kv_cache_381_b200")


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_381_b200 import build
    return build.build()


def test_header_and_host_calls_from_c(lib, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    exe = str(tmp_path / "host_abi")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "host_abi.c"), "-L", PKG, "-lpa", f"-Wl,-rpath,{PKG}",
                    "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
