"""The device entry points have no CPU fallback: given host tensors they
refuse before any library call, and the package never imports the oracle."""

import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    return pa


def test_device_calls_refuse_host_tensors(pa):
    S, Hq, Hkv, D, bs, nb = 2, 4, 2, 64, 16, 4
    q = torch.zeros(S, Hq, D, dtype=torch.float16)
    out = torch.zeros_like(q)
    kc = torch.zeros(nb, bs, Hkv, D, dtype=torch.float16)
    vc = torch.zeros_like(kc)
    tables = torch.zeros(S, 1, dtype=torch.int32)
    lens = torch.ones(S, dtype=torch.int32)
    k = torch.zeros(S, Hkv, D, dtype=torch.float16)
    slots = torch.zeros(S, dtype=torch.int64)
    before = pa.launch_count()
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_cache_write(k, k, kc, vc, slots)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_decode(out, q, kc, vc, tables, lens, 0.125)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_verify(out.view(S, 1, Hq, D), q.view(S, 1, Hq, D), kc, vc, tables, lens, 0.125)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_write_decode(k, k, slots, out, q, kc, vc, tables, lens, 0.125)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_copy_blocks(kc, vc, torch.zeros(1, 2, dtype=torch.int32))
    assert pa.launch_count() == before


def test_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_381_b200")
    for d, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                src = open(os.path.join(d, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", src, re.M), f
