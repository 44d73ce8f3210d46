"""The serving-loop driver behind the bench's per-step trace timing
(paged_kv_cache_381_b200.trace): the continuous-batching trace's device work
replayed step by step through the library's calls.  Its arithmetic is the same
calls the trace parity test checks against the oracle; here the driver itself
must run every step, time it, and leave no device error."""

import dataclasses

import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import trace, workloads as wl

pytestmark = pytest.mark.gpu


def test_trace_driver_times_every_step():
    assert torch.cuda.is_available()
    from paged_kv_cache_381_b200 import build
    build.build()
    pa.pa_get_device_error()
    tc = dataclasses.replace(wl.TRACE, steps=40)
    r = trace.run(tc, seed=5)
    assert r["steps"] == 40 and len(r["host_ms"]) == 40
    assert all(ms > 0 for ms in r["device_ms"])
    assert all(b > 0 for b in r["kv_bytes"])
    assert r["admitted"] >= tc.max_running
    assert pa.pa_get_device_error() == 0
