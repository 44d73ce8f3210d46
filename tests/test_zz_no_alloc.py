"""pa_decode_noalloc: paged decode for callers that cannot allocate device memory.

Who needs it: a serving engine usually gives almost all GPU memory to its KV
block pool when it starts and allocates nothing afterwards, and some callers
sit on a latency-critical path where cudaMalloc (which can synchronise the
device) is not allowed.  Neither can hand pa_decode the scratch workspace its
split-K path asks for, so the library offers this entry point, whose scratch
is a fixed array built into the library.

The test calls it through the C ABI twice in a row on a batch that uses the
split-K path, and compares each result with the existing pa_decode entry point
(given a caller-allocated workspace) within the tolerance the other GPU tests
use; it also checks the oracle and the rejection of a batch too large for the
built-in array.  It does not depend on any other test having run.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from oracle.numerics import widen
from tests.gpu_harness import DeviceBatch, assert_close, oracle_outputs, to_storage

pytestmark = pytest.mark.gpu

PA_ERR_UNSUPPORTED = 2


def _call_noalloc(b, out, max_context_len, num_seqs=None, partition_size=0, tables=None):
    S, Hq, D = b.q.shape
    tables = b.block_tables if tables is None else tables
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return pa.lib().pa_decode_noalloc(
        out.data_ptr(), b.q.data_ptr(), b.k_cache.data_ptr(), b.v_cache.data_ptr(), tables.data_ptr(),
        b.context_lens.data_ptr(), b.cfg.scale, b.bs, b.cfg.num_kv_heads, S if num_seqs is None else num_seqs, Hq, D,
        tables.shape[1], max_context_len, b.nb, {"f32": 0, "f16": 1, "bf16": 2}[b.dtype], partition_size,
        stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    from paged_kv_cache_381_b200 import build
    build.build()
    # Llama-3-70B-shaped heads (64 query / 8 kv, head_dim 128, bf16), contexts
    # long enough to be split into 512-token partitions and merged.
    cfg = wl.DecodeConfig("noalloc", "bf16", 8, 64, 8, 128, 16, "fixed")
    lens = (4096, 1, 700, 513, 2000, 33, 3000, 8192)
    inp = wl.make_decode_inputs(cfg, 17, context_lens=lens)
    b = DeviceBatch(inp)
    b.step_write()
    mcl = int(max(lens))
    need = pa.pa_decode_workspace_size(len(lens), cfg.num_heads, cfg.head_dim, mcl)
    assert 0 < need <= 32 * 1024 * 1024

    ref = torch.empty_like(b.q)
    pa.pa_decode(ref, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, cfg.scale, b.bs,
                 cfg.num_kv_heads, max_context_len=mcl)
    torch.cuda.synchronize()
    ref_bits = to_storage(ref, "bf16")
    oracle = oracle_outputs(inp)

    for call in range(2):
        out = torch.full_like(b.q, float("nan"))
        assert _call_noalloc(b, out, mcl) == 0, call
        torch.cuda.synchronize()
        got = to_storage(out, "bf16")
        assert_close(got, widen(ref_bits, "bf16"), "bf16", f"call {call} vs pa_decode")
        assert_close(got, oracle, "bf16", f"call {call} vs oracle")
    assert pa.pa_get_device_error() == 0


def test_noalloc_single_pass_and_rejection():
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    cfg = wl.DecodeConfig("noalloc1", "f16", 3, 32, 32, 128, 16, "fixed")
    inp = wl.make_decode_inputs(cfg, 18, context_lens=(100, 1, 512))
    b = DeviceBatch(inp)
    b.step_write()
    ref = torch.empty_like(b.q)
    pa.pa_decode(ref, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, cfg.scale, b.bs,
                 cfg.num_kv_heads, max_context_len=512)
    out = torch.empty_like(b.q)
    assert _call_noalloc(b, out, 512) == 0          # one partition: no scratch needed
    torch.cuda.synchronize()
    assert_close(to_storage(out, "f16"), widen(to_storage(ref, "f16"), "f16"), "f16", "single pass")
    # a batch whose scratch need exceeds the built-in array is refused before any
    # launch: the same sequences with block tables wide enough for 30000 tokens
    # (padded with -1) and that bound, in 32-token partitions, would need ~47 MB
    # of scratch
    big = pa.pa_decode_workspace_size(3, 32, 128, 30000, 32)
    assert big > 32 * 1024 * 1024
    wide = torch.full((3, 30000 // b.bs + 1), -1, dtype=torch.int32, device="cuda")
    wide[:, :b.block_tables.shape[1]] = b.block_tables
    n0 = pa.launch_count()
    assert _call_noalloc(b, out, 30000, partition_size=32, tables=wide) == PA_ERR_UNSUPPORTED
    assert pa.launch_count() == n0
    assert pa.pa_get_device_error() == 0


def test_noalloc_bound_above_table_capacity():
    """A declared max_context_len far above what the block tables can hold is
    capped at the table capacity, as pa_decode caps it, so the scratch need
    fits the built-in array and the call matches pa_decode."""
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    cfg = wl.DecodeConfig("noalloc2", "bf16", 4, 64, 8, 128, 16, "fixed")
    lens = (3000, 17, 1200, 4096)
    inp = wl.make_decode_inputs(cfg, 19, context_lens=lens)
    b = DeviceBatch(inp)
    b.step_write()
    bound = 10 ** 6
    assert pa.pa_decode_workspace_size(len(lens), cfg.num_heads, cfg.head_dim, bound) > 32 * 1024 * 1024
    ref = torch.empty_like(b.q)
    pa.pa_decode(ref, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, cfg.scale, b.bs,
                 cfg.num_kv_heads, max_context_len=bound,
                 workspace=torch.empty(pa.pa_decode_workspace_size(len(lens), cfg.num_heads, cfg.head_dim,
                                                                   b.block_tables.shape[1] * b.bs),
                                       dtype=torch.uint8, device="cuda"))
    out = torch.full_like(b.q, float("nan"))
    assert _call_noalloc(b, out, bound) == 0
    torch.cuda.synchronize()
    assert np.array_equal(to_storage(out, "bf16"), to_storage(ref, "bf16"))
    assert_close(to_storage(out, "bf16"), oracle_outputs(inp), "bf16", "bound above table capacity")
    assert pa.pa_get_device_error() == 0
