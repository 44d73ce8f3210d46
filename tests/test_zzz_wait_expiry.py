"""The kernels' bounded waits give up instead of hanging.

Every mbarrier wait in the library's kernels is bounded by %globaltimer; on
expiry a CTA sets PA_DEVERR_TIMEOUT and leaves.  pa_check_wait_expiry runs
that wait on a barrier that nothing arrives at (a flag that is never set), so
the limit must run out: the call must return, the error word must hold
exactly the timeout bit, and the context must stay usable (a decode after it
matches the oracle).
"""

import time

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from paged_kv_cache_381_b200.batch import PagedBatch
from oracle import attention as oa
from oracle.numerics import widen

pytestmark = pytest.mark.gpu


def test_wait_expires_and_context_stays_usable():
    assert torch.cuda.is_available()
    from paged_kv_cache_381_b200 import build
    build.build()
    pa.pa_get_device_error()                      # clear the error word
    t0 = time.perf_counter()
    pa.pa_check_wait_expiry()
    flags = pa.pa_get_device_error()              # synchronizes the stream
    waited = time.perf_counter() - t0
    assert flags == pa.DEVERR_TIMEOUT, hex(flags)
    assert 1.5 < waited < 30.0, waited            # the 2 s limit, not an early exit
    # the context still runs kernels correctly
    cfg = wl.CONFIGS["tiny"]
    inp = wl.make_decode_inputs(cfg, 0)
    dev = torch.device("cuda")
    hist_k = torch.from_numpy(np.concatenate(inp.k_hist)).to(dev)
    hist_v = torch.from_numpy(np.concatenate(inp.v_hist)).to(dev)
    offsets = np.concatenate([[0], np.cumsum(inp.context_lens)])
    batch = PagedBatch(hist_k, hist_v, offsets, inp.context_lens, inp.num_blocks, cfg.block_size,
                       np.random.default_rng(0).permutation(inp.num_blocks))
    q = torch.from_numpy(inp.q).to(dev)
    out = torch.empty_like(q)
    batch.write_new_tokens()
    batch.decode(out, q, cfg.scale)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    for s in range(len(inp.context_lens)):
        ref = oa.decode_history(widen(inp.q[s], "f32"), widen(inp.k_hist[s], "f32"), widen(inp.v_hist[s], "f32"),
                                cfg.scale)
        assert np.all(np.abs(got[s] - ref) <= 1e-5 + 1e-5 * np.abs(ref)), s
