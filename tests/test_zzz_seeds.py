"""Full-size parity on further seeds (1-4) of the decode workloads.

The bench times seed 0; these draws change the context lengths (the 70b
batch's power-law mix, the 7b batch's uniform mix) and every value, so the
kernels meet other length mixes, table layouts and outliers in the same launch
configuration.  Checked like seed 0: sampled (sequence, head) rows against the
fp64 oracle, plus finiteness of every output.  The file runs last: it adds
draws, not code paths.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from paged_kv_cache_381_b200.batch import PagedBatch
from tests.gpu_harness import assert_close, to_storage
from oracle import attention as oa
from oracle.numerics import widen

pytestmark = pytest.mark.gpu

SEEDS = [1, 2, 3, 4]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_381_b200 import build
    build.build()
    pa.pa_get_device_error()          # clear the error word
    yield


def _batch(cfg, seed):
    d = wl.draw_device(cfg, seed)
    batch = PagedBatch(d.k_hist, d.v_hist, d.offsets, d.context_lens, d.num_blocks, cfg.block_size,
                       d.free_order)
    batch.write_new_tokens()
    return d, batch


def _ref(d, cfg, s, g, upto, qrow):
    a = int(d.offsets[s])
    K = widen(to_storage(d.k_hist[a:a + upto, g], cfg.dtype), cfg.dtype)
    V = widen(to_storage(d.v_hist[a:a + upto, g], cfg.dtype), cfg.dtype)
    return oa.attend(widen(qrow, cfg.dtype), K, V, cfg.scale)


@pytest.mark.parametrize("seed", SEEDS)
@pytest.mark.parametrize("name", ["7b", "70b", "long"])
def test_decode_other_seeds(name, seed):
    cfg = wl.CONFIGS[name]
    d, batch = _batch(cfg, seed)
    out = torch.empty_like(d.q)
    batch.decode(out, d.q, cfg.scale, partition_size=cfg.partition_size)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    lens = d.context_lens
    S, Hq = len(lens), cfg.num_heads
    r = np.random.default_rng([seed, 21])
    rows = {(int(np.argmax(lens)), 0), (int(np.argmin(lens)), Hq - 1)}
    while len(rows) < 24:
        rows.add((int(r.integers(S)), int(r.integers(Hq))))
    G = Hq // cfg.num_kv_heads
    qs, got = to_storage(d.q, cfg.dtype), to_storage(out, cfg.dtype)
    rows = sorted(rows)
    ref = [_ref(d, cfg, s, h // G, int(lens[s]), qs[s, h]) for s, h in rows]
    assert_close(np.stack([got[s, h] for s, h in rows]), np.stack(ref), cfg.dtype, f"{name} seed {seed}")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("seed", SEEDS)
def test_verify_other_seeds(seed):
    """The 70b batch verifying 6 candidate tokens, the kernel chosen as in the bench."""
    cfg = wl.CONFIGS["70b"]
    Q = 6
    d, batch = _batch(cfg, seed)
    lens = d.context_lens
    assert int(lens.min()) >= Q
    S, Hq, D = len(lens), cfg.num_heads, cfg.head_dim
    g = torch.Generator(device="cuda").manual_seed(100 + seed)
    q = torch.randn((S, Q, Hq, D), generator=g, device="cuda", dtype=torch.float32).to(d.q.dtype)
    out = torch.empty_like(q)
    pa.pa_verify(out, q, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens, cfg.scale,
                 max_context_len=batch.max_context_len)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    r = np.random.default_rng([seed, 22])
    picks = {(int(np.argmax(lens)), Q - 1, 0), (int(np.argmin(lens)), 0, Hq - 1)}
    while len(picks) < 20:
        picks.add((int(r.integers(S)), int(r.integers(Q)), int(r.integers(Hq))))
    G = Hq // cfg.num_kv_heads
    qs, got = to_storage(q, cfg.dtype), to_storage(out, cfg.dtype)
    for s, i, h in sorted(picks):
        ref = _ref(d, cfg, s, h // G, int(lens[s]) - Q + i + 1, qs[s, i, h])
        assert_close(got[s, i, h], ref, cfg.dtype, f"70b seed {seed} row {(s, i, h)}")
    assert torch.isfinite(out.float()).all()
