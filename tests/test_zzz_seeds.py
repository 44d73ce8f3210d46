"""Full-size parity on further seeds (1-4) of the decode workloads.

The bench times seed 0; these draws change the context lengths (the 70b
batch's power-law mix, the 7b batch's uniform mix) and every value, so the
kernels meet other length mixes, table layouts and outliers in the same launch
configuration.  Checked like seed 0: every (sequence, head) row against the
fp64 oracle, element by element.  The file runs late: it adds draws, not code
paths.
"""

import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from paged_kv_cache_381_b200.batch import PagedBatch
from tests.full_size import assert_every_row, oracle_all_rows

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


@pytest.mark.parametrize("seed", SEEDS)
@pytest.mark.parametrize("name", ["7b", "70b", "long"])
def test_decode_other_seeds(name, seed):
    cfg = wl.CONFIGS[name]
    d, batch = _batch(cfg, seed)
    out = torch.empty_like(d.q)
    batch.decode(out, d.q, cfg.scale, partition_size=cfg.partition_size)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    ref = oracle_all_rows(d.q, d, cfg)
    assert_every_row(out, ref, cfg.dtype, f"{name} seed {seed}")


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
    ref = oracle_all_rows(q, d, cfg, verify=True)
    assert_every_row(out, ref, cfg.dtype, f"70b verify seed {seed}")
