"""GPU parity of pa_verify, the multi-query (speculative verification) pass,
against the fp64 oracle (oracle.attention.paged_verify).

Tolerance as for decode: 2e-3 absolute + 1e-2 relative for fp16 / bf16.  The
cache is filled through the product path (host block manager slots +
pa_cache_write); the Q candidate tokens are the last Q rows of each history.
Full-size shapes are checked on every (sequence, query, head) row.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from paged_kv_cache_381_b200.batch import PagedBatch
from tests.gpu_harness import DeviceBatch, assert_close, to_device, to_storage
from tests.full_size import assert_every_row, oracle_all_rows
from oracle import attention as oa
from oracle import cache as oc
from oracle.numerics import widen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_381_b200 import build
    build.build()
    pa.pa_get_device_error()
    yield


@pytest.fixture(autouse=True, params=["mma_sync", "tcgen05"])
def verify_kind(request):
    """Every case runs on both tensor-core paths of pa_verify."""
    before = pa.get_verify_kernel()
    pa.set_verify_kernel(pa.VERIFY_TCGEN05 if request.param == "tcgen05" else pa.VERIFY_MMA_SYNC)
    yield request.param
    pa.set_verify_kernel(before)


def _cfg(dtype="bf16", Hq=16, Hkv=2, D=128, bs=16, lens=(6, 17, 40, 100)):
    return wl.DecodeConfig("verify", dtype, len(lens), Hq, Hkv, D, bs, "fixed", fixed_lengths=tuple(lens))


def _run(cfg, Q, seed=0, partition_size=0, lens=None, tables=None, num_blocks=None, inp=None):
    inp = wl.make_decode_inputs(cfg, seed, context_lens=lens) if inp is None else inp
    b = DeviceBatch(inp, tables=tables, num_blocks=num_blocks)
    b.step_write()                         # every history row is now in the pool
    r = np.random.default_rng(1000 + seed)
    S = len(inp.context_lens)
    q_store = wl.to_storage(r.standard_normal((S, Q, cfg.num_heads, cfg.head_dim), dtype=np.float32), cfg.dtype)
    q = to_device(q_store, cfg.dtype)
    out = torch.full_like(q, float("nan"))
    pa.pa_verify(out, q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, cfg.scale,
                 max_context_len=int(max(inp.context_lens)), partition_size=partition_size)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    return inp, b, q_store, to_storage(out, cfg.dtype)


def _pool(inp, b):
    """The histories placed in a pool by the oracle's own scatter (nothing is
    read back from the device)."""
    cfg = inp.cfg
    sd = np.float32 if cfg.dtype == "f32" else np.uint16
    kc = np.zeros((b.nb, b.bs, cfg.num_kv_heads, cfg.head_dim), dtype=sd)
    vc = np.zeros_like(kc)
    for s in range(len(inp.context_lens)):
        kc, vc = oc.scatter_history(inp.k_hist[s], inp.v_hist[s], b.tables[s], kc, vc)
    return kc, vc


def _oracle(inp, b, q_store):
    kc, vc = _pool(inp, b)
    return oa.paged_verify(q_store, kc, vc, b.tables, inp.context_lens, inp.cfg.scale, b.bs, inp.cfg.dtype)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_shape_grid(dtype, D, bs):
    cfg = _cfg(dtype, 16, 2, D, bs, lens=(6, 7, 33, 70, 129))
    inp, b, q, got = _run(cfg, 6)
    assert_close(got, _oracle(inp, b, q), dtype, f"verify {dtype} D{D} bs{bs}")


@pytest.mark.parametrize("G,Q", [(1, 1), (1, 6), (1, 17), (1, 64), (4, 5), (8, 6), (8, 8), (8, 16), (6, 7)])
def test_groups_and_query_counts(G, Q):
    """Rows per kv head G*Q from 1 to 128: one, two and four 16-row tiles per
    chunk (warps split the slots or the rows) and two 64-row chunks."""
    lens = (Q, Q + 1, 3 * Q + 5, 300)
    cfg = _cfg("bf16", 2 * G, 2, 128, 16, lens=lens)
    inp, b, q, got = _run(cfg, Q, seed=G * 100 + Q)
    assert_close(got, _oracle(inp, b, q), "bf16", f"G{G} Q{Q}")


@pytest.mark.parametrize("P", [32, 64, 512])
def test_split_partitions(P):
    """Long contexts split into partitions, including last partitions shorter
    than Q (some rows see nothing there) and merged by the reduce kernel."""
    lens = (1030, 2049, 513, 40, 6)
    cfg = _cfg("f16", 64, 8, 128, 16, lens=lens)
    inp, b, q, got = _run(cfg, 6, seed=P, partition_size=P)
    assert_close(got, _oracle(inp, b, q), "f16", f"P{P}")


@pytest.mark.parametrize("P,bs", [(1024, 16), (2048, 16), (2048, 32)])
def test_large_partitions(P, bs):
    """1024- and 2048-token partitions (the sizes pa_verify picks for many query
    rows per kv head): contexts of one to three partitions and a last partition
    shorter than Q, merged by the reduce kernel."""
    lens = (4099, 2049, 2048, 1030, 6)
    cfg = _cfg("bf16", 64, 8, 128, bs, lens=lens)
    inp, b, q, got = _run(cfg, 6, seed=P + bs, partition_size=P)
    assert_close(got, _oracle(inp, b, q), "bf16", f"P{P} bs{bs}")


def test_partition_beyond_the_block_table_is_refused():
    """A partition of more than 128 blocks (2048 tokens of 8-token blocks) does
    not fit the kernels' block-id table: pa_verify refuses it."""
    cfg = _cfg("bf16", 64, 8, 128, 8, lens=(3000, 40))
    with pytest.raises(pa.PagedAttentionError):
        _run(cfg, 6, partition_size=2048)


def test_single_query_matches_decode_oracle():
    cfg = _cfg("bf16", 32, 8, 128, 16, lens=(1, 16, 17, 90, 777))
    inp, b, q, got = _run(cfg, 1)
    ref = oa.paged_decode(q[:, 0], *_pool(inp, b), b.tables, inp.context_lens, cfg.scale, 16, "bf16")
    assert_close(got[:, 0], ref, "bf16", "Q=1")


def test_short_and_empty_contexts_give_zero_rows():
    """Contexts shorter than Q: rows before position 0 are zero; an empty
    context (a padded batch slot) is all zero."""
    lens = (0, 2, 5, 64)
    cfg = _cfg("bf16", 8, 2, 64, 8, lens=lens)
    inp, b, q, got = _run(cfg, 5)
    ref = _oracle(inp, b, q)
    assert_close(got, ref, "bf16", "short")
    g = widen(got, "bf16")
    assert not g[0].any() and not g[1, :3].any() and g[1, 3:].all()


def test_physical_placement_is_bitwise_invariant():
    """The same histories under two different shuffles of the pool give the
    same bits (every reduction order depends on logical positions only)."""
    lens = (6, 600, 1500)
    cfg = _cfg("bf16", 64, 8, 128, 16, lens=lens)
    inp = wl.make_decode_inputs(cfg, 3, context_lens=lens)
    nb2, t2 = wl.shuffled_tables(np.random.default_rng(123), wl.blocks_for(lens, 16), inp.num_blocks + 37, 0)
    _, _, q1, g1 = _run(cfg, 6, seed=3, inp=inp)
    _, b2, q2, g2 = _run(cfg, 6, seed=3, inp=inp, tables=t2, num_blocks=nb2)
    assert np.array_equal(q1, q2)
    assert np.array_equal(g1, g2)
    assert_close(g2, _oracle(inp, b2, q2), "bf16", "shuffled")


@pytest.mark.parametrize("name", ["70b", "7b"])
def test_full_size_every_row(name):
    """The decode workload's batch verifying 6 candidate tokens per sequence
    (the bench's verification configuration): every (sequence, query, head)
    row against the fp64 oracle."""
    cfg = wl.CONFIGS[name]
    Q = 6
    d = wl.draw_device(cfg, 0)
    assert int(d.context_lens.min()) >= Q
    batch = PagedBatch(d.k_hist, d.v_hist, d.offsets, d.context_lens, d.num_blocks, cfg.block_size, d.free_order)
    batch.write_new_tokens()
    S, Hq, D = len(d.context_lens), cfg.num_heads, cfg.head_dim
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn((S, Q, Hq, D), generator=g, device="cuda", dtype=torch.float32).to(d.q.dtype)
    out = torch.empty_like(q)
    pa.pa_verify(out, q, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens, cfg.scale,
                 max_context_len=batch.max_context_len)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    ref = oracle_all_rows(q, d, cfg, verify=True)
    assert_every_row(out, ref, cfg.dtype, f"{name} verify")
