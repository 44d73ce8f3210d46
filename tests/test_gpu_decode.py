"""GPU parity tests: the CUDA path through the C ABI against the fp64 oracle.

Tolerances (stated by the task's contract for this path): fp16 / bf16 outputs
within 2e-3 absolute + 1e-2 relative of the unrounded fp64 oracle; fp32 within
1e-5 absolute + 1e-5 relative.  Cache writes, block copies and bookkeeping are
bit-exact.  Full-size workloads (the bench's launch configuration) are checked
on every (sequence, head) row, element by element.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from paged_kv_cache_381_b200.batch import PagedBatch
from tests.gpu_harness import (DeviceBatch, assert_cache_exact, assert_close, free_order_for, oracle_outputs,
                               to_device, to_storage, TORCH_DTYPE)
from tests.full_size import assert_every_row, oracle_all_rows
from oracle import attention as oa
from oracle.numerics import widen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_381_b200 import build
    build.build()
    pa.pa_get_device_error()          # clear the error word
    yield


@pytest.fixture(params=["auto", "simt"])
def math_path(request):
    """Run a test with the tensor-core (auto) and the CUDA-core decode path."""
    pa.set_decode_math(pa.MATH_AUTO if request.param == "auto" else pa.MATH_SIMT)
    yield request.param
    pa.set_decode_math(pa.MATH_AUTO)


@pytest.fixture(params=["fused", "kernel"])
def merge_mode(request):
    """Merge split partitions in the decode kernel (fused) or in the reduce kernel."""
    pa.set_split_merge(pa.MERGE_FUSED if request.param == "fused" else pa.MERGE_KERNEL)
    yield request.param
    pa.set_split_merge(pa.MERGE_KERNEL)


def _no_device_error():
    assert pa.pa_get_device_error() == 0


def _run(inp, partition_size=0, block_size=None):
    b = DeviceBatch(inp, block_size=block_size)
    b.step_write()
    out = b.decode(partition_size=partition_size)
    torch.cuda.synchronize()
    return b, to_storage(out, inp.cfg.dtype)


def test_tiny_config_fp32():
    """4 sequences {1,16,17,90}, MHA 4/4, D=64, 16-token blocks, 32-block pool."""
    inp = wl.make_decode_inputs(wl.CONFIGS["tiny"], 0)
    b, got = _run(inp)
    assert_close(got, oracle_outputs(inp), "f32", "tiny")
    assert_cache_exact(b)
    # a single-token context returns its value row exactly
    assert np.array_equal(got[0], inp.v_hist[0][0])
    _no_device_error()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_single_token_context_returns_value_exactly(dtype, math_path):
    cfg = _grid_cfg(dtype, 128, 16, 8)
    inp = wl.make_decode_inputs(cfg, 40, context_lens=(1, 1, 300))
    b, got = _run(inp)
    G = cfg.num_heads // cfg.num_kv_heads
    for s in (0, 1):
        for h in range(cfg.num_heads):
            assert np.array_equal(got[s, h], inp.v_hist[s][0, h // G]), (s, h)


def _grid_cfg(dtype, D, bs, G, hkv=2):
    return wl.DecodeConfig("grid", dtype, 0, G * hkv, hkv, D, bs, "fixed")


GRID_LENS = (0, 1, 2, 31, 32, 33, 100, 511, 512, 513, 1100)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_shape_grid(dtype, D, bs, G, math_path):
    if dtype == "f32" and math_path != "auto":
        pytest.skip("fp32 always uses the CUDA-core path")
    cfg = _grid_cfg(dtype, D, bs, G)
    inp = wl.make_decode_inputs(cfg, 1000 + D + bs + G, context_lens=GRID_LENS)
    b, got = _run(inp)
    assert_close(got, oracle_outputs(inp), dtype, f"{dtype} D{D} bs{bs} G{G}")
    _no_device_error()


@pytest.mark.parametrize("G", [3, 6, 12, 16])
def test_uneven_and_wide_groups(G, math_path):
    """Groups that are not a power of two, or wider than one query chunk."""
    cfg = _grid_cfg("bf16", 128, 16, G)
    inp = wl.make_decode_inputs(cfg, 77 + G, context_lens=(5, 700, 64, 1))
    b, got = _run(inp)
    assert_close(got, oracle_outputs(inp), "bf16", f"G{G}")
    _no_device_error()


@pytest.mark.parametrize("P", [32, 64, 96, 512, 1024])
def test_partition_sizes(P, math_path, merge_mode):
    cfg = _grid_cfg("f16", 128, 16, 4)
    inp = wl.make_decode_inputs(cfg, 5, context_lens=(1, 95, 96, 97, 1023, 1024, 1025, 2500))
    b, got = _run(inp, partition_size=P)
    assert_close(got, oracle_outputs(inp), "f16", f"P{P}")
    _no_device_error()


def test_split_vs_single_pass(math_path, merge_mode):
    cfg = _grid_cfg("bf16", 128, 16, 8)
    inp = wl.make_decode_inputs(cfg, 6, context_lens=(1000, 17, 640, 1024))
    ref = oracle_outputs(inp)
    b = DeviceBatch(inp)
    b.step_write()
    single = to_storage(b.decode(partition_size=1024), "bf16")
    split = to_storage(b.decode(partition_size=64), "bf16")
    assert_close(single, ref, "bf16", "single")
    assert_close(split, ref, "bf16", "split")
    assert_close(split, widen(single, "bf16"), "bf16", "split vs single")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("P", [64, 0])
def test_write_decode_equals_write_then_decode(dtype, P, math_path, merge_mode):
    """pa_write_decode (the write and the plan in one kernel when the batch is
    split) gives the bits of pa_cache_write followed by pa_decode: the same
    pools and the same outputs, and those match the oracle."""
    if dtype == "f32" and math_path != "auto":
        pytest.skip("fp32 always uses the CUDA-core path")
    cfg = _grid_cfg(dtype, 128, 16, 4)
    lens = (0, 1, 33, 300, 700, 1100) if P else (0, 1, 33, 300, 511, 17)
    inp = wl.make_decode_inputs(cfg, 60 + P, context_lens=lens)
    a = DeviceBatch(inp)
    a.step_write()
    out_a = a.decode(partition_size=P)
    b = DeviceBatch(inp)
    # the same rows and slots as DeviceBatch.step_write, through the fused call
    S = len(b.lens)
    hkv, d = cfg.num_kv_heads, cfg.head_dim
    sd = inp.k_hist[0].dtype
    slots = np.full(S, -1, dtype=np.int64)
    k = np.zeros((S, hkv, d), dtype=sd)
    v = np.zeros((S, hkv, d), dtype=sd)
    for s_ in range(S):
        n = int(b.lens[s_])
        if n > 0:
            slots[s_] = b.bm.slots(s_, n - 1, 1)[0]
            k[s_] = inp.k_hist[s_][n - 1]
            v[s_] = inp.v_hist[s_][n - 1]
    out_b = torch.empty_like(b.q)
    n0 = pa.launch_count()
    pa.pa_write_decode(to_device(k, dtype), to_device(v, dtype), torch.from_numpy(slots).cuda(), out_b, b.q,
                       b.k_cache, b.v_cache, b.block_tables, b.context_lens, cfg.scale,
                       max_context_len=int(b.lens.max()), partition_size=P)
    torch.cuda.synchronize()
    launches = pa.launch_count() - n0
    _no_device_error()
    split = max(lens) > (P or 512)
    fused = merge_mode == "fused"
    # split: write+plan, decode (+ reduce); one partition: write, decode
    assert launches == ((2 if fused else 3) if split else 2)
    # bit patterns (the untouched pool cells hold a NaN sentinel)
    bits = lambda t: np.ascontiguousarray(to_storage(t, dtype)).view(np.uint8)      # noqa: E731
    assert np.array_equal(bits(out_a), bits(out_b))
    assert np.array_equal(bits(a.k_cache), bits(b.k_cache))
    assert np.array_equal(bits(a.v_cache), bits(b.v_cache))
    assert_close(to_storage(out_b, dtype), oracle_outputs(inp), dtype, f"write_decode {dtype} P{P}")
    assert_cache_exact(b)


def test_cache_write_bit_exact_all_dtypes():
    for dtype in ("f32", "f16", "bf16"):
        cfg = _grid_cfg(dtype, 128, 8, 2)
        inp = wl.make_decode_inputs(cfg, 9, context_lens=(0, 1, 7, 8, 9, 130))
        b = DeviceBatch(inp)
        b.step_write()
        torch.cuda.synchronize()
        assert_cache_exact(b)
    _no_device_error()


def test_block_permutation_is_bitwise_invariant(math_path):
    cfg = _grid_cfg("bf16", 128, 16, 8)
    lens = (3, 200, 777, 1500)
    inp = wl.make_decode_inputs(cfg, 10, context_lens=lens)
    r = np.random.default_rng(123)
    nb2, t2 = wl.shuffled_tables(r, wl.blocks_for(lens, 16), inp.num_blocks + 37, 0)
    outs = []
    for tables, nb in ((inp.block_tables, inp.num_blocks), (t2, nb2)):
        b = DeviceBatch(inp, tables=tables, num_blocks=nb)
        b.step_write()
        outs.append(to_storage(b.decode(), "bf16"))
    assert np.array_equal(outs[0], outs[1])
    assert_close(outs[0], oracle_outputs(inp), "bf16")


def test_shared_prefix_matches_private_copies_bitwise(math_path):
    """Sequences that fork a prefix holder (shared blocks, copy-on-write on the
    first divergent write) give the same bits as sequences holding copies."""
    cfg = _grid_cfg("f16", 128, 16, 4)
    hkv, D, bs = cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    r = np.random.default_rng(31)
    prefix = 100                                      # not block aligned: 6 full + 4 rows
    tails = [40, 1, 300]
    Kp = wl.normal_storage(r, (prefix, hkv, D), "f16")
    Vp = wl.normal_storage(r, (prefix, hkv, D), "f16")
    Kt = [wl.normal_storage(r, (n, hkv, D), "f16") for n in tails]
    Vt = [wl.normal_storage(r, (n, hkv, D), "f16") for n in tails]
    q = to_device(wl.normal_storage(r, (3, cfg.num_heads, D), "f16"), "f16")
    nb = 200
    kc = torch.zeros((nb, bs, hkv, D), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    bm = pa.BlockManager(nb, bs, r.permutation(nb).tolist())
    holder = 1000
    bm.allocate(holder, prefix)
    pa.pa_cache_write(to_device(Kp, "f16"), to_device(Vp, "f16"), kc, vc,
                      torch.from_numpy(bm.slots(holder, 0, prefix)).cuda())
    for s in range(3):
        bm.fork(holder, s)
        for i in range(tails[s]):
            slot, src, dst = bm.append_slot(s)
            if src >= 0:
                pa.pa_copy_blocks(kc, vc, torch.tensor([[src, dst]], dtype=torch.int32, device="cuda"))
            pa.pa_cache_write(to_device(Kt[s][i:i + 1], "f16"), to_device(Vt[s][i:i + 1], "f16"), kc, vc,
                              torch.tensor([slot], dtype=torch.int64, device="cuda"))
    width = max(len(bm.block_table(s)) for s in range(3))
    tabs, lens = bm.pack([0, 1, 2], width)
    out_shared = torch.empty_like(q)
    pa.pa_decode(out_shared, q, kc, vc, torch.from_numpy(tabs).cuda(), torch.from_numpy(lens).cuda(), cfg.scale,
                 bs, hkv, max_context_len=int(lens.max()))
    # private copies: every sequence allocates its own blocks
    kc2 = torch.zeros_like(kc)
    vc2 = torch.zeros_like(vc)
    bm2 = pa.BlockManager(nb, bs, list(range(nb)))
    for s in range(3):
        n = prefix + tails[s]
        bm2.allocate(s, n)
        Kh = np.concatenate([Kp, Kt[s]])
        Vh = np.concatenate([Vp, Vt[s]])
        pa.pa_cache_write(to_device(Kh, "f16"), to_device(Vh, "f16"), kc2, vc2,
                          torch.from_numpy(bm2.slots(s, 0, n)).cuda())
    tabs2, lens2 = bm2.pack([0, 1, 2], width)
    out_priv = torch.empty_like(q)
    pa.pa_decode(out_priv, q, kc2, vc2, torch.from_numpy(tabs2).cuda(), torch.from_numpy(lens2).cuda(), cfg.scale,
                 bs, hkv, max_context_len=int(lens2.max()))
    assert np.array_equal(to_storage(out_shared, "f16"), to_storage(out_priv, "f16"))
    ref = np.stack([oa.decode_history(widen(to_storage(q[s], "f16"), "f16"),
                                      widen(np.concatenate([Kp, Kt[s]]), "f16"),
                                      widen(np.concatenate([Vp, Vt[s]]), "f16"), cfg.scale) for s in range(3)])
    assert_close(to_storage(out_shared, "f16"), ref, "f16")
    _no_device_error()


def test_copy_blocks_bit_exact():
    nb, bs, hkv, D = 12, 16, 4, 64
    g = torch.Generator(device="cuda").manual_seed(3)
    kc = torch.randn((nb, bs, hkv, D), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn((nb, bs, hkv, D), generator=g, device="cuda").to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    pairs = torch.tensor([[1, 7], [3, 0], [11, 5]], dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(kc, vc, pairs)
    exp_k, exp_v = k0.clone(), v0.clone()
    for s, d in [(1, 7), (3, 0), (11, 5)]:
        exp_k[d] = k0[s]
        exp_v[d] = v0[s]
    assert torch.equal(kc.view(torch.int16), exp_k.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), exp_v.view(torch.int16))
    _no_device_error()


def test_long_context_with_outlier_keys(math_path, merge_mode):
    """Two 8192-token sequences, 1% of K rows scaled by 8, 512-token partitions."""
    cfg = wl.DecodeConfig("longsmall", "bf16", 2, 64, 8, 128, 16, "const", len_lo=8192, len_hi=8192,
                          partition_size=512, outlier_frac=0.01)
    inp = wl.make_decode_inputs(cfg, 3)
    b, got = _run(inp, partition_size=512)
    assert_close(got, oracle_outputs(inp), "bf16", "long")
    _no_device_error()


def test_device_errors_are_flagged_not_faulted():
    cfg = _grid_cfg("bf16", 128, 16, 8)
    inp = wl.make_decode_inputs(cfg, 12, context_lens=(40, 70))
    b = DeviceBatch(inp)
    b.step_write()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    # block id past the pool: clamped and flagged
    bad = b.block_tables.clone()
    bad[1, 2] = b.nb + 5
    out = torch.empty_like(b.q)
    pa.pa_decode(out, b.q, b.k_cache, b.v_cache, bad, b.context_lens, cfg.scale, 16, cfg.num_kv_heads,
                 max_context_len=70)
    assert pa.pa_get_device_error() & pa.DEVERR_BLOCK_ID
    # context longer than max_context_len: clamped and flagged
    pa.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, cfg.scale, 16,
                 cfg.num_kv_heads, max_context_len=50)
    assert pa.pa_get_device_error() & pa.DEVERR_CONTEXT_LEN
    # slot past the pool: skipped and flagged
    k1 = b.q[:1, :cfg.num_kv_heads].contiguous()
    pa.pa_cache_write(k1, k1, b.k_cache, b.v_cache,
                      torch.tensor([b.nb * 16 + 3], dtype=torch.int64, device="cuda"))
    assert pa.pa_get_device_error() & pa.DEVERR_SLOT
    # everything still works afterwards
    got = to_storage(b.decode(), "bf16")
    assert_close(got, oracle_outputs(inp), "bf16")
    _no_device_error()


def test_argument_errors_are_synchronous():
    cfg = _grid_cfg("bf16", 128, 16, 8)
    inp = wl.make_decode_inputs(cfg, 13, context_lens=(10,))
    b = DeviceBatch(inp)
    out = torch.empty_like(b.q)
    wide = torch.zeros((1, 400), dtype=torch.int32, device="cuda")    # valid ids, wide enough for 5000 tokens
    ptrs = (out.data_ptr(), b.q.data_ptr(), b.k_cache.data_ptr(), b.v_cache.data_ptr(),
            wide.data_ptr(), b.context_lens.data_ptr())

    def call(bs=16, hkv=2, hq=16, D=128, mcl=10):
        return pa.lib().pa_decode(*ptrs, 0.1, bs, hkv, 1, hq, D, 400, mcl, b.nb, 2, 0, None, 0, None)

    assert call(D=96) == 2           # head_dim 96 unsupported
    assert call(hkv=3) == 1          # 16 query heads are not a multiple of 3 kv heads
    assert call(mcl=5000) == 1       # split-K needed but no workspace given
    assert call(bs=12) == 2          # block size 12 unsupported
    torch.cuda.synchronize()
    _no_device_error()


def test_pa_step_from_host_buffers_matches_device_path():
    cfg = wl.CONFIGS["70b"]
    inp = wl.make_decode_inputs(cfg, 21, context_lens=np.array([3000, 17, 600, 1, 4096, 250]))
    b = DeviceBatch(inp)
    # device path
    b.step_write()
    ref_dev = to_storage(b.decode(), "bf16")
    # host path: same step again from pinned host buffers (rewrites identical rows)
    S, Hq, D = b.q.shape
    hkv = cfg.num_kv_heads
    slots = np.array([b.bm.slots(s, int(n) - 1, 1)[0] for s, n in enumerate(b.lens)], dtype=np.int64)
    k_new = np.stack([inp.k_hist[s][-1] for s in range(S)])
    v_new = np.stack([inp.v_hist[s][-1] for s in range(S)])
    pin = lambda t: t.pin_memory()
    host = {"q": pin(b.q.cpu()), "k": pin(to_device(k_new, "bf16", "cpu")), "v": pin(to_device(v_new, "bf16", "cpu")),
            "slot_mapping": pin(torch.from_numpy(slots)), "block_tables": pin(b.block_tables.cpu()),
            "context_lens": pin(b.context_lens.cpu()), "out": pin(torch.empty_like(b.q, device="cpu"))}
    dev = {k: torch.empty_like(v, device="cuda") for k, v in host.items()}
    mcl = int(b.lens.max())
    dev["workspace"] = torch.empty(max(1, pa.pa_decode_workspace_size(S, Hq, D, mcl)), dtype=torch.uint8,
                                   device="cuda")
    pa.pa_step(host, dev, b.k_cache, b.v_cache, cfg.scale, mcl)
    torch.cuda.synchronize()
    assert np.array_equal(to_storage(host["out"], "bf16"), ref_dev)
    assert_close(ref_dev, oracle_outputs(inp), "bf16")
    _no_device_error()


def test_pipeline_overlapped_steps_match_device_path():
    """pa_pipeline over 5 steps with 2 staging sets, a different query per step
    (own pinned host buffers): every step's host output equals the device
    path's decode of the same query, bit for bit."""
    cfg = wl.CONFIGS["70b"]
    inp = wl.make_decode_inputs(cfg, 22, context_lens=np.array([3000, 17, 600, 1, 4096, 250, 70]))
    b = DeviceBatch(inp)
    b.step_write()
    S, Hq, D = b.q.shape
    slots = np.array([b.bm.slots(s, int(n) - 1, 1)[0] for s, n in enumerate(b.lens)], dtype=np.int64)
    k_new = np.stack([inp.k_hist[s][-1] for s in range(S)])
    v_new = np.stack([inp.v_hist[s][-1] for s in range(S)])
    pin = lambda t: t.pin_memory()
    mcl = int(b.lens.max())
    g = torch.Generator(device="cuda").manual_seed(5)
    qs = [torch.randn((S, Hq, D), generator=g, device="cuda").to(torch.bfloat16) for _ in range(5)]
    refs = []
    for q in qs:
        out = torch.empty_like(q)
        pa.pa_decode(out, q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, cfg.scale, max_context_len=mcl)
        refs.append(to_storage(out, "bf16"))
    common = {"k": pin(to_device(k_new, "bf16", "cpu")), "v": pin(to_device(v_new, "bf16", "cpu")),
              "slot_mapping": pin(torch.from_numpy(slots)), "block_tables": pin(b.block_tables.cpu()),
              "context_lens": pin(b.context_lens.cpu())}
    hosts = [dict(common, q=pin(q.cpu()), out=pin(torch.full_like(q, float("nan"), device="cpu"))) for q in qs]
    ws = torch.empty(max(1, pa.pa_decode_workspace_size(S, Hq, D, mcl)), dtype=torch.uint8, device="cuda")
    sets = []
    for _ in range(2):
        d = {k: torch.empty_like(v, device="cuda") for k, v in hosts[0].items()}
        d["workspace"] = ws
        sets.append(d)
    pipe = pa.Pipeline(2)
    pipe.begin(b.k_cache)
    for i, h in enumerate(hosts):
        pipe.step(i % 2, h, sets[i % 2], b.k_cache, b.v_cache, cfg.scale, mcl)
    pipe.end(b.k_cache)
    torch.cuda.synchronize()
    for h, ref in zip(hosts, refs):
        assert np.array_equal(to_storage(h["out"], "bf16"), ref)
    _no_device_error()


def test_launch_count_and_profile(merge_mode):
    cfg = _grid_cfg("bf16", 128, 16, 8)
    inp = wl.make_decode_inputs(cfg, 14, context_lens=(2000, 30))
    b = DeviceBatch(inp)
    n0 = pa.launch_count()
    pa.profile_begin()
    b.step_write()
    b.decode()
    prof = pa.profile_end()
    fused = merge_mode == "fused"
    # cache write, plan, decode (+ reduce when partitions are merged by their own kernel)
    assert pa.launch_count() - n0 == (3 if fused else 4)
    assert prof["decode"][1] == 1 and prof["decode"][0] > 0
    assert prof["plan"][1] == 1 and prof["cache_write"][1] == 1
    assert prof["reduce"][1] == (0 if fused else 1)


# -- full-size workloads, every row, in the bench's launch configuration ----------

@pytest.mark.parametrize("name", ["7b", "70b", "long"])
def test_full_size_every_row(name, math_path, merge_mode):
    """Every (sequence, head) row of the full-size batch against the fp64
    oracle, element by element."""
    cfg = wl.CONFIGS[name]
    d = wl.draw_device(cfg, 0)
    batch = PagedBatch(d.k_hist, d.v_hist, d.offsets, d.context_lens, d.num_blocks, cfg.block_size,
                       d.free_order)
    batch.write_new_tokens()
    out = torch.empty_like(d.q)
    batch.decode(out, d.q, cfg.scale, partition_size=cfg.partition_size)
    torch.cuda.synchronize()
    _no_device_error()
    ref = oracle_all_rows(d.q, d, cfg)
    assert_every_row(out, ref, cfg.dtype, f"{name} ({math_path}, {merge_mode})")
