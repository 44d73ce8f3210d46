"""GPU tests of the host swap path: pa_swap_blocks between a device pool and a
pinned host pool (bit-exact both ways), and a decode batch whose sequences are
swapped out, their GPU blocks reused and overwritten, then swapped back in:
the decode output is bit-identical to the output before the swap."""

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from tests.gpu_harness import DeviceBatch, to_device, to_storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_381_b200 import build
    build.build()
    pa.pa_get_device_error()
    yield


def _pools(nb, bs, hkv, d, dtype, device):
    tt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    if device == "pinned":
        k = torch.empty((nb, bs, hkv, d), dtype=tt).pin_memory()
        v = torch.empty((nb, bs, hkv, d), dtype=tt).pin_memory()
        k.view(torch.uint8).fill_(0xAB)
        v.view(torch.uint8).fill_(0xCD)
        return k, v
    k = torch.randn((nb, bs, hkv, d), device="cuda").to(tt)
    v = torch.randn((nb, bs, hkv, d), device="cuda").to(tt)
    return k, v


@pytest.mark.parametrize("dtype,bs,hkv,d", [("bf16", 16, 8, 128), ("f16", 8, 32, 128), ("f32", 32, 4, 64)])
def test_round_trip_bit_exact(dtype, bs, hkv, d):
    r = np.random.default_rng(3)
    nb_dev, nb_host, n = 300, 200, 120
    dk, dv = _pools(nb_dev, bs, hkv, d, dtype, "cuda")
    hk, hv = _pools(nb_host, bs, hkv, d, dtype, "pinned")
    src = r.choice(nb_dev, n, replace=False).astype(np.int32)
    dst = r.choice(nb_host, n, replace=False).astype(np.int32)
    pairs = torch.from_numpy(np.stack([src, dst], 1).copy()).cuda()
    pa.pa_swap_blocks(hk, hv, dk, dv, pairs)                 # device -> host
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    idx_s, idx_d = torch.from_numpy(src).long(), torch.from_numpy(dst).long()
    assert torch.equal(hk[idx_d].view(torch.uint8), dk.cpu()[idx_s].view(torch.uint8))
    assert torch.equal(hv[idx_d].view(torch.uint8), dv.cpu()[idx_s].view(torch.uint8))
    untouched = np.setdiff1d(np.arange(nb_host), dst)
    assert (hk[torch.from_numpy(untouched).long()].view(torch.uint8) == 0xAB).all()
    # host -> device into other blocks, pairs given in pinned host memory
    back = r.choice(nb_dev, n, replace=False).astype(np.int32)
    pairs_h = torch.from_numpy(np.stack([dst, back], 1).copy()).pin_memory()
    ref_k, ref_v = dk.clone(), dv.clone()
    pa.pa_swap_blocks(dk, dv, hk, hv, pairs_h)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    idx_b = torch.from_numpy(back).long().cuda()
    assert torch.equal(dk[idx_b].view(torch.uint8), ref_k[idx_s.cuda()].view(torch.uint8))
    assert torch.equal(dv[idx_b].view(torch.uint8), ref_v[idx_s.cuda()].view(torch.uint8))
    keep = torch.from_numpy(np.setdiff1d(np.arange(nb_dev), back)).long().cuda()
    assert torch.equal(dk[keep].view(torch.uint8), ref_k[keep].view(torch.uint8))


def test_pageable_host_memory_is_rejected():
    dk, dv = _pools(16, 16, 2, 64, "bf16", "cuda")
    hk = torch.empty((16, 16, 2, 64), dtype=torch.bfloat16)          # pageable: not reachable from kernels
    hv = torch.empty_like(hk)
    pairs = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    lib = pa.lib()
    from paged_kv_cache_381_b200 import _native
    desc = _native.CacheDesc(0, 16, 2, 64, 2)
    import ctypes
    st = lib.pa_swap_blocks(ctypes.c_void_p(hk.data_ptr()), ctypes.c_void_p(hv.data_ptr()), 16,
                            ctypes.c_void_p(dk.data_ptr()), ctypes.c_void_p(dv.data_ptr()), 16,
                            ctypes.c_void_p(pairs.data_ptr()), 1, ctypes.byref(desc), ctypes.c_void_p(0))
    assert st == 1
    with pytest.raises(ValueError):
        pa.pa_swap_blocks(hk, hv, dk, dv, pairs)


def test_out_of_range_ids_are_flagged_not_faulted():
    dk, dv = _pools(8, 16, 2, 64, "bf16", "cuda")
    hk, hv = _pools(4, 16, 2, 64, "bf16", "pinned")
    before = hk.clone()
    pairs = torch.tensor([[0, 4], [8, 0], [-1, 1]], dtype=torch.int32, device="cuda")
    pa.pa_get_device_error()
    pa.pa_swap_blocks(hk, hv, dk, dv, pairs)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() & 2
    assert torch.equal(hk.view(torch.uint8), before.view(torch.uint8))


def test_swapped_sequences_decode_bit_identical():
    """Swap out half the batch, let another sequence take and overwrite the
    freed GPU blocks, release it, swap back in (other blocks), decode again."""
    cfg = wl.DecodeConfig("swap", "bf16", 6, 32, 8, 128, 16, "fixed", fixed_lengths=(1, 17, 100, 300, 640, 1500),
                          num_blocks=0, spare=0.6)
    inp = wl.make_decode_inputs(cfg, 4)
    b = DeviceBatch(inp)
    b.step_write()
    before = to_storage(b.decode(), "bf16")
    bm = b.bm
    bm.set_cpu_blocks(200)
    hk = torch.empty((200,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_seqs = [1, 3, 5]
    for s in out_seqs:
        pairs = bm.swap_out(s)
        assert len(pairs) == len(bm.block_table(s))
        pa.pa_swap_blocks(hk, hv, b.k_cache, b.v_cache, torch.from_numpy(pairs).cuda())
    # another request takes every free GPU block and fills it with other values
    filler = 99
    nfree = bm.num_free
    bm.allocate(filler, nfree * b.bs)
    vacated = {int(x) for s in out_seqs for x in inp.block_tables[s] if x >= 0}
    assert vacated <= set(bm.block_table(filler))        # every block the swap freed is overwritten
    slots = torch.from_numpy(bm.slots(filler, 0, nfree * b.bs)).cuda()
    junk = torch.randn((nfree * b.bs, 8, 128), device="cuda").to(torch.bfloat16)
    pa.pa_cache_write(junk, junk, b.k_cache, b.v_cache, slots)
    bm.free(filler)
    for s in out_seqs:
        pairs = bm.swap_in(s)
        pa.pa_swap_blocks(b.k_cache, b.v_cache, hk, hv, torch.from_numpy(pairs).cuda())
    tabs, lens = bm.pack(list(range(len(inp.context_lens))), b.block_tables.shape[1])
    b.block_tables = torch.from_numpy(np.ascontiguousarray(tabs)).cuda()
    after = to_storage(b.decode(), "bf16")
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    assert np.array_equal(before, after)
