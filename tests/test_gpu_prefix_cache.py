"""Prefix cache on the GPU: multi-turn conversations over shared system prompts.

Prefix caching ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
section "Prefix Caching前缀复用优化"): a request whose prompt begins with cached
KV references those blocks and skips their prefill.

The workload (tests/prefix_workload.py) drives the C++ block manager with the
cache on.  On the device: K/V rows are written with pa_cache_write only past
the cached prefix of each prompt, and one row per sequence per decode step;
pa_decode runs over the batch.  Checked:
  * the reused rows in the device pools equal freshly drawn rows bit for bit;
  * decode outputs against the fp64 oracle computed from freshly drawn rows
    for the full token sequence (no cache involved);
  * rows written = tokens - cached tokens, the cached share is large, and some
    continued conversations lost blocks to eviction.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from oracle import attention as oa
from oracle.numerics import widen
from tests.gpu_harness import assert_close, sentinel_pool, to_device, to_storage
from tests.prefix_workload import BS, D, HKV, HQ, SEED, run_conversations

pytestmark = pytest.mark.gpu


def _rows(tokens, start, dtype, salt):
    return wl.prefix_rows(SEED, tokens, start, HKV, D, dtype, salt)


class _Device:
    def __init__(self, dtype, num_blocks):
        self.dtype = dtype
        self.kc = sentinel_pool(num_blocks, BS, HKV, D, dtype)
        self.vc = sentinel_pool(num_blocks, BS, HKV, D, dtype)
        self.r = np.random.default_rng(99)
        self.checks = 0
        self.reused_checked = 0

    def prefill(self, bm, seq, toks, cached):
        dt, n = self.dtype, len(toks)
        if n > cached:
            slots = torch.from_numpy(bm.slots(seq, cached, n - cached)).cuda()
            pa.pa_cache_write(to_device(_rows(toks, cached, dt, 0), dt), to_device(_rows(toks, cached, dt, 1), dt),
                              self.kc, self.vc, slots)
        if cached:
            # the reused rows are the rows a fresh prefill would have written
            sl = bm.slots(seq, 0, cached)
            pos = np.unique(np.concatenate([np.arange(min(4, cached)), np.arange(cached - min(4, cached), cached),
                                            self.r.integers(0, cached, 8)]))
            idx = torch.from_numpy(sl[pos]).cuda()
            kd = to_storage(self.kc.view(-1, HKV, D)[idx], dt)
            vd = to_storage(self.vc.view(-1, HKV, D)[idx], dt)
            assert np.array_equal(kd, _rows(toks, 0, dt, 0)[pos])
            assert np.array_equal(vd, _rows(toks, 0, dt, 1)[pos])
            self.reused_checked += len(pos)

    def append(self, bm, batch, slots):
        dt = self.dtype
        k = np.concatenate([_rows(toks, len(toks) - 1, dt, 0) for _, _, _, toks in batch])
        v = np.concatenate([_rows(toks, len(toks) - 1, dt, 1) for _, _, _, toks in batch])
        pa.pa_cache_write(to_device(k, dt), to_device(v, dt), self.kc, self.vc,
                          torch.tensor(slots, dtype=torch.int64, device="cuda"))

    def decode(self, bm, batch, step):
        dt = self.dtype
        ids = [b[0] for b in batch]
        width = max(len(bm.block_table(s)) for s in ids)
        tabs, lens = bm.pack(ids, width)
        q_store = np.stack([wl.token_rows(SEED, 7, [s * 1000 + step], HQ, D, dt, salt=2)[0] for s in ids])
        q = to_device(q_store, dt)
        out = torch.empty_like(q)
        scale = 1.0 / np.sqrt(D)
        pa.pa_decode(out, q, self.kc, self.vc, torch.from_numpy(np.ascontiguousarray(tabs)).cuda(),
                     torch.from_numpy(lens).cuda(), scale, BS, HKV, max_context_len=int(lens.max()))
        got = to_storage(out, dt)
        G = HQ // HKV
        for i, (s, _, _, toks) in enumerate(batch):
            K = widen(_rows(toks, 0, dt, 0), dt)
            V = widen(_rows(toks, 0, dt, 1), dt)
            qq = widen(q_store[i], dt)
            ref = np.stack([oa.attend(qq[h], K[:, h // G, :], V[:, h // G, :], scale) for h in range(HQ)])
            assert_close(got[i], ref, dt, f"seq {s} step {step}")
            self.checks += 1

    def finish_wave(self):
        assert pa.pa_get_device_error() == 0


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_multi_turn_prefix_reuse(dtype):
    dev = _Device(dtype, 300)
    st = run_conversations(dev, num_blocks=300)
    assert st["written"] + st["cached"] == st["total"]
    assert st["cached"] > 0.4 * st["total"], st
    assert st["short"] > 0 and st["cache_stats"][2] > 0
    assert dev.checks > 0 and dev.reused_checked > 0
