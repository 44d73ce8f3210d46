"""Helpers shared by the GPU parity tests.

Inputs come from the seeded generators; the device cache is filled through the
product's own path (host block manager slots + pa_cache_write); expected values
come only from the oracle, computed from the generators' histories."""

import numpy as np
import torch

import paged_kv_cache_381_b200 as pa
from oracle import attention as oa
from oracle import cache as oc
from oracle.numerics import widen

TORCH_DTYPE = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
TOL = {"f32": (1e-5, 1e-5), "f16": (2e-3, 1e-2), "bf16": (2e-3, 1e-2)}   # (abs, rel)
SENTINEL = {"f32": 0x7FC00000, "f16": 0x7E00, "bf16": 0x7FC0}              # quiet NaN bit patterns


def to_device(stored, dtype, device="cuda"):
    """Storage-form numpy array -> CUDA tensor of the dtype (bit-exact)."""
    a = np.ascontiguousarray(stored)
    if dtype == "f32":
        return torch.from_numpy(a.view(np.float32)).to(device)
    t = torch.from_numpy(a.view(np.int16))
    return t.to(device).view(TORCH_DTYPE[dtype])


def to_storage(t, dtype):
    """CUDA tensor -> storage-form numpy array (bit-exact)."""
    if dtype == "f32":
        return t.detach().cpu().numpy().astype(np.float32)
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def sentinel_pool(nb, bs, hkv, d, dtype, device="cuda"):
    if dtype == "f32":
        return torch.full((nb, bs, hkv, d), SENTINEL["f32"], dtype=torch.int32, device=device).view(torch.float32)
    return torch.full((nb, bs, hkv, d), SENTINEL[dtype], dtype=torch.int16, device=device).view(TORCH_DTYPE[dtype])


def free_order_for(tables, num_blocks):
    """Free-list order under which allocating the sequences in order reproduces
    ``tables`` (blocks are taken from the end of the list)."""
    used = [int(b) for row in tables for b in row if b >= 0]
    taken = set(used)
    rest = [b for b in range(num_blocks) if b not in taken]
    return list(reversed(used + rest))


class DeviceBatch:
    """A decode batch resident on the GPU, filled through the product path.

    All history rows but the last are written first ("prefill"); the step then
    writes each sequence's newest token with pa_cache_write and decodes.
    """

    def __init__(self, inp, block_size=None, tables=None, num_blocks=None, device="cuda"):
        cfg = inp.cfg
        self.inp, self.cfg, self.dtype = inp, cfg, cfg.dtype
        self.bs = block_size or cfg.block_size
        self.tables = inp.block_tables if tables is None else tables
        self.nb = inp.num_blocks if num_blocks is None else num_blocks
        self.lens = np.asarray(inp.context_lens, dtype=np.int64)
        S = len(self.lens)
        self.bm = pa.BlockManager(self.nb, self.bs, free_order_for(self.tables, self.nb))
        for s in range(S):
            self.bm.allocate(s, int(self.lens[s]))
            assert self.bm.block_table(s) == [int(b) for b in self.tables[s] if b >= 0]
        hkv, d = cfg.num_kv_heads, cfg.head_dim
        self.k_cache = sentinel_pool(self.nb, self.bs, hkv, d, self.dtype, device)
        self.v_cache = sentinel_pool(self.nb, self.bs, hkv, d, self.dtype, device)
        # prefill: positions [0, ctx-1)
        slots, krows, vrows = [], [], []
        for s in range(S):
            n = int(self.lens[s])
            if n > 1:
                slots.append(self.bm.slots(s, 0, n - 1))
                krows.append(inp.k_hist[s][:n - 1])
                vrows.append(inp.v_hist[s][:n - 1])
        if slots:
            self._write(np.concatenate(slots), np.concatenate(krows), np.concatenate(vrows))
        width = max(1, self.tables.shape[1])
        tabs, ctx = self.bm.pack(list(range(S)), width)
        self.block_tables = torch.from_numpy(np.ascontiguousarray(tabs)).to(device)
        self.context_lens = torch.from_numpy(ctx).to(device)
        self.q = to_device(inp.q, self.dtype, device)

    def _write(self, slots, k, v):
        dt = self.dtype
        pa.pa_cache_write(to_device(k, dt), to_device(v, dt), self.k_cache, self.v_cache,
                          torch.from_numpy(np.asarray(slots, dtype=np.int64)).cuda())

    def step_write(self):
        """Write every sequence's newest token (slot -1 for empty sequences)."""
        S = len(self.lens)
        hkv, d = self.cfg.num_kv_heads, self.cfg.head_dim
        sd = self.inp.k_hist[0].dtype if self.inp.k_hist else np.float32
        slots = np.full(S, -1, dtype=np.int64)
        k = np.zeros((S, hkv, d), dtype=sd)
        v = np.zeros((S, hkv, d), dtype=sd)
        for s in range(S):
            n = int(self.lens[s])
            if n > 0:
                slots[s] = self.bm.slots(s, n - 1, 1)[0]
                k[s] = self.inp.k_hist[s][n - 1]
                v[s] = self.inp.v_hist[s][n - 1]
        self._write(slots, k, v)

    def decode(self, partition_size=0, max_context_len=None, out=None):
        if out is None:
            out = torch.empty_like(self.q)
        mcl = int(self.lens.max()) if max_context_len is None else max_context_len
        pa.pa_decode(out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                     self.cfg.scale, self.bs, self.cfg.num_kv_heads, max_context_len=mcl,
                     partition_size=partition_size)
        return out


def oracle_outputs(inp, rows=None):
    """fp64 oracle from the histories, through the oracle's own paged path."""
    cfg = inp.cfg
    bs = cfg.block_size
    S = len(inp.context_lens)
    sd = np.float32 if cfg.dtype == "f32" else np.uint16
    hkv, d = cfg.num_kv_heads, cfg.head_dim
    if rows is None:
        nb = inp.num_blocks
        kc = np.zeros((nb, bs, hkv, d), dtype=sd)
        vc = np.zeros((nb, bs, hkv, d), dtype=sd)
        for s in range(S):
            kc, vc = oc.scatter_history(inp.k_hist[s], inp.v_hist[s], inp.block_tables[s], kc, vc)
        return oa.paged_decode(inp.q, kc, vc, inp.block_tables, inp.context_lens, cfg.scale, bs, cfg.dtype)
    G = cfg.num_heads // hkv
    res = []
    for s, h in rows:
        g = h // G
        K = widen(inp.k_hist[s][:, g, :], cfg.dtype)
        V = widen(inp.v_hist[s][:, g, :], cfg.dtype)
        res.append(oa.attend(widen(inp.q[s, h], cfg.dtype), K, V, cfg.scale))
    return np.stack(res)


def assert_close(got_storage, ref, dtype, what=""):
    atol, rtol = TOL[dtype]
    got = widen(got_storage, dtype)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first {idx.tolist()}; "
                             f"max err {float(np.nanmax(err))}")


def assert_cache_exact(batch):
    """Every live token's K/V row in the device pools equals its history row
    bit for bit; every other cell still holds the sentinel."""
    dt = batch.dtype
    kc = to_storage(batch.k_cache, dt)
    vc = to_storage(batch.v_cache, dt)
    sent = np.array(SENTINEL[dt], dtype=kc.dtype if dt != "f32" else np.uint32)
    kcb = kc.view(np.uint32) if dt == "f32" else kc
    vcb = vc.view(np.uint32) if dt == "f32" else vc
    live = np.zeros(kc.shape[:2], dtype=bool)
    for s, n in enumerate(batch.lens.tolist()):
        for t in range(n):
            b, o = int(batch.tables[s][t // batch.bs]), t % batch.bs
            live[b, o] = True
            assert np.array_equal(kc[b, o], batch.inp.k_hist[s][t]), (s, t)
            assert np.array_equal(vc[b, o], batch.inp.v_hist[s][t]), (s, t)
    assert (kcb[~live] == sent).all() and (vcb[~live] == sent).all()
