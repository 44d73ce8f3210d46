"""A decode batch resident in paged device pools, built through the library.

``PagedBatch`` takes each sequence's contiguous K/V history on the device,
lets the native block manager assign physical blocks (from a given free-list
order), writes all history rows but each sequence's newest one into the pools
with ``pa_cache_write`` (a synthetic prefill), and keeps the newest rows plus
their slots for the decode step, which writes them and then decodes:

    batch.write_new_tokens()      # pa_cache_write of one token per sequence
    batch.decode(out)             # pa_decode over the block tables

With ``new_tokens = Q > 1`` the last Q rows of each history are held back
instead (a speculative step's candidate tokens), written together by
``write_new_tokens`` and attended by ``verify`` (pa_verify).
"""

import numpy as np
import torch

from . import (BlockManager, pa_cache_write, pa_decode, pa_decode_workspace_size, pa_verify,
               pa_verify_workspace_size, pa_write_decode)


class PagedBatch:
    def __init__(self, k_hist, v_hist, offsets, context_lens, num_blocks, block_size, free_order=None,
                 table_width=None, fill=None, new_tokens=1):
        dev = k_hist.device
        self.lens = np.asarray(context_lens, dtype=np.int64)
        self.offsets = np.asarray(offsets, dtype=np.int64)
        S = len(self.lens)
        self.num_seqs = S
        self.block_size = bs = int(block_size)
        self.num_blocks = int(num_blocks)
        _, hkv, d = k_hist.shape
        self.num_kv_heads, self.head_dim = hkv, d
        self.bm = BlockManager(self.num_blocks, bs, free_order)
        for s in range(S):
            self.bm.allocate(s, int(self.lens[s]))
        shape = (self.num_blocks, bs, hkv, d)
        if fill is None:
            self.k_cache = torch.empty(shape, dtype=k_hist.dtype, device=dev)
            self.v_cache = torch.empty(shape, dtype=k_hist.dtype, device=dev)
        else:
            self.k_cache, self.v_cache = fill(shape)
        # prefill: every history row except each sequence's newest Q ones, which the
        # step writes (rows ordered [sequence][i]; slot -1 where a context is shorter than Q)
        Q = self.new_tokens = int(new_tokens)
        rows, slots = [], []
        newest_rows, newest_slots = [], []
        for s in range(S):
            n = int(self.lens[s])
            sl = self.bm.slots(s, 0, n) if n else np.zeros(0, np.int64)
            k = min(n, Q)
            if n > k:
                rows.append(np.arange(self.offsets[s], self.offsets[s] + n - k))
                slots.append(sl[:n - k])
            for i in range(Q):
                p = n - Q + i
                newest_rows.append(int(self.offsets[s] + p) if p >= 0 else -1)
                newest_slots.append(int(sl[p]) if p >= 0 else -1)
        if rows:
            r = torch.from_numpy(np.concatenate(rows)).to(dev)
            sm = torch.from_numpy(np.concatenate(slots).astype(np.int64)).to(dev)
            chunk = 1 << 20
            for i in range(0, int(r.numel()), chunk):
                idx = r[i:i + chunk]
                pa_cache_write(k_hist.index_select(0, idx), v_hist.index_select(0, idx), self.k_cache,
                               self.v_cache, sm[i:i + chunk].contiguous())
        nr = torch.tensor([max(x, 0) for x in newest_rows], dtype=torch.int64, device=dev)
        self.k_new = k_hist.index_select(0, nr).contiguous()
        self.v_new = v_hist.index_select(0, nr).contiguous()
        self.slot_mapping = torch.tensor(newest_slots, dtype=torch.int64, device=dev)
        width = table_width or max(1, max(-(-int(n) // bs) for n in self.lens) if S else 1)
        tables, ctx = self.bm.pack(list(range(S)), width)
        self.tables_host = tables
        self.block_tables = torch.from_numpy(np.ascontiguousarray(tables)).to(dev)
        self.context_lens = torch.from_numpy(ctx).to(dev)
        self.max_context_len = int(self.lens.max()) if S else 0
        self.workspace = None

    def write_new_tokens(self, stream=None):
        pa_cache_write(self.k_new, self.v_new, self.k_cache, self.v_cache, self.slot_mapping, stream=stream)

    def ensure_workspace(self, num_heads, partition_size=0):
        if self.new_tokens > 1:
            need = pa_verify_workspace_size(self.num_seqs, self.new_tokens, num_heads, self.head_dim,
                                            self.max_context_len, partition_size)
        else:
            need = pa_decode_workspace_size(self.num_seqs, num_heads, self.head_dim, self.max_context_len,
                                            partition_size)
        if need and (self.workspace is None or self.workspace.numel() < need):
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.k_cache.device)
        return self.workspace

    def decode(self, out, q, scale, partition_size=0, stream=None):
        ws = self.ensure_workspace(q.shape[1], partition_size)
        return pa_decode(out, q, self.k_cache, self.v_cache, self.block_tables, self.context_lens, scale,
                         self.block_size, self.num_kv_heads, max_context_len=self.max_context_len,
                         partition_size=partition_size, workspace=ws, stream=stream)

    def step(self, out, q, scale, partition_size=0, stream=None):
        """write_new_tokens then decode, in one library call (pa_write_decode)."""
        ws = self.ensure_workspace(q.shape[1], partition_size)
        return pa_write_decode(self.k_new, self.v_new, self.slot_mapping, out, q, self.k_cache, self.v_cache,
                               self.block_tables, self.context_lens, scale, self.block_size, self.num_kv_heads,
                               max_context_len=self.max_context_len, partition_size=partition_size, workspace=ws,
                               stream=stream)

    def verify(self, out, q, scale, partition_size=0, stream=None):
        """q, out: [S, Q, Hq, D] with Q = new_tokens."""
        ws = self.ensure_workspace(q.shape[2], partition_size)
        return pa_verify(out, q, self.k_cache, self.v_cache, self.block_tables, self.context_lens, scale,
                         self.block_size, self.num_kv_heads, max_context_len=self.max_context_len,
                         partition_size=partition_size, workspace=ws, stream=stream)
