"""The continuous-batching trace as a serving loop: per-step host and device
time.

[P1] "大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解"
section 2 and [P3] "连续批处理Continuous Batching配置": every iteration, finished
sequences leave and free their blocks, waiting requests are admitted while
blocks suffice, and the running batch takes one decode step.  This module
drives that loop with the library's own parts: the native scheduler decides
each step (admissions, the slots of every K/V row to write, copy-on-write
pairs, preemption), and the device runs the step's work in issue order --
copy-on-write copies (pa_copy_blocks), writes of newly admitted prompts
(pa_cache_write) and, last, the append of each running sequence's new token
with the decode over the running batch (pa_write_decode).

``run(tc, seed)`` first runs the scheduler alone for every step (timing each
scheduling step and its table packing on the host), then replays the device
work of each step between two CUDA events on one stream, with the step's
metadata copied from pinned host memory inside the timed region and L2
flushed between steps outside it.  K/V and q values are seeded device draws:
the values do not change the work.
"""

import math
import time

import numpy as np

from . import (BlockManager, Scheduler, pa_cache_write, pa_copy_blocks, pa_decode_workspace_size, pa_write_decode)
from . import workloads as wl


def dry_peak(tc, reqs):
    """Peak blocks in use over the trace with an unbounded pool."""
    big = 1 << 20
    bm = BlockManager(big, tc.block_size)
    bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = Scheduler(bm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        sch.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    peak = 0
    for _ in range(tc.steps):
        sch.step(raw=True)
        peak = max(peak, bm.stats()[1])
    return peak


def _runs(kind, a, b, c):
    """Split a step's ops into runs in issue order: ("w", slots) for consecutive
    writes, ("c", pairs) for consecutive copy-on-write copies."""
    runs = []
    i, n = 0, len(kind)
    while i < n:
        k = int(kind[i])
        j = i
        while j < n and int(kind[j]) == k:
            j += 1
        if k == 0:
            runs.append(("w", np.ascontiguousarray(c[i:j], dtype=np.int64)))
        elif k == 1:
            runs.append(("c", np.ascontiguousarray(np.stack([a[i:j], b[i:j]], 1), dtype=np.int32)))
        else:
            raise ValueError("swap ops need a host pool; the trace runs with recompute preemption")
        i = j
    return runs


def schedule(tc=wl.TRACE, seed=5):
    """The scheduler alone over every step of the trace (host only): per step
    its device ops in issue order, packed tables and context lengths, and the
    host time of the scheduling step and its table packing."""
    reqs = wl.make_trace_requests(tc, seed)
    nb = int(math.ceil(tc.pool_frac * dry_peak(tc, reqs)))
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    bm = BlockManager(nb, tc.block_size, order)
    bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = Scheduler(bm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        sch.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    prefix_slots = np.asarray(bm.slots(wl.PREFIX_SEQ, 0, tc.prefix_len), dtype=np.int64)
    steps, host_ms = [], []
    preempted = admitted = 0
    for _ in range(tc.steps):
        t0 = time.perf_counter()
        rec = sch.step(raw=True)
        running = rec["running"]
        if running:
            # a table holds exactly ceil(context / block size) blocks
            width = -(-max(rec["context_lens"]) // tc.block_size)
            tables, lens = bm.pack(running, width)
        host_ms.append((time.perf_counter() - t0) * 1e3)
        preempted += len(rec["preempted"])
        admitted += len(rec["admitted"])
        if not running:
            steps.append(None)
            continue
        runs = _runs(rec["op_kind"], rec["op_a"], rec["op_b"], rec["op_c"])
        steps.append((runs, np.ascontiguousarray(tables), np.ascontiguousarray(lens), int(lens.max())))
    return {"steps": steps, "host_ms": host_ms, "num_blocks": nb, "prefix_slots": prefix_slots,
            "preempted": preempted, "admitted": admitted}


def run(tc=wl.TRACE, seed=5, device="cuda", flush_bytes=256 << 20, partition_size=0):
    """Run the trace; returns per-step host and device times and the work done."""
    import torch
    dev = torch.device(device)
    sc = schedule(tc, seed)
    steps, host_ms, nb, prefix_slots = sc["steps"], sc["host_ms"], sc["num_blocks"], sc["prefix_slots"]
    max_rows = max([len(prefix_slots)] + [len(x) for st in steps if st is not None for k, x in st[0] if k == "w"])
    max_running = max([1] + [len(st[2]) for st in steps if st is not None])

    # ---- device buffers: pools, seeded rows, pinned metadata
    H, Hq, D, bs = tc.num_kv_heads, tc.num_heads, tc.head_dim, tc.block_size
    tt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[tc.dtype]
    g = torch.Generator(device=dev).manual_seed(seed)
    kc = torch.zeros((nb, bs, H, D), dtype=tt, device=dev)
    vc = torch.zeros_like(kc)
    krows = torch.randn((max_rows, H, D), generator=g, device=dev, dtype=torch.float32).to(tt)
    vrows = torch.randn((max_rows, H, D), generator=g, device=dev, dtype=torch.float32).to(tt)
    qall = torch.randn((max_running, Hq, D), generator=g, device=dev, dtype=torch.float32).to(tt)
    out_all = torch.empty_like(qall)
    max_ctx = max(s[3] for s in steps if s is not None)
    ws_bytes = pa_decode_workspace_size(max_running, Hq, D, max_ctx, partition_size)
    workspace = torch.empty(max(1, ws_bytes), dtype=torch.uint8, device=dev)
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device=dev)
    slots_d = torch.empty(max_rows, dtype=torch.int64, device=dev)
    pin = lambda a: torch.from_numpy(a).pin_memory()          # noqa: E731
    host_steps = []
    for s in steps:
        if s is None:
            host_steps.append(None)
            continue
        runs, tables, lens, mcl = s
        host_steps.append(([(k, pin(x)) for k, x in runs], pin(tables), pin(lens), mcl))
    pa_cache_write(krows[:len(prefix_slots)], vrows[:len(prefix_slots)], kc, vc, torch.from_numpy(prefix_slots).to(dev))
    torch.cuda.synchronize()

    # ---- the device work of every step, in issue order, between two events
    ev = []
    kv_bytes = []
    elt = wl.ELEMENT_BYTES[tc.dtype]
    for s in host_steps:
        if s is None:
            continue
        runs, tables_h, lens_h, mcl = s
        R = int(lens_h.numel())
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        tables_d = tables_h.to(dev, non_blocking=True)
        lens_d = lens_h.to(dev, non_blocking=True)
        last = len(runs) - 1
        final_slots = None
        for i, (kind, x) in enumerate(runs):
            if kind == "c":
                pa_copy_blocks(kc, vc, x.to(dev, non_blocking=True))
                continue
            n = int(x.numel())
            sd = slots_d[:n]
            sd.copy_(x, non_blocking=True)
            if i == last:
                final_slots = sd
            else:
                pa_cache_write(krows[:n], vrows[:n], kc, vc, sd)
        q, out = qall[:R], out_all[:R]
        if final_slots is None:          # no write after the last copy: decode alone
            final_slots = slots_d[:0]
        n = int(final_slots.numel())
        pa_write_decode(krows[:n], vrows[:n], final_slots, out, q, kc, vc, tables_d, lens_d, tc.scale, bs, H,
                        max_context_len=mcl, partition_size=partition_size, workspace=workspace)
        b.record()
        flush.zero_()
        ev.append((a, b))
        kv_bytes.append(int(lens_h.sum()) * 2 * H * D * elt)
    torch.cuda.synchronize()
    dev_ms = [x.elapsed_time(y) for x, y in ev]
    return {"device_ms": dev_ms, "host_ms": host_ms, "kv_bytes": kv_bytes, "num_blocks": nb,
            "preempted": sc["preempted"], "admitted": sc["admitted"], "steps": len(dev_ms)}
