"""Continuous-batching trace on the GPU (fp16, 8-token blocks, 32/32 heads,
head_dim 128, at most 128 running sequences, 200 decode steps).

Half the requests share a 1024-token system prefix held in reference-counted
blocks; one in eight forks a parallel-sampling child right after its prompt
(copy-on-write on the first divergent write); unique prompts are 1-512
tokens and output lengths geometric with mean 256.  The pool holds 75% of the
peak demand of an unbounded dry run, so admission blocks and sequences get
preempted (both asserted).

Every step: the native scheduler and the oracle's Python model agree on the
step record bit for bit; its writes and copies are applied on the device in
issue order (pa_cache_write / pa_copy_blocks); the decode runs over the
running batch.  Checked: every row written this step, bit-exact; the decode
output of every running sequence at every step against the fp64 oracle
(computed on spawned worker processes that draw each history from the
generators); the full cache contents of sampled sequences, bit-exact, and
every 50 steps those of the whole batch.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from oracle import block_manager as obm
from oracle import scheduler as osch
from tests.gpu_harness import assert_close, to_device, to_storage
from tests.trace_oracle import TraceOracle

pytestmark = pytest.mark.gpu

SEED = 5


class Streams:
    """Which history stream (request, parent or prefix holder) owns a position."""

    def __init__(self, tc, reqs):
        self.prefix = tc.prefix_len
        self.share = {q.seq_id: q.shares_prefix for q in reqs}
        self.parent = {}
        self.fork_pos = {}
        for q in reqs:
            if q.fork_child >= 0:
                self.parent[q.fork_child] = q.seq_id
                self.share[q.fork_child] = q.shares_prefix
                self.fork_pos[q.fork_child] = (tc.prefix_len if q.shares_prefix else 0) + q.prompt_len

    def of(self, seq, pos):
        while seq in self.parent and pos < self.fork_pos[seq]:
            seq = self.parent[seq]
        if seq != wl.PREFIX_SEQ and self.share.get(seq, False) and pos < self.prefix:
            return wl.PREFIX_SEQ
        return seq

    def rows(self, seq, positions, tc, salt):
        positions = np.asarray(positions, dtype=np.int64)
        out = np.empty((len(positions), tc.num_kv_heads, tc.head_dim), dtype=np.uint16)
        owners = np.array([self.of(seq, int(p)) for p in positions], dtype=np.int64)
        for o in np.unique(owners):
            sel = owners == o
            out[sel] = wl.token_rows(SEED, int(o), positions[sel], tc.num_kv_heads, tc.head_dim, tc.dtype, salt)
        return out


def _rows_for_writes(writes, streams, tc, salt):
    out = np.empty((len(writes), tc.num_kv_heads, tc.head_dim), dtype=np.uint16)
    keys = {}
    for i, (seq, pos, _) in enumerate(writes):
        keys.setdefault(streams.of(seq, pos), []).append((i, pos))
    for owner, lst in keys.items():
        idx = np.array([i for i, _ in lst])
        out[idx] = wl.token_rows(SEED, owner, [p for _, p in lst], tc.num_kv_heads, tc.head_dim, tc.dtype, salt)
    return out


def _dry_peak(tc, reqs):
    big = 1 << 20
    bm = pa.BlockManager(big, tc.block_size)
    bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = pa.Scheduler(bm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        sch.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    peak = 0
    for _ in range(tc.steps):
        sch.step()
        free, used, _ = bm.stats()
        peak = max(peak, used)
    return peak


@pytest.mark.parametrize("preempt", ["recompute", "swap"])
def test_continuous_batching_trace(preempt):
    """With preempt="swap", victims move to a pinned host pool (a quarter of the
    GPU pool) and come back before new admissions; the swap copies run with
    pa_swap_blocks in issue order among the writes and copy-on-write copies."""
    assert torch.cuda.is_available()
    from paged_kv_cache_381_b200 import build
    build.build()
    pa.pa_get_device_error()
    tc = wl.TRACE
    reqs = wl.make_trace_requests(tc, SEED)
    streams = Streams(tc, reqs)
    nb = int(math.ceil(tc.pool_frac * _dry_peak(tc, reqs)))
    order = np.random.default_rng(SEED).permutation(nb).astype(np.int32)
    ncpu = nb // 4 if preempt == "swap" else 0
    bm = pa.BlockManager(nb, tc.block_size, order)
    bm.set_cpu_blocks(ncpu)
    if preempt == "swap":
        model_bm = obm.SwappingBlockManager(nb, tc.block_size, ncpu, order.tolist())
    else:
        model_bm = obm.BlockManager(nb, tc.block_size, order.tolist())
    for m in (bm, model_bm):
        m.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = pa.Scheduler(bm, tc.max_running, wl.PREFIX_SEQ, preempt=preempt)
    model = osch.Scheduler(model_bm, tc.max_running, wl.PREFIX_SEQ, preempt=preempt)
    for q in reqs:
        sch.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
        model.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child,
                                       q.fork_output_len))
    H, D, bs = tc.num_kv_heads, tc.head_dim, tc.block_size
    dev = torch.device("cuda")
    kc = torch.zeros((nb, bs, H, D), dtype=torch.float16, device=dev)
    vc = torch.zeros_like(kc)
    hk = torch.zeros((max(ncpu, 1), bs, H, D), dtype=torch.float16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    kflat, vflat = kc.view(nb * bs, H, D), vc.view(nb * bs, H, D)

    def write(ws):
        if not ws:
            return
        k = _rows_for_writes(ws, streams, tc, 0)
        v = _rows_for_writes(ws, streams, tc, 1)
        slots = torch.tensor([w[2] for w in ws], dtype=torch.int64, device=dev)
        pa.pa_cache_write(to_device(k, "f16"), to_device(v, "f16"), kc, vc, slots)

    # the shared prefix is written once
    pre = [(wl.PREFIX_SEQ, p, int(s)) for p, s in enumerate(bm.slots(wl.PREFIX_SEQ, 0, tc.prefix_len))]
    write(pre)
    oracle = TraceOracle(SEED, tc, (tc.prefix_len, wl.PREFIX_SEQ, dict(streams.share), dict(streams.parent),
                                    dict(streams.fork_pos)))
    try:
        _trace_steps(tc, sch, model, bm, streams, kc, vc, hk, hv, kflat, vflat, write, oracle, preempt)
    finally:
        oracle.close()


def _trace_steps(tc, sch, model, bm, streams, kc, vc, hk, hv, kflat, vflat, write, oracle, preempt):
    H, D, bs = tc.num_kv_heads, tc.head_dim, tc.block_size
    dev = torch.device("cuda")

    r = np.random.default_rng(11)
    saw = {"preempt": 0, "cow": 0, "blocked": 0, "finish": 0, "so": 0, "si": 0}
    checked = {"rows": 0, "steps": 0}
    for step in range(tc.steps):
        rec = sch.step()
        mrec = model.step()
        assert rec["finished"] == mrec.finished and rec["admitted"] == mrec.admitted, step
        assert rec["preempted"] == mrec.preempted and rec["ops"] == [tuple(o) for o in mrec.ops], step
        assert rec["running"] == mrec.running and rec["context_lens"] == mrec.context_lens, step
        assert rec["swapped_out"] == mrec.swapped_out and rec["swapped_in"] == mrec.swapped_in, step
        saw["preempt"] += len(rec["preempted"])
        saw["finish"] += len(rec["finished"])
        if rec["num_waiting"] > 0 and len(rec["running"]) < tc.max_running:
            saw["blocked"] += 1
        # apply writes, copies and swap copies in issue order
        run = []
        for op in rec["ops"]:
            if op[0] == "w":
                run.append(op[1:])
                continue
            write(run)
            run = []
            pair = torch.tensor([[op[1], op[2]]], dtype=torch.int32, device=dev)
            if op[0] == "c":
                saw["cow"] += 1
                pa.pa_copy_blocks(kc, vc, pair)
            elif op[0] == "so":
                saw["so"] += 1
                pa.pa_swap_blocks(hk, hv, kc, vc, pair)
            else:
                saw["si"] += 1
                pa.pa_swap_blocks(kc, vc, hk, hv, pair)
        write(run)
        running, ctx = rec["running"], rec["context_lens"]
        if not running:
            continue
        width = max(len(bm.block_table(s)) for s in running)
        tables, lens = bm.pack(running, width)
        assert lens.tolist() == ctx
        q = np.stack([wl.token_rows(SEED, s, [c], tc.num_heads, D, tc.dtype, 2)[0] for s, c in zip(running, ctx)])
        qd = to_device(q, "f16")
        out = torch.empty_like(qd)
        pa.pa_decode(out, qd, kc, vc, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev), tc.scale,
                     bs, H, max_context_len=int(lens.max()))
        # every running sequence, every step: the oracle works while the GPU does
        oracle.submit([(s, c, q[i]) for i, (s, c) in enumerate(zip(running, ctx))])
        torch.cuda.synchronize()
        # rows written this step, still owned by their writer: bit-exact
        live = {s: set() for s in running}
        checks = [w for w in (o[1:] for o in rec["ops"] if o[0] == "w") if w[0] in live]
        if checks:
            slots = torch.tensor([w[2] for w in checks], dtype=torch.int64, device=dev)
            gotk = to_storage(kflat.index_select(0, slots), "f16")
            gotv = to_storage(vflat.index_select(0, slots), "f16")
            owned = np.array([bm.slots(w[0], w[1], 1)[0] == w[2] for w in checks])
            assert np.array_equal(gotk[owned], _rows_for_writes(checks, streams, tc, 0)[owned]), step
            assert np.array_equal(gotv[owned], _rows_for_writes(checks, streams, tc, 1)[owned]), step
        got = to_storage(out, "f16")
        refs = oracle.results()
        assert_close(got, np.stack(refs), "f16", f"step {step}, all {len(running)} running sequences")
        # sampled sequences: their whole cache, bit-exact (every 50 steps: every sequence)
        sample = set(r.choice(len(running), size=min(4, len(running)), replace=False).tolist())
        if step % 50 == 49:
            sample = set(range(len(running)))
        for i in sorted(sample):
            s, n = running[i], ctx[i]
            sl = torch.from_numpy(bm.slots(s, 0, n)).to(dev)
            K = streams.rows(s, range(n), tc, 0)
            V = streams.rows(s, range(n), tc, 1)
            assert np.array_equal(to_storage(kflat.index_select(0, sl), "f16"), K), (step, s)
            assert np.array_equal(to_storage(vflat.index_select(0, sl), "f16"), V), (step, s)
        checked["rows"] += len(running)
        checked["steps"] += 1
        assert pa.pa_get_device_error() == 0
    assert saw["preempt"] >= 1, saw
    assert saw["cow"] >= 1, saw
    assert saw["blocked"] >= 1, saw
    assert saw["finish"] >= 1, saw
    if preempt == "swap":
        assert saw["so"] >= 1 and saw["si"] >= 1, saw
    # every step decoded a running batch, and every row of it was checked
    assert checked["steps"] == tc.steps and checked["rows"] >= 100 * tc.steps, checked
