"""Pins for the oracle's numerics, cache writes, block manager and scheduler
(CPU only).

* widening of stored bf16 / fp16 values is checked over all 65536 bit
  patterns against torch's own conversions (a library routine);
* cache writes are checked cell by cell against an explicit map built from the
  block tables, with untouched cells keeping a sentinel;
* the block manager and scheduler replay hand-derived traces stored under
  tests/golden/ (derivations and page citations there), and random op streams
  keep every bookkeeping invariant.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import block_manager as obm
from oracle import cache as oc
from oracle import scheduler as osch
from oracle.numerics import widen
from paged_kv_cache_381_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# -- numerics -----------------------------------------------------------------

@pytest.mark.parametrize("dtype,tt", [("bf16", torch.bfloat16), ("f16", torch.float16)])
def test_widen_all_bit_patterns(dtype, tt):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = widen(bits, dtype)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(tt).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_widen_f32_identity():
    x = np.random.default_rng(0).standard_normal(1000).astype(np.float32)
    assert np.array_equal(widen(x, "f32"), x.astype(np.float64))


def test_generator_rounding_is_nearest_even():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7: ties to even -> 1
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32)
    got = widen(wl.to_storage(x, "bf16"), "bf16")
    assert got.tolist() == [1.0, 1.0 + 2.0 ** -6]


# -- cache writes ---------------------------------------------------------------

def test_cache_write_cell_by_cell():
    r = np.random.default_rng(1)
    nb, bs, Hkv, D = 9, 4, 3, 8
    lens = [5, 0, 11, 4]
    _, tables = wl.shuffled_tables(r, wl.blocks_for(lens, bs), nb, 0)
    hist_k = [r.integers(0, 60000, size=(n, Hkv, D)).astype(np.uint16) for n in lens]
    hist_v = [r.integers(0, 60000, size=(n, Hkv, D)).astype(np.uint16) for n in lens]
    sentinel = np.uint16(0xFFFF)
    kc = np.full((nb, bs, Hkv, D), sentinel, np.uint16)
    vc = kc.copy()
    ks, vs, slots = [], [], []
    for s, n in enumerate(lens):
        for t in range(n):
            ks.append(hist_k[s][t]); vs.append(hist_v[s][t])
            slots.append(oc.slot_of(tables[s], t, bs))
    # padding tokens (slot -1) are not written
    ks.append(np.zeros((Hkv, D), np.uint16)); vs.append(np.zeros((Hkv, D), np.uint16)); slots.append(-1)
    kc, vc = oc.cache_write(np.array(ks), np.array(vs), kc, vc, np.array(slots))
    owner = {}
    for s, n in enumerate(lens):
        for j in range(-(-n // bs)):
            for o in range(bs):
                if j * bs + o < n:
                    owner[(int(tables[s][j]), o)] = (s, j * bs + o)
    for b in range(nb):
        for o in range(bs):
            if (b, o) in owner:
                s, t = owner[(b, o)]
                assert np.array_equal(kc[b, o], hist_k[s][t]) and np.array_equal(vc[b, o], hist_v[s][t])
            else:
                assert (kc[b, o] == sentinel).all() and (vc[b, o] == sentinel).all()


def test_copy_blocks():
    r = np.random.default_rng(2)
    kc = r.integers(0, 1000, size=(6, 2, 1, 3)).astype(np.uint16)
    vc = r.integers(0, 1000, size=(6, 2, 1, 3)).astype(np.uint16)
    k2, v2 = oc.copy_blocks(kc, vc, [[1, 4], [2, 5]])
    for b in range(6):
        src = {4: 1, 5: 2}.get(b, b)
        assert np.array_equal(k2[b], kc[src]) and np.array_equal(v2[b], vc[src])


# -- block manager ----------------------------------------------------------------

def _apply(bm, op):
    kind = op["op"]
    if kind == "allocate":
        return bm.allocate(op["seq"], op["tokens"])
    if kind == "fork":
        return bm.fork(op["parent"], op["child"])
    if kind == "append":
        return bm.append_slot(op["seq"])
    if kind == "free":
        return bm.free(op["seq"])
    raise ValueError(kind)


def test_block_manager_golden_trace():
    with open(os.path.join(GOLDEN, "block_manager_trace.json")) as f:
        g = json.load(f)
    bm = obm.BlockManager(g["num_blocks"], g["block_size"], g["initial_free_order"])
    for op in g["ops"]:
        exp = op["expect"]
        seq = op.get("seq", op.get("child"))
        if "error" in exp:
            err = {"no_blocks": obm.NoBlocks, "invalid_arg": obm.InvalidArg}[exp["error"]]
            with pytest.raises(err):
                _apply(bm, op)
        else:
            res = _apply(bm, op)
            if "slot" in exp:
                assert res[0] == exp["slot"], op
                assert [res[1], res[2]] == exp["cow"], op
        if "table" in exp:
            assert bm.block_table(seq) == exp["table"], op
        if "free" in exp:
            assert bm.free_list == exp["free"], op
        if "ref" in exp:
            for b, c in exp["ref"].items():
                assert bm.ref[int(b)] == c, op
        if "ctx" in exp:
            assert bm.context_len(seq) == exp["ctx"], op
        bm.check()


def test_block_manager_random_streams_keep_invariants():
    r = np.random.default_rng(3)
    for trial in range(20):
        nb, bs = int(r.integers(4, 40)), int(r.choice([1, 2, 4, 8]))
        bm = obm.BlockManager(nb, bs, r.permutation(nb).tolist())
        live, next_id = [], 0
        for _ in range(300):
            c = r.random()
            try:
                if c < 0.25 or not live:
                    bm.allocate(next_id, int(r.integers(0, 3 * bs)))
                    live.append(next_id); next_id += 1
                elif c < 0.4:
                    bm.fork(live[int(r.integers(len(live)))], next_id)
                    live.append(next_id); next_id += 1
                elif c < 0.85:
                    s = live[int(r.integers(len(live)))]
                    before = list(bm.block_table(s))
                    pos = bm.context_len(s)
                    slot, src, dst = bm.append_slot(s)
                    t = bm.block_table(s)
                    assert slot == t[pos // bs] * bs + pos % bs
                    assert bm.ref[t[pos // bs]] == 1          # written block is private
                    if src >= 0:
                        assert before[-1] == src and t[-1] == dst and pos % bs != 0
                else:
                    s = live.pop(int(r.integers(len(live))))
                    bm.free(s)
            except obm.NoBlocks:
                pass
            bm.check()
        for s in live:
            bm.free(s)
        bm.check()
        assert bm.num_free == nb


def test_block_manager_errors_leave_state_unchanged():
    bm = obm.BlockManager(2, 4, [0, 1])
    bm.allocate(1, 8)
    snap = (list(bm.free_list), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.ctx))
    with pytest.raises(obm.NoBlocks):
        bm.append_slot(1)
    with pytest.raises(obm.NoBlocks):
        bm.allocate(2, 1)
    with pytest.raises(obm.InvalidArg):
        bm.allocate(1, 1)
    with pytest.raises(obm.InvalidArg):
        bm.fork(7, 8)
    assert snap == (list(bm.free_list), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.ctx))


# -- scheduler ----------------------------------------------------------------------

def _load_traces():
    with open(os.path.join(GOLDEN, "scheduler_traces.json")) as f:
        return json.load(f)["traces"]


def _build(tr):
    if tr.get("preempt") == "swap":
        bm = obm.SwappingBlockManager(tr["num_blocks"], tr["block_size"], tr["num_cpu_blocks"],
                                      tr["initial_free_order"])
    else:
        bm = obm.BlockManager(tr["num_blocks"], tr["block_size"], tr["initial_free_order"])
    prefix = -1
    if tr["prefix"]:
        prefix = tr["prefix"]["seq"]
        bm.allocate(prefix, tr["prefix"]["tokens"])
    sch = osch.Scheduler(bm, tr["max_running"], prefix, preempt=tr.get("preempt", "recompute"))
    for q in tr["requests"]:
        sch.add_request(osch.Request(q["seq"], q["prompt"], q["output"], q.get("shares_prefix", False),
                                     q.get("fork_child", -1), q.get("fork_output", 0)))
    return bm, sch


@pytest.mark.parametrize("tr", _load_traces(), ids=lambda t: t["name"])
def test_scheduler_golden_traces(tr):
    bm, sch = _build(tr)
    for i, exp in enumerate(tr["steps"]):
        rec = sch.step()
        assert rec.finished == exp["finished"], (i, rec.finished)
        assert rec.admitted == exp["admitted"], (i, rec.admitted)
        assert rec.preempted == exp["preempted"], (i, rec.preempted)
        assert [list(o) for o in rec.ops] == exp["ops"], (i, rec.ops)
        assert rec.running == exp["running"], (i, rec.running)
        assert rec.context_lens == exp["context_lens"], (i, rec.context_lens)
        if "swapped_out" in exp:
            assert (rec.swapped_out, rec.swapped_in) == (exp["swapped_out"], exp["swapped_in"]), i
        bm.check()


def test_scheduler_random_trace_invariants():
    """A scaled-down continuous-batching trace: invariants every step.

    Every live sequence's blocks hold exactly the positions written for it
    (checked through a shadow cache of (stream, position) tags replayed from
    the ops), the running count never exceeds the cap, first admissions follow
    arrival order, and the pool is conserved.
    """
    tc = wl.TraceConfig(block_size=4, max_running=12, num_requests=40, steps=120, prefix_len=10,
                        prompt_hi=30, output_mean=12.0, fork_every=4)
    reqs = wl.make_trace_requests(tc, 5)
    nb = 70
    bm = obm.BlockManager(nb, tc.block_size, np.random.default_rng(9).permutation(nb).tolist())
    bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = osch.Scheduler(bm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        sch.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix,
                                     q.fork_child, q.fork_output_len))
    shadow = {}
    for p, sl in enumerate(bm.slots(wl.PREFIX_SEQ, 0, tc.prefix_len)):
        shadow[sl] = (wl.PREFIX_SEQ, p)
    parent_of = {q.fork_child: q.seq_id for q in reqs if q.fork_child >= 0}
    fork_pos = {q.fork_child: (tc.prefix_len if q.shares_prefix else 0) + q.prompt_len
                for q in reqs if q.fork_child >= 0}
    share = {q.seq_id: q.shares_prefix for q in reqs}

    def stream_of(seq, pos):
        if seq in parent_of and pos < fork_pos[seq]:
            return stream_of(parent_of[seq], pos)
        if share.get(seq, False) and pos < tc.prefix_len:
            return wl.PREFIX_SEQ
        return seq

    first_admit = []
    saw_preempt = saw_cow = False
    for _ in range(tc.steps):
        rec = sch.step()
        for op in rec.ops:
            if op[0] == "c":
                bs = tc.block_size
                for o in range(bs):
                    if op[1] * bs + o in shadow:
                        shadow[op[2] * bs + o] = shadow[op[1] * bs + o]
                saw_cow = True
            else:
                _, seq, pos, slot = op
                shadow[slot] = (stream_of(seq, pos), pos)
        slots = [w[2] for w in rec.writes]
        assert len(slots) == len(set(slots)), "a slot written twice in one step"
        saw_preempt |= bool(rec.preempted)
        for a in rec.admitted:
            if a < tc.num_requests and a not in first_admit:
                first_admit.append(a)
        assert len(rec.running) <= tc.max_running
        bm.check()
        for seq, n in zip(rec.running, rec.context_lens):
            assert bm.context_len(seq) == n
            for p, sl in enumerate(bm.slots(seq, 0, n)):
                assert shadow.get(sl) == (stream_of(seq, p), p), (seq, p)
    assert first_admit == sorted(first_admit)
    assert saw_preempt and saw_cow


def _swap_trace_run(tc, reqs, nb, ncpu, seed, record_cls=None):
    """Run the scheduler model with preemption by swap; replay its ops on a
    shadow of GPU and host slots; check every sequence's content each step."""
    bm = obm.SwappingBlockManager(nb, tc.block_size, ncpu, np.random.default_rng(seed).permutation(nb).tolist())
    bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = osch.Scheduler(bm, tc.max_running, wl.PREFIX_SEQ, preempt="swap")
    for q in reqs:
        sch.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix,
                                     q.fork_child, q.fork_output_len))
    bs = tc.block_size
    gpu, cpu = {}, {}
    for p, sl in enumerate(bm.slots(wl.PREFIX_SEQ, 0, tc.prefix_len)):
        gpu[sl] = (wl.PREFIX_SEQ, p)
    parent_of = {q.fork_child: q.seq_id for q in reqs if q.fork_child >= 0}
    fork_pos = {q.fork_child: (tc.prefix_len if q.shares_prefix else 0) + q.prompt_len
                for q in reqs if q.fork_child >= 0}
    share = {q.seq_id: q.shares_prefix for q in reqs}

    def stream_of(seq, pos):
        if seq in parent_of and pos < fork_pos[seq]:
            return stream_of(parent_of[seq], pos)
        if share.get(seq, False) and pos < tc.prefix_len:
            return wl.PREFIX_SEQ
        return seq

    saw = {"so": 0, "si": 0, "recompute": 0}
    for _ in range(tc.steps):
        rec = sch.step()
        run = []
        for op in rec.ops:
            if op[0] == "w":
                run.append(op[3])
                gpu[op[3]] = (stream_of(op[1], op[2]), op[2])
                continue
            assert len(run) == len(set(run)), "a slot written twice in one run of writes"
            run = []
            src, dst = (gpu, gpu) if op[0] == "c" else (gpu, cpu) if op[0] == "so" else (cpu, gpu)
            for o in range(bs):
                if op[1] * bs + o in src:
                    dst[op[2] * bs + o] = src[op[1] * bs + o]
            if op[0] in saw:
                saw[op[0]] += 1
        assert len(run) == len(set(run))
        saw["recompute"] += len(rec.preempted) - len(rec.swapped_out)
        bm.check()
        for seq, n in zip(rec.running, rec.context_lens):
            for p, sl in enumerate(bm.slots(seq, 0, n)):
                assert gpu.get(sl) == (stream_of(seq, p), p), (seq, p)
        for s in sch.swapped:             # swapped out: host blocks it moved, GPU blocks it shares
            t, loc = bm.tables[s.seq_id], bm.on_cpu[s.seq_id]
            for p in range(bm.ctx[s.seq_id]):
                store = cpu if loc[p // bs] else gpu
                assert store.get(t[p // bs] * bs + p % bs) == (stream_of(s.seq_id, p), p), (s.seq_id, p)
    return saw


SWAP_TC = wl.TraceConfig(block_size=4, max_running=12, num_requests=40, steps=150, prefix_len=10,
                         prompt_hi=30, output_mean=14.0, fork_every=4)


@pytest.mark.parametrize("ncpu", [6, 40, 400])
def test_scheduler_swap_trace_content(ncpu):
    """Preemption by swap on a scaled-down trace: every running sequence reads
    its own tokens every step, and so does every swapped-out one where its
    table says (host or shared GPU blocks); consecutive writes never repeat a
    slot.  A small host pool also forces recompute fallbacks."""
    reqs = wl.make_trace_requests(SWAP_TC, 5)
    saw = _swap_trace_run(SWAP_TC, reqs, 60, ncpu, 9)
    assert saw["so"] > 0 and saw["si"] > 0, saw
    if ncpu == 6:
        assert saw["recompute"] > 0, saw
