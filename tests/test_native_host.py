"""CPU tests of libpa.so: it loads without a GPU, exports every function that
include/pa.h declares, and its host block manager and scheduler agree
bit-exactly with the oracle's Python models (golden traces and random op
streams).  No CUDA call is made here."""

import ctypes
import json
import os
import re

import numpy as np
import pytest

from oracle import block_manager as obm
from oracle import scheduler as osch
from paged_kv_cache_381_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    return pa


def _declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if not f.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(pa_\w+)\s*\(", src):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol(pa):
    names = _declared_functions()
    assert len(names) >= 20
    lib = pa.lib()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    from paged_kv_cache_381_b200 import _native
    assert names == set(_native.SIGNATURES), names ^ set(_native.SIGNATURES)


def test_status_strings(pa):
    assert pa.lib().pa_status_string(0) == b"ok"
    assert pa.lib().pa_status_string(3) == b"no free blocks"


def test_workspace_size_rules(pa):
    assert pa.pa_decode_workspace_size(8, 64, 128, 512, 512) == 0      # one partition: no scratch
    n = pa.pa_decode_workspace_size(8, 64, 128, 32768, 512)
    parts = 8 * 64 * 64
    assert n >= parts * 128 * 4 + 2 * parts * 4 + 8 * 64 * 8
    assert n % 256 == 0
    assert pa.pa_decode_workspace_size(8, 64, 128, 32768, 100) == 0    # invalid partition size


class _Native:
    """Adapter giving the C++ manager the oracle model's interface."""

    def __init__(self, pa, nb, bs, order):
        self.bm = pa.BlockManager(nb, bs, order)
        self.pa = pa

    def apply(self, op):
        k = op["op"]
        if k == "allocate":
            return self.bm.allocate(op["seq"], op["tokens"])
        if k == "fork":
            return self.bm.fork(op["parent"], op["child"])
        if k == "append":
            return self.bm.append_slot(op["seq"])
        return self.bm.free(op["seq"])


def test_block_manager_golden_trace(pa):
    with open(os.path.join(GOLDEN, "block_manager_trace.json")) as f:
        g = json.load(f)
    nat = _Native(pa, g["num_blocks"], g["block_size"], g["initial_free_order"])
    for op in g["ops"]:
        exp = op["expect"]
        seq = op.get("seq", op.get("child"))
        if "error" in exp:
            with pytest.raises(pa.PagedAttentionError) as ei:
                nat.apply(op)
            assert ei.value.status == {"no_blocks": 3, "invalid_arg": 1}[exp["error"]]
        else:
            res = nat.apply(op)
            if "slot" in exp:
                assert res[0] == exp["slot"] and [res[1], res[2]] == exp["cow"], op
        if "table" in exp:
            assert nat.bm.block_table(seq) == exp["table"], op
        if "free" in exp:
            assert nat.bm.free_list() == exp["free"], op
        if "ref" in exp:
            for b, c in exp["ref"].items():
                assert nat.bm.ref_count(int(b)) == c
        if "ctx" in exp:
            assert nat.bm.context_len(seq) == exp["ctx"]


def test_block_manager_matches_model_on_random_streams(pa):
    r = np.random.default_rng(12)
    for trial in range(25):
        nb, bs = int(r.integers(3, 50)), int(r.choice([1, 2, 4, 8, 16]))
        order = r.permutation(nb).tolist()
        model = obm.BlockManager(nb, bs, order)
        nat = pa.BlockManager(nb, bs, order)
        live, nid = [], 0
        for _ in range(400):
            c = r.random()
            if c < 0.2 or not live:
                op = ("allocate", nid, int(r.integers(0, 4 * bs)))
            elif c < 0.35:
                op = ("fork", live[int(r.integers(len(live)))], nid)
            elif c < 0.85:
                op = ("append", live[int(r.integers(len(live)))])
            else:
                op = ("free", live[int(r.integers(len(live)))])
            m_err = n_err = None
            m_res = n_res = None
            try:
                m_res = getattr(model, {"append": "append_slot"}.get(op[0], op[0]))(*op[1:])
            except (obm.NoBlocks, obm.InvalidArg) as e:
                m_err = type(e).__name__
            try:
                n_res = getattr(nat, {"append": "append_slot"}.get(op[0], op[0]))(*op[1:])
            except pa.PagedAttentionError as e:
                n_err = {3: "NoBlocks", 1: "InvalidArg"}[e.status]
            assert m_err == n_err, (op, m_err, n_err)
            if op[0] == "append" and m_err is None:
                assert tuple(m_res) == tuple(n_res), op
            if m_err is None:
                if op[0] in ("allocate", "fork"):
                    live.append(op[-1] if op[0] == "fork" else op[1])
                    nid += 1
                elif op[0] == "free":
                    live.remove(op[1])
            assert model.free_list == nat.free_list(), op
        for s in live:
            assert model.block_table(s) == nat.block_table(s)
            assert model.context_len(s) == nat.context_len(s)
        assert [model.ref[b] for b in range(nb)] == [nat.ref_count(b) for b in range(nb)]


def test_pack_layout(pa):
    bm = pa.BlockManager(10, 4, list(range(10)))
    bm.allocate(1, 9)
    bm.allocate(2, 0)
    bm.allocate(3, 4)
    tables, lens = bm.pack([3, 1, 2], 4)
    assert lens.tolist() == [4, 9, 0]
    assert tables.tolist() == [[6, -1, -1, -1], [9, 8, 7, -1], [-1, -1, -1, -1]]
    with pytest.raises(pa.PagedAttentionError):
        bm.pack([1], 2)          # table wider than the requested width


def _load_traces():
    with open(os.path.join(GOLDEN, "scheduler_traces.json")) as f:
        return json.load(f)["traces"]


@pytest.mark.parametrize("tr", _load_traces(), ids=lambda t: t["name"])
def test_scheduler_golden_traces(pa, tr):
    bm = pa.BlockManager(tr["num_blocks"], tr["block_size"], tr["initial_free_order"])
    bm.set_cpu_blocks(tr.get("num_cpu_blocks", 0))
    prefix = -1
    if tr["prefix"]:
        prefix = tr["prefix"]["seq"]
        bm.allocate(prefix, tr["prefix"]["tokens"])
    sch = pa.Scheduler(bm, tr["max_running"], prefix, preempt=tr.get("preempt", "recompute"))
    for q in tr["requests"]:
        sch.add_request(q["seq"], q["prompt"], q["output"], q.get("shares_prefix", False),
                        q.get("fork_child", -1), q.get("fork_output", 0))
    for i, exp in enumerate(tr["steps"]):
        rec = sch.step()
        for key in ("finished", "admitted", "preempted", "running", "context_lens", "swapped_out", "swapped_in"):
            if key in exp:
                assert rec[key] == exp[key], (i, key, rec[key])
        assert [list(o) for o in rec["ops"]] == exp["ops"], (i, rec["ops"])


def test_scheduler_matches_model_on_trace(pa):
    """Scaled-down continuous-batching trace: C++ and Python agree every step."""
    tc = wl.TraceConfig(block_size=8, max_running=32, num_requests=80, steps=150, prefix_len=36,
                        prompt_hi=100, output_mean=30.0, fork_every=5)
    reqs = wl.make_trace_requests(tc, 3)
    nb = 160
    order = np.random.default_rng(4).permutation(nb).tolist()
    mb = obm.BlockManager(nb, tc.block_size, order)
    nbm = pa.BlockManager(nb, tc.block_size, order)
    mb.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    nbm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    ms = osch.Scheduler(mb, tc.max_running, wl.PREFIX_SEQ)
    ns = pa.Scheduler(nbm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        ms.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child,
                                    q.fork_output_len))
        ns.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    seen = set()
    for step in range(tc.steps):
        a = ms.step()
        b = ns.step()
        assert a.finished == b["finished"], step
        assert a.admitted == b["admitted"], step
        assert a.preempted == b["preempted"], step
        assert [tuple(o) for o in a.ops] == b["ops"], step
        assert a.running == b["running"] and a.context_lens == b["context_lens"], step
        assert mb.free_list == nbm.free_list(), step
        seen |= {"preempt"} if a.preempted else set()
        seen |= {"cow"} if a.cow else set()
        seen |= {"finish"} if a.finished else set()
    assert seen == {"preempt", "cow", "finish"}


def test_full_trace_host_side_lockstep(pa):
    """The full-size continuous-batching trace's bookkeeping (no device work):
    native scheduler == oracle model every step, slots unique within a step."""
    import math
    tc = wl.TRACE
    reqs = wl.make_trace_requests(tc, 5)
    big = pa.BlockManager(1 << 20, tc.block_size)
    big.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    dry = pa.Scheduler(big, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        dry.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    peak = 0
    for _ in range(tc.steps):
        dry.step()
        peak = max(peak, big.stats()[1])
    nb = int(math.ceil(tc.pool_frac * peak))
    order = np.random.default_rng(5).permutation(nb).tolist()
    mb = obm.BlockManager(nb, tc.block_size, order)
    nbm = pa.BlockManager(nb, tc.block_size, order)
    mb.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    nbm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    ms = osch.Scheduler(mb, tc.max_running, wl.PREFIX_SEQ)
    ns = pa.Scheduler(nbm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        ms.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child,
                                    q.fork_output_len))
        ns.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    preempted = 0
    for step in range(tc.steps):
        a = ms.step()
        b = ns.step()
        assert [tuple(o) for o in a.ops] == b["ops"] and a.running == b["running"], step
        assert a.context_lens == b["context_lens"] and a.preempted == b["preempted"], step
        slots = [w[2] for w in a.writes]
        assert len(slots) == len(set(slots)), step
        preempted += len(a.preempted)
        mb.check()
    assert preempted > 0


def test_verify_workspace_and_argument_rules(pa):
    """pa_verify's scratch is decode's with Q x heads rows; its argument checks
    return before any device work (so they run without a GPU)."""
    lib = pa.lib()
    assert pa.pa_verify_workspace_size(8, 6, 64, 128, 32768) == pa.pa_decode_workspace_size(8, 6 * 64, 128, 32768)
    assert pa.pa_verify_workspace_size(8, 6, 64, 128, 512) == 0
    assert pa.pa_verify_workspace_size(8, 0, 64, 128, 32768) == 0
    nul = ctypes.c_void_p(0)
    args = lambda Q, dt, hq=64: (nul, nul, nul, nul, nul, nul, 0.1, 16, 8, 4, Q, hq, 128, 8, 128, 64, dt, 0, nul, 0,
                                 nul)
    assert lib.pa_verify(*args(6, 0)) == 2            # fp32: unsupported (tensor cores only)
    assert lib.pa_verify(*args(65, 2)) == 2           # more than 64 query rows per sequence
    assert lib.pa_verify(*args(0, 2)) == 1            # no query rows
    assert lib.pa_verify(*args(6, 2, hq=60)) == 1     # heads not a multiple of kv heads
    assert lib.pa_verify(*args(6, 2)) == 1            # null pointers


def test_verify_partition_choice(pa):
    """partition_size 0, R query rows per kv head, C = ceil(R / 64), items(P) =
    seqs x ceil(ctx / P) x kv heads x C: 2048 tokens when R >= 32, blocks of 16
    or more, seqs x kv heads x C >= 592 and items(2048) >= 1776; 1024 when
    R >= 32 and items(1024) >= 1776; else 512.  An explicit size is kept; the
    0-partition workspace covers every choice."""
    P = pa.pa_verify_partition_size
    assert P(256, 6, 64, 8, 7918, 16) == 2048       # 70b-shaped: 48 rows, items(2048) = 8192
    assert P(256, 6, 64, 8, 7918, 8) == 1024        # 8-token blocks: 2048 tokens would be 256 blocks
    assert P(8, 6, 64, 8, 32768, 16) == 1024        # long contexts: items(2048) = 1024, items(1024) = 2048
    assert P(8, 6, 64, 8, 16384, 16) == 512         # items(1024) = 1024
    assert P(64, 6, 32, 32, 2049, 16) == 512        # 7b-shaped: 6 rows
    assert P(256, 3, 64, 8, 8192, 16) == 512        # 24 rows
    assert P(73, 4, 64, 8, 8192, 16) == 1024        # 32 rows, 584 unsplit items: no 2048
    assert P(74, 4, 64, 8, 8192, 16) == 2048        # 592 unsplit items, items(2048) = 2368
    assert P(74, 4, 64, 8, 6144, 16) == 2048        # items(2048) = 74 x 3 x 8 = 1776, the bound itself
    assert P(74, 4, 64, 8, 4096, 16) == 1024        # items(2048) = 1184, items(1024) = 2368
    assert P(256, 6, 64, 8, 8192, 16, 256) == 256
    for S, Q, Hq, D, ctx in ((256, 6, 64, 128, 8192), (64, 6, 32, 128, 2048), (8, 4, 64, 64, 32768)):
        for p in (1024, 2048):
            assert pa.pa_verify_workspace_size(S, Q, Hq, D, ctx, 0) >= pa.pa_verify_workspace_size(S, Q, Hq, D, ctx, p)


def test_verify_kernel_selection(pa):
    """The process-wide tensor-core path of pa_verify: AUTO by default, the
    three named kinds accepted, anything else rejected with nothing changed."""
    assert pa.get_verify_kernel() == pa.VERIFY_AUTO
    try:
        for k in (pa.VERIFY_MMA_SYNC, pa.VERIFY_TCGEN05, pa.VERIFY_AUTO):
            pa.set_verify_kernel(k)
            assert pa.get_verify_kernel() == k
        pa.set_verify_kernel(pa.VERIFY_TCGEN05)
        assert pa.lib().pa_set_verify_kernel(3) == 1
        assert pa.lib().pa_set_verify_kernel(-1) == 1
        assert pa.get_verify_kernel() == pa.VERIFY_TCGEN05
    finally:
        pa.set_verify_kernel(pa.VERIFY_AUTO)


@pytest.mark.parametrize("ncpu,nb", [(6, 60), (40, 60), (400, 50)])
def test_scheduler_swap_matches_model(pa, ncpu, nb):
    """Preemption by swap: C++ and Python agree every step (ops incl. swap
    copies, swapped ids, free lists of both pools)."""
    tc = wl.TraceConfig(block_size=4, max_running=12, num_requests=40, steps=150, prefix_len=10,
                        prompt_hi=30, output_mean=14.0, fork_every=4)
    reqs = wl.make_trace_requests(tc, 5)
    order = np.random.default_rng(9).permutation(nb).tolist()
    mb = obm.SwappingBlockManager(nb, tc.block_size, ncpu, order)
    nbm = pa.BlockManager(nb, tc.block_size, order)
    nbm.set_cpu_blocks(ncpu)
    for m in (mb, nbm):
        m.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    ms = osch.Scheduler(mb, tc.max_running, wl.PREFIX_SEQ, preempt="swap")
    ns = pa.Scheduler(nbm, tc.max_running, wl.PREFIX_SEQ, preempt="swap")
    for q in reqs:
        ms.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child,
                                    q.fork_output_len))
        ns.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    n_so = 0
    for step in range(tc.steps):
        a, b = ms.step(), ns.step()
        assert [tuple(o) for o in a.ops] == b["ops"], step
        assert (a.finished, a.admitted, a.preempted) == (b["finished"], b["admitted"], b["preempted"]), step
        assert (a.swapped_out, a.swapped_in) == (b["swapped_out"], b["swapped_in"]), step
        assert a.running == b["running"] and a.context_lens == b["context_lens"], step
        assert len(ms.swapped) == b["num_swapped"], step
        assert mb.free_list == nbm.free_list() and mb.cpu_free == nbm.cpu_free_list(), step
        n_so += len(a.swapped_out)
    assert n_so > 0


def test_decode_and_cache_write_argument_rules(pa):
    """pa_decode and pa_cache_write return their argument errors synchronously,
    before any device work, so these run without a GPU (status codes: 0 ok,
    1 invalid argument, 2 unsupported)."""
    lib = pa.lib()
    nul = ctypes.c_void_p(0)

    def dec(S=4, Hq=64, Hkv=8, D=128, bs=16, dt=2, P=0, scale=0.1):
        return lib.pa_decode(nul, nul, nul, nul, nul, nul, scale, bs, Hkv, S, Hq, D, 8, 128, 64, dt, P, nul, 0, nul)

    assert dec(S=0) == 0                               # nothing to do
    assert dec() == 1                                  # null pointers
    assert dec(Hq=60) == 1                             # heads not a multiple of kv heads
    assert dec(D=96) == 2                              # head_dim outside {64, 128}
    assert dec(bs=12) == 2                             # block size outside {8, 16, 32}
    assert dec(P=100) == 1                             # partition not a multiple of 32
    assert dec(dt=7) == 1                              # unknown dtype
    assert dec(scale=float("nan")) == 1

    def cw(T=4, nb=64, bs=16, Hkv=8, D=128, dt=2):
        desc = pa._native.CacheDesc(nb, bs, Hkv, D, dt)
        return lib.pa_cache_write(nul, nul, nul, nul, nul, T, ctypes.byref(desc), nul)

    assert cw(T=0) == 0
    assert cw() == 1                                   # null pointers
    assert cw(T=-1) == 1
    assert cw(bs=12) == 2 and cw(D=96) == 2
    assert cw(nb=0) == 1 and cw(dt=9) == 1
    assert lib.pa_cache_write(nul, nul, nul, nul, nul, 4, None, nul) == 1


def test_write_decode_argument_rules(pa):
    """pa_write_decode checks every argument of the cache write and of the
    decode before anything is launched (so these run without a GPU)."""
    lib = pa.lib()
    nul = ctypes.c_void_p(0)
    before = pa.launch_count()

    def wd(T=4, S=4, Hq=64, Hkv=8, D=128, bs=16, dt=2, P=0, scale=0.1, nb=64):
        return lib.pa_write_decode(nul, nul, nul, T, nul, nul, nul, nul, nul, nul, scale, bs, Hkv, S, Hq, D, 8, 128,
                                   nb, dt, P, nul, 0, nul)

    assert wd() == 1                                   # null write pointers
    assert wd(T=-1) == 1
    assert wd(T=0) == 1                                # no write: the decode's own checks (null pointers)
    assert wd(T=0, S=0) == 0                           # nothing at all to do
    assert wd(bs=12) == 2 and wd(D=96) == 2            # unsupported shapes (write checks first)
    assert wd(T=0, Hq=60) == 1                         # decode checks: heads not a multiple of kv heads
    assert wd(T=0, P=100) == 1 and wd(T=0, scale=float("nan")) == 1
    assert wd(dt=7) == 1
    assert pa.launch_count() == before


def test_noalloc_scratch_need_uses_the_table_capacity(pa):
    """pa_decode_noalloc sizes its scratch need as pa_decode does, from
    max_context_len capped by the block table's capacity: a generous bound over
    a small table is not refused, a batch that really needs more than the
    built-in array is (both decided before any device call)."""
    lib = pa.lib()
    nul = ctypes.c_void_p(0)

    def na(mcl, maxb, S=8, Hq=64, D=128, P=0):
        return lib.pa_decode_noalloc(nul, nul, nul, nul, nul, nul, 0.1, 16, 8, S, Hq, D, maxb, mcl, 64, 2, P, nul)

    assert pa.pa_decode_workspace_size(8, 64, 128, 10 ** 6) > 32 * 1024 * 1024
    assert na(10 ** 6, 8) == 1          # table holds 128 tokens: one partition, no scratch; then null pointers
    assert pa.pa_decode_workspace_size(32, 64, 128, 2048 * 16) > 32 * 1024 * 1024
    assert na(10 ** 6, 2048, S=32) == 2  # 32768 tokens of table, 32 sequences: the scratch exceeds the array


def test_scheduler_raw_record_matches_tuples(pa):
    """step(raw=True) gives the same ops as arrays."""
    tc = wl.TraceConfig(block_size=4, max_running=12, num_requests=40, steps=80, prefix_len=10,
                        prompt_hi=30, output_mean=10.0, fork_every=4)
    reqs = wl.make_trace_requests(tc, 2)
    order = np.random.default_rng(2).permutation(70).tolist()
    pair = []
    for _ in range(2):
        bm = pa.BlockManager(70, tc.block_size, order)
        bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
        s = pa.Scheduler(bm, tc.max_running, wl.PREFIX_SEQ)
        for q in reqs:
            s.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
        pair.append(s)
    names = {"w": 0, "c": 1, "so": 2, "si": 3}
    n_ops = 0
    for step in range(tc.steps):
        a, b = pair[0].step(), pair[1].step(raw=True)
        assert b["ops"] is None and a["running"] == b["running"], step
        assert [names[o[0]] for o in a["ops"]] == b["op_kind"].tolist(), step
        assert [o[1] for o in a["ops"]] == b["op_a"].tolist(), step
        assert [o[2] for o in a["ops"]] == b["op_b"].tolist(), step
        assert [o[3] if o[0] == "w" else -1 for o in a["ops"]] == b["op_c"].tolist(), step
        n_ops += len(a["ops"])
    assert n_ops > 0
