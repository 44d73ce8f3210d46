"""Reserved versus used KV slots (CPU only): pa_bm_usage and the trace study
against the oracle's accounting, which is pinned by closed forms."""

import numpy as np
import pytest

from oracle import block_manager as obm
from oracle import fragmentation as ofr
from oracle import scheduler as osch
from paged_kv_cache_381_b200 import workloads as wl


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    return pa


# ---- the oracle's accounting against closed forms ----------------------------------

@pytest.mark.parametrize("n,bs", [(1, 16), (16, 16), (17, 16), (100, 8), (1000, 32)])
def test_single_sequence_wastes_only_its_last_block_tail(n, bs):
    bm = obm.BlockManager(200, bs)
    bm.allocate(1, n)
    reserved, used = ofr.paged_step(bm)
    assert reserved == -(-n // bs) * bs and used == n
    assert reserved - used < bs


def test_shared_blocks_count_once_until_copied():
    bs = 4
    bm = obm.BlockManager(20, bs)
    bm.allocate(1, 10)                      # blocks: 4 + 4 + 2 filled
    bm.fork(1, 2)
    assert ofr.paged_step(bm) == (12, 10)   # same three blocks, same ten slots
    bm.append_slot(2)                       # copy-on-write of the shared last block
    # blocks: 2 shared full, parent's last (2 filled), child's copy (3 filled)
    assert ofr.paged_step(bm) == (16, 4 + 4 + 2 + 3)


def test_contiguous_and_static_by_hand():
    # two sequences: admitted with contexts 9 and 4 (their first steps show 10 and 5)
    steps = [([1, 2], [10, 5]), ([1, 2], [11, 6]), ([1], [12])]
    # reserved per step: (9 + 8) + (4 + 8), then again, then 17
    assert ofr.contiguous_trace(steps, 8) == (29 + 29 + 17, 15 + 17 + 12)
    # static: one batch of prompts 3 and 5, outputs 1 and 2 -> pad 5 + 2 = 7, lasts 2 steps
    assert ofr.static_trace([(3, 1), (5, 2)], 2, 10) == (7 * 2 * 2, (3 + 1 + 5 + 1) + (3 + 1 + 5 + 2))
    assert ofr.static_trace([(3, 1), (5, 2)], 2, 1) == (7 * 2, 3 + 1 + 5 + 1)


# ---- pa_bm_usage against the oracle ------------------------------------------------------

def test_native_usage_matches_oracle_on_random_streams(pa):
    r = np.random.default_rng(41)
    for trial in range(20):
        nb, bs = int(r.integers(4, 60)), int(r.choice([1, 2, 4, 8, 16]))
        order = r.permutation(nb).tolist()
        model, nat = obm.BlockManager(nb, bs, order), pa.BlockManager(nb, bs, order)
        live, nid = [], 0
        for _ in range(300):
            c = r.random()
            try:
                if c < 0.2 or not live:
                    model.allocate(nid, int(r.integers(0, 4 * bs)))
                    nat.allocate(nid, model.context_len(nid))
                    live.append(nid)
                    nid += 1
                elif c < 0.35:
                    p = live[int(r.integers(len(live)))]
                    model.fork(p, nid)
                    nat.fork(p, nid)
                    live.append(nid)
                    nid += 1
                elif c < 0.85:
                    s = live[int(r.integers(len(live)))]
                    model.append_slot(s)
                    nat.append_slot(s)
                else:
                    s = live.pop(int(r.integers(len(live))))
                    model.free(s)
                    nat.free(s)
            except obm.NoBlocks:
                continue
            reserved, used = ofr.paged_step(model)
            held, filled = nat.usage()
            assert (held * bs, filled) == (reserved, used)


# ---- the trace study against the oracle ------------------------------------------------

def _oracle_trace(tc, seed, steps):
    reqs = wl.make_trace_requests(tc, seed)
    bs = tc.block_size
    peak = sum(-(-(tc.prefix_len + q.prompt_len + q.output_len) // bs) + 1 for q in reqs)
    peak += sum(-(-(tc.prefix_len + q.prompt_len + q.fork_output_len) // bs) + 1 for q in reqs if q.fork_child >= 0)
    bm = obm.BlockManager(peak + -(-tc.prefix_len // bs), bs)
    bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = osch.Scheduler(bm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        sch.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child,
                                     q.fork_output_len))
    paged, timeline = [], []
    for _ in range(steps):
        rec = sch.step()
        paged.append(ofr.paged_step(bm))
        timeline.append((rec.running, rec.context_lens))
    members = []
    for q in reqs:
        pre = tc.prefix_len if q.shares_prefix else 0
        members.append((pre + q.prompt_len, q.output_len))
        if q.fork_child >= 0:
            members.append((pre + q.prompt_len, q.fork_output_len))
    return paged, timeline, members


def test_study_matches_oracle_on_the_trace(pa):
    from paged_kv_cache_381_b200 import fragmentation as fr
    tc, steps = wl.TRACE, 80
    paged, timeline, members = _oracle_trace(tc, 0, steps)
    rows = fr.paged_usage(tc, 0, steps)
    assert [(h * tc.block_size, f) for h, f, _, _ in rows] == paged
    res = fr.study(tc, 0, steps, max_new_tokens=(2048, 512))
    assert (res["paged"]["reserved"], res["paged"]["used"]) == tuple(map(sum, zip(*paged)))
    for m in (2048, 512):
        c = res["contiguous"][str(m)]
        assert (c["reserved"], c["used"]) == ofr.contiguous_trace(timeline, m)
    st = res["static"]
    assert (st["reserved"], st["used"]) == ofr.static_trace(members, tc.max_running, steps)


def test_paged_waste_is_small_on_the_trace(pa):
    """The pages report under 5% KV fragmentation with paging against tens of
    percent with contiguous reservation; the synthetic trace shows the same
    ordering."""
    from paged_kv_cache_381_b200 import fragmentation as fr
    res = fr.study(wl.TRACE, 0, 120)
    assert res["paged"]["waste"] < 0.05
    assert res["contiguous"]["2048"]["waste"] > 0.3 and res["static"]["waste"] > 0.3
    assert res["paged"]["waste"] < res["contiguous"]["exact"]["waste"]
