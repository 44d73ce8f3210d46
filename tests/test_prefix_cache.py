"""Prefix cache of the block manager (CPU only).

Prefix caching ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
section "Prefix Caching前缀复用优化"): a request whose prompt begins with KV
that is already cached references those blocks and skips their prefill.

The oracle's model is pinned by
  * a hand-derived golden trace (tests/golden/prefix_cache_trace.json);
  * a content check: the test keeps its own picture of every slot, written
    the way prefill and decode would write it (a slot holds the whole token
    prefix its K/V depends on), and after every operation each live sequence
    must read, through its block table, exactly the prefixes of its tokens;
  * closed forms for shared system prompts and repeated conversations;
  * planted mistakes (a key without the prefix, eviction that keeps the name)
    that the content check must catch.
The C++ manager (libpa.so) is then checked against the model op by op.
"""

import json
import os

import numpy as np
import pytest

from oracle import block_manager as obm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    return pa


# ---- adapters: one interface over the model and the C++ manager --------------

class _Model:
    NoBlocks = obm.NoBlocks

    def __init__(self, nb, bs, order=None, cls=obm.PrefixCachingBlockManager):
        self.bm = cls(nb, bs, order)
        self.bs = bs

    def allocate_prefix(self, seq, toks):
        return self.bm.allocate_prefix(seq, toks)

    def allocate(self, seq, n):
        self.bm.allocate(seq, n)

    def append_token(self, seq, t):
        return self.bm.append_token(seq, t)

    def append_slot(self, seq):
        return self.bm.append_slot(seq)

    def fork(self, p, c):
        self.bm.fork(p, c)

    def free(self, seq):
        self.bm.free(seq)

    def table(self, seq):
        return self.bm.block_table(seq)

    def free_list(self):
        return list(self.bm.free_list)

    def evictable(self):
        return list(self.bm.evictable)

    def ref(self, b):
        return self.bm.ref[b]

    def stats(self):
        return self.bm.num_cached, len(self.bm.evictable), self.bm.hits, self.bm.lookups

    def num_free(self):
        return self.bm.num_free

    def invariants(self):
        self.bm.check()


class _Native(_Model):
    def __init__(self, pa, nb, bs, order=None):
        self.pa = pa
        self.bm = pa.BlockManager(nb, bs, order)
        self.bm.enable_prefix_cache(True)
        self.bs = bs
        self.NoBlocks = pa.NoBlocksError

    def table(self, seq):
        return self.bm.block_table(seq)

    def free_list(self):
        return self.bm.free_list()

    def evictable(self):
        return self.bm.evictable()

    def ref(self, b):
        return self.bm.ref_count(b)

    def stats(self):
        return self.bm.cache_stats()

    def num_free(self):
        return self.bm.num_free

    def invariants(self):
        cached, ev, hits, lookups = self.bm.cache_stats()
        assert ev == len(self.bm.evictable()) and ev <= cached and hits <= lookups
        assert self.bm.num_free == len(self.bm.free_list()) + ev


# ---- golden trace ---------------------------------------------------------------

def _replay_golden(m):
    with open(os.path.join(GOLDEN, "prefix_cache_trace.json")) as f:
        g = json.load(f)
    for op in g["ops"]:
        exp, k = op["expect"], op["op"]
        res = None
        if "error" in exp:
            with pytest.raises(m.NoBlocks):
                if k == "allocate_prefix":
                    m.allocate_prefix(op["seq"], op["tokens"])
                else:
                    m.append_token(op["seq"], op["token"])
        elif k == "allocate_prefix":
            res = m.allocate_prefix(op["seq"], op["tokens"])
            assert res == exp["cached"], op
        elif k == "append_token":
            res = m.append_token(op["seq"], op["token"])
            assert res[0] == exp["slot"] and [res[1], res[2]] == exp["cow"], op
        elif k == "free":
            m.free(op["seq"])
        if "table" in exp:
            assert m.table(op["seq"]) == exp["table"], op
        if "free" in exp:
            assert m.free_list() == exp["free"], op
        if "evictable" in exp:
            assert m.evictable() == exp["evictable"], op
        if "num_free" in exp:
            assert m.num_free() == exp["num_free"], op
        if "ref" in exp:
            for b, c in exp["ref"].items():
                assert m.ref(int(b)) == c, op
        st = m.stats()
        if "cached_blocks" in exp:
            assert st[0] == exp["cached_blocks"], op
        if k == "stats":
            assert st == (exp["cached_blocks"], exp["evictable_count"], exp["hits"], exp["lookups"])
    return g


def test_model_golden_trace():
    g = json.load(open(os.path.join(GOLDEN, "prefix_cache_trace.json")))
    m = _Model(g["num_blocks"], g["block_size"], g["initial_free_order"])
    _replay_golden(m)
    m.bm.check()


def test_native_golden_trace(pa):
    g = json.load(open(os.path.join(GOLDEN, "prefix_cache_trace.json")))
    _replay_golden(_Native(pa, g["num_blocks"], g["block_size"], g["initial_free_order"]))


# ---- content check ---------------------------------------------------------------

class _Driver:
    """Runs operations on an adapter and keeps the test's own picture of the
    slots: a slot written for position p of a sequence holds tuple(tokens[:p+1]),
    which is what that position's K/V depends on."""

    def __init__(self, m):
        self.m = m
        self.bs = m.bs
        self.store = {}
        self.toks = {}              # the test's record of each live sequence's tokens
        self.fresh = -1             # ids for tokens the manager is not told

    def _unique(self):
        self.fresh -= 1
        return self.fresh

    def _write(self, seq, start):
        t = self.m.table(seq)
        toks = self.toks[seq]
        for p in range(start, len(toks)):
            self.store[t[p // self.bs] * self.bs + p % self.bs] = tuple(toks[:p + 1])

    def allocate_prefix(self, seq, toks):
        c = self.m.allocate_prefix(seq, toks)
        assert c % self.bs == 0 and 0 <= c <= len(toks)
        self.toks[seq] = list(toks)
        self._write(seq, c)
        return c

    def allocate(self, seq, n):
        self.m.allocate(seq, n)
        self.toks[seq] = [self._unique() for _ in range(n)]
        self._write(seq, 0)

    def _append(self, seq, tok, known):
        res = self.m.append_token(seq, tok) if known else self.m.append_slot(seq)
        slot, src, dst = res
        if src >= 0:                      # copy-on-write: the caller copies the block
            for i in range(self.bs):
                if src * self.bs + i in self.store:
                    self.store[dst * self.bs + i] = self.store[src * self.bs + i]
        self.toks[seq].append(tok)
        t = self.m.table(seq)
        p = len(self.toks[seq]) - 1
        assert slot == t[p // self.bs] * self.bs + p % self.bs
        self.store[slot] = tuple(self.toks[seq])
        return res

    def append_token(self, seq, tok):
        return self._append(seq, tok, True)

    def append_slot(self, seq):
        return self._append(seq, self._unique(), False)

    def fork(self, p, c):
        self.m.fork(p, c)
        self.toks[c] = list(self.toks[p])

    def free(self, seq):
        self.m.free(seq)
        del self.toks[seq]

    def check(self):
        for seq, toks in self.toks.items():
            t = self.m.table(seq)
            for p in range(len(toks)):
                got = self.store.get(t[p // self.bs] * self.bs + p % self.bs)
                assert got == tuple(toks[:p + 1]), (seq, p, got, toks[:p + 1])
        self.m.invariants()


def _run_stream(drivers, seed, n_ops=300, vocab=4):
    """Apply one seeded operation stream to every driver (errors must agree)
    and check every driver's content after each operation.

    Prompts overlap heavily: a shared system prompt, a replay of an earlier
    conversation, or random tokens, plus a random suffix; decode appends
    tokens from a small vocabulary so identical blocks also arise
    independently.  Returns the operations applied and their outcomes."""
    r = np.random.default_rng(seed)
    bs = drivers[0].bs
    systems = [[int(x) for x in r.integers(0, vocab, int(r.integers(1, 4)) * bs)] for _ in range(3)]
    history, live, nid, log = [], [], 0, []
    for _ in range(n_ops):
        c = r.random()
        if c < 0.25 or not live:
            kind = r.random()
            if kind < 0.4:
                toks = list(systems[int(r.integers(3))])
            elif kind < 0.7 and history:
                toks = list(history[int(r.integers(len(history)))])
            else:
                toks = []
            toks += [int(x) for x in r.integers(0, vocab, int(r.integers(0, 2 * bs + 1)))]
            op = ("allocate_prefix", nid, toks)
        elif c < 0.28:
            op = ("allocate", nid, int(r.integers(0, 2 * bs)))
        elif c < 0.36:
            op = ("fork", live[int(r.integers(len(live)))], nid)
        elif c < 0.80:
            op = ("append_token", live[int(r.integers(len(live)))], int(r.integers(0, vocab)))
        elif c < 0.84:
            op = ("append_slot", live[int(r.integers(len(live)))])
        else:
            op = ("free", live[int(r.integers(len(live)))])
        outs = []
        for d in drivers:
            try:
                outs.append(getattr(d, op[0])(*op[1:]))
            except d.m.NoBlocks:
                outs.append("no_blocks")
        assert all(o == outs[0] for o in outs), (op, outs)
        log.append((op, outs[0]))
        if outs[0] != "no_blocks":
            if op[0] in ("allocate_prefix", "allocate", "fork"):
                live.append(nid)
                nid += 1
            elif op[0] == "free":
                live.remove(op[1])
            else:
                seq = op[1]
                known = [t for t in drivers[0].toks[seq] if t >= 0]
                if len(known) == len(drivers[0].toks[seq]) and r.random() < 0.15:
                    history.append(known)       # a conversation to continue later
        for d in drivers:
            d.check()
    return log


@pytest.mark.parametrize("seed", range(12))
def test_model_content_on_random_streams(seed):
    r = np.random.default_rng(100 + seed)
    nb, bs = int(r.integers(4, 40)), int(r.choice([1, 2, 4]))
    d = _Driver(_Model(nb, bs, r.permutation(nb).tolist()))
    log = _run_stream([d], seed)
    d.m.bm.check()
    # the stream must exercise the cache: hits, evictions and refusals all occur
    assert d.m.bm.hits > 0
    assert any(o == "no_blocks" for _, o in log) or nb > 30


# ---- planted mistakes: the content check must catch each -----------------------

class _KeyByBlockOnly(obm.PrefixCachingBlockManager):
    """Mistake: a block is named by its own tokens only, not the whole prefix."""

    def _key(self, toks, j):
        return tuple(toks[j * self.block_size:(j + 1) * self.block_size])

    def check(self):
        pass


class _EvictKeepsName(obm.PrefixCachingBlockManager):
    """Mistake: eviction reuses a block but leaves its name in the cache."""

    def _take(self):
        if self.free_list:
            return self.free_list.pop()
        return self.evictable.pop(0)

    def check(self):
        pass


@pytest.mark.parametrize("cls", [_KeyByBlockOnly, _EvictKeepsName])
def test_content_check_catches_planted_mistakes(cls):
    caught = 0
    for seed in range(12):
        r = np.random.default_rng(100 + seed)
        nb, bs = int(r.integers(4, 40)), int(r.choice([1, 2, 4]))
        d = _Driver(_Model(nb, bs, r.permutation(nb).tolist(), cls=cls))
        try:
            _run_stream([d], seed)
        except AssertionError:
            caught += 1
    assert caught >= 3, caught


def test_partial_block_is_never_shared():
    """Two prompts that agree on a partly filled last block share no block
    there: the second request writes its own copy."""
    m = _Model(8, 4)
    assert m.allocate_prefix(1, [1, 2, 3, 4, 5, 6]) == 0
    m.free(1)
    assert m.allocate_prefix(2, [1, 2, 3, 4, 5, 6]) == 4     # only the full block is found
    t2 = m.table(2)
    assert m.allocate_prefix(3, [1, 2, 3, 4, 5, 6]) == 4
    t3 = m.table(3)
    assert t2[0] == t3[0] and t2[1] != t3[1]
    m.bm.check()


# ---- closed forms ---------------------------------------------------------------

@pytest.mark.parametrize("bs,sys_blocks,n_req", [(16, 8, 10), (4, 3, 7), (1, 5, 4)])
def test_shared_system_prompt_hits(bs, sys_blocks, n_req):
    """n_req prompts = one system prompt of L = sys_blocks*bs tokens + distinct
    suffixes, in a pool with room for all: the first request finds nothing,
    every later one finds the L system tokens; hits = (n_req-1)*sys_blocks."""
    L = sys_blocks * bs
    system = list(range(1000, 1000 + L))
    m = _Model(4 * n_req * (sys_blocks + 2), bs)
    cached = [m.allocate_prefix(i, system + [i, i + 1, i + 2]) for i in range(n_req)]
    assert cached == [0] + [L] * (n_req - 1)
    st = m.stats()
    assert st[2] == (n_req - 1) * sys_blocks
    # probes: the first request stops at its first block; a later one walks the
    # system blocks and, when the 3-token suffix fills a block, one miss more
    assert st[3] == 1 + (n_req - 1) * (sys_blocks + (1 if bs <= 3 else 0))
    # the system prompt's blocks are referenced by every request
    for j in range(sys_blocks):
        assert m.ref(m.table(0)[j]) == n_req
    m.bm.check()


def test_multi_turn_conversation_reuses_all_full_blocks():
    """A conversation continued after its request finished finds every full
    block it had filled (prompt and decoded tokens alike)."""
    bs = 4
    m = _Model(64, bs)
    turn1 = list(range(10))                  # 2 full blocks + 2 tokens
    assert m.allocate_prefix(1, turn1) == 0
    out = [50, 51, 52, 53, 54, 55, 56]       # decode fills block 3 and 4 partially
    for t in out:
        m.append_token(1, t)
    conv = turn1 + out                       # 17 tokens = 4 full blocks + 1
    m.free(1)
    assert m.stats()[1] == 4                 # the 4 full blocks wait on the evictable list
    turn2 = conv + [60, 61, 62]
    assert m.allocate_prefix(2, turn2) == 16
    m.bm.check()


def test_cache_off_behaves_like_plain_manager(pa):
    """With the cache disabled, allocate_prefix finds nothing and the pool
    evolves exactly as the plain manager's."""
    bm = pa.BlockManager(10, 2, list(range(10)))
    plain = obm.BlockManager(10, 2, list(range(10)))
    assert bm.allocate_prefix(1, [1, 2, 3, 4, 5]) == 0
    plain.allocate(1, 5)
    bm.free(1)
    plain.free(1)
    assert bm.allocate_prefix(2, [1, 2, 3, 4, 5]) == 0
    plain.allocate(2, 5)
    assert bm.block_table(2) == plain.block_table(2)
    assert bm.free_list() == plain.free_list
    assert bm.cache_stats() == (0, 0, 0, 0)


# ---- the C++ manager against the model ----------------------------------------

@pytest.mark.parametrize("seed", range(16))
def test_native_matches_model_op_by_op(pa, seed):
    r = np.random.default_rng(300 + seed)
    nb, bs = int(r.integers(3, 48)), int(r.choice([1, 2, 4, 8]))
    order = r.permutation(nb).tolist()
    model, nat = _Driver(_Model(nb, bs, order)), _Driver(_Native(pa, nb, bs, order))
    _run_stream([model, nat], seed, n_ops=400)
    assert model.m.free_list() == nat.m.free_list()
    assert model.m.evictable() == nat.m.evictable()
    assert model.m.stats() == nat.m.stats()
    for s in model.toks:
        assert model.m.table(s) == nat.m.table(s)
    assert [model.m.ref(b) for b in range(nb)] == [nat.m.ref(b) for b in range(nb)]


def test_conversation_workload_host_side(pa):
    """The multi-turn workload the GPU test runs, host side only: it reuses
    most K/V rows and some continued conversations lose blocks to eviction."""
    import sys
    sys.path.insert(0, ROOT)
    from tests.prefix_workload import NullDevice, run_conversations
    st = run_conversations(NullDevice())
    assert st["written"] + st["cached"] == st["total"]
    assert st["cached"] > 0.4 * st["total"] and st["short"] > 0, st
