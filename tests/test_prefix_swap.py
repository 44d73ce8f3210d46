"""Prefix cache and host swap pool together (CPU only).

The two sections of "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置"
("Prefix Caching前缀复用优化", "生产部署注意事项") at once: a swapped-out
sequence's named blocks stay reusable on the GPU until evicted, and come back
without a copy while the cache still names them.

The oracle's model (oracle.block_manager.PrefixSwappingBlockManager) is pinned
by a hand-derived golden trace (tests/golden/prefix_swap_trace.json) and by a
content check over random operation streams: the test keeps its own picture
of every GPU and host slot (a slot holds the whole token prefix its K/V
depends on), applies each copy the manager reports, and after every operation
each live sequence must read exactly its prefixes through its table (host
blocks for the blocks a swapped-out sequence moved).  Planted mistakes fail
that check.  The C++ manager is then checked against the model op by op.
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


class _Model:
    NoBlocks, Invalid = obm.NoBlocks, obm.InvalidArg

    def __init__(self, nb, bs, ncpu, order=None, cls=obm.PrefixSwappingBlockManager):
        self.bm = cls(nb, bs, ncpu, order)
        self.bs = bs

    def allocate_prefix(self, s, toks):
        return self.bm.allocate_prefix(s, toks)

    def allocate(self, s, n):
        self.bm.allocate(s, n)

    def fork(self, p, c):
        self.bm.fork(p, c)

    def append_token(self, s, t):
        return self.bm.append_token(s, t)

    def append_slot(self, s):
        return self.bm.append_slot(s)

    def free(self, s):
        self.bm.free(s)

    def swap_out(self, s):
        return [tuple(p) for p in self.bm.swap_out(s)]

    def swap_in(self, s):
        return [tuple(p) for p in self.bm.swap_in(s)]

    def table(self, s):
        return list(self.bm.tables[s])

    def free_list(self):
        return list(self.bm.free_list)

    def evictable(self):
        return list(self.bm.evictable)

    def cpu_free(self):
        return list(self.bm.cpu_free)

    def ref(self, b):
        return self.bm.ref[b]

    def swapped(self, s):
        return self.bm.swapped(s)

    def num_free(self):
        return self.bm.num_free

    def num_cached(self):
        return self.bm.num_cached

    def invariants(self):
        self.bm.check()


class _Native(_Model):
    def __init__(self, pa, nb, bs, ncpu, order=None):
        self.bm = pa.BlockManager(nb, bs, order)
        self.bm.enable_prefix_cache(True)
        self.bm.set_cpu_blocks(ncpu)
        self.bs = bs
        self.NoBlocks, self.Invalid = pa.NoBlocksError, pa.PagedAttentionError

    def swap_out(self, s):
        return [tuple(int(x) for x in p) for p in self.bm.swap_out(s)]

    def swap_in(self, s):
        return [tuple(int(x) for x in p) for p in self.bm.swap_in(s)]

    def table(self, s):
        return self.bm.block_table(s)

    def free_list(self):
        return self.bm.free_list()

    def evictable(self):
        return self.bm.evictable()

    def cpu_free(self):
        return self.bm.cpu_free_list()

    def ref(self, b):
        return self.bm.ref_count(b)

    def swapped(self, s):
        return self.bm.swapped(s)

    def num_free(self):
        return self.bm.num_free

    def num_cached(self):
        return self.bm.cache_stats()[0]

    def invariants(self):
        cached, ev, hits, lookups = self.bm.cache_stats()
        assert ev == len(self.bm.evictable()) and ev <= cached and hits <= lookups
        assert self.bm.num_free == len(self.bm.free_list()) + ev


# ---- golden trace ---------------------------------------------------------------

def _replay(m):
    with open(os.path.join(GOLDEN, "prefix_swap_trace.json")) as f:
        g = json.load(f)
    for op in g["ops"]:
        exp, k = op["expect"], op["op"]
        call = {"allocate_prefix": lambda: m.allocate_prefix(op["seq"], op["tokens"]),
                "allocate": lambda: m.allocate(op["seq"], op["tokens"]),
                "append_token": lambda: m.append_token(op["seq"], op["token"]),
                "free": lambda: m.free(op["seq"]),
                "swap_out": lambda: m.swap_out(op["seq"]),
                "swap_in": lambda: m.swap_in(op["seq"])}[k]
        if "error" in exp:
            with pytest.raises(m.NoBlocks):
                call()
        else:
            res = call()
            if "cached" in exp:
                assert res == exp["cached"], op
            if "pairs" in exp:
                assert res == [tuple(p) for p in exp["pairs"]], op
            if "slot" in exp:
                assert res[0] == exp["slot"] and [res[1], res[2]] == exp["cow"], op
        if "table" in exp:
            assert m.table(op["seq"]) == exp["table"], op
        if "free" in exp:
            assert m.free_list() == exp["free"], op
        if "evictable" in exp:
            assert m.evictable() == exp["evictable"], op
        if "cpu_free" in exp:
            assert m.cpu_free() == exp["cpu_free"], op
        if "num_free" in exp:
            assert m.num_free() == exp["num_free"], op
        if "cached_blocks" in exp:
            assert m.num_cached() == exp["cached_blocks"], op
        if "ref" in exp:
            for b, c in exp["ref"].items():
                assert m.ref(int(b)) == c, op
        m.invariants()


def test_model_golden_trace():
    g = json.load(open(os.path.join(GOLDEN, "prefix_swap_trace.json")))
    _replay(_Model(g["num_blocks"], g["block_size"], g["num_cpu_blocks"]))


def test_native_golden_trace(pa):
    g = json.load(open(os.path.join(GOLDEN, "prefix_swap_trace.json")))
    _replay(_Native(pa, g["num_blocks"], g["block_size"], g["num_cpu_blocks"]))


# ---- content check ---------------------------------------------------------------

class _Driver:
    """Runs operations and keeps the test's own picture of the GPU and host
    slots: a slot written for position p of a sequence holds tuple(tokens[:p+1])."""

    def __init__(self, m):
        self.m, self.bs = m, m.bs
        self.gpu, self.cpu = {}, {}
        self.toks = {}             # live sequence -> its tokens (negative ids: not told to the manager)
        self.loc = {}              # swapped sequence -> per logical block, True = host block
        self.fresh = -1

    def _unique(self):
        self.fresh -= 1
        return self.fresh

    def _write(self, s, start):
        t, toks = self.m.table(s), self.toks[s]
        for p in range(start, len(toks)):
            self.gpu[(t[p // self.bs], p % self.bs)] = tuple(toks[:p + 1])

    def allocate_prefix(self, s, toks):
        c = self.m.allocate_prefix(s, toks)
        self.toks[s] = list(toks)
        self._write(s, c)
        return c

    def allocate(self, s, n):
        self.m.allocate(s, n)
        self.toks[s] = [self._unique() for _ in range(n)]
        self._write(s, 0)

    def fork(self, p, c):
        self.m.fork(p, c)
        self.toks[c] = list(self.toks[p])

    def _append(self, s, tok, known):
        res = self.m.append_token(s, tok) if known else self.m.append_slot(s)
        slot, src, dst = res
        if src >= 0:
            for o in range(self.bs):
                if (src, o) in self.gpu:
                    self.gpu[(dst, o)] = self.gpu[(src, o)]
        self.toks[s].append(tok)
        self.gpu[(slot // self.bs, slot % self.bs)] = tuple(self.toks[s])
        return res

    def append_token(self, s, tok):
        return self._append(s, tok, True)

    def append_slot(self, s):
        return self._append(s, self._unique(), False)

    def free(self, s):
        self.m.free(s)
        del self.toks[s]
        self.loc.pop(s, None)

    def _copy(self, pairs, src, dst):
        moved = {(d, o): src[(a, o)] for a, d in pairs for o in range(self.bs) if (a, o) in src}
        dst.update(moved)

    def swap_out(self, s):
        before = self.m.table(s)
        pairs = self.m.swap_out(s)
        self._copy(pairs, self.gpu, self.cpu)
        loc, k = [], 0
        for b in before:                     # pairs come in logical order
            moved = k < len(pairs) and pairs[k][0] == b
            loc.append(moved)
            k += moved
        assert k == len(pairs)
        self.loc[s] = loc
        return pairs

    def swap_in(self, s):
        pairs = self.m.swap_in(s)
        self._copy(pairs, self.cpu, self.gpu)
        del self.loc[s]
        return pairs

    def check(self):
        for s, toks in self.toks.items():
            t = self.m.table(s)
            assert self.m.swapped(s) == (s in self.loc)
            loc = self.loc.get(s, [False] * len(t))
            for p in range(len(toks)):
                store = self.cpu if loc[p // self.bs] else self.gpu
                got = store.get((t[p // self.bs], p % self.bs))
                assert got == tuple(toks[:p + 1]), (s, p, got, toks[:p + 1])
        self.m.invariants()


def _stream(drivers, seed, n_ops=400, vocab=3):
    """One seeded operation stream applied to every driver (outcomes must
    agree), the content checked after every operation.  Prompts overlap (shared
    system prompts, replayed conversations), so swapped-out sequences' named
    blocks are hit by new requests, evicted, and taken back."""
    r = np.random.default_rng(seed)
    bs = drivers[0].bs
    systems = [[int(x) for x in r.integers(0, vocab, int(r.integers(1, 4)) * bs)] for _ in range(3)]
    history, live, nid, log = [], [], 0, []
    for _ in range(n_ops):
        res = [s for s in live if not drivers[0].m.swapped(s)]
        out = [s for s in live if drivers[0].m.swapped(s)]
        c = r.random()
        if c < 0.2 or not live:
            kind = r.random()
            if kind < 0.4:
                toks = list(systems[int(r.integers(3))])
            elif kind < 0.7 and history:
                toks = list(history[int(r.integers(len(history)))])
            else:
                toks = []
            toks += [int(x) for x in r.integers(0, vocab, int(r.integers(0, 2 * bs + 1)))]
            op = ("allocate_prefix", nid, toks)
        elif c < 0.23:
            op = ("allocate", nid, int(r.integers(0, 2 * bs)))
        elif c < 0.28 and res:
            op = ("fork", res[int(r.integers(len(res)))], nid)
        elif c < 0.62 and res:
            op = ("append_token", res[int(r.integers(len(res)))], int(r.integers(0, vocab)))
        elif c < 0.65 and res:
            op = ("append_slot", res[int(r.integers(len(res)))])
        elif c < 0.76 and res:
            op = ("swap_out", res[int(r.integers(len(res)))])
        elif c < 0.88 and out:
            op = ("swap_in", out[int(r.integers(len(out)))])
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
            elif op[0] in ("append_token", "append_slot"):
                known = [t for t in drivers[0].toks[op[1]] if t >= 0]
                if len(known) == len(drivers[0].toks[op[1]]) and r.random() < 0.15:
                    history.append(known)
        for d in drivers:
            d.check()
    return log


@pytest.mark.parametrize("seed", range(16))
def test_model_content_on_random_streams(seed):
    r = np.random.default_rng(900 + seed)
    nb, bs, ncpu = int(r.integers(4, 40)), int(r.choice([1, 2, 4])), int(r.integers(0, 30))
    d = _Driver(_Model(nb, bs, ncpu, r.permutation(nb).tolist()))
    log = _stream([d], seed)
    d.m.bm.check()
    assert any(op[0] == "swap_in" and o != "no_blocks" for op, o in log) or ncpu == 0


def test_streams_take_blocks_back_without_a_copy():
    """Across the streams, swap-in finds remembered blocks still cached (no
    copy) and evicted ones (copy), and swapped-out blocks are hit by new
    requests while their owner is away."""
    taken_back = copied = 0
    for seed in range(16):
        r = np.random.default_rng(900 + seed)
        nb, bs, ncpu = int(r.integers(4, 40)), int(r.choice([1, 2, 4])), int(r.integers(0, 30))
        m = _Model(nb, bs, ncpu, r.permutation(nb).tolist())
        d = _Driver(m)
        orig = m.bm.swap_in

        def counting(seq, orig=orig, m=m):
            nonlocal taken_back, copied
            host = sum(m.bm.on_cpu[seq])
            pairs = orig(seq)
            copied += len(pairs)
            taken_back += host - len(pairs)
            return pairs

        m.bm.swap_in = counting
        _stream([d], seed)
    assert taken_back > 0 and copied > 0


# ---- planted mistakes: the content check must catch each -----------------------

class _TakeBackWithoutNameCheck(obm.PrefixSwappingBlockManager):
    """Mistake: swap-in takes a remembered block back even after it was evicted."""

    def swap_in(self, seq):
        table, loc, left = self.tables[seq], self.on_cpu[seq], self.left[seq]
        if sum(loc) > self.num_free:
            raise obm.NoBlocks("no blocks")
        pairs = []
        for j, here in enumerate(loc):
            if not here:
                continue
            c, kept = table[j], left[j]
            if kept is not None:
                g = kept[0]
                if g in self.evictable:
                    self.evictable.remove(g)
                if g in self.free_list:
                    self.free_list.remove(g)
                self.ref[g] += 1
            else:
                g = self._take()
                self.ref[g] = 1
                pairs.append((c, g))
            self.cpu_free.append(c)
            table[j] = g
        del self.on_cpu[seq], self.left[seq]
        return pairs

    def check(self):
        pass


class _SwapOutFreesNamed(obm.PrefixSwappingBlockManager):
    """Mistake: swap-out frees named blocks outright but leaves their names."""

    def swap_out(self, seq):
        pairs = super().swap_out(seq)
        for g, _ in pairs:
            if g in self.evictable:
                self.evictable.remove(g)
                self.free_list.append(g)
        return pairs

    def check(self):
        pass


@pytest.mark.parametrize("cls", [_TakeBackWithoutNameCheck, _SwapOutFreesNamed])
def test_planted_mistakes_fail_the_content_check(cls):
    caught = 0
    for seed in range(16):
        r = np.random.default_rng(900 + seed)
        nb, bs, ncpu = int(r.integers(4, 40)), int(r.choice([1, 2, 4])), int(r.integers(0, 30))
        d = _Driver(_Model(nb, bs, ncpu, r.permutation(nb).tolist(), cls=cls))
        try:
            _stream([d], seed)
        except AssertionError:
            caught += 1
    assert caught > 0


# ---- the C++ manager against the model -------------------------------------------

@pytest.mark.parametrize("seed", range(16))
def test_native_matches_model_op_by_op(pa, seed):
    r = np.random.default_rng(900 + seed)
    nb, bs, ncpu = int(r.integers(4, 40)), int(r.choice([1, 2, 4])), int(r.integers(0, 30))
    order = r.permutation(nb).tolist()
    model, nat = _Driver(_Model(nb, bs, ncpu, order)), _Driver(_Native(pa, nb, bs, ncpu, order))
    _stream([model, nat], seed)
    assert model.m.free_list() == nat.m.free_list()
    assert model.m.evictable() == nat.m.evictable()
    assert model.m.cpu_free() == nat.m.cpu_free()
    assert model.m.num_cached() == nat.m.num_cached()
    for s in model.toks:
        assert model.m.table(s) == nat.m.table(s)
        assert model.m.swapped(s) == nat.m.swapped(s)
    assert [model.m.ref(b) for b in range(nb)] == [nat.m.ref(b) for b in range(nb)]
