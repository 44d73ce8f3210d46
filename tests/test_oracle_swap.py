"""Host swap pool: the oracle's block-manager model (CPU only).

Swap ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
"生产部署注意事项"): when GPU memory runs short, the KV cache of some requests
moves out to CPU memory and comes back once GPU memory is free.

Pins for the oracle's model: a hand-derived golden trace
(tests/golden/swap_trace.json) and a content check -- the test keeps its own
picture of every GPU and host slot, applies each copy the manager asks for,
and after every operation each resident sequence must read its own tokens
through its table, while each swapped-out one must find them in the GPU
blocks it still shares and the host blocks it was given.  Planted mistakes
must fail that check.  The helpers here also drive the C++ manager in
tests/test_swap.py.
"""

import json
import os

import numpy as np
import pytest

from oracle import block_manager as obm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


class _Model:
    NoBlocks, Invalid = obm.NoBlocks, obm.InvalidArg

    def __init__(self, nb, bs, ncpu, order=None, cls=obm.SwappingBlockManager):
        self.bm = cls(nb, bs, ncpu, order)
        self.bs = bs

    def allocate(self, s, n):
        self.bm.allocate(s, n)

    def fork(self, p, c):
        self.bm.fork(p, c)

    def append(self, s):
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

    def cpu_free(self):
        return list(self.bm.cpu_free)

    def ref(self, b):
        return self.bm.ref[b]

    def swapped(self, s):
        return self.bm.swapped(s)

    def invariants(self):
        self.bm.check()


def _replay(m):
    g = json.load(open(os.path.join(GOLDEN, "swap_trace.json")))
    for op in g["ops"]:
        exp, k = op["expect"], op["op"]
        seq = op.get("seq", op.get("child"))
        call = {"allocate": lambda: m.allocate(op["seq"], op["tokens"]),
                "fork": lambda: m.fork(op["parent"], op["child"]),
                "append": lambda: m.append(op["seq"]),
                "free": lambda: m.free(op["seq"]),
                "swap_out": lambda: m.swap_out(op["seq"]),
                "swap_in": lambda: m.swap_in(op["seq"])}[k]
        if "error" in exp:
            err = m.NoBlocks if exp["error"] == "no_blocks" else m.Invalid
            with pytest.raises(err):
                call()
        else:
            res = call()
            if "pairs" in exp:
                assert res == [tuple(p) for p in exp["pairs"]], op
            if "slot" in exp:
                assert res[0] == exp["slot"] and [res[1], res[2]] == exp["cow"], op
        if "table" in exp:
            assert m.table(seq) == exp["table"], op
        if "free" in exp:
            assert m.free_list() == exp["free"], op
        if "cpu_free" in exp:
            assert m.cpu_free() == exp["cpu_free"], op
        if "ref" in exp:
            for b, c in exp["ref"].items():
                assert m.ref(int(b)) == c, op
        m.invariants()


def test_model_golden_trace():
    g = json.load(open(os.path.join(GOLDEN, "swap_trace.json")))
    _replay(_Model(g["num_blocks"], g["block_size"], g["num_cpu_blocks"]))


class _Driver:
    """Applies operations and the copies they report to the test's own
    picture of the slots: gpu[(block, offset)] and cpu[(block, offset)] hold
    (sequence lineage, position) tags written the way decode writes them."""

    def __init__(self, m):
        self.m, self.bs = m, m.bs
        self.gpu, self.cpu = {}, {}
        self.toks = {}             # seq -> list of tags, one per position
        self.loc = {}              # swapped seq -> per logical block, True = host block
        self.next_tag = 0

    def _tag(self):
        self.next_tag += 1
        return self.next_tag

    def allocate(self, s, n):
        self.m.allocate(s, n)
        self.toks[s] = [self._tag() for _ in range(n)]
        t = self.m.table(s)
        for p, tag in enumerate(self.toks[s]):
            self.gpu[(t[p // self.bs], p % self.bs)] = tag

    def fork(self, p, c):
        self.m.fork(p, c)
        self.toks[c] = list(self.toks[p])

    def append(self, s):
        slot, src, dst = self.m.append(s)
        if src >= 0:
            for o in range(self.bs):
                if (src, o) in self.gpu:
                    self.gpu[(dst, o)] = self.gpu[(src, o)]
        tag = self._tag()
        self.toks[s].append(tag)
        self.gpu[(slot // self.bs, slot % self.bs)] = tag

    def free(self, s):
        self.m.free(s)
        del self.toks[s]
        self.loc.pop(s, None)

    def _copy(self, pairs, src, dst):
        # all sources are read before any destination is written (one launch)
        moved = {(d, o): src[(s_, o)] for s_, d in pairs for o in range(self.bs) if (s_, o) in src}
        dst.update(moved)

    def swap_out(self, s):
        before = self.m.table(s)
        pairs = self.m.swap_out(s)
        self._copy(pairs, self.gpu, self.cpu)
        # the pairs come in logical order: match them to the table's entries
        loc, k = [], 0
        for b in before:
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
            for p, tag in enumerate(toks):
                # a swapped-out sequence: host blocks for the ones it moved, GPU for the shared ones
                store = self.cpu if loc[p // self.bs] else self.gpu
                assert store.get((t[p // self.bs], p % self.bs)) == tag, (s, p)
        self.m.invariants()


def _stream(drivers, seed, n_ops=400):
    r = np.random.default_rng(seed)
    bs = drivers[0].bs
    live, nid, log = [], 0, []
    for _ in range(n_ops):
        c = r.random()
        res = [s for s in live if not drivers[0].m.swapped(s)]
        out = [s for s in live if drivers[0].m.swapped(s)]
        if c < 0.15 or not live:
            op = ("allocate", nid, int(r.integers(0, 4 * bs)))
        elif c < 0.25 and res:
            op = ("fork", res[int(r.integers(len(res)))], nid)
        elif c < 0.60 and res:
            op = ("append", res[int(r.integers(len(res)))])
        elif c < 0.72 and res:
            op = ("swap_out", res[int(r.integers(len(res)))])
        elif c < 0.86 and out:
            op = ("swap_in", out[int(r.integers(len(out)))])
        elif c < 0.90:
            op = ("append", live[int(r.integers(len(live)))])     # may hit a swapped sequence
        else:
            op = ("free", live[int(r.integers(len(live)))])
        outs = []
        for d in drivers:
            try:
                outs.append(getattr(d, op[0])(*op[1:]))
            except d.m.NoBlocks:
                outs.append("no_blocks")
            except d.m.Invalid:
                outs.append("invalid")
        assert all(o == outs[0] for o in outs), (op, outs)
        log.append((op, outs[0]))
        if outs[0] not in ("no_blocks", "invalid"):
            if op[0] == "allocate":
                live.append(op[1])
                nid += 1
            elif op[0] == "fork":
                live.append(op[2])
                nid += 1
            elif op[0] == "free":
                live.remove(op[1])
        for d in drivers:
            d.check()
    return log


@pytest.mark.parametrize("seed", range(10))
def test_model_content_on_random_streams(seed):
    r = np.random.default_rng(500 + seed)
    nb, bs, ncpu = int(r.integers(4, 40)), int(r.choice([1, 2, 4])), int(r.integers(0, 30))
    d = _Driver(_Model(nb, bs, ncpu, r.permutation(nb).tolist()))
    log = _stream([d], seed)
    kinds = {op[0] for op, o in log if o not in ("no_blocks", "invalid")}
    assert {"swap_out", "swap_in"} <= kinds or ncpu == 0


class _MovesShared(obm.SwappingBlockManager):
    """Mistake: shared blocks move to the host too (and leave the GPU)."""

    def swap_out(self, seq):
        if seq in self.tables and seq not in self.on_cpu:
            for b in self.tables[seq]:
                self.ref[b] = 1               # pretend every block is held alone
        return super().swap_out(seq)

    def check(self):
        pass


class _ForgetsCopy(obm.SwappingBlockManager):
    """Mistake: swap_in reports no copies for the second and later blocks."""

    def swap_in(self, seq):
        return super().swap_in(seq)[:1]

    def check(self):
        pass


@pytest.mark.parametrize("cls", [_MovesShared, _ForgetsCopy])
def test_content_check_catches_planted_mistakes(cls):
    caught = 0
    for seed in range(10):
        r = np.random.default_rng(500 + seed)
        nb, bs, ncpu = int(r.integers(4, 40)), int(r.choice([1, 2, 4])), int(r.integers(0, 30))
        try:
            _stream([_Driver(_Model(nb, bs, ncpu, r.permutation(nb).tolist(), cls=cls))], seed)
        except (AssertionError, KeyError, IndexError, ValueError):
            caught += 1
    assert caught >= 3, caught
