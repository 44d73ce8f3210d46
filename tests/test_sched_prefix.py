"""Scheduler admissions through the prefix cache (CPU only).

[P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
"Prefix Caching前缀复用优化": a request whose prompt begins with cached KV
references those blocks and skips their prefill.  The scheduler's model
(oracle.scheduler.Scheduler with ``prefix_cache=True``) is pinned by a content
check: the test replays every step's record (cache writes, copy-on-write
copies, swap copies) on its own picture of the GPU and host slots -- a slot
written for position p of a sequence holds that sequence's token prefix up to
p, from the test's own record of prompts and generated tokens -- and after
every step each running sequence must read its prefixes through its table.
Writes skipped for cached positions are only correct if the blocks found hold
exactly those prefixes.  Planted mistakes fail the check.  The C++ scheduler
is then checked against the model step by step.
"""

import numpy as np
import pytest

from oracle import block_manager as obm
from oracle import scheduler as osch
from paged_kv_cache_381_b200 import workloads as wl

VOCAB = 4


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    return pa


def token_fn(seq, pos):
    return wl.generated_token(seq, pos, VOCAB)


def _trace(seed, bs, n_requests=40, prefix_len=10):
    """Requests of the continuous-batching trace with prompt token ids: the
    prefix-sharing ones start with the system prefix; a third of the others
    replay an earlier request's prompt (a continued conversation)."""
    tc = wl.TraceConfig(block_size=bs, max_running=12, num_requests=n_requests, steps=120,
                        prefix_len=prefix_len, prompt_hi=30, output_mean=10.0, fork_every=4)
    reqs = wl.make_trace_requests(tc, seed)
    r = np.random.default_rng([seed, 77])
    prefix = [int(x) for x in r.integers(0, VOCAB, prefix_len)]
    prompts = []
    for q in reqs:
        if prompts and r.random() < 0.33:
            base = prompts[int(r.integers(len(prompts)))]
            toks = (base + [int(x) for x in r.integers(0, VOCAB, q.prompt_len)])[:q.prompt_len]
        else:
            toks = [int(x) for x in r.integers(0, VOCAB, q.prompt_len)]
        prompts.append(toks)
    return tc, reqs, prefix, prompts


class _Content:
    """The test's picture of the slots, updated from each step's record."""

    def __init__(self, bs, prefix, reqs, prompts):
        self.bs = bs
        self.gpu, self.cpu = {}, {}
        self.toks = {}
        self.prefix_holder = list(prefix)
        for q, p in zip(reqs, prompts):
            own = (list(prefix) if q.shares_prefix else []) + list(p)
            self.toks[q.seq_id] = own
            if q.fork_child >= 0:
                self.toks[q.fork_child] = list(own)       # the child shares the prompt
        self.known = {s: len(t) for s, t in self.toks.items()}

    def tokens(self, seq, n):
        t = self.toks[seq]
        while len(t) < n:
            t.append(token_fn(seq, len(t)))
        return t[:n]

    def place_prefix(self, table):
        for p in range(len(self.prefix_holder)):
            self.gpu[(table[p // self.bs], p % self.bs)] = tuple(self.prefix_holder[:p + 1])

    def apply(self, ops):
        for op in ops:
            if op[0] == "w":
                _, seq, pos, slot = op
                self.gpu[(slot // self.bs, slot % self.bs)] = tuple(self.tokens(seq, pos + 1))
            elif op[0] == "c":
                _, src, dst = op
                for o in range(self.bs):
                    if (src, o) in self.gpu:
                        self.gpu[(dst, o)] = self.gpu[(src, o)]
            else:
                kind, a, b = op
                src, dst = (self.gpu, self.cpu) if kind == "so" else (self.cpu, self.gpu)
                for o in range(self.bs):
                    if (a, o) in src:
                        dst[(b, o)] = src[(a, o)]

    def check(self, table_of, running, context_lens):
        for seq, n in zip(running, context_lens):
            t = table_of(seq)
            toks = self.tokens(seq, n)
            for p in range(n):
                got = self.gpu.get((t[p // self.bs], p % self.bs))
                assert got == tuple(toks[:p + 1]), (seq, p, got)


def _model(seed, bs, nb, ncpu, swap, cls_sched=osch.Scheduler, cls_bm=None):
    tc, reqs, prefix, prompts = _trace(seed, bs)
    order = np.random.default_rng(seed).permutation(nb).tolist()
    if cls_bm is None:
        cls_bm = obm.PrefixSwappingBlockManager if swap else obm.PrefixCachingBlockManager
    bm = cls_bm(nb, bs, ncpu, order) if swap else cls_bm(nb, bs, order)
    bm.allocate_prefix(wl.PREFIX_SEQ, prefix)
    sch = cls_sched(bm, tc.max_running, wl.PREFIX_SEQ, preempt="swap" if swap else "recompute",
                    prefix_cache=True, prefix_tokens=prefix, token_fn=token_fn)
    for q, p in zip(reqs, prompts):
        sch.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child,
                                     q.fork_output_len, tokens=p))
    content = _Content(bs, prefix, reqs, prompts)
    content.place_prefix(bm.block_table(wl.PREFIX_SEQ))
    return tc, bm, sch, content


def _run_model(seed, bs, nb, ncpu=0, swap=False, steps=120, **kw):
    tc, bm, sch, content = _model(seed, bs, nb, ncpu, swap, **kw)
    stats = {"preempted": 0, "swapped": 0, "written": 0, "readmit_skips": 0}
    preempted = set()
    for _ in range(steps):
        rec = sch.step()
        content.apply(rec.ops)
        content.check(bm.block_table, rec.running, rec.context_lens)
        bm.check()
        for seq in rec.admitted:
            if seq in preempted:
                first = min((o[2] for o in rec.ops if o[0] == "w" and o[1] == seq), default=None)
                held = sch_prefix_blocks(sch, seq) * bs
                stats["readmit_skips"] += first is not None and first > held
        preempted |= set(rec.preempted) - set(rec.swapped_out)
        stats["preempted"] += len(rec.preempted)
        stats["swapped"] += len(rec.swapped_out)
        stats["written"] += sum(1 for o in rec.ops if o[0] == "w")
    stats["hits"] = bm.hits
    return stats


def sch_prefix_blocks(sch, seq):
    """Full blocks of the system prefix a sequence holds through the cache."""
    s = next(x for x in sch.running + list(sch.waiting) + list(sch.swapped) if x.seq_id == seq)
    return (sch.prefix_len // sch.bm.block_size) if s.shares_prefix else 0


CASES = [(s, bs, nb) for s, (bs, nb) in enumerate([(2, 40), (4, 30), (2, 60), (1, 50), (4, 80), (2, 35)])]


@pytest.mark.parametrize("seed,bs,nb", CASES)
def test_model_content_recompute(seed, bs, nb):
    st = _run_model(seed, bs, nb)
    assert st["hits"] > 0


@pytest.mark.parametrize("seed,bs,nb", CASES)
def test_model_content_swap(seed, bs, nb):
    st = _run_model(seed, bs, nb, ncpu=nb // 2, swap=True)
    assert st["hits"] > 0


def test_streams_exercise_preemption_and_hits():
    """The traces preempt both ways, and a recomputed sequence coming back finds
    K/V it wrote before its preemption (the blocks kept their keys)."""
    pre = sw = back = 0
    for seed, bs, nb in CASES:
        st = _run_model(seed, bs, nb)
        pre += st["preempted"]
        back += st["readmit_skips"]
        sw += _run_model(seed, bs, nb, ncpu=nb // 2, swap=True)["swapped"]
    assert pre > 0 and sw > 0 and back > 0


# ---- planted mistakes ---------------------------------------------------------

class _KeepAbandonedNames(osch.Scheduler):
    """Mistake: a recompute preemption drops the step's dead writes but leaves
    the names of the blocks they targeted."""

    def _preempt_last(self, rec):
        real = self.bm.forget
        self.bm.forget = lambda b: None
        try:
            return super()._preempt_last(rec)
        finally:
            self.bm.forget = real


class _NoCachePrefill(osch.Scheduler):
    """Mistake: admission finds the cached blocks but writes nothing at all for
    the prompt (skips the uncached part too)."""

    def _admit(self, s, rec):
        n = len(rec.ops)
        super()._admit(s, rec)
        del rec.ops[n:]


class _CachedOffByOne(osch.Scheduler):
    """Mistake: admission skips one position more than the cache holds."""

    def _admit(self, s, rec):
        n = len(rec.ops)
        super()._admit(s, rec)
        for k in range(n, len(rec.ops)):
            if rec.ops[k][0] == "w" and rec.ops[k][1] == s.seq_id:
                del rec.ops[k]
                break


class _LooseBlockManager(obm.PrefixCachingBlockManager):
    def check(self):
        pass


@pytest.mark.parametrize("cls", [_KeepAbandonedNames, _NoCachePrefill, _CachedOffByOne])
def test_planted_mistakes_fail_the_content_check(cls):
    caught = 0
    for seed, bs, nb in CASES:
        try:
            _run_model(seed, bs, nb, cls_sched=cls, cls_bm=_LooseBlockManager)
        except AssertionError:
            caught += 1
    assert caught > 0


# ---- the C++ scheduler against the model ---------------------------------------

def _native_pair(pa, seed, bs, nb, ncpu, swap):
    tc, mbm, ms, content = _model(seed, bs, nb, ncpu, swap)
    _, reqs, prefix, prompts = _trace(seed, bs)
    order = np.random.default_rng(seed).permutation(nb).tolist()
    nbm = pa.BlockManager(nb, bs, order)
    nbm.enable_prefix_cache()
    if swap:
        nbm.set_cpu_blocks(ncpu)
    nbm.allocate_prefix(wl.PREFIX_SEQ, prefix)
    ns = pa.Scheduler(nbm, tc.max_running, wl.PREFIX_SEQ, preempt="swap" if swap else "recompute",
                      prefix_cache=True, prefix_tokens=prefix, token_fn=token_fn)
    for q, p in zip(reqs, prompts):
        ns.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len,
                       tokens=p)
    return mbm, ms, nbm, ns, content


@pytest.mark.parametrize("swap", [False, True])
@pytest.mark.parametrize("seed,bs,nb", CASES)
def test_native_scheduler_matches_model(pa, seed, bs, nb, swap):
    """Every step: the same record (ops in issue order, events, batch), the same
    free, evictable and host lists, the same cache counters; and the C++
    record passes the content check on its own."""
    ncpu = nb // 2 if swap else 0
    mbm, ms, nbm, ns, content = _native_pair(pa, seed, bs, nb, ncpu, swap)
    for step in range(120):
        a, b = ms.step(), ns.step()
        assert [tuple(o) for o in a.ops] == b["ops"], step
        assert (a.finished, a.admitted, a.preempted) == (b["finished"], b["admitted"], b["preempted"]), step
        assert (a.swapped_out, a.swapped_in) == (b["swapped_out"], b["swapped_in"]), step
        assert a.running == b["running"] and a.context_lens == b["context_lens"], step
        assert mbm.free_list == nbm.free_list(), step
        assert mbm.evictable == nbm.evictable(), step
        if swap:
            assert mbm.cpu_free == nbm.cpu_free_list(), step
        c, e, h, lk = nbm.cache_stats()
        assert (c, e, h, lk) == (len(mbm.name), len(mbm.evictable), mbm.hits, mbm.lookups), step
        content.apply(b["ops"])
        content.check(lambda s: nbm.block_table(s), b["running"], b["context_lens"])


def test_forget_rules(pa):
    """pa_bm_forget takes only cached blocks with count zero, like the model."""
    bs, nb = 2, 8
    for m in (obm.PrefixCachingBlockManager(nb, bs), pa.BlockManager(nb, bs)):
        if isinstance(m, pa.BlockManager):
            m.enable_prefix_cache()
        m.allocate_prefix(1, [5, 6, 7, 8, 9])        # two full blocks named, one partial
        t = m.block_table(1)
        for b in (t[0], t[2], nb, -1):               # referenced, partial, out of range
            with pytest.raises(Exception):
                m.forget(b)
        m.free(1)
        ev = list(m.evictable if isinstance(m, obm.PrefixCachingBlockManager) else m.evictable())
        assert sorted(ev) == sorted(t[:2])
        with pytest.raises(Exception):
            m.forget(t[2])                             # back on the free list, not cached
        m.forget(t[1])
        fl = m.free_list if isinstance(m, obm.PrefixCachingBlockManager) else m.free_list()
        assert fl[-1] == t[1]
        assert m.allocate_prefix(2, [5, 6, 7, 8]) == bs  # the first block is still found
        m.free(2)


def test_prefix_mode_argument_rules(pa):
    bs, nb = 2, 16
    plain = pa.BlockManager(nb, bs)
    with pytest.raises(pa.PagedAttentionError):        # block manager without the cache
        pa.Scheduler(plain, 4, prefix_cache=True, token_fn=token_fn)
    bm = pa.BlockManager(nb, bs)
    bm.enable_prefix_cache()
    bm.allocate_prefix(wl.PREFIX_SEQ, [1, 2, 3])
    with pytest.raises(pa.PagedAttentionError):        # prefix ids disagree with the holder's length
        pa.Scheduler(bm, 4, wl.PREFIX_SEQ, prefix_cache=True, prefix_tokens=[1, 2], token_fn=token_fn)
    with pytest.raises(ValueError):
        pa.Scheduler(bm, 4, wl.PREFIX_SEQ, prefix_cache=True, prefix_tokens=[1, 2, 3])
    s = pa.Scheduler(bm, 4, wl.PREFIX_SEQ, prefix_cache=True, prefix_tokens=[1, 2, 3], token_fn=token_fn)
    with pytest.raises(pa.PagedAttentionError):        # prompt ids are required
        s.add_request(1, 3, 2)
    with pytest.raises(ValueError):
        s.add_request(1, 3, 2, tokens=[1, 2])
    s.add_request(1, 3, 2, shares_prefix=True, tokens=[3, 0, 1])
    rec = s.step()
    # prefix 1 2 3 + 3 0 1: the holder's full block (1 2) is found; positions 2.. are written
    assert [o[2] for o in rec["ops"] if o[0] == "w"] == [2, 3, 4, 5, 6]
    plain_s = pa.Scheduler(plain, 4)
    with pytest.raises(pa.PagedAttentionError):        # tokens without the prefix-cache mode
        plain_s.add_request(1, 2, 2, tokens=[1, 2])


def test_no_holder_replayed_prompts(pa):
    """Admission through the cache with no prefix holder: repeated prompts alone
    make the hits; C++ and model agree and the content check holds."""
    bs, nb = 2, 40
    r = np.random.default_rng(11)
    base = [int(x) for x in r.integers(0, VOCAB, 12)]
    order = r.permutation(nb).tolist()
    mbm = obm.PrefixCachingBlockManager(nb, bs, order)
    nbm = pa.BlockManager(nb, bs, order)
    nbm.enable_prefix_cache()
    ms = osch.Scheduler(mbm, 6, prefix_cache=True, token_fn=token_fn)
    ns = pa.Scheduler(nbm, 6, prefix_cache=True, prefix_tokens=[], token_fn=token_fn)
    reqs, prompts = [], []
    for i in range(24):
        n = int(r.integers(3, 16))
        p = (base + [int(x) for x in r.integers(0, VOCAB, n)])[:n] if i % 2 else \
            [int(x) for x in r.integers(0, VOCAB, n)]
        q = wl.TraceRequest(seq_id=i, prompt_len=n, output_len=int(r.integers(1, 9)), shares_prefix=False,
                            fork_child=-1, fork_output_len=0)
        reqs.append(q)
        prompts.append(p)
        ms.add_request(osch.Request(i, n, q.output_len, tokens=p))
        ns.add_request(i, n, q.output_len, tokens=p)
    content = _Content(bs, [], reqs, prompts)
    for step in range(60):
        a, b = ms.step(), ns.step()
        assert [tuple(o) for o in a.ops] == b["ops"], step
        assert a.running == b["running"] and a.context_lens == b["context_lens"], step
        assert mbm.free_list == nbm.free_list() and mbm.evictable == nbm.evictable(), step
        content.apply(b["ops"])
        content.check(lambda s: nbm.block_table(s), b["running"], b["context_lens"])
    assert mbm.hits > 0 and not ms.running and not ms.waiting


def test_holder_must_be_cached_under_the_prefix_ids(pa):
    """A holder made without the cache, or prefix ids other than the holder's,
    are refused by both schedulers: a sharer would then take more blocks than
    its budget charge."""
    bs, nb = 4, 32
    ids = [0, 1, 2, 3, 1, 1, 2, 0, 3, 3]
    wrong = ids[:5] + [2] + ids[6:]                 # differs in the second block
    for make_model in (True, False):
        def manager(cached):
            if make_model:
                m = obm.PrefixCachingBlockManager(nb, bs)
            else:
                m = pa.BlockManager(nb, bs)
                m.enable_prefix_cache()
            if cached:
                m.allocate_prefix(wl.PREFIX_SEQ, ids)
            else:
                m.allocate(wl.PREFIX_SEQ, len(ids))
            return m

        def sched(m, toks):
            if make_model:
                return osch.Scheduler(m, 4, wl.PREFIX_SEQ, prefix_cache=True, prefix_tokens=toks, token_fn=token_fn)
            return pa.Scheduler(m, 4, wl.PREFIX_SEQ, prefix_cache=True, prefix_tokens=toks, token_fn=token_fn)

        err = ValueError if make_model else pa.PagedAttentionError
        with pytest.raises(err):
            sched(manager(False), ids)
        with pytest.raises(err):
            sched(manager(True), wrong)
        sched(manager(True), ids)
