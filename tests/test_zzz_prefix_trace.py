"""Continuous batching with admission through the prefix cache, on the GPU.

[P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
"Prefix Caching前缀复用优化": a request whose prompt begins with cached KV
references those blocks and skips their prefill.  Here the scheduler admits
every request through the cache (pa_sched_enable_prefix_cache): requests that
share a 200-token system prefix (not block aligned) or replay an earlier
prompt find its full blocks, only the rest is written, and the pool is small
enough that sequences are preempted (by recompute or by swap).

Every K/V row is drawn from a key of the whole token prefix ending at its
position (workloads.prefix_rows' keys), as a model's K/V would be, so a
cached block is right only if it holds exactly that prefix's rows.  Every
step: the native scheduler and the oracle's model agree on the record; the
ops run on the device in issue order (pa_cache_write, pa_copy_blocks,
pa_swap_blocks); sampled sequences' whole cache contents equal freshly drawn
rows bit for bit, and their decode outputs match the fp64 oracle on those
rows.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_381_b200 as pa
from paged_kv_cache_381_b200 import workloads as wl
from oracle import attention as oa
from oracle import block_manager as obm
from oracle import scheduler as osch
from oracle.numerics import widen
from tests.gpu_harness import assert_close, to_device, to_storage

pytestmark = pytest.mark.gpu

SEED = 13
VOCAB = 3
DEV = "cuda"
TC = wl.TraceConfig(dtype="f16", num_heads=16, num_kv_heads=4, head_dim=128, block_size=16, max_running=32,
                    num_requests=96, steps=150, prefix_len=200, prompt_lo=1, prompt_hi=160, output_mean=24.0,
                    fork_every=6, pool_frac=0.6)


def token_fn(seq, pos):
    return wl.generated_token(seq, pos, VOCAB)


def _prompts(reqs):
    """System prefix ids and each request's own prompt ids; a third of the
    requests replay the start of an earlier prompt."""
    r = np.random.default_rng([SEED, 3])
    prefix = [int(x) for x in r.integers(0, VOCAB, TC.prefix_len)]
    prompts = []
    for q in reqs:
        if prompts and r.random() < 0.33:
            base = prompts[int(r.integers(len(prompts)))]
            p = (base + [int(x) for x in r.integers(0, VOCAB, q.prompt_len)])[:q.prompt_len]
        else:
            p = [int(x) for x in r.integers(0, VOCAB, q.prompt_len)]
        prompts.append(p)
    return prefix, prompts


class Tokens:
    """Each sequence's token ids (prompt, then generated) and prefix keys."""

    def __init__(self, prefix, reqs, prompts):
        self.toks = {wl.PREFIX_SEQ: list(prefix)}
        for q, p in zip(reqs, prompts):
            own = (list(prefix) if q.shares_prefix else []) + list(p)
            self.toks[q.seq_id] = own
            if q.fork_child >= 0:
                self.toks[q.fork_child] = list(own)
        self.keys = {}

    def key_list(self, seq, n):
        t = self.toks[seq]
        while len(t) < n:
            t.append(token_fn(seq, len(t)))
        k = self.keys.get(seq)
        if k is None or len(k) < n:
            k = wl.prefix_keys(t[:max(n, len(t))])
            self.keys[seq] = k
        return k[:n]

    def rows(self, seq, positions, salt):
        keys = self.key_list(seq, max(positions) + 1)[np.asarray(positions, dtype=np.int64)]
        return wl.token_rows(SEED, 0x9F, keys, TC.num_kv_heads, TC.head_dim, TC.dtype, salt)

    def rows_for_writes(self, ws, salt):
        out = np.empty((len(ws), TC.num_kv_heads, TC.head_dim), dtype=np.uint16)
        by_seq = {}
        for i, (seq, pos, _) in enumerate(ws):
            by_seq.setdefault(seq, []).append((i, pos))
        for seq, lst in by_seq.items():
            out[np.array([i for i, _ in lst])] = self.rows(seq, [p for _, p in lst], salt)
        return out


def _managers(nb, ncpu, prefix, order=None):
    nbm = pa.BlockManager(nb, TC.block_size, order)
    nbm.enable_prefix_cache()
    if ncpu:
        nbm.set_cpu_blocks(ncpu)
    nbm.allocate_prefix(wl.PREFIX_SEQ, prefix)
    return nbm


def _scheduler(bm, preempt, prefix, reqs, prompts, native=True):
    if native:
        s = pa.Scheduler(bm, TC.max_running, wl.PREFIX_SEQ, preempt=preempt, prefix_cache=True,
                         prefix_tokens=prefix, token_fn=token_fn)
        for q, p in zip(reqs, prompts):
            s.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len,
                          tokens=p)
        return s
    s = osch.Scheduler(bm, TC.max_running, wl.PREFIX_SEQ, preempt=preempt, prefix_cache=True,
                       prefix_tokens=prefix, token_fn=token_fn)
    for q, p in zip(reqs, prompts):
        s.add_request(osch.Request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child,
                                   q.fork_output_len, tokens=p))
    return s


def _dry_peak(prefix, reqs, prompts):
    bm = _managers(1 << 18, 0, prefix)
    sch = _scheduler(bm, "recompute", prefix, reqs, prompts)
    peak = 0
    for _ in range(TC.steps):
        sch.step()
        peak = max(peak, bm.usage()[0])
    return peak


@pytest.mark.parametrize("preempt", ["recompute", "swap"])
def test_prefix_cache_admission_trace(preempt):
    if DEV == "cuda":
        assert torch.cuda.is_available()
        from paged_kv_cache_381_b200 import build
        build.build()
        pa.pa_get_device_error()
    reqs = wl.make_trace_requests(TC, SEED)
    prefix, prompts = _prompts(reqs)
    toks = Tokens(prefix, reqs, prompts)
    nb = int(math.ceil(TC.pool_frac * _dry_peak(prefix, reqs, prompts)))
    order = np.random.default_rng(SEED).permutation(nb).astype(np.int32)
    ncpu = nb // 4 if preempt == "swap" else 0
    bm = _managers(nb, ncpu, prefix, order)
    model_bm = (obm.PrefixSwappingBlockManager(nb, TC.block_size, ncpu, order.tolist()) if ncpu else
                obm.PrefixCachingBlockManager(nb, TC.block_size, order.tolist()))
    model_bm.allocate_prefix(wl.PREFIX_SEQ, prefix)
    sch = _scheduler(bm, preempt, prefix, reqs, prompts)
    model = _scheduler(model_bm, preempt, prefix, reqs, prompts, native=False)

    H, D, bs = TC.num_kv_heads, TC.head_dim, TC.block_size
    dev = torch.device(DEV)
    kc = torch.zeros((nb, bs, H, D), dtype=torch.float16, device=dev)
    vc = torch.zeros_like(kc)
    hk = torch.zeros((max(ncpu, 1), bs, H, D), dtype=torch.float16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    kflat, vflat = kc.view(nb * bs, H, D), vc.view(nb * bs, H, D)

    def write(ws):
        if ws:
            slots = torch.tensor([w[2] for w in ws], dtype=torch.int64, device=dev)
            pa.pa_cache_write(to_device(toks.rows_for_writes(ws, 0), "f16", DEV),
                              to_device(toks.rows_for_writes(ws, 1), "f16", DEV), kc, vc, slots)

    write([(wl.PREFIX_SEQ, p, int(s)) for p, s in enumerate(bm.slots(wl.PREFIX_SEQ, 0, TC.prefix_len))])

    r = np.random.default_rng(17)
    saw = {"preempt": 0, "cow": 0, "so": 0, "si": 0, "finish": 0, "written": 0, "admitted_rows": 0}
    for step in range(TC.steps):
        rec = sch.step()
        mrec = model.step()
        assert rec["ops"] == [tuple(o) for o in mrec.ops], step
        assert (rec["finished"], rec["admitted"], rec["preempted"]) == (mrec.finished, mrec.admitted,
                                                                         mrec.preempted), step
        assert rec["running"] == mrec.running and rec["context_lens"] == mrec.context_lens, step
        assert rec["swapped_out"] == mrec.swapped_out and rec["swapped_in"] == mrec.swapped_in, step
        assert bm.evictable() == model_bm.evictable and bm.free_list() == model_bm.free_list, step
        saw["preempt"] += len(rec["preempted"])
        saw["finish"] += len(rec["finished"])
        run = []
        for op in rec["ops"]:
            if op[0] == "w":
                run.append(op[1:])
                saw["written"] += 1
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
        saw["admitted_rows"] += sum(c for s, c in zip(running, ctx) if s in rec["admitted"])
        width = max(len(bm.block_table(s)) for s in running)
        tables, lens = bm.pack(running, width)
        assert lens.tolist() == ctx
        q = np.stack([wl.token_rows(SEED, s, [c], TC.num_heads, D, TC.dtype, 2)[0] for s, c in zip(running, ctx)])
        qd = to_device(q, "f16", DEV)
        out = torch.empty_like(qd)
        pa.pa_decode(out, qd, kc, vc, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev), TC.scale,
                     bs, H, max_context_len=int(lens.max()))
        if DEV == "cuda":
            torch.cuda.synchronize()
        got = to_storage(out, "f16")
        # sampled sequences, and every one admitted this step (its cached part
        # was never written by it): whole cache contents and output
        sample = set(r.choice(len(running), size=min(3, len(running)), replace=False).tolist())
        sample |= {i for i, s in enumerate(running) if s in rec["admitted"]}
        for i in sorted(sample):
            s, n = running[i], ctx[i]
            sl = torch.from_numpy(bm.slots(s, 0, n)).to(dev)
            K, V = toks.rows(s, range(n), 0), toks.rows(s, range(n), 1)
            assert np.array_equal(to_storage(kflat.index_select(0, sl), "f16"), K), (step, s)
            assert np.array_equal(to_storage(vflat.index_select(0, sl), "f16"), V), (step, s)
            ref = oa.decode_history(widen(q[i], "f16"), widen(K, "f16"), widen(V, "f16"), TC.scale)
            assert_close(got[i], ref, "f16", f"step {step} seq {s}")
        if DEV == "cuda":
            assert pa.pa_get_device_error() == 0
    cached, _, hits, _ = bm.cache_stats()
    assert hits * bs > 0.2 * saw["admitted_rows"], (hits, saw)     # the cache saves real prefill
    assert saw["preempt"] >= 1 and saw["finish"] >= 1 and saw["cow"] >= 1, saw
    if preempt == "swap":
        assert saw["so"] >= 1 and saw["si"] >= 1, saw
