"""Multi-turn conversation workload for the prefix cache (host side).

Conversations start from one of a few shared system prompts; each turn adds
20-199 user tokens to the whole conversation so far and decodes n_dec new
tokens.  Jobs run in waves of up to `wave` sequences; a job that does not fit
the pool waits for the next wave.  The pool is sized so that cached blocks
must be evicted before the last turns.

`run_conversations` drives the C++ block manager (prefix cache on) and hands
every device action to `dev`: `dev.prefill(seq, toks, cached)` after a
sequence is allocated, `dev.append(batch, slots)` after each decode step's
slots are reserved, and `dev.decode(batch, step)` on the steps in
`decode_steps`.  With `NullDevice` the same schedule runs on the CPU, so the
counts it is built to produce can be checked without a GPU.

Every K/V row of the workload is drawn from a key of the whole token prefix
that ends at its position (workloads.prefix_rows), as a model's K/V would be.
"""

import numpy as np

import paged_kv_cache_381_b200 as pa

HQ, HKV, D, BS = 32, 8, 128, 16
SEED = 21


class NullDevice:
    def prefill(self, bm, seq, toks, cached):
        pass

    def append(self, bm, batch, slots):
        pass

    def decode(self, bm, batch, step):
        pass

    def finish_wave(self):
        pass


def run_conversations(dev, n_conv=12, n_turns=3, wave=8, n_dec=16, num_blocks=300, decode_steps=None,
                      seed=SEED):
    r = np.random.default_rng(seed)
    decode_steps = (0, n_dec - 1) if decode_steps is None else decode_steps
    systems = [[int(x) for x in r.integers(1, 32000, n)] for n in (512, 333, 800)]
    convs = {c: list(systems[c % 3]) for c in range(n_conv)}
    pending = [(c, 0) for c in range(n_conv)]
    bm = pa.BlockManager(num_blocks, BS, r.permutation(num_blocks).tolist())
    bm.enable_prefix_cache(True)
    st = dict(written=0, total=0, cached=0, short=0, jobs=0, waves=0)
    seq_id = 0
    while pending:
        batch, deferred = [], []
        for c, t in pending:
            if len(batch) == wave:
                deferred.append((c, t))
                continue
            toks = convs[c] + [int(x) for x in r.integers(1, 32000, int(r.integers(20, 200)))]
            # admit only with room for this prompt (as if nothing were cached) and
            # for every admitted sequence's decode blocks
            grow = -(-n_dec // BS) + 1
            if bm.num_free < -(-len(toks) // BS) + (len(batch) + 1) * grow:
                deferred.append((c, t))
                continue
            try:
                cached = bm.allocate_prefix(seq_id, toks)
            except pa.NoBlocksError:
                deferred.append((c, t))
                continue
            assert cached % BS == 0 and cached <= len(toks)
            if t > 0:
                # the earlier turns sit in full blocks that are found again
                # unless they were evicted meanwhile
                full = (len(convs[c]) // BS) * BS
                assert cached <= full
                st["short"] += cached < full
            dev.prefill(bm, seq_id, toks, cached)
            st["written"] += len(toks) - cached
            st["total"] += len(toks)
            st["cached"] += cached
            st["jobs"] += 1
            batch.append((seq_id, c, t, toks))
            seq_id += 1
        assert batch, "no job fits the pool"
        st["waves"] += 1
        for step in range(n_dec):
            slots = []
            for s, c, t, toks in batch:
                tok = int(r.integers(1, 32000))
                slot, src, dst = bm.append_token(s, tok)
                assert src < 0                       # nothing forks here: no copy-on-write
                toks.append(tok)
                slots.append(slot)
            dev.append(bm, batch, slots)
            st["written"] += len(batch)
            st["total"] += len(batch)
            if step in decode_steps:
                dev.decode(bm, batch, step)
        dev.finish_wave()
        for s, c, t, toks in batch:
            bm.free(s)
            convs[c] = toks
            if t + 1 < n_turns:
                deferred.append((c, t + 1))
        pending = deferred
    st["cache_stats"] = bm.cache_stats()
    return st
