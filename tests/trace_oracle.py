"""fp64 oracle of every running sequence of the continuous-batching trace,
on spawned worker processes (test infrastructure).

Each K/V row of the trace is a counter-keyed draw (workloads.token_rows) of
its owner stream -- the request itself, its fork parent below the fork
point, or the shared-prefix holder below the prefix length -- and its
position.  A worker owns the sequences whose id is its index modulo the
number of workers, keeps the rows it has drawn (per owner stream, in storage
form) and for every step rebuilds each of its sequences' histories from them
and runs the unchanged oracle (oracle.attention.decode_history).  Spawned
workers start from a fresh interpreter, so they are safe to start after the
first CUDA call.
"""

import multiprocessing as mp
import os

import numpy as np


def owners(state, seq, n):
    """Owner stream of positions 0 .. n-1 of sequence `seq`: moving up the fork
    chain while the position lies below the fork point, then to the
    prefix holder below the shared-prefix length."""
    prefix, prefix_seq, share, parent, fork_pos = state
    pos = np.arange(n, dtype=np.int64)
    own = np.full(n, seq, dtype=np.int64)
    active = np.ones(n, dtype=bool)
    cur = seq
    while cur in parent:
        move = active & (pos < fork_pos[cur])
        own[move] = parent[cur]
        active = move
        cur = parent[cur]
    shares = np.array([share.get(int(o), False) and int(o) != prefix_seq for o in own.tolist()], dtype=bool) \
        if n else np.zeros(0, dtype=bool)
    own[shares & (pos < prefix)] = prefix_seq
    return own


def _worker(conn, seed, tc, state):
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except ImportError:
        pass
    from oracle import attention as oa
    from oracle.numerics import widen
    from paged_kv_cache_381_b200 import workloads as wl
    cache = {}

    def rows(owner, upto, salt):
        have = cache.get((owner, salt))
        m = 0 if have is None else len(have)
        if m < upto:
            new = wl.token_rows(seed, owner, np.arange(m, upto), tc.num_kv_heads, tc.head_dim, tc.dtype, salt)
            have = new if have is None else np.concatenate([have, new])
            cache[(owner, salt)] = have
        return have

    def history(seq, n, salt):
        own = owners(state, seq, n)
        out = np.empty((n, tc.num_kv_heads, tc.head_dim), dtype=np.uint16)
        pos = np.arange(n)
        for o in np.unique(own):
            sel = own == o
            out[sel] = rows(int(o), int(pos[sel].max()) + 1, salt)[pos[sel]]
        return out

    while True:
        msg = conn.recv()
        if msg is None:
            break
        res = []
        for i, seq, n, q in msg:
            K, V = history(seq, n, 0), history(seq, n, 1)
            res.append((i, oa.decode_history(widen(q, tc.dtype), widen(K, tc.dtype), widen(V, tc.dtype), tc.scale)))
        conn.send(res)
    conn.close()


class TraceOracle:
    """Worker processes holding the trace's histories; decode(tasks) returns
    the oracle's output of each (sequence, context length, q rows) task."""

    def __init__(self, seed, tc, state, workers=None):
        if workers is None:
            cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
            workers = max(1, min(16, cores))
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for _ in range(workers):
            a, b = ctx.Pipe()
            p = ctx.Process(target=_worker, args=(b, seed, tc, state), daemon=True)
            p.start()
            b.close()
            self.conns.append(a)
            self.procs.append(p)

    def submit(self, tasks):
        """Send (seq, n, q_storage) tasks; collect with results()."""
        n = len(self.conns)
        parts = [[] for _ in range(n)]
        for i, (seq, ctx, q) in enumerate(tasks):
            parts[int(seq) % n].append((i, int(seq), int(ctx), q))
        for c, part in zip(self.conns, parts):
            c.send(part)
        self._count = len(tasks)

    def results(self):
        out = [None] * self._count
        for c in self.conns:
            for i, r in c.recv():
                out[i] = r
        return out

    def close(self):
        for c in self.conns:
            try:
                c.send(None)
            except (BrokenPipeError, OSError):
                pass
        for p in self.procs:
            p.join(timeout=10)
            if p.is_alive():
                p.terminate()
