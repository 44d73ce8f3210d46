"""Full-size parity helpers: every output row of a full-size batch against the
fp64 oracle.

The device draws of a full-size workload are copied to the host once; the
oracle (``oracle.attention.decode_history``, unchanged) then runs one
sequence per task on a pool of spawned worker processes, one BLAS thread
each, so that every (sequence, head) row of the 70B-, 7B-shaped and long
batches is checked in seconds.  Spawned workers start from a fresh
interpreter, so the pool is safe to start after the first CUDA call.
Results are kept per input fingerprint: the math-path and merge-mode variants
of one workload reuse one oracle pass.
"""

import hashlib
import multiprocessing as mp
import os

import numpy as np

from tests.gpu_harness import assert_close, to_storage

_POOL = None
_CACHE = {}


def _init_worker():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except ImportError:
        pass


def pool():
    """The oracle's worker pool (spawned on first use, one process per core,
    at most 16)."""
    global _POOL
    if _POOL is None:
        cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
        _POOL = mp.get_context("spawn").Pool(max(1, min(16, cores)), initializer=_init_worker)
    return _POOL


def _decode_task(task):
    """fp64 oracle of one sequence: q [Hq, D], K/V [n, Hkv, D] in storage form."""
    from oracle import attention as oa
    from oracle.numerics import widen
    q, k, v, dtype, scale = task
    return oa.decode_history(widen(q, dtype), widen(k, dtype), widen(v, dtype), scale)


def _verify_task(task):
    """fp64 oracle of one sequence's Q candidate rows: query i sits at position
    n - Q + i and attends to positions 0 .. n - Q + i (a context cut after the
    query's own position); a row with no visible position is zero."""
    from oracle import attention as oa
    from oracle.numerics import widen
    q, k, v, dtype, scale = task
    Q = q.shape[0]
    n = k.shape[0]
    K, V = widen(k, dtype), widen(v, dtype)
    out = np.zeros(q.shape, dtype=np.float64)
    for i in range(Q):
        p = n - Q + i
        if p >= 0:
            out[i] = oa.decode_history(widen(q[i], dtype), K[:p + 1], V[:p + 1], scale)
    return out


def _fingerprint(*arrays):
    h = hashlib.blake2b(digest_size=16)
    for a in arrays:
        a = np.ascontiguousarray(a)
        h.update(str((a.dtype.str, a.shape)).encode())
        h.update(memoryview(a).cast("B"))
    return h.hexdigest()


def oracle_all_rows(q_dev, d, cfg, verify=False):
    """fp64 oracle of every output row of a full-size batch drawn by
    ``workloads.draw_device`` (histories d.k_hist / d.v_hist on the device,
    sequence s at rows d.offsets[s] .. d.offsets[s + 1]).  q_dev: [S, Hq, D]
    (decode) or [S, Q, Hq, D] (verify) on the device."""
    q = to_storage(q_dev, cfg.dtype)
    k = to_storage(d.k_hist, cfg.dtype)
    v = to_storage(d.v_hist, cfg.dtype)
    lens = np.asarray(d.context_lens, dtype=np.int64)
    # the whole input is hashed: a cached result is only reused for bit-identical inputs
    key = (cfg.name, cfg.dtype, verify, _fingerprint(q, k, v, lens))
    if key in _CACHE:
        return _CACHE[key]
    offs = np.asarray(d.offsets, dtype=np.int64)
    tasks = [(q[s], k[offs[s]:offs[s + 1]], v[offs[s]:offs[s + 1]], cfg.dtype, cfg.scale) for s in range(len(lens))]
    # longest first, so the pool's tail is short
    order = np.argsort(-lens, kind="stable")
    res = pool().map(_verify_task if verify else _decode_task, [tasks[s] for s in order], chunksize=1)
    ref = np.empty(q.shape, dtype=np.float64)
    for s, r in zip(order, res):
        ref[s] = r
    _CACHE[key] = ref                 # results only (tens of MB at most), not the histories
    return ref


def assert_every_row(out_dev, ref, dtype, what):
    """Every element of the device output within the dtype's tolerance of the
    oracle (and therefore finite)."""
    assert_close(to_storage(out_dev, dtype), ref, dtype, what)
