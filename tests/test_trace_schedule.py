"""Host side of the trace driver behind the bench's per-step trace timing:
the scheduler's step records turned into device work in issue order."""

import numpy as np

from paged_kv_cache_381_b200 import trace, workloads as wl


def test_schedule_gives_every_step_its_work_in_issue_order():
    sc = trace.schedule(wl.TRACE, 5)
    steps = sc["steps"]
    assert len(steps) == wl.TRACE.steps and len(sc["host_ms"]) == wl.TRACE.steps
    assert sc["preempted"] >= 1 and sc["admitted"] >= wl.TRACE.max_running
    bs = wl.TRACE.block_size
    seen_copy = False
    for st in steps:
        assert st is not None
        runs, tables, lens, mcl = st
        assert mcl == int(lens.max())
        # every table holds ceil(context / block size) blocks, the rest is padding
        nblk = -(-lens.astype(np.int64) // bs)
        assert tables.shape[1] == int(nblk.max())
        for r, n in enumerate(nblk):
            assert (tables[r, :n] >= 0).all() and (tables[r, n:] == -1).all()
        # runs alternate kinds; slots within a write run are distinct and inside the pool
        for (k0, _), (k1, _) in zip(runs, runs[1:]):
            assert k0 != k1
        for kind, x in runs:
            if kind == "w":
                assert len(np.unique(x)) == len(x) and x.min() >= 0 and x.max() < sc["num_blocks"] * bs
            else:
                seen_copy = True
                assert x.shape[1] == 2 and (x >= 0).all() and (x < sc["num_blocks"]).all()
        # the step's last run writes (the decode tokens): fused with the decode
        assert runs[-1][0] == "w"
    assert seen_copy
