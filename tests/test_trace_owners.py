"""Host check of the trace oracle's ownership map: the vectorised owner of
every position of every sequence of the GPU trace equals the plain rule
(up the fork chain while below the fork point, then the prefix holder below
the shared-prefix length), and the rows a worker assembles equal rows drawn
position by position."""

import numpy as np

from paged_kv_cache_381_b200 import workloads as wl
from tests.trace_oracle import owners


def _plain_owner(prefix, share, parent, fork_pos, seq, pos):
    while seq in parent and pos < fork_pos[seq]:
        seq = parent[seq]
    if seq != wl.PREFIX_SEQ and share.get(seq, False) and pos < prefix:
        return wl.PREFIX_SEQ
    return seq


def test_owner_map_matches_the_plain_rule():
    tc = wl.TRACE
    reqs = wl.make_trace_requests(tc, 5)
    share = {q.seq_id: q.shares_prefix for q in reqs}
    parent, fork_pos = {}, {}
    for q in reqs:
        if q.fork_child >= 0:
            parent[q.fork_child] = q.seq_id
            share[q.fork_child] = q.shares_prefix
            fork_pos[q.fork_child] = (tc.prefix_len if q.shares_prefix else 0) + q.prompt_len
    state = (tc.prefix_len, wl.PREFIX_SEQ, share, parent, fork_pos)
    seqs = sorted(share)
    assert any(s in parent for s in seqs) and any(share[s] for s in seqs) and any(not share[s] for s in seqs)
    for seq in seqs:
        n = 1300
        got = owners(state, seq, n)
        want = np.array([_plain_owner(tc.prefix_len, share, parent, fork_pos, seq, p) for p in range(n)])
        assert np.array_equal(got, want), seq
    # a planted mistake (the prefix rule dropped) is caught
    bad = (0, wl.PREFIX_SEQ, share, parent, fork_pos)
    s0 = next(s for s in seqs if share[s])
    assert not np.array_equal(owners(bad, s0, 50),
                              [_plain_owner(tc.prefix_len, share, parent, fork_pos, s0, p) for p in range(50)])
