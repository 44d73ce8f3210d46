"""The refill rule of the tcgen05 verification kernel's K/V ring, checked on
the host against the kernel's own constants.

The producer refills a ring slot by waiting on the commit barrier of the
element that last used it (S done for a K chunk, P.V done for a V chunk),
NSLOTS stream positions back.  Those barriers come in NPH copies (chunk g
uses copy g % NPH) and the wait tests a phase parity, so it is exact only if
the same copy's next use -- the element of the same kind NPH chunks later --
is issued no earlier than the refill, i.e. at least NSLOTS positions later in
the stream.  The stream order per item is K0, then K(c+1), V(c) for each
chunk c; this test enumerates item mixes and checks the rule for the
kernel's NSLOTS and NPH.
"""

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "paged_kv_cache_381_b200", "csrc", "device", "verify_tc.cuh")


def _constants():
    """Ring depths the default build can take (one per q-tile mode), NPH and the
    static_assert bound on NSLOTS."""
    src = open(SRC).read()
    m = re.search(r"#define PA_VERIFY_TC_SLOTS \(PA_VERIFY_TC_QTMA \? (\d+) : (\d+)\)", src)
    nslots = [int(m.group(1)), int(m.group(2))] if m else \
        [int(re.search(r"#define PA_VERIFY_TC_SLOTS (\d+)", src).group(1))]
    nph = int(re.search(r"static constexpr int NPH = (\d+);", src).group(1))
    limit = int(re.search(r"static_assert\(NSLOTS >= 3 && NSLOTS <= (\d+)", src).group(1))
    return nslots, nph, limit


def _stream(chunks_per_item):
    out, g = [], 0
    for nc in chunks_per_item:
        out.append(("K", g))
        for c in range(nc):
            if c + 1 < nc:
                out.append(("K", g + c + 1))
            out.append(("V", g + c))
        g += nc
    return out


def _min_distance(step, trials=3000, seed=0):
    r = np.random.default_rng(seed)
    worst = None
    for _ in range(trials):
        mix = [int(x) for x in r.choice([1, 1, 2, 3, 4, 5, 8, 16], size=int(r.integers(1, 12)))]
        st = _stream(mix)
        pos = {e: i for i, e in enumerate(st)}
        for i, (kind, g) in enumerate(st):
            j = pos.get((kind, g + step))
            if j is not None:
                d = j - i
                worst = d if worst is None else min(worst, d)
    return worst


def test_stream_order_matches_the_kernel_description():
    assert _stream([1]) == [("K", 0), ("V", 0)]
    assert _stream([3]) == [("K", 0), ("K", 1), ("V", 0), ("K", 2), ("V", 1), ("V", 2)]


def test_refill_rule_holds_for_the_kernel_constants():
    nslots, nph, limit = _constants()
    d = _min_distance(nph)
    assert all(d >= n for n in nslots), (d, nslots, nph)
    # the static_assert bound on NSLOTS is exactly what the rule allows
    assert d == limit, (d, limit)


def test_two_barrier_copies_would_allow_only_three_slots():
    # with the S / P.V barriers in two copies the same copy returns three
    # positions later, which is why four copies are used
    assert _min_distance(2) == 3
