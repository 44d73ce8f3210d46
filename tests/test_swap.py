"""Host swap pool of the C++ block manager against the oracle's model (CPU
only): the hand-derived golden trace and random operation streams, op by op,
with the slot-content check of tests/test_oracle_swap.py on both."""

import json
import os

import numpy as np
import pytest

from tests.test_oracle_swap import GOLDEN, _Driver, _Model, _replay, _stream


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_381_b200 import build
    build.build()
    import paged_kv_cache_381_b200 as pa
    return pa


class _Native(_Model):
    def __init__(self, pa, nb, bs, ncpu, order=None):
        self.bm = pa.BlockManager(nb, bs, order)
        self.bm.set_cpu_blocks(ncpu)
        self.bs = bs
        self.NoBlocks = pa.NoBlocksError
        self.Invalid = pa.PagedAttentionError

    def append(self, s):
        return self.bm.append_slot(s)

    def swap_out(self, s):
        return [tuple(int(x) for x in p) for p in self.bm.swap_out(s)]

    def swap_in(self, s):
        return [tuple(int(x) for x in p) for p in self.bm.swap_in(s)]

    def table(self, s):
        return self.bm.block_table(s)

    def free_list(self):
        return self.bm.free_list()

    def cpu_free(self):
        return self.bm.cpu_free_list()

    def ref(self, b):
        return self.bm.ref_count(b)

    def swapped(self, s):
        return self.bm.swapped(s)

    def invariants(self):
        pass


def test_native_golden_trace(pa):
    g = json.load(open(os.path.join(GOLDEN, "swap_trace.json")))
    _replay(_Native(pa, g["num_blocks"], g["block_size"], g["num_cpu_blocks"]))


@pytest.mark.parametrize("seed", range(12))
def test_native_matches_model_op_by_op(pa, seed):
    r = np.random.default_rng(700 + seed)
    nb, bs, ncpu = int(r.integers(3, 48)), int(r.choice([1, 2, 4, 8])), int(r.integers(0, 40))
    order = r.permutation(nb).tolist()
    model, nat = _Driver(_Model(nb, bs, ncpu, order)), _Driver(_Native(pa, nb, bs, ncpu, order))
    _stream([model, nat], seed, n_ops=500)
    assert model.m.free_list() == nat.m.free_list()
    assert model.m.cpu_free() == nat.m.cpu_free()
    for s in model.toks:
        assert model.m.table(s) == nat.m.table(s)
        assert model.m.swapped(s) == nat.m.swapped(s)
    assert [model.m.ref(b) for b in range(nb)] == [nat.m.ref(b) for b in range(nb)]
