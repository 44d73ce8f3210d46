"""Pins for the oracle's multi-query (speculative verification) attention.

* torch's float64 scaled_dot_product_attention with is_causal=True over the
  whole square history (every position queries its own prefix), of which the
  last Q rows are the verification queries -- the library's own causal rule,
  not a mask written here;
* Q = 1 is the decode oracle;
* every query row equals the decode oracle on the context cut after its
  position;
* a planted off-by-one in the causal bound fails the library pin.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as oa
from oracle import cache as oc
from paged_kv_cache_381_b200 import workloads as wl


def _paged(r, S, Q, Hq, Hkv, D, bs, lens, dtype="f32"):
    nb = sum(-(-n // bs) for n in lens) + 3
    order = r.permutation(nb)
    tables = np.full((S, max(-(-n // bs) for n in lens)), -1, dtype=np.int64)
    k = np.zeros((nb, bs, Hkv, D), np.float32)
    v = np.zeros((nb, bs, Hkv, D), np.float32)
    hist = []
    used = 0
    for s, n in enumerate(lens):
        m = -(-n // bs)
        tables[s, :m] = order[used:used + m]
        used += m
        K = r.standard_normal((n, Hkv, D)).astype(np.float32)
        V = r.standard_normal((n, Hkv, D)).astype(np.float32)
        k, v = oc.scatter_history(K, V, tables[s], k, v)
        hist.append((K, V))
    q = r.standard_normal((S, Q, Hq, D)).astype(np.float32)
    return q, k, v, tables, hist


@pytest.mark.parametrize("G,Q", [(1, 1), (1, 6), (4, 5), (8, 6)])
def test_matches_library_causal_sdpa(G, Q):
    r = np.random.default_rng(10 * G + Q)
    Hkv, D, bs = 2, 32, 4
    Hq = G * Hkv
    lens = [Q, Q + 1, 37, 100]
    q, k, v, tables, hist = _paged(r, len(lens), Q, Hq, Hkv, D, bs, lens)
    scale = 1.0 / math.sqrt(D)
    out = oa.paged_verify(q, k, v, tables, lens, scale, bs, "f32")
    for s, n in enumerate(lens):
        K, V = (torch.from_numpy(x.astype(np.float64)).permute(1, 0, 2)[None] for x in hist[s])
        # every position of the history queries its own prefix; the last Q rows carry q
        allq = torch.zeros((1, Hq, n, D), dtype=torch.float64)
        allq[0, :, n - Q:, :] = torch.from_numpy(q[s].astype(np.float64)).permute(1, 0, 2)
        ref = F.scaled_dot_product_attention(allq, K, V, is_causal=True, scale=scale, enable_gqa=True)
        ref = ref[0, :, n - Q:, :].permute(1, 0, 2).numpy()
        np.testing.assert_allclose(out[s], ref, rtol=1e-12, atol=1e-13)


def test_single_query_is_decode():
    r = np.random.default_rng(2)
    lens = [1, 16, 17, 90]
    q, k, v, tables, _ = _paged(r, 4, 1, 8, 2, 16, 8, lens)
    a = oa.paged_verify(q, k, v, tables, lens, 0.25, 8, "f32")
    b = oa.paged_decode(q[:, 0], k, v, tables, lens, 0.25, 8, "f32")
    np.testing.assert_array_equal(a[:, 0], b)


def test_rows_equal_decode_on_cut_contexts():
    r = np.random.default_rng(3)
    Q, lens = 5, [5, 9, 33]
    q, k, v, tables, _ = _paged(r, 3, Q, 4, 4, 16, 4, lens)
    out = oa.paged_verify(q, k, v, tables, lens, 0.3, 4, "f32")
    for i in range(Q):
        cut = [n - Q + i + 1 for n in lens]
        ref = oa.paged_decode(q[:, i], k, v, tables, cut, 0.3, 4, "f32")
        np.testing.assert_array_equal(out[:, i], ref)


def test_short_context_rows_are_zero():
    r = np.random.default_rng(4)
    q, k, v, tables, _ = _paged(r, 1, 4, 2, 2, 8, 4, [2])
    out = oa.paged_verify(q, k, v, tables, [2], 0.5, 4, "f32")
    assert not out[0, :2].any() and out[0, 2:].any()


def test_planted_off_by_one_is_caught(monkeypatch):
    real = oa.attend

    def sees_one_less(q, K, V, scale):
        return real(q, K[:-1] if K.shape[0] > 1 else K, V[:-1] if V.shape[0] > 1 else V, scale)

    monkeypatch.setattr(oa, "attend", sees_one_less)
    with pytest.raises(AssertionError):
        test_matches_library_causal_sdpa(4, 5)
