"""Pins for the oracle's decode attention (CPU only).

The oracle is pinned to things other than itself:
* hand-derived closed forms stored under tests/golden/ (cited there);
* brute force on tiny inputs in plain Python scalars, with no max shift,
  reading the logical history directly (not through block tables);
* a library attention routine (torch's scaled_dot_product_attention in
  float64, with its own grouped-query mapping) on contiguous histories;
* closed forms that hold at any size (single token, zero query, constant
  values, one dominating score);
* paging invariants: physical placement, block size and sharing by reference
  change nothing;
* planted mistakes (a wrong kv-head mapping, a dropped scale, an off-by-one
  gather) each fail at least one of the pins above.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as oa
from oracle import cache as oc
from oracle.numerics import widen
from paged_kv_cache_381_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _num(x):
    return math.log(3.0) if x == "ln3" else float(x)


def _golden_cases():
    with open(os.path.join(GOLDEN, "attention_closed_forms.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_closed_forms_contiguous(case):
    q = np.array([[_num(x) for x in row] for row in case["q"]])
    K = np.array(case["k"], dtype=np.float64)
    V = np.array(case["v"], dtype=np.float64)
    out = oa.decode_history(q, K, V, case["scale"])
    np.testing.assert_allclose(out, np.array(case["expected"]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
@pytest.mark.parametrize("block_size", [1, 2, 3])
def test_golden_closed_forms_paged(case, block_size):
    """Same cases with the history scattered over a shuffled pool."""
    q = np.array([[[_num(x) for x in row] for row in case["q"]]], dtype=np.float64)
    K = np.array(case["k"], dtype=np.float64)
    V = np.array(case["v"], dtype=np.float64)
    n, Hkv, D = K.shape
    nblk = -(-n // block_size)
    pool = nblk + 3
    r = np.random.default_rng(7)
    table = r.permutation(pool)[:nblk]
    kc = np.full((pool, block_size, Hkv, D), np.nan)
    vc = np.full((pool, block_size, Hkv, D), np.nan)
    for t in range(n):
        kc[table[t // block_size], t % block_size] = K[t]
        vc[table[t // block_size], t % block_size] = V[t]
    out = oa.paged_decode(q.astype(np.float32), kc.astype(np.float32), vc.astype(np.float32), table[None, :],
                          [n], case["scale"], block_size, "f32")
    # f32 storage rounds ln 3; compare with the float32-rounded inputs' exact result
    ref = oa.decode_history(q[0].astype(np.float32).astype(np.float64),
                            K.astype(np.float32).astype(np.float64),
                            V.astype(np.float32).astype(np.float64), case["scale"])
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[0], np.array(case["expected"]), rtol=0, atol=1e-6)


def _brute(q, Khist, Vhist, scale):
    """Direct softmax in Python scalars: exp(z_i) / sum_j exp(z_j), no shift."""
    Hq, D = len(q), len(q[0])
    Hkv = len(Khist[0]) if Khist else 1
    G = Hq // Hkv
    out = []
    for h in range(Hq):
        g = h // G
        n = len(Khist)
        if n == 0:
            out.append([0.0] * D)
            continue
        e = []
        for t in range(n):
            z = scale * math.fsum(q[h][d] * Khist[t][g][d] for d in range(D))
            e.append(math.exp(z))
        den = math.fsum(e)
        out.append([math.fsum(e[t] * Vhist[t][g][d] for t in range(n)) / den for d in range(D)])
    return out


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_tiny_paged(seed):
    r = np.random.default_rng(100 + seed)
    Hkv = int(r.integers(1, 3))
    G = int(r.choice([1, 2, 4]))
    Hq, D = Hkv * G, int(r.integers(1, 5))
    bs = int(r.choice([1, 2, 4]))
    lens = r.integers(0, 6, size=3)
    nb, tables = wl.shuffled_tables(r, wl.blocks_for(lens, bs), 0, 1.0)
    q = r.standard_normal((3, Hq, D)).astype(np.float32)
    kc = r.standard_normal((nb, bs, Hkv, D)).astype(np.float32)
    vc = r.standard_normal((nb, bs, Hkv, D)).astype(np.float32)
    scale = 0.37
    got = oa.paged_decode(q, kc, vc, tables, lens, scale, bs, "f32")
    for s in range(3):
        # logical history built cell by cell from the table, independently of gather()
        Kh = [[[float(kc[tables[s][t // bs], t % bs, g, d]) for d in range(D)] for g in range(Hkv)]
              for t in range(int(lens[s]))]
        Vh = [[[float(vc[tables[s][t // bs], t % bs, g, d]) for d in range(D)] for g in range(Hkv)]
              for t in range(int(lens[s]))]
        qs = [[float(q[s, h, d]) for d in range(D)] for h in range(Hq)]
        ref = np.array(_brute(qs, Kh, Vh, scale))
        np.testing.assert_allclose(got[s], ref, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("G", [1, 2, 8])
def test_matches_library_sdpa(G):
    """torch's float64 SDPA with enable_gqa on contiguous histories."""
    r = np.random.default_rng(5 + G)
    Hkv, D, n = 2, 32, 300
    Hq = G * Hkv
    q = r.standard_normal((Hq, D))
    K = r.standard_normal((n, Hkv, D)) * 2.0
    V = r.standard_normal((n, Hkv, D))
    scale = 1.0 / math.sqrt(D)
    out = oa.decode_history(q, K, V, scale)
    tq = torch.from_numpy(q)[None, :, None, :]
    tk = torch.from_numpy(K).permute(1, 0, 2)[None]
    tv = torch.from_numpy(V).permute(1, 0, 2)[None]
    ref = F.scaled_dot_product_attention(tq, tk, tv, scale=scale, enable_gqa=True)[0, :, 0, :].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_matches_library_sdpa_long_contiguous():
    r = np.random.default_rng(11)
    D, n = 64, 1024
    q = r.standard_normal((4, D))
    K = r.standard_normal((n, 4, D))
    V = r.standard_normal((n, 4, D))
    scale = 1.0 / 8.0
    out = oa.decode_history(q, K, V, scale)
    tq = torch.from_numpy(q)[None, :, None, :]
    tk = torch.from_numpy(K).permute(1, 0, 2)[None]
    tv = torch.from_numpy(V).permute(1, 0, 2)[None]
    ref = F.scaled_dot_product_attention(tq, tk, tv, scale=scale)[0, :, 0, :].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_closed_form_single_token_exact():
    r = np.random.default_rng(3)
    for _ in range(20):
        D = int(r.integers(1, 129))
        q = r.standard_normal(D) * 50
        k = r.standard_normal((1, D)) * 50
        v = r.standard_normal((1, D))
        assert np.array_equal(oa.attend(q, k, v, 0.9), v[0])


def test_closed_form_constant_values_and_zero_query():
    r = np.random.default_rng(4)
    K = r.standard_normal((77, 16)) * 3
    c = r.standard_normal(16)
    V = np.tile(c, (77, 1))
    np.testing.assert_allclose(oa.attend(r.standard_normal(16), K, V, 0.5), c, rtol=1e-14, atol=1e-15)
    V2 = r.standard_normal((77, 16))
    np.testing.assert_allclose(oa.attend(np.zeros(16), K, V2, 0.5), V2.mean(axis=0), rtol=1e-13, atol=1e-14)
    Kc = np.tile(r.standard_normal(16), (77, 1))
    np.testing.assert_allclose(oa.attend(r.standard_normal(16), Kc, V2, 0.5), V2.mean(axis=0), rtol=1e-13, atol=1e-14)


def test_closed_form_dominating_score():
    """One score above the rest by 50: weight of the others < 33 * e^-50."""
    D, n = 8, 33
    r = np.random.default_rng(8)
    q = np.zeros(D); q[0] = 1.0
    K = np.zeros((n, D)); K[17, 0] = 50.0
    V = r.standard_normal((n, D))
    out = oa.attend(q, K, V, 1.0)
    bound = 33 * math.exp(-50) * np.abs(V).max() * 2
    assert np.abs(out - V[17]).max() <= bound + 1e-16


def test_empty_context_is_zero():
    assert np.array_equal(oa.attend(np.ones(4), np.zeros((0, 4)), np.zeros((0, 4)), 1.0), np.zeros(4))


def _paged_case(seed, dtype="bf16"):
    cfg = wl.DecodeConfig("t", dtype, 5, 8, 2, 16, 4, "uniform", len_lo=1, len_hi=40)
    inp = wl.make_decode_inputs(cfg, seed)
    return cfg, inp


def _fill(inp, block_size, tables, nb):
    Hkv, D = inp.k_hist[0].shape[1:]
    sd = inp.k_hist[0].dtype
    kc = np.zeros((nb, block_size, Hkv, D), dtype=sd)
    vc = np.zeros((nb, block_size, Hkv, D), dtype=sd)
    for s in range(len(inp.context_lens)):
        kc, vc = oc.scatter_history(inp.k_hist[s], inp.v_hist[s], tables[s], kc, vc)
    return kc, vc


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_invariant_physical_placement(dtype):
    cfg, inp = _paged_case(21, dtype)
    bs = cfg.block_size
    kc, vc = _fill(inp, bs, inp.block_tables, inp.num_blocks)
    a = oa.paged_decode(inp.q, kc, vc, inp.block_tables, inp.context_lens, cfg.scale, bs, dtype)
    r = np.random.default_rng(99)
    nb2, t2 = wl.shuffled_tables(r, wl.blocks_for(inp.context_lens, bs), inp.num_blocks + 9, 0)
    kc2, vc2 = _fill(inp, bs, t2, nb2)
    b = oa.paged_decode(inp.q, kc2, vc2, t2, inp.context_lens, cfg.scale, bs, dtype)
    assert np.array_equal(a, b)


def test_invariant_block_size_and_contiguous():
    cfg, inp = _paged_case(22)
    outs = []
    for bs in (8, 16, 64):
        r = np.random.default_rng(bs)
        nb, t = wl.shuffled_tables(r, wl.blocks_for(inp.context_lens, bs), 0, 0.5)
        kc, vc = _fill(inp, bs, t, nb)
        outs.append(oa.paged_decode(inp.q, kc, vc, t, inp.context_lens, cfg.scale, bs, "bf16"))
    # fully contiguous: decode straight from the histories
    contig = np.stack([oa.decode_history(widen(inp.q[s], "bf16"), widen(inp.k_hist[s], "bf16"),
                                         widen(inp.v_hist[s], "bf16"), cfg.scale)
                       for s in range(len(inp.context_lens))])
    for o in outs:
        assert np.array_equal(o, contig)


def test_invariant_shared_prefix_by_reference():
    """Two sequences pointing at the same prefix blocks == private copies."""
    r = np.random.default_rng(23)
    bs, Hkv, D, Hq = 4, 2, 16, 4
    prefix = 12
    tail = [5, 9]
    Kp = wl.normal_storage(r, (prefix, Hkv, D), "f16")
    Vp = wl.normal_storage(r, (prefix, Hkv, D), "f16")
    Kt = [wl.normal_storage(r, (n, Hkv, D), "f16") for n in tail]
    Vt = [wl.normal_storage(r, (n, Hkv, D), "f16") for n in tail]
    q = wl.normal_storage(r, (2, Hq, D), "f16")
    lens = [prefix + n for n in tail]
    nb = 20
    kc = np.zeros((nb, bs, Hkv, D), np.uint16)
    vc = np.zeros((nb, bs, Hkv, D), np.uint16)
    shared = [0, 1, 2]
    kc, vc = oc.scatter_history(Kp, Vp, shared, kc, vc)
    tabs_shared = [[0, 1, 2, 3, 4], [0, 1, 2, 5, 6, 7]]
    for s in range(2):
        tb = tabs_shared[s]
        for i in range(tail[s]):
            p = prefix + i
            kc[tb[p // bs], p % bs] = Kt[s][i]
            vc[tb[p // bs], p % bs] = Vt[s][i]
    T = np.full((2, 6), -1, np.int32)
    T[0, :5] = tabs_shared[0]
    T[1, :6] = tabs_shared[1]
    a = oa.paged_decode(q, kc, vc, T, lens, 0.25, bs, "f16")
    # private copies in other blocks
    kc2 = np.zeros_like(kc); vc2 = np.zeros_like(vc)
    priv = [[8, 9, 10, 3, 4], [11, 12, 13, 5, 6, 7]]
    for s in range(2):
        Kh = np.concatenate([Kp, Kt[s]]); Vh = np.concatenate([Vp, Vt[s]])
        kc2, vc2 = oc.scatter_history(Kh, Vh, priv[s], kc2, vc2)
    T2 = np.full((2, 6), -1, np.int32)
    T2[0, :5] = priv[0]
    T2[1, :6] = priv[1]
    b = oa.paged_decode(q, kc2, vc2, T2, lens, 0.25, bs, "f16")
    assert np.array_equal(a, b)


def test_rows_variant_matches_full():
    cfg, inp = _paged_case(24)
    kc, vc = _fill(inp, cfg.block_size, inp.block_tables, inp.num_blocks)
    full = oa.paged_decode(inp.q, kc, vc, inp.block_tables, inp.context_lens, cfg.scale, cfg.block_size, "bf16")
    rows = [(0, 0), (4, 7), (2, 3)]
    part = oa.paged_decode_rows(inp.q, kc, vc, inp.block_tables, inp.context_lens, cfg.scale,
                                cfg.block_size, "bf16", rows)
    for i, (s, h) in enumerate(rows):
        assert np.array_equal(part[i], full[s, h])


# -- planted mistakes: each must be caught by a pin above -------------------------

def _golden_gqa_fails(decode_fn):
    case = [c for c in _golden_cases() if c["name"].startswith("grouped")][0]
    q = np.array([[_num(x) for x in row] for row in case["q"]])
    out = decode_fn(q, np.array(case["k"], float), np.array(case["v"], float), case["scale"])
    return not np.allclose(out, np.array(case["expected"]), atol=1e-12)


def test_planted_interleaved_grouping_is_caught():
    def wrong(q, K, V, scale):
        Hq, Hkv = q.shape[0], K.shape[1]
        return np.stack([oa.attend(q[h], K[:, h % Hkv], V[:, h % Hkv], scale) for h in range(Hq)])
    assert _golden_gqa_fails(wrong)


def test_planted_missing_scale_is_caught():
    def wrong(q, K, V, scale):
        return oa.decode_history(q, K, V, 1.0)
    assert _golden_gqa_fails(wrong)


def test_planted_off_by_one_gather_is_caught(monkeypatch):
    def wrong_gather(cache, table_row, context_len, block_size):
        t = np.arange(int(context_len)) + 1
        blocks = np.asarray(table_row, dtype=np.int64)[np.minimum(t // block_size, len(table_row) - 1)]
        return cache[blocks, t % block_size]
    monkeypatch.setattr(oa, "gather", wrong_gather)
    with pytest.raises(AssertionError):
        test_brute_force_tiny_paged(1)
