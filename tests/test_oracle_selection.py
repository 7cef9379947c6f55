"""Pins for the oracle's indexer scores, Top-K, block pool, Reindex and Reuse
(no GPU).  References: exact rational arithmetic, numpy lexsort brute force,
the invariants the readings guarantee, and the worked example of the three
CSA2 modes (tests/golden/toy_example.txt)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _cache_from_rows(x_rows, W, m=1):
    """Host cache of len(x_rows) entries appended one token at a time."""
    n, D = x_rows.shape
    dI = W.shape[1]
    c = oracle.MainCache(1, n, D, dI, m)
    kv = bits(x_rows.to(torch.bfloat16))[None]
    oracle.append(c, kv, None, bits(W), None, None, np.zeros(1, np.int32), n)
    return c


def _rand_cache(n, D, dI, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, D, generator=g)
    W = (torch.randn(D, dI, generator=g) / D ** 0.5).to(torch.bfloat16)
    return _cache_from_rows(x, W), W


# ---------------------------------------------------------------- scores


def _exact_score(c, j, q, w):
    """score_j from the definition with exact rationals."""
    H_I, dI = q.shape
    s = Fraction(0)
    for h in range(H_I):
        q8, sq = oracle.quant_query(q[h])
        dot = sum(Fraction(oracle.e4m3_value(int(q8[i]))) * Fraction(oracle.e4m3_value(int(c.ik[0, j, i])))
                  for i in range(dI))
        logit = Fraction(float(sq)) * Fraction(float(c.ik_scale[0, j])) * dot
        s += Fraction(float(w[h])) * max(Fraction(0), logit)
    return s


def test_scores_match_exact_rationals():
    c, _ = _rand_cache(24, 64, 32, seed=10)
    g = torch.Generator().manual_seed(11)
    q = bits(torch.randn(3, 32, generator=g).to(torch.bfloat16))
    w = torch.rand(3, generator=g).numpy()
    got = oracle.index_scores(c, 0, q, w, 24)
    for j in range(24):
        ref = float(_exact_score(c, j, q, w))
        assert abs(got[j] - ref) <= 1e-12 * abs(ref) + 1e-300, (j, got[j], ref)


def test_single_head_unit_weight_is_relu_of_dot():
    c, _ = _rand_cache(40, 64, 32, seed=12)
    g = torch.Generator().manual_seed(13)
    q = bits(torch.randn(1, 32, generator=g).to(torch.bfloat16))
    got = oracle.index_scores(c, 0, q, np.ones(1, np.float32), 40)
    q8, sq = oracle.quant_query(q[0])
    qd = np.array([oracle.e4m3_value(int(v)) for v in q8]) * float(sq)
    for j in range(40):
        kd = np.array([oracle.e4m3_value(int(v)) for v in c.ik[0, j]]) * float(c.ik_scale[0, j])
        ref = max(0.0, float(qd @ kd))
        assert abs(got[j] - ref) <= 1e-12 * abs(ref) + 1e-300
    assert np.all(got >= 0) and np.any(got == 0) and np.any(got > 0)


def test_negative_weights_and_zero_query():
    c, _ = _rand_cache(16, 32, 32, seed=14)
    q = np.zeros((2, 32), np.uint16)
    got = oracle.index_scores(c, 0, q, np.array([1.0, -1.0], np.float32), 16)
    assert np.all(got == 0)


# ---------------------------------------------------------------- top-k


def _brute_topk(s, K):
    s = np.asarray(s, np.float64)
    ok = np.flatnonzero(np.isfinite(s))
    order = ok[np.lexsort((ok, -s[ok]))]     # score desc, index asc
    pick = np.sort(order[:K])
    return np.concatenate([pick, -np.ones(K - pick.size, np.int64)]).astype(np.int32)


@pytest.mark.parametrize("n,K,levels", [(1000, 64, None), (5000, 512, 7), (100, 512, None), (3000, 17, 3),
                                        (1, 4, None), (0, 4, None)])
def test_topk_matches_bruteforce(n, K, levels):
    rng = np.random.default_rng(n + K)
    s = rng.standard_normal(n)
    if levels:
        s = np.round(s * levels) / levels       # many exact ties
    if n > 10:
        s[rng.choice(n, n // 10, replace=False)] = -np.inf
        s[3] = np.nan
    np.testing.assert_array_equal(oracle.topk(s, K), _brute_topk(s, K))


def test_block_pool_matches_bruteforce_and_contains_topk():
    rng = np.random.default_rng(20)
    n, P, K = 70001, 512, 256
    s = rng.standard_normal(n)
    s[rng.choice(n, 3000, replace=False)] = -np.inf
    pool = oracle.block_pool(s, P)
    nb = (n + 7) // 8
    sp = np.concatenate([s, np.full(nb * 8 - n, -np.inf)]).reshape(nb, 8)
    bmax = np.where(np.isfinite(sp), sp, -np.inf).max(axis=1)
    np.testing.assert_array_equal(pool, _brute_topk(bmax, P))
    top = oracle.topk(s, K)
    assert set((top // 8).tolist()) <= set(pool.tolist())


def test_block_pool_small_context_is_every_block():
    s = np.random.default_rng(21).standard_normal(16000)
    pool = oracle.block_pool(s, 2048)
    assert pool[:2000].tolist() == list(range(2000)) and np.all(pool[2000:] == -1)


# ---------------------------------------------------------------- reindex / reuse


def test_reindex_over_full_pool_with_full_query_reproduces_full():
    c, _ = _rand_cache(1000, 64, 32, seed=22)
    g = torch.Generator().manual_seed(23)
    q = bits(torch.randn(4, 32, generator=g).to(torch.bfloat16))
    w = torch.rand(4, generator=g).numpy()
    n_vis = 997
    full = oracle.index_scores(c, 0, q, w, n_vis)
    top = oracle.topk(full, 64)
    pool = oracle.block_pool(full, 2048)
    rs = oracle.reindex_scores(c, 0, q, w, n_vis, pool)
    cols = oracle.topk(rs, 64)
    np.testing.assert_array_equal(oracle.columns_to_entries(cols, pool), top)


def test_reindex_selection_lies_in_pool():
    c, _ = _rand_cache(2000, 64, 32, seed=24)
    g = torch.Generator().manual_seed(25)
    q1 = bits(torch.randn(4, 32, generator=g).to(torch.bfloat16))
    q2 = bits(torch.randn(4, 32, generator=g).to(torch.bfloat16))
    w = torch.rand(4, generator=g).numpy()
    full = oracle.index_scores(c, 0, q1, w, 2000)
    pool = oracle.block_pool(full, 32)          # 256 candidates
    rs = oracle.reindex_scores(c, 0, q2, w, 2000, pool)
    sel = oracle.columns_to_entries(oracle.topk(rs, 64), pool)
    assert set((sel[sel >= 0] // 8).tolist()) <= set(pool[pool >= 0].tolist())
    # brute force over the pool's entries
    ent = np.array([b * 8 + r for b in pool if b >= 0 for r in range(8)])
    sc = oracle.index_scores(c, 0, q2, w, 2000, entries=ent)
    ref = ent[_brute_topk(sc, 64)]
    np.testing.assert_array_equal(sel, np.sort(ref))


def test_toy_example_modes():
    """Full keeps t3,t7; Reuse inherits them; Reindex rescoring keeps t2,t5."""
    cfg = dict(line.split(":") for line in read_golden("toy_example.txt"))
    n, K = int(cfg["tokens"]), int(cfg["topk"])
    D = dI = 32
    x = torch.zeros(n, D)
    for j in range(n):
        x[j, j] = 4.0                      # entry j points along channel j
    W = torch.eye(D).to(torch.bfloat16)    # indexer key = the entry itself
    c = _cache_from_rows(x, W)

    def query(*ents):
        q = torch.zeros(1, dI)
        for e in ents:
            q[0, e] = 1.0
        return bits(q.to(torch.bfloat16))

    w = np.ones(1, np.float32)
    full = oracle.index_scores(c, 0, query(2, 6), w, n)
    sel_full = oracle.topk(full, K)
    assert sel_full.tolist() == [int(v) for v in cfg["full"].split()]
    reuse = sel_full.copy()                # a Reuse layer runs no indexer
    assert reuse.tolist() == [int(v) for v in cfg["reuse"].split()]
    pool = oracle.block_pool(full, 2048)
    rs = oracle.reindex_scores(c, 0, query(1, 4), w, n, pool)
    sel_re = oracle.columns_to_entries(oracle.topk(rs, K), pool)
    assert sel_re.tolist() == [int(v) for v in cfg["reindex"].split()]
