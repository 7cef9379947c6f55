"""Parity at the full workload sizes, in the launch configuration bench.py
times (runner.Step: the same calls, grids, splits and cluster shapes).

- dec_full and enc_prefill: the oracle rebuilds the whole cache from the same
  seeded inputs (sequences in parallel threads), so everything is compared:
  cache bytes and window rows bit-exact, every score within the fp32 bar, the
  Top-K sets and the pool equal up to the 1e-3 band around the K-th oracle
  score, and the attention of every (sampled) query row whose Top-K set
  matches within the tolerance.
- dec_group and long (contexts of 262,144 and 1,048,576 entries): the oracle
  computes sampled outputs one by one (cache bytes and indexer keys of sampled
  entries, Full and Reindex scores at sampled entries); the selections are
  checked by properties that hold at any size (the Top-K / pool of the
  scores the kernel was given, the column -> entry map, Reuse inheritance,
  planted-key recall), the Reindex selection of one sequence against the
  oracle's scores of all pool columns, and every layer's attention of every
  sequence against the oracle (it needs only the K selected entries and the
  window rows, so it costs the same at any context length).
No expected value comes from the CUDA path: the oracle's inputs are the
seeded generators of fp4_kv_cache_append_b200.inputs.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_append_b200 import csa2 as C
from fp4_kv_cache_append_b200 import inputs as I
from fp4_kv_cache_append_b200 import runner

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SCORE_RTOL, SCORE_ATOL_REL = 1e-4, 1e-6
BAND = 1e-3


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    C.csa2_device_status(clear=True)
    yield
    torch.cuda.synchronize()


def _pool():
    return cf.ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 8))


def _np(t):
    return t.detach().cpu().numpy()


def _check_scores(got, ref):
    ref = np.asarray(ref)
    atol = SCORE_ATOL_REL * np.abs(ref).max()
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= SCORE_RTOL * np.abs(ref) + atol), f"max err {err.max()} (max ref {np.abs(ref).max()})"


def _check_attn(got_bf16, ref_bits):
    ref = oracle.bf16_to_f32(ref_bits).astype(np.float64)
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    print(f"attention error: max {err.max() / np.abs(ref).max():.2e} of max|ref|, "
          f"mean rel {err.sum() / np.abs(ref).sum():.2e}")
    assert err.max() <= 1e-2 * np.abs(ref).max(), f"max err {err.max()} vs {np.abs(ref).max()}"
    assert err.sum() <= 1e-3 * np.abs(ref).sum(), f"mean rel err {err.sum() / np.abs(ref).sum()}"


def _band_equal(got, ref, ref_scores):
    """Index sets equal except for entries whose oracle score is within BAND of
    the K-th oracle score; returns whether the sets are identical."""
    g = set(int(x) for x in got if x >= 0)
    r = set(int(x) for x in ref if x >= 0)
    assert len(g) == len(r)
    if g == r:
        return True
    kth = min(ref_scores[e] for e in r)
    for e in g ^ r:
        assert abs(ref_scores[e] - kth) <= BAND * abs(kth), f"entry {e}: {ref_scores[e]} vs K-th {kth}"
    return False


def _oracle_sequence(wl, seed, b, layers):
    """Oracle main cache (one sequence) and window caches after the step."""
    om = oracle.MainCache(1, runner.cap_for(wl), wl.D, wl.dI, wl.m)
    kv = I.context_kv(wl, seed, b)
    gate = I.context_gate(wl, seed, b) if wl.m == 2 else None
    oracle.append(om, I.bits(kv)[None], I.bits(gate)[None] if gate is not None else None,
                  I.bits(I.w_ik(wl, seed)), None, None, np.zeros(1, np.int32), kv.shape[0])
    sws = {}
    lo = I.window_lo(wl)
    for l in layers:
        sw = oracle.SwaCache(1, runner.w_cap_for(wl), wl.D, window=wl.window)
        rows = I.window_kv(wl, seed, l, b)
        oracle.append(None, None, None, None, sw, I.bits(rows)[None], np.array([lo], np.int32), rows.shape[0])
        sws[l] = sw
    return om, sws


def _assert_cache_rows(gm, b, om, entries=None):
    sl = slice(None) if entries is None else entries
    for name in ("codes", "scales", "ik"):
        np.testing.assert_array_equal(_np(getattr(gm, name)[b])[sl], getattr(om, name)[0][sl], err_msg=name)
    np.testing.assert_array_equal(_np(gm.ik_scale[b])[sl].view(np.uint32), om.ik_scale[0][sl].view(np.uint32))


def _entry_oracle(wl, seed, b, entries, kv_all, W):
    """Oracle bytes of the given entries of sequence b, one by one (m = 1)."""
    om = oracle.MainCache(1, runner.cap_for(wl), wl.D, wl.dI, wl.m)
    for e in entries:
        codes, scales = oracle.quant_fp4_row(oracle.bf16_to_f32(I.bits(kv_all[e])))
        ik, s = oracle.index_key(codes, scales, W)
        om.codes[0, e], om.scales[0, e], om.ik[0, e], om.ik_scale[0, e] = codes, scales, ik, s
    return om


def _topk_property(scores, K, got):
    """got = the K best finite scores (ties -> smaller column), ascending, -1 padded."""
    s = scores.astype(np.float64)
    fin = np.isfinite(s)
    cols = np.nonzero(fin)[0]
    order = cols[np.lexsort((cols, -s[cols]))][:K]
    want = np.full(K, -1, np.int64)
    want[: order.size] = np.sort(order)
    np.testing.assert_array_equal(np.asarray(got, np.int64), want)


def _pool_property(scores, P, got):
    s = scores.astype(np.float64).copy()
    s[~np.isfinite(s)] = -np.inf
    nb = (s.size + 7) // 8
    pad = np.full(nb * 8, -np.inf)
    pad[: s.size] = s
    bmax = pad.reshape(nb, 8).max(axis=1)
    _topk_property(bmax, P, got)


def _attn_sane(out, main, b):
    o = out.float()
    assert torch.isfinite(o).all()
    assert o.abs().max() > 0
    # a convex combination of dequantised rows: |o| <= max |FP4 value| x max scale (448 * 6)
    assert o.abs().max() <= 448.0 * 6.0


# ---------------------------------------------------------------------------- dec_full


def test_fullsize_dec_full_step():
    wl = I.WORKLOADS["dec_full"]
    seed = 0
    st = runner.Step(wl, seed=seed, copies=1)
    st.prefill()
    st.run(copy=0)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    with _pool() as ex:
        ref = list(ex.map(lambda b: _oracle_sequence(wl, seed, b, [0]), range(wl.B)))
    gm, gs = st.main[0], st.swa[0][0]
    t = wl.first_new
    for b, (om, sws) in enumerate(ref):
        _assert_cache_rows(gm, b, om)
        assert int(gm.n_entries[b]) == int(om.n_entries[0])
        np.testing.assert_array_equal(_np(gs.rows[b]), sws[0].rows[0])

    def row(b):
        om = ref[b][0]
        qi, w = I.index_queries(wl, seed, 0, b, 1)
        n_vis = oracle.n_visible(int(om.n_entries[0]), t, wl.m)
        sc = oracle.index_scores(om, 0, I.bits(qi[0]), w[0].numpy(), n_vis)
        return n_vis, sc, oracle.topk(sc, wl.K), oracle.block_pool(sc, wl.P)

    with _pool() as ex:
        rows = list(ex.map(row, range(wl.B)))
    scores, nval, idx, pool = _np(st.scores), _np(st.n_valid), _np(st.idx), _np(st.pool)
    compared = 0
    for b, (n_vis, sc, ref_idx, ref_pool) in enumerate(rows):
        assert nval[b] == n_vis
        _check_scores(scores[b, :n_vis], sc)
        same = _band_equal(idx[b], ref_idx, sc)
        bs = np.full((n_vis + 7) // 8 * 8, -np.inf)
        bs[:n_vis] = sc
        _band_equal(pool[b], ref_pool, bs.reshape(-1, 8).max(axis=1))
        if same:
            q = I.queries(wl, seed, 0, b, 1)[0]
            out = oracle.attention(ref[b][0], ref[b][1][0], 0, I.bits(q), ref_idx, t, st.scale)
            _check_attn(st.out[0][b, 0], out)
            compared += 1
    assert compared >= wl.B - 2


# ---------------------------------------------------------------------------- enc_prefill


def test_fullsize_enc_prefill_chunk():
    wl = I.WORKLOADS["enc_prefill"]
    seed = 0
    st = runner.Step(wl, seed=seed, copies=1)
    st.prefill()
    st.run(copy=0)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    om, sws = _oracle_sequence(wl, seed, 0, st.layers)
    gm = st.main[0]
    _assert_cache_rows(gm, 0, om)
    assert int(gm.n_entries[0]) == int(om.n_entries[0])
    np.testing.assert_array_equal(gm.pending_kv[0].cpu().view(torch.int16).numpy().view(np.uint16), om.pending_kv[0])
    for l in st.layers:
        np.testing.assert_array_equal(_np(st.swa[0][l].rows[0]), sws[l].rows[0])
    qi, w = I.index_queries(wl, seed, 0, 0, wl.T)
    qs = {l: I.queries(wl, seed, l, 0, wl.T) for l in st.layers}
    rows = [0, 1, 2047, 4096, wl.T - 1]

    def row(j):
        t = wl.first_new + j
        n_vis = oracle.n_visible(int(om.n_entries[0]), t, wl.m)
        sc = oracle.index_scores(om, 0, I.bits(qi[j]), w[j].numpy(), n_vis)
        return t, n_vis, sc, oracle.topk(sc, wl.K)

    with _pool() as ex:
        res = list(ex.map(row, rows))
    scores, nval, idx = _np(st.scores), _np(st.n_valid), _np(st.idx)
    compared = 0
    for j, (t, n_vis, sc, ref_idx) in zip(rows, res):
        assert nval[j] == n_vis
        _check_scores(scores[j, :n_vis], sc)
        if _band_equal(idx[j], ref_idx, sc):
            for l in st.layers:
                out = oracle.attention(om, sws[l], 0, I.bits(qs[l][j]), ref_idx, t, st.scale)
                _check_attn(st.out[l][0, j], out)
            compared += 1
    assert compared >= len(rows) - 1
    # every row's selection is the Top-K of the scores it was given
    for j in range(0, wl.T, 1021):
        _topk_property(scores[j, : nval[j]], wl.K, idx[j])


# ---------------------------------------------------------------------------- dec_group, long


def _check_group(st, wl, seed, sample=256):
    """Reindex + Reuse layers of a decoder group, by samples and properties."""
    gm = st.main[0]
    kv_ctx = st._kv_ctx
    W = I.bits(I.w_ik(wl, seed))
    g = np.random.default_rng(7)
    t = wl.first_new
    scores, pool_scores, idx = _np(st.scores), _np(st.pool_scores), _np(st.idx)
    gpool = _np(st.group_pool) if wl.mode == "group" else _np(st.pool)
    lo = I.window_lo(wl)

    picks = []   # sampled entries (with the step's new one) and sampled pool entries, per sequence
    for b in range(wl.B):
        n_vis = int(gm.n_entries[b])
        ent = np.unique(np.concatenate([g.choice(n_vis, sample, replace=False), [n_vis - 1]])).astype(np.int32)
        pool_ent = (gpool[b][gpool[b] >= 0][:, None] * 8 + np.arange(8)[None, :]).ravel()
        pool_ent = pool_ent[pool_ent < n_vis]
        pool_ent = np.unique(g.choice(pool_ent, min(sample, pool_ent.size), replace=False)).astype(np.int32)
        picks.append((ent, pool_ent))

    def seq(b):
        ent, pool_ent = picks[b]
        return ent, pool_ent, _entry_oracle(wl, seed, b, np.union1d(ent, pool_ent), kv_ctx[b], W)

    with _pool() as ex:
        per = list(ex.map(seq, range(wl.B)))
    for b, (ent, pool_ent, om) in enumerate(per):
        _assert_cache_rows(gm, b, om, ent)
        n_vis = oracle.n_visible(int(gm.n_entries[b]), t, wl.m)
        # the pool layer's Full scan at sampled entries, and the pool it built
        head = runner.POOL_LAYER if wl.mode == "group" else 0
        qi, w = I.index_queries(wl, seed, head, b, 1)
        _check_scores(scores[b][ent], oracle.index_scores(om, 0, I.bits(qi[0]), w[0].numpy(), n_vis, entries=ent))
        _pool_property(scores[b][:n_vis], wl.P, gpool[b])
        # Reindex: its own query over the pool's columns
        rl = [l for k, l in st.plan if k == "reindex"][0]
        qi, w = I.index_queries(wl, seed, rl, b, 1)
        colmap = oracle.columns_to_entries(np.arange(wl.P * 8, dtype=np.int32) % (wl.P * 8), gpool[b])
        sel = np.nonzero(np.isin(colmap, pool_ent))[0]
        ref = oracle.index_scores(om, 0, I.bits(qi[0]), w[0].numpy(), n_vis, entries=colmap[sel].astype(np.int32))
        _check_scores(pool_scores[b][sel], ref)
        # the Reindex Top-K is the Top-K of its columns, mapped to entries
        cols = np.full(wl.K, -1, np.int64)
        s = pool_scores[b].astype(np.float64)
        fin = np.nonzero(np.isfinite(s))[0]
        best = fin[np.lexsort((fin, -s[fin]))][: wl.K]
        cols[: best.size] = np.sort(best)
        np.testing.assert_array_equal(idx[b], oracle.columns_to_entries(cols.astype(np.int32), gpool[b]))
        # window rows of every layer
        for l in st.layers:
            sw = oracle.SwaCache(1, runner.w_cap_for(wl), wl.D, window=wl.window)
            rows = I.window_kv(wl, seed, l, b)
            oracle.append(None, None, None, None, sw, I.bits(rows)[None], np.array([lo], np.int32), rows.shape[0])
            np.testing.assert_array_equal(_np(st.swa[0][l].rows[b]), sw.rows[0])
        for l in st.layers:   # Reuse layers read the same indices; their outputs are sane
            _attn_sane(st.out[l][b, 0], gm, b)
    _check_group_attention(st, wl, seed)
    _check_reindex_selection(st, wl, seed, 0)


def _oracle_window(wl, seed, l, b):
    sw = oracle.SwaCache(1, runner.w_cap_for(wl), wl.D, window=wl.window)
    rows = I.window_kv(wl, seed, l, b)
    oracle.append(None, None, None, None, sw, I.bits(rows)[None], np.array([I.window_lo(wl)], np.int32),
                  rows.shape[0])
    return sw


def _check_group_attention(st, wl, seed):
    """The Reindex layer's and every Reuse layer's attention against the
    oracle, for every sequence, with the step's own selection (the oracle
    needs only the K selected entries and the layer's window rows)."""
    t = wl.first_new
    W = I.bits(I.w_ik(wl, seed))
    idx = _np(st.idx)
    layers = [l for k, l in st.plan if k != "full"]

    def one(b):
        sel = idx[b][idx[b] >= 0]
        om = _entry_oracle(wl, seed, b, np.unique(sel), st._kv_ctx[b], W)
        out = []
        for l in layers:
            q = I.queries(wl, seed, l, b, 1)[0]
            out.append((l, oracle.attention(om, _oracle_window(wl, seed, l, b), 0, I.bits(q), idx[b], t, st.scale)))
        return out

    with _pool() as ex:
        res = list(ex.map(one, range(wl.B)))
    for b, per in enumerate(res):
        for l, ref in per:
            _check_attn(st.out[l][b, 0], ref)


def _check_reindex_selection(st, wl, seed, b):
    """The Reindex layer's Top-K of sequence b against the oracle's scores of
    all P x 8 pool columns, equal up to the 1e-3 band around the K-th score."""
    gm = st.main[0]
    gpool = _np(st.group_pool) if wl.mode == "group" else _np(st.pool)
    n_vis = oracle.n_visible(int(gm.n_entries[b]), wl.first_new, wl.m)
    colmap = oracle.columns_to_entries(np.arange(wl.P * 8, dtype=np.int32), gpool[b])
    ents = np.unique(colmap[(colmap >= 0) & (colmap < n_vis)]).astype(np.int32)
    om = _entry_oracle(wl, seed, b, ents, st._kv_ctx[b], I.bits(I.w_ik(wl, seed)))
    rl = [l for k, l in st.plan if k == "reindex"][0]
    qi, w = I.index_queries(wl, seed, rl, b, 1)
    col_scores = oracle.reindex_scores(om, 0, I.bits(qi[0]), w[0].numpy(), n_vis, gpool[b])
    ref = oracle.columns_to_entries(oracle.topk(col_scores, wl.K), gpool[b])
    by_entry = {int(e): float(v) for e, v in zip(colmap, col_scores) if e >= 0}
    _band_equal(_np(st.idx)[b], ref, by_entry)


def test_fullsize_dec_group():
    wl = I.WORKLOADS["dec_group"]
    st = runner.Step(wl, seed=0, copies=1)
    st.prefill()
    st.run(copy=0)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    _check_group(st, wl, 0)


def test_fullsize_long_context():
    wl = I.WORKLOADS["long"]
    st = runner.Step(wl, seed=0, copies=1)
    st.prefill()
    st.run(copy=0)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    scores, nval = _np(st.scores), _np(st.n_valid)
    pool_step = _np(st.pool)
    # the Full layer's selection (the Reindex layer reuses the idx buffer, so
    # select again with the step's call and buffers): the Top-K and pool of its
    # 1,048,576 scores, the planted keys among them
    idx2 = torch.empty_like(st.idx)
    pool2 = torch.empty_like(st.pool)
    C.csa2_topk(st.scores, st.cap, wl.K, idx2, n_valid=st.n_valid, P_out=wl.P, out_pool=pool2, ws=st.ws_topk)
    torch.cuda.synchronize()
    idx2, pool2 = _np(idx2), _np(pool2)
    np.testing.assert_array_equal(pool2, pool_step)
    for b in range(wl.B):
        n_vis = int(nval[b])
        _topk_property(scores[b, :n_vis], wl.K, idx2[b])
        _pool_property(scores[b, :n_vis], wl.P, pool2[b])
        planted = I.planted_positions(wl, 0, b).numpy()
        assert np.isin(planted, idx2[b]).mean() >= 0.9
    # the Full layer's own attention (layer 0) over the Full selection
    W = I.bits(I.w_ik(wl, 0))
    for b in range(wl.B):
        om = _entry_oracle(wl, 0, b, np.unique(idx2[b][idx2[b] >= 0]), st._kv_ctx[b], W)
        ref = oracle.attention(om, _oracle_window(wl, 0, 0, b), 0, I.bits(I.queries(wl, 0, 0, b, 1)[0]), idx2[b],
                               wl.first_new, st.scale)
        _check_attn(st.out[0][b, 0], ref)
    _check_group(st, wl, 0)
