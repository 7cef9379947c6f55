"""Pins for the oracle's append and sparse attention (no GPU): a dense
brute-force formulation of the same attention (every cache row scored, the
unselected ones masked), closed-form special cases, append invariants and the
planted-key recall of the Tiny workload."""
import math

import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_append_b200 import inputs as I


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _setup(n=300, D=64, W_cap=128, window=128, s_swa=0.75, seed=30):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, D, generator=g)
    W = (torch.randn(D, 32, generator=g) / D ** 0.5).to(torch.bfloat16)
    c = oracle.MainCache(1, n, D, 32, 1)
    oracle.append(c, bits(x.to(torch.bfloat16))[None], None, bits(W), None, None, np.zeros(1, np.int32), n)
    swa = oracle.SwaCache(1, W_cap, D, scale=s_swa, window=window)
    xs = torch.randn(n, D, generator=g).to(torch.bfloat16)
    oracle.append(None, None, None, None, swa, bits(xs)[None], np.zeros(1, np.int32), n)
    return c, swa, g


def _dense(c, swa, q, idx, t, scale):
    """Dense formulation: score every FP4 row and every ring row, mask out the
    rows outside the attended set, softmax in float64."""
    H, D = q.shape
    n = c.cap
    fp4 = np.array([oracle.fp4_dequant_row(c.codes[0, j], c.scales[0, j], D) for j in range(n)])
    ring = np.array([[oracle.e4m3_value(int(v)) for v in row] for row in swa.rows[0]]) * swa.scale
    keys = np.concatenate([fp4, ring])
    mult = np.zeros(len(keys))
    for k in idx:
        if 0 <= k < n:
            mult[k] += 1
    lo = max(0, t - swa.window + 1)
    for p in range(lo, t + 1):
        mult[n + p % swa.W_cap] += 1
    qf = oracle.bf16_to_f32(q).astype(np.float64)
    lg = scale * (qf @ keys.T)
    lg = np.where(mult[None] > 0, lg, -np.inf)
    lg -= lg.max(axis=1, keepdims=True)
    p = np.exp(lg) * mult[None]
    out = (p @ keys) / p.sum(axis=1, keepdims=True)
    return out


@pytest.mark.parametrize("t,window,W_cap", [(299, 128, 128), (50, 128, 128), (299, 64, 160), (0, 128, 128)])
def test_attention_matches_dense_bruteforce(t, window, W_cap):
    c, swa, g = _setup(W_cap=W_cap, window=window)
    q = bits(torch.randn(4, 64, generator=g).to(torch.bfloat16))
    idx = I.random_indices(t + 1, 40, g, n_missing=3).numpy()
    scale = 1 / math.sqrt(64)
    got = oracle.attention(c, swa, 0, q, idx, t, scale)
    ref = _dense(c, swa, q, idx, t, scale)
    gf = oracle.bf16_to_f32(got).astype(np.float64)
    # both round the same float64 result to bf16; allow one bf16 ulp for summation order
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-38
    assert np.all(np.abs(gf - ref) <= ulp)


def test_attention_single_key_returns_it():
    c, swa, g = _setup()
    swa_empty = oracle.SwaCache(1, 128, 64, window=0)
    q = bits(torch.randn(3, 64, generator=g).to(torch.bfloat16))
    idx = np.array([-1, 17, -1], np.int32)
    got = oracle.attention(c, swa_empty, 0, q, idx, 100, 0.1)
    x = oracle.fp4_dequant_row(c.codes[0, 17], c.scales[0, 17], 64)
    for h in range(3):   # values (a -0 code accumulates to +0)
        np.testing.assert_array_equal(oracle.bf16_to_f32(got[h]), oracle.bf16_to_f32(oracle.f64_to_bf16(x)))


def test_attention_zero_query_is_mean_of_values():
    c, swa, g = _setup()
    q = np.zeros((2, 64), np.uint16)
    idx = np.array([3, 9, 200], np.int32)
    t = 250
    got = oracle.attention(c, swa, 0, q, idx, t, 0.125)
    rows = [oracle.fp4_dequant_row(c.codes[0, j], c.scales[0, j], 64) for j in idx]
    rows += [np.array([oracle.e4m3_value(int(v)) for v in swa.rows[0, p % 128]]) * 0.75
             for p in range(t - 127, t + 1)]
    mean = np.mean(rows, axis=0)
    gf = oracle.bf16_to_f32(got[0]).astype(np.float64)
    assert np.all(np.abs(gf - mean) <= np.abs(mean) * 2.0 ** -8 + 1e-30)


def test_attention_empty_set_is_zero():
    c, _, g = _setup()
    swa_empty = oracle.SwaCache(1, 128, 64, window=0)
    q = bits(torch.randn(2, 64, generator=g).to(torch.bfloat16))
    got = oracle.attention(c, swa_empty, 0, q, np.full(8, -1, np.int32), 10, 0.1)
    assert not got.any()


# ---------------------------------------------------------------- append


def test_append_m1_rows_and_ring():
    g = torch.Generator().manual_seed(31)
    B, T, D = 2, 200, 64
    x = torch.randn(B, T, D, generator=g).to(torch.bfloat16)
    xs = torch.randn(B, T, D, generator=g).to(torch.bfloat16)
    W = (torch.randn(D, 32, generator=g) / 8).to(torch.bfloat16)
    c = oracle.MainCache(B, 512, D, 32, 1)
    swa = oracle.SwaCache(B, 128, D, scale=0.5)
    pos0 = np.array([0, 37], np.int32)
    oracle.append(c, bits(x), None, bits(W), swa, bits(xs), pos0, T)
    assert c.n_entries.tolist() == [200, 237]
    for b in range(B):
        for tau in (0, 77, T - 1):
            e = pos0[b] + tau
            codes, scales = oracle.quant_fp4_row(x[b, tau].float().numpy())
            assert np.array_equal(c.codes[b, e], codes) and np.array_equal(c.scales[b, e], scales)
            ik, s = oracle.index_key(codes, scales, bits(W))
            assert np.array_equal(c.ik[b, e], ik) and c.ik_scale[b, e] == s
        for tau in range(T - 128, T):
            p = pos0[b] + tau
            ref = oracle.e4m3_encode(xs[b, tau].float().numpy() / np.float32(0.5))
            assert np.array_equal(swa.rows[b, p % 128], ref)
    assert not c.codes[0, 200:].any() and not c.codes[1, :37].any()


def test_append_m2_chunking_invariance():
    """Appending in chunks that split pairs (pending token) equals one call."""
    g = torch.Generator().manual_seed(32)
    B, T, D = 1, 41, 32
    x = torch.randn(B, T, D, generator=g).to(torch.bfloat16)
    z = torch.randn(B, T, D, generator=g).to(torch.bfloat16)
    W = (torch.randn(D, 32, generator=g) / 6).to(torch.bfloat16)
    one = oracle.MainCache(B, 64, D, 32, 2)
    oracle.append(one, bits(x), bits(z), bits(W), None, None, np.zeros(1, np.int32), T)
    many = oracle.MainCache(B, 64, D, 32, 2)
    start = 0
    for ln in (1, 4, 7, 1, 1, 10, 17):
        oracle.append(many, bits(x[:, start:start + ln]), bits(z[:, start:start + ln]), bits(W),
                      None, None, np.array([start], np.int32), ln)
        start += ln
    assert start == T
    assert one.n_entries[0] == many.n_entries[0] == 20
    for a in ("codes", "scales", "ik", "ik_scale", "pending_kv", "pending_gate"):
        assert np.array_equal(getattr(one, a), getattr(many, a)), a
    # entry e pools tokens 2e, 2e+1
    pooled = oracle.pool_pair(bits(x[0, 10]), bits(x[0, 11]), bits(z[0, 10]), bits(z[0, 11]))
    codes, scales = oracle.quant_fp4_row(pooled)
    assert np.array_equal(one.codes[0, 5], codes) and np.array_equal(one.scales[0, 5], scales)


def test_visibility_rule():
    assert oracle.n_visible(100, 99, 1) == 100
    assert oracle.n_visible(100, 50, 1) == 51
    assert oracle.n_visible(100, 50, 2) == 25      # tokens 0..50: 25 complete pairs
    assert oracle.n_visible(100, 51, 2) == 26
    assert oracle.n_visible(10, 51, 2) == 10


# ---------------------------------------------------------------- whole step, Tiny


def test_tiny_planted_keys_are_recalled():
    wl = I.WORKLOADS["tiny"]
    seed, b = 0, 0
    c = oracle.MainCache(1, wl.entries, wl.D, wl.dI, 1)
    kv = I.context_kv(wl, seed, b)
    W = I.w_ik(wl, seed)
    oracle.append(c, bits(kv)[None], None, bits(W), None, None, np.zeros(1, np.int32), wl.total_tokens)
    qi, w = I.index_queries(wl, seed, 0, b)
    t = wl.total_tokens - 1
    n_vis = oracle.n_visible(int(c.n_entries[0]), t, 1)
    assert n_vis == 4096
    scores = oracle.index_scores(c, b, bits(qi[0]), w[0].numpy(), n_vis)
    top = oracle.topk(scores, wl.K)
    planted = I.planted_positions(wl, seed, b).numpy()
    assert set(planted.tolist()) <= set(top.tolist())
    pool = oracle.block_pool(scores, wl.P)
    assert set((top // 8).tolist()) <= set(pool.tolist())
