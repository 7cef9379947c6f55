"""GPU parity of every libcsa2 entry point against the oracle (same seeded
inputs, calls through the C ABI).

Bars: cache bytes (FP4 codes, E4M3 scales, window FP8 rows, indexer-key FP8
codes and f32 scales) bit-exact; Top-K of identical fp32 scores exact; Top-K of
the whole scoring chain equal up to the 1e-3 tie band around the K-th oracle
score; attention max|err| <= 1e-2 max|ref| and sum|err|/sum|ref| <= 1e-3.
Indexer scores: |gpu - oracle| <= 1e-4 |oracle| + 1e-6 max|oracle| (fp32
accumulation of exact FP8 products over <= 64 heads: ~64 * 2^-24 relative,
with headroom for the tensor-core accumulation order).
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_append_b200 import csa2 as C
from fp4_kv_cache_append_b200 import inputs as I

pytestmark = pytest.mark.gpu

SCORE_RTOL, SCORE_ATOL_REL = 1e-4, 1e-6
BAND = 1e-3


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def gen(seed):
    return torch.Generator().manual_seed(seed)


@pytest.fixture(autouse=True)
def _clean_status():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    C.csa2_device_status(clear=True)
    yield
    torch.cuda.synchronize()


def build_pair(B, cap, D, dI, m, T, pos0, seed, W_cap=128, s_swa=1.0, window=128, swa=True):
    """Same append on GPU and oracle; returns (gpu caches, oracle caches, inputs)."""
    g = gen(seed)
    kv = torch.randn(B, T, D, generator=g).to(torch.bfloat16)
    gate = torch.randn(B, T, D, generator=g).mul(2).to(torch.bfloat16) if m == 2 else None
    W = (torch.randn(D, dI, generator=g) / math.sqrt(D)).to(torch.bfloat16)
    kvs = torch.randn(B, T, D, generator=g).to(torch.bfloat16)
    pos = np.asarray(pos0, np.int32)
    gm = C.MainCache(B, cap, D, dI, m)
    gs = C.SwaCache(B, W_cap, D, scale=s_swa, window=window) if swa else None
    C.csa2_append_quant(gm, kv.cuda(), gate.cuda() if gate is not None else None, W.cuda(), gs,
                        kvs.cuda() if swa else None, torch.from_numpy(pos).cuda(), T)
    om = oracle.MainCache(B, cap, D, dI, m)
    osw = oracle.SwaCache(B, W_cap, D, scale=s_swa, window=window) if swa else None
    oracle.append(om, bits(kv), bits(gate) if gate is not None else None, bits(W), osw,
                  bits(kvs) if swa else None, pos, T)
    torch.cuda.synchronize()
    return gm, gs, om, osw, W


def assert_cache_equal(gm, om, gs=None, osw=None):
    for name in ("codes", "scales", "ik", "n_entries"):
        np.testing.assert_array_equal(getattr(gm, name).cpu().numpy(), getattr(om, name), err_msg=name)
    np.testing.assert_array_equal(gm.ik_scale.cpu().numpy().view(np.uint32), om.ik_scale.view(np.uint32))
    if gm.m == 2:
        np.testing.assert_array_equal(bits(gm.pending_kv), om.pending_kv)
        np.testing.assert_array_equal(bits(gm.pending_gate), om.pending_gate)
    if gs is not None:
        np.testing.assert_array_equal(gs.rows.cpu().numpy(), osw.rows)


# ------------------------------------------------------------------ A1 / A1' / A2 append


@pytest.mark.parametrize("D,dI", [(128, 64), (256, 128), (512, 128), (512, 64)])
def test_append_m1_bit_exact(D, dI):
    gm, gs, om, osw, _ = build_pair(B=3, cap=512, D=D, dI=dI, m=1, T=300, pos0=[0, 17, 200], seed=D + dI,
                                    s_swa=0.5)
    assert_cache_equal(gm, om, gs, osw)
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("D,dI,with_window", [(512, 128, True), (256, 64, True), (128, 64, False), (512, 64, True)])
def test_append_decode_single_token_and_ring_wrap(D, dI, with_window):
    # one token per sequence per call: the decode path (an 8-block cluster per entry)
    B, cap = 3, 1024
    gm, gs, om, osw, W = build_pair(B=B, cap=cap, D=D, dI=dI, m=1, T=700, pos0=[0, 5, 9], seed=3 + D + dI)
    g = gen(4)
    for step in range(3):
        kv = torch.randn(B, 1, D, generator=g).to(torch.bfloat16)
        kv[1, 0, : D // 2] = 0   # all-zero groups: scale byte 0, codes 0
        kvs = torch.randn(B, 1, D, generator=g).to(torch.bfloat16)
        pos = np.array([700 + step, 705 + step, 709 + step], np.int32)
        C.csa2_append_quant(gm, kv.cuda(), None, W.cuda(), gs if with_window else None,
                            kvs.cuda() if with_window else None, torch.from_numpy(pos).cuda(), 1)
        oracle.append(om, bits(kv), None, bits(W), osw if with_window else None, bits(kvs) if with_window else None,
                      pos, 1)
    torch.cuda.synchronize()
    if with_window:
        assert_cache_equal(gm, om, gs, osw)
    else:
        assert_cache_equal(gm, om)


@pytest.mark.parametrize("D,s_swa", [(512, 1.0), (256, 0.5)])
def test_swa_replay_rebuild_matches_incremental_ring(D, s_swa):
    """SWA bounded replay: re-encoding the last 128 tokens' window rows with
    one window-only append (no main cache) into an empty ring gives the same
    ring bytes as the ring built token by token, and as the oracle's."""
    B, W_cap, n = 2, 128, 300
    g = gen(61 + D)
    kvs = torch.randn(B, n, D, generator=g).to(torch.bfloat16)
    inc = C.SwaCache(B, W_cap, D, scale=s_swa)
    osw = oracle.SwaCache(B, W_cap, D, s_swa, 128)
    for t in range(n):   # decode-style: one token per call
        pos = torch.full((B,), t, dtype=torch.int32)
        C.csa2_append_quant(None, None, None, None, inc, kvs[:, t:t + 1].contiguous().cuda(), pos.cuda(), 1)
    oracle.append(None, None, None, None, osw, bits(kvs), np.zeros(B, np.int32), n)
    reb = C.SwaCache(B, W_cap, D, scale=s_swa)
    first = n - W_cap
    C.csa2_append_quant(None, None, None, None, reb, kvs[:, first:].contiguous().cuda(),
                        torch.full((B,), first, dtype=torch.int32).cuda(), W_cap)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(reb.rows.cpu().numpy(), inc.rows.cpu().numpy())
    np.testing.assert_array_equal(reb.rows.cpu().numpy(), osw.rows)
    assert C.csa2_device_status() == 0


def test_append_m2_pending_across_calls():
    B, D, dI, cap = 2, 256, 64, 256
    g = gen(5)
    T_all = 77
    kv = torch.randn(B, T_all, D, generator=g).to(torch.bfloat16)
    gate = torch.randn(B, T_all, D, generator=g).mul(3).to(torch.bfloat16)
    W = (torch.randn(D, dI, generator=g) / 16).to(torch.bfloat16)
    gm = C.MainCache(B, cap, D, dI, 2)
    om = oracle.MainCache(B, cap, D, dI, 2)
    start = 0
    for ln in (1, 5, 2, 1, 30, 38):
        sl = slice(start, start + ln)
        pos = np.array([start, start], np.int32)
        C.csa2_append_quant(gm, kv[:, sl].contiguous().cuda(), gate[:, sl].contiguous().cuda(), W.cuda(), None,
                            None, torch.from_numpy(pos).cuda(), ln)
        oracle.append(om, bits(kv[:, sl]), bits(gate[:, sl]), bits(W), None, None, pos, ln)
        start += ln
    torch.cuda.synchronize()
    assert start == T_all
    assert_cache_equal(gm, om)


def test_append_m2_bulk_prefill_chunk():
    gm, gs, om, osw, _ = build_pair(B=1, cap=2048, D=512, dI=128, m=2, T=2000, pos0=[100], seed=6,
                                    W_cap=2176, s_swa=2.0)
    assert_cache_equal(gm, om, gs, osw)


# ------------------------------------------------------------------ A3 Full scoring


def _rows_queries(B, T_q, H_I, dI, seed):
    g = gen(seed)
    q = torch.randn(B, T_q, H_I, dI, generator=g).to(torch.bfloat16)
    w = torch.rand(B, T_q, H_I, generator=g)
    return q, w


def _check_scores(got, ref):
    ref = np.asarray(ref)
    atol = SCORE_ATOL_REL * np.abs(ref).max()
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= SCORE_RTOL * np.abs(ref) + atol), f"max err {err.max()} (max ref {np.abs(ref).max()})"


@pytest.mark.parametrize("D,dI,H_I,n,T_q,m", [(128, 64, 4, 1000, 1, 1), (512, 128, 64, 2047, 3, 1),
                                              (256, 128, 17, 700, 2, 1), (512, 128, 64, 900, 4, 2)])
def test_index_full_vs_oracle(D, dI, H_I, n, T_q, m):
    B = 2
    cap = (n // m + 127) // 128 * 128 + 128
    T = n
    gm, _, om, _, _ = build_pair(B=B, cap=cap, D=D, dI=dI, m=m, T=T, pos0=[0, 0], seed=n + dI, swa=False)
    q, w = _rows_queries(B, T_q, H_I, dI, seed=7)
    # causal positions: the last T_q tokens, and one early query
    qpos = np.stack([np.arange(n - T_q, n) for _ in range(B)]).astype(np.int32)
    qpos[1, 0] = 300
    scores = torch.full((B * T_q, cap), float("nan"), device="cuda")
    nval = torch.zeros(B * T_q, dtype=torch.int32, device="cuda")
    C.csa2_index_full(gm, q.cuda(), w.cuda(), torch.from_numpy(qpos).cuda(), scores, nval)
    torch.cuda.synchronize()
    sc = scores.cpu().numpy()
    nv = nval.cpu().numpy()
    for b in range(B):
        for j in range(T_q):
            r = b * T_q + j
            n_vis = oracle.n_visible(int(om.n_entries[b]), int(qpos[b, j]), m)
            assert nv[r] == n_vis
            ref = oracle.index_scores(om, b, bits(q[b, j]), w[b, j].numpy(), n_vis)
            _check_scores(sc[r, :n_vis], ref)
            assert np.all(np.isnan(sc[r, n_vis:])), "columns beyond n_vis must not be written"
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("D,dI,H_I,T_q", [(512, 128, 64, 1), (256, 64, 17, 3)])
def test_index_full_prepared_by_the_append(D, dI, H_I, T_q):
    """Append + query preparation in one launch, then the prepared scan: the
    cache bytes of the appended token, and scores bit-identical to the plain
    scan (which itself is checked against the oracle above)."""
    B, n = 2, 3000
    cap = (n + 1 + 127) // 128 * 128
    gm, gs, om, osw, W = build_pair(B=B, cap=cap, D=D, dI=dI, m=1, T=n, pos0=[0, 0], seed=31 + D)
    q, w = _rows_queries(B, T_q, H_I, dI, seed=32)
    g = gen(33)
    kv = torch.randn(B, 1, D, generator=g).to(torch.bfloat16)
    kvs = torch.randn(B, 1, D, generator=g).to(torch.bfloat16)
    pos = np.array([n, n], np.int32)
    qpos = np.array([[n - T_q + 1 + j for j in range(T_q)] for _ in range(B)], np.int32)
    qpos[:, -1] = n
    ws = C.workspace(C.csa2_index_workspace_size(B * T_q, dI))
    C.csa2_append_quant_ex(gm, kv.cuda(), None, W.cuda(), gs, kvs.cuda(), torch.from_numpy(pos).cuda(), 1,
                           q.cuda(), w.cuda(), ws)
    oracle.append(om, bits(kv), None, bits(W), osw, bits(kvs), pos, 1)
    got = torch.full((B * T_q, cap), float("nan"), device="cuda")
    nv = torch.empty(B * T_q, dtype=torch.int32, device="cuda")
    C.csa2_index_full_prepared(gm, torch.from_numpy(qpos).cuda(), got, nv, ws=ws)
    plain = torch.full((B * T_q, cap), float("nan"), device="cuda")
    C.csa2_index_full(gm, q.cuda(), w.cuda(), torch.from_numpy(qpos).cuda(), plain, nv)
    torch.cuda.synchronize()
    assert_cache_equal(gm, om, gs, osw)
    a, b_ = got.cpu().numpy(), plain.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b_.view(np.uint32))
    # preparation only (T = 0): the same workspace contents
    ws2 = C.workspace(C.csa2_index_workspace_size(B * T_q, dI))
    C.csa2_append_quant_ex(gm, None, None, None, None, None, torch.from_numpy(pos).cuda(), 0, q.cuda(), w.cuda(), ws2)
    torch.cuda.synchronize()
    assert torch.equal(ws.cpu(), ws2.cpu())
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("T_q", [1, 4])
def test_index_scan_wait_that_runs_out_flags_and_recovers(T_q):
    """Failure detection without a fault: with csa2_debug_inject_timeout the
    scan's MMA issuer waits on a barrier that nothing arrives on; the wait
    runs out, the scan sets CSA2_DEV_TIMEOUT, stops every role, drains its
    copies and MMAs, frees its tensor memory and returns.  The context stays
    usable: the next scans give the reference scores again."""
    B, n, D, dI, H_I = 2, 3000, 256, 128, 64
    gm, _, om, _, _ = build_pair(B=B, cap=3072, D=D, dI=dI, m=1, T=n, pos0=[0, 0], seed=91, swa=False)
    g = gen(92)
    qi = torch.randn(B, T_q, H_I, dI, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(B, T_q, H_I, generator=g).cuda()
    qpos = torch.tensor(np.stack([np.arange(n - T_q, n)] * B), dtype=torch.int32).cuda()
    ref = torch.zeros(B * T_q, 3072, device="cuda")
    C.csa2_index_full(gm, qi, w, qpos, ref)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    bad = torch.zeros_like(ref)
    C.csa2_debug_inject_timeout(64)
    try:
        C.csa2_index_full(gm, qi, w, qpos, bad)
        torch.cuda.synchronize()
    finally:
        C.csa2_debug_inject_timeout(0)
    assert C.csa2_device_status(clear=True) & C.DEV_TIMEOUT
    assert not torch.equal(bad, ref)   # the scan gave up before writing its scores
    again = torch.zeros_like(ref)
    for _ in range(2):
        C.csa2_index_full(gm, qi, w, qpos, again)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    assert torch.equal(again, ref)


@pytest.mark.parametrize("T_q,m", [(8, 1), (6, 1), (4, 2)])
def test_index_full_row_groups_match_single_rows(T_q, m):
    """T_q a multiple of 4 (or 2) takes the multi-row scan, which puts 4 (or 2)
    query rows on one MMA; every row's scores must equal, bit for bit, those
    of the one-row scan of that row alone (same per-entry head reduction)."""
    B, D, dI, H_I, n = 2, 512, 128, 64, 5000
    cap = (n // m + 127) // 128 * 128 + 128
    gm, _, om, _, _ = build_pair(B=B, cap=cap, D=D, dI=dI, m=m, T=n, pos0=[0, 0], seed=41 + T_q, swa=False)
    q, w = _rows_queries(B, T_q, H_I, dI, seed=42)
    qpos = np.stack([np.arange(n - T_q, n) for _ in range(B)]).astype(np.int32)
    qpos[1, 1] = 777   # rows of one group with different causal limits
    grouped = torch.full((B * T_q, cap), float("nan"), device="cuda")
    nval = torch.zeros(B * T_q, dtype=torch.int32, device="cuda")
    C.csa2_index_full(gm, q.cuda(), w.cuda(), torch.from_numpy(qpos).cuda(), grouped, nval)
    single = torch.full((B * T_q, cap), float("nan"), device="cuda")
    nv1 = torch.zeros(B, dtype=torch.int32, device="cuda")
    for j in range(T_q):
        out = torch.full((B, cap), float("nan"), device="cuda")
        C.csa2_index_full(gm, q[:, j:j + 1].contiguous().cuda(), w[:, j:j + 1].contiguous().cuda(),
                          torch.from_numpy(qpos[:, j:j + 1].copy()).cuda(), out, nv1)
        single[j::T_q] = out
    torch.cuda.synchronize()
    a, b_ = grouped.cpu().numpy(), single.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b_.view(np.uint32))
    nv = nval.cpu().numpy()
    for b in range(B):
        for j in (0, T_q - 1):
            r = b * T_q + j
            n_vis = oracle.n_visible(int(om.n_entries[b]), int(qpos[b, j]), m)
            assert nv[r] == n_vis
            _check_scores(a[r, :n_vis], oracle.index_scores(om, b, bits(q[b, j]), w[b, j].numpy(), n_vis))
    assert C.csa2_device_status() == 0


# ------------------------------------------------------------------ projected append (CED producer)


def _decisions(x, D):
    """FP4 decisions (scale bytes [rows][D/16], codes [rows][D]) of binary32 rows."""
    rows = x.shape[0]
    g = x.reshape(rows, D // 16, 16)
    amax = np.abs(g).max(axis=2).astype(np.float32)
    sb = np.where(amax == 0, 0, oracle.e4m3_encode(amax / np.float32(6)))
    sv = np.vectorize(oracle.e4m3_value)(sb.astype(np.int64)).astype(np.float32)
    safe = np.where(sv == 0, np.float32(1), sv)
    codes = np.where(sv[..., None] == 0, 0, oracle.e2m1_encode((g / safe[..., None]).astype(np.float32)))
    return sb, codes.reshape(rows, D)


def _codes_with(x, sb, D):
    """E2M1 codes [rows][D] of binary32 rows under given scale bytes [rows][D/16]."""
    rows = x.shape[0]
    sv = np.vectorize(oracle.e4m3_value)(sb.astype(np.int64)).astype(np.float32)
    safe = np.where(sv == 0, np.float32(1), sv)
    g = x.reshape(rows, D // 16, 16)
    return np.where(sv[..., None] == 0, 0, oracle.e2m1_encode((g / safe[..., None]).astype(np.float32))).reshape(rows, D)


def _unpack(codes_rows):
    lo, hi = codes_rows & 0xF, codes_rows >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes_rows.shape[0], -1)


@pytest.mark.parametrize("B,T,d,D,dI,pos", [(2, 300, 1024, 512, 128, [0, 100]), (1, 129, 256, 256, 64, [7]),
                                            (3, 8, 4096, 512, 128, [5, 0, 60])])
def test_append_project_vs_oracle(B, T, d, D, dI, pos):
    """kv = H W_KV in fp32 on the tensor cores, FP4-quantised in the epilogue,
    against the oracle's correctly rounded projection.  The tensor core's
    accumulation order is its own, so a byte may differ only where the exact
    value lies within the fp32 accumulation bound of a rounding boundary:
    every differing scale byte or code must be one whose decision changes
    inside [exact - eps, exact + eps] (eps = (d/16 + 16) x 2^-22 x sum |h w|),
    and such values must be rare.  Indexer keys follow from the stored bytes
    bit-exactly."""
    g = gen(d + D + T)
    cap = 512
    H = torch.randn(B, T, d, generator=g).to(torch.bfloat16)
    Wkv = (torch.randn(d, D, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    Wik = (torch.randn(D, dI, generator=g) / math.sqrt(D)).to(torch.bfloat16)
    pos0 = np.array(pos, np.int32)
    gm = C.MainCache(B, cap, D, dI, 1)
    C.csa2_append_project(gm, H.cuda(), Wkv.cuda(), Wik.cuda(), torch.from_numpy(pos0).cuda())
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    om = oracle.MainCache(B, cap, D, dI, 1)
    oracle.append_project(om, bits(H), bits(Wkv), bits(Wik), pos0, T)
    np.testing.assert_array_equal(gm.n_entries.cpu().numpy(), pos0 + T)
    codes, scales = gm.codes.cpu().numpy(), gm.scales.cpu().numpy()
    ik, iks = gm.ik.cpu().numpy(), gm.ik_scale.cpu().numpy()
    Hd, Wd = H.double().numpy(), Wkv.double().numpy()
    n_diff = n_vals = 0
    for b in range(B):
        rows = slice(pos0[b], pos0[b] + T)
        exact = Hd[b] @ Wd
        eps = (d / 16 + 16) * 2.0 ** -22 * (np.abs(Hd[b]) @ np.abs(Wd))
        shrink = np.where(exact >= 0, np.maximum(exact - eps, 0), np.minimum(exact + eps, 0))
        grow = np.where(exact >= 0, exact + eps, exact - eps)
        s_lo, s_hi = _decisions(shrink, D)[0], _decisions(grow, D)[0]
        gs, os_ = scales[b, rows], om.scales[b, rows]
        gc, oc = _unpack(codes[b, rows]), _unpack(om.codes[b, rows])
        # a scale byte differs only where the group's decision moves within the bound
        sdiff = gs != os_
        assert np.all(s_lo[sdiff] != s_hi[sdiff]), "a scale byte differs away from a rounding boundary"
        # with equal scales, a code differs only where its decision moves within the bound
        same_s = np.repeat(~sdiff, 16, axis=1)
        cdiff = (gc != oc) & same_s
        lo_c, hi_c = _codes_with(exact - eps, os_, D), _codes_with(exact + eps, os_, D)
        assert np.all((lo_c != hi_c)[cdiff]), "a code differs away from a rounding boundary"
        n_diff += int((gc != oc).sum()) + 16 * int(sdiff.sum())
        n_vals += gc.size
        # indexer keys: from the stored bytes, exactly as the oracle forms them
        same = (gc == oc).reshape(T, D // 16, 16).all(axis=2) & ~sdiff
        for t in range(T):
            e = pos0[b] + t
            if same[t].all():
                ref_ik, ref_s = om.ik[b, e], om.ik_scale[b, e]
            else:
                ref_ik, ref_s = oracle.index_key(codes[b, e], scales[b, e], bits(Wik))
            np.testing.assert_array_equal(ik[b, e], ref_ik)
            assert iks[b, e].view(np.uint32) == np.float32(ref_s).view(np.uint32)
    assert n_diff <= 0.01 * n_vals, f"{n_diff} of {n_vals} values differ from the oracle's"
    # entries outside the appended range are untouched
    for b in range(B):
        assert not codes[b, :pos0[b]].any() and not codes[b, pos0[b] + T:].any()


# ------------------------------------------------------------------ A4 Top-K


def _ref_topk_rows(s, n_valid, K):
    return np.stack([oracle.topk(s[r, :n_valid[r]].astype(np.float64), K) for r in range(s.shape[0])])


@pytest.mark.parametrize("B,n,T_q,m,K,P,mode", [(8, 20000, 1, 1, 512, 2048, "plain"),
                                                 (4, 65536, 1, 1, 512, 2048, "prepared"),
                                                 (2, 131072, 1, 1, 512, 2048, "plain"),
                                                 (1, 9000, 8, 2, 512, 0, "plain"),
                                                 (2, 3000, 4, 1, 512, 256, "plain"),
                                                 (3, 500, 1, 1, 512, 2048, "plain"),
                                                 (2, 12000, 1, 1, 100, 64, "constant")])
def test_index_topk_equals_scan_then_topk(B, n, T_q, m, K, P, mode):
    """csa2_index_topk (block maxima from the scan's epilogue, selection from
    them) gives bit for bit the scores, n_valid, Top-K and pool of
    csa2_index_full followed by csa2_topk -- on ordinary rows, on a short
    context (fewer blocks than K), with several query rows per sequence, and
    on a cache of identical entries (every block ties: the whole-row path)."""
    D, dI, H_I = 256, 128, 64
    cap = (n // m + 127) // 128 * 128
    g = gen(n + K + T_q)
    gm = C.MainCache(B, cap, D, dI, m)
    if mode == "constant":
        kv = torch.randn(1, 1, D, generator=g).to(torch.bfloat16).expand(B, n, D).contiguous()
    else:
        kv = torch.randn(B, n, D, generator=g).to(torch.bfloat16)
    gate = torch.randn(B, n, D, generator=g).to(torch.bfloat16) if m == 2 else None
    W = (torch.randn(D, dI, generator=g) / math.sqrt(D)).to(torch.bfloat16)
    C.csa2_append_quant(gm, kv.cuda(), gate.cuda() if gate is not None else None, W.cuda(), None, None,
                        torch.zeros(B, dtype=torch.int32).cuda(), n)
    qi = torch.randn(B, T_q, H_I, dI, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(B, T_q, H_I, generator=g).cuda()
    qpos = torch.tensor(np.stack([np.arange(n - T_q, n) - 3 * b for b in range(B)]), dtype=torch.int32).cuda()
    rows = B * T_q
    s1 = torch.full((rows, cap), float("nan"), device="cuda")
    nv1 = torch.empty(rows, dtype=torch.int32, device="cuda")
    i1 = torch.empty(rows, K, dtype=torch.int32, device="cuda")
    p1 = torch.empty(rows, max(P, 1), dtype=torch.int32, device="cuda")
    C.csa2_index_full(gm, qi, w, qpos, s1, nv1)
    wst = C.workspace(C.csa2_topk_workspace_size(rows, cap, K, P))
    C.csa2_topk(s1, cap, K, i1, n_valid=nv1, P_out=P, out_pool=p1 if P else None, ws=wst)
    s2 = torch.full((rows, cap), float("nan"), device="cuda")
    nv2 = torch.empty(rows, dtype=torch.int32, device="cuda")
    i2 = torch.full((rows, K), -7, dtype=torch.int32, device="cuda")
    p2 = torch.full((rows, max(P, 1)), -7, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_index_topk_workspace_size(rows, cap, dI))
    if mode == "prepared":
        C.csa2_append_quant_ex(gm, None, None, None, None, None, torch.full((B,), n, dtype=torch.int32).cuda(), 0,
                               qi, w, ws)
        C.csa2_index_topk(gm, None, None, qpos, s2, K, i2, n_valid=nv2, P_out=P, out_pool=p2 if P else None, ws=ws)
    else:
        C.csa2_index_topk(gm, qi, w, qpos, s2, K, i2, n_valid=nv2, P_out=P, out_pool=p2 if P else None, ws=ws)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    assert torch.equal(nv1, nv2)
    for r in range(rows):
        k = int(nv1[r])
        assert torch.equal(s1[r, :k].view(torch.int32), s2[r, :k].view(torch.int32))
    assert torch.equal(i1, i2)
    if P:
        assert torch.equal(p1, p2)


@pytest.mark.parametrize("rows,n,K,P,levels", [(3, 4096, 64, 2048, None), (2, 65536, 512, 2048, None),
                                               (4, 20000, 512, 2048, 50), (2, 300, 512, 2048, None),
                                               (1, 262144, 512, 2048, None), (2, 9000, 2048, 0, 3),
                                               (2, 70000, 17, 64, None)])
def test_topk_exact_on_same_scores(rows, n, K, P, levels):
    rng = np.random.default_rng(rows * n + K)
    s = rng.standard_normal((rows, n)).astype(np.float32)
    if levels:
        s = (np.round(s * levels) / levels).astype(np.float32)
    s[:, rng.choice(n, n // 20, replace=False)] = -np.inf
    s[0, 5] = np.nan
    s[0, 6] = np.inf
    n_valid = np.array([n - 7 * r for r in range(rows)], np.int32)
    ld = n + 32
    sd = torch.full((rows, ld), 12345.0)
    sd[:, :n] = torch.from_numpy(s)
    out = torch.empty(rows, K, dtype=torch.int32, device="cuda")
    pool = torch.empty(rows, max(P, 1), dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_topk_workspace_size(rows, n, K, P))
    C.csa2_topk(sd.cuda(), n, K, out, n_valid=torch.from_numpy(n_valid).cuda(), P_out=P,
                out_pool=pool if P else None, ws=ws)
    torch.cuda.synchronize()
    ref = _ref_topk_rows(s, n_valid, K)
    np.testing.assert_array_equal(out.cpu().numpy(), ref)
    if P:
        refp = np.stack([oracle.block_pool(s[r, :n_valid[r]].astype(np.float64), P) for r in range(rows)])
        np.testing.assert_array_equal(pool.cpu().numpy(), refp)


def _hard_scores(kind, rows, n, rng):
    s = rng.standard_normal((rows, n)).astype(np.float32)
    if kind == "outlier":            # one huge score: every other score shares the first value bin
        s[:, n // 3] = 1e30
    elif kind == "constant":         # a single value: ties decided by column only
        s[:] = 0.75
    elif kind == "huge_range":       # the value range overflows binary32
        s[:, 1] = -3e38
        s[:, 2] = 3e38
    elif kind == "two_clusters":     # two narrow groups far apart, the K-th inside the upper one
        s = np.where(rng.random((rows, n)) < 0.02, 1000.0 + 1e-3 * s, 1e-3 * s).astype(np.float32)
    elif kind == "tiny":             # subnormal and tiny normal magnitudes
        s = (s * np.float32(1e-39)).astype(np.float32)
    elif kind == "few_values":       # 5 distinct values, many ties at the K-th
        s = np.round(s).astype(np.float32)
    return s


@pytest.mark.parametrize("kind", ["outlier", "constant", "huge_range", "two_clusters", "tiny", "few_values"])
@pytest.mark.parametrize("n", [65536, 20000])
def test_topk_exact_on_hard_distributions(kind, n):
    rows, K, P = 2, 512, 2048
    rng = np.random.default_rng(zlib.crc32(f"{kind}/{n}".encode()))
    s = _hard_scores(kind, rows, n, rng)
    s[1, rng.choice(n, n // 10, replace=False)] = -np.inf
    n_valid = np.array([n, n - 5], np.int32)
    out = torch.empty(rows, K, dtype=torch.int32, device="cuda")
    pool = torch.empty(rows, P, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_topk_workspace_size(rows, n, K, P))
    C.csa2_topk(torch.from_numpy(s).cuda(), n, K, out, n_valid=torch.from_numpy(n_valid).cuda(), P_out=P,
                out_pool=pool, ws=ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), _ref_topk_rows(s, n_valid, K))
    refp = np.stack([oracle.block_pool(s[r, :n_valid[r]].astype(np.float64), P) for r in range(rows)])
    np.testing.assert_array_equal(pool.cpu().numpy(), refp)


@pytest.mark.parametrize("kind,n,P", [("normal", 65536, 2048), ("few_values", 40000, 2048), ("normal", 30001, 0)])
def test_topk_cluster_rows_past_one_wave(kind, n, P):
    """Rows of at most 65,536 columns go through one 8-block thread-block
    cluster per row; 160 rows run as several waves of clusters, exact against
    the oracle with ragged n_valid, absent scores and empty rows."""
    rows, K = 160, 512
    rng = np.random.default_rng(zlib.crc32(f"wave/{kind}/{n}".encode()))
    s = rng.standard_normal((rows, n)).astype(np.float32) if kind == "normal" else _hard_scores(kind, rows, n, rng)
    s[3, rng.choice(n, n // 10, replace=False)] = -np.inf
    n_valid = rng.integers(n // 2, n + 1, rows).astype(np.int32)
    n_valid[5], n_valid[6] = 100, 0
    out = torch.empty(rows, K, dtype=torch.int32, device="cuda")
    pool = torch.empty(rows, max(P, 1), dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_topk_workspace_size(rows, n, K, P))
    C.csa2_topk(torch.from_numpy(s).cuda(), n, K, out, n_valid=torch.from_numpy(n_valid).cuda(), P_out=P,
                out_pool=pool if P else None, ws=ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), _ref_topk_rows(s, n_valid, K))
    if P:
        refp = np.stack([oracle.block_pool(s[r, :n_valid[r]].astype(np.float64), P) for r in range(rows)])
        np.testing.assert_array_equal(pool.cpu().numpy(), refp)
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("kind", ["normal", "outlier", "constant", "huge_range", "two_clusters", "tiny", "few_values"])
@pytest.mark.parametrize("pad", [3, 0])
def test_topk_many_long_rows(kind, pad):
    """128 or more rows of more than 65,536 columns (prefill chunks) take the
    one-block-per-row kernel, which needs no workspace: exact against the
    oracle with ragged n_valid, absent scores, rows shorter than K or empty,
    and a row pitch that is (pad 3: 70,004) or is not (pad 0: 70,001) a
    multiple of 4."""
    rows, n, K = 136, 70001, 512
    ld = n + pad
    rng = np.random.default_rng(zlib.crc32(f"rows/{kind}/{pad}".encode()))
    s = rng.standard_normal((rows, n)).astype(np.float32) if kind == "normal" else _hard_scores(kind, rows, n, rng)
    s[1, rng.choice(n, n // 10, replace=False)] = -np.inf
    n_valid = rng.integers(n // 2, n + 1, rows).astype(np.int32)
    n_valid[2], n_valid[3], n_valid[4] = 300, 0, n
    buf = np.full((rows, ld), np.nan, np.float32)
    buf[:, :n] = s
    assert C.csa2_topk_workspace_size(rows, n, K, 0) == 0
    out = torch.empty(rows, K, dtype=torch.int32, device="cuda")
    C.csa2_topk(torch.from_numpy(buf).cuda(), n, K, out, n_valid=torch.from_numpy(n_valid).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), _ref_topk_rows(s, n_valid, K))
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("rows,n,K", [(128, 131072, 2048), (200, 65537, 1), (128, 100000, 2000)])
def test_topk_many_long_rows_extremes(rows, n, K):
    rng = np.random.default_rng(zlib.crc32(f"rowsx/{rows}/{n}/{K}".encode()))
    s = rng.standard_normal((rows, n)).astype(np.float32)
    s[:, : n // 7] = np.round(s[:, : n // 7] * 4) / 4   # a tied stretch
    n_valid = np.full(rows, n, np.int32)
    out = torch.empty(rows, K, dtype=torch.int32, device="cuda")
    C.csa2_topk(torch.from_numpy(s).cuda(), n, K, out, n_valid=torch.from_numpy(n_valid).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), _ref_topk_rows(s, n_valid, K))


def test_topk_pool_mapping_for_reindex_rows():
    rows, P, K = 3, 64, 40
    rng = np.random.default_rng(11)
    pool = np.sort(rng.choice(5000, size=(rows, P), replace=False), axis=1).astype(np.int32)
    pool[2, 50:] = -1
    s = rng.standard_normal((rows, P * 8)).astype(np.float32)
    s[2, 400:] = -np.inf
    out = torch.empty(rows, K, dtype=torch.int32, device="cuda")
    ws = C.workspace(C.csa2_topk_workspace_size(rows, P * 8, K, 0))
    C.csa2_topk(torch.from_numpy(s).cuda(), P * 8, K, out, pool_blocks=torch.from_numpy(pool).cuda(), ws=ws)
    torch.cuda.synchronize()
    for r in range(rows):
        cols = oracle.topk(s[r].astype(np.float64), K)
        np.testing.assert_array_equal(out[r].cpu().numpy(), oracle.columns_to_entries(cols, pool[r]))


# ------------------------------------------------------------------ A6 Reindex


def test_index_reindex_vs_oracle():
    B, D, dI, H_I, n = 2, 512, 128, 64, 5000
    cap = 5120
    gm, _, om, _, _ = build_pair(B=B, cap=cap, D=D, dI=dI, m=1, T=n, pos0=[0, 0], seed=21, swa=False)
    rng = np.random.default_rng(22)
    P = 256
    pool = np.stack([np.sort(rng.choice(cap // 8, P, replace=False)) for _ in range(B)]).astype(np.int32)
    pool[1, -10:] = -1
    q, w = _rows_queries(B, 1, H_I, dI, seed=23)
    qpos = np.array([[n - 1], [n - 400]], np.int32)
    out = torch.empty(B, P * 8, device="cuda")
    C.csa2_index_reindex(gm, q.cuda(), w.cuda(), torch.from_numpy(qpos).cuda(), torch.from_numpy(pool).cuda(), out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for b in range(B):
        n_vis = oracle.n_visible(int(om.n_entries[b]), int(qpos[b, 0]), 1)
        ref = oracle.reindex_scores(om, b, bits(q[b, 0]), w[b, 0].numpy(), n_vis, pool[b])
        fin = np.isfinite(ref)
        assert np.array_equal(np.isfinite(got[b]), fin)
        _check_scores(got[b][fin], ref[fin])


# ------------------------------------------------------------------ A5 attention


def _check_attn(got_bf16, ref_bits):
    ref = oracle.bf16_to_f32(ref_bits).astype(np.float64)
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    print(f"attention error: max {err.max() / np.abs(ref).max():.2e} of max|ref|, "
          f"mean rel {err.sum() / np.abs(ref).sum():.2e}")
    assert err.max() <= 1e-2 * np.abs(ref).max(), f"max err {err.max()} vs {np.abs(ref).max()}"
    assert err.sum() <= 1e-3 * np.abs(ref).sum(), f"mean rel err {err.sum() / np.abs(ref).sum()}"


@pytest.mark.parametrize("D,H,K,T_q,window,W_cap,use_ws", [(512, 64, 512, 1, 128, 128, True),
                                                           (512, 64, 512, 1, 128, 128, False),
                                                           (128, 8, 64, 1, 128, 128, True),
                                                           (256, 19, 100, 3, 128, 200, True),
                                                           (512, 64, 512, 5, 128, 256, False)])
def test_attention_vs_oracle(D, H, K, T_q, window, W_cap, use_ws):
    B, n = 2, 1500
    cap = 1536
    gm, gs, om, osw, _ = build_pair(B=B, cap=cap, D=D, dI=64, m=1, T=n, pos0=[0, 0], seed=D + H, W_cap=W_cap,
                                    s_swa=0.75, window=window)
    g = gen(31)
    q = torch.randn(B, T_q, H, D, generator=g).to(torch.bfloat16)
    qpos = np.stack([np.arange(n - T_q, n) for _ in range(B)]).astype(np.int32)
    qpos[0, 0] = 60   # window shorter than 128
    idx = torch.stack([torch.stack([I.random_indices(int(qpos[b, j]) + 1, K, g, n_missing=(b + j) % 5)
                                    for j in range(T_q)]) for b in range(B)])
    out = torch.empty(B, T_q, H, D, dtype=torch.bfloat16, device="cuda")
    ws = C.workspace(C.csa2_attn_workspace_size(B, T_q, H, D, K, window)) if use_ws else None
    scale = 1 / math.sqrt(D)
    C.csa2_sparse_attn_decode(gm, gs, q.cuda(), torch.from_numpy(qpos).cuda(), idx.cuda(), scale, out, ws=ws)
    torch.cuda.synchronize()
    for b in range(B):
        for j in range(T_q):
            ref = oracle.attention(om, osw, b, bits(q[b, j]), idx[b, j].numpy(), int(qpos[b, j]), scale)
            _check_attn(out[b, j], ref)
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("B,T_q", [(8, 4), (16, 4), (40, 4)])
def test_attention_multi_tile_splits(B, T_q):
    """Row counts where the launch plan gives splits of several key tiles
    each (32 rows: 3 splits of 2 tiles; 64 rows: 2 splits of 3; 160 rows:
    one block per row over all 5 tiles): sampled rows against the oracle."""
    D, H, K, n, cap = 512, 64, 512, 2000, 2048
    gm, gs, om, osw, _ = build_pair(B=B, cap=cap, D=D, dI=64, m=1, T=n, pos0=[0] * B, seed=77 + B, s_swa=0.5)
    g = gen(78)
    q = torch.randn(B, T_q, H, D, generator=g).to(torch.bfloat16)
    qpos = np.stack([np.arange(n - T_q, n) for _ in range(B)]).astype(np.int32)
    idx = torch.stack([torch.stack([I.random_indices(int(qpos[b, j]) + 1, K, g, n_missing=(b + j) % 3)
                                    for j in range(T_q)]) for b in range(B)])
    out = torch.empty(B, T_q, H, D, dtype=torch.bfloat16, device="cuda")
    ws = C.workspace(C.csa2_attn_workspace_size(B, T_q, H, D, K, 128))
    scale = 1 / math.sqrt(D)
    C.csa2_sparse_attn_decode(gm, gs, q.cuda(), torch.from_numpy(qpos).cuda(), idx.cuda(), scale, out, ws=ws)
    torch.cuda.synchronize()
    for b, j in [(0, 0), (B // 2, 1), (B - 1, T_q - 1)]:
        ref = oracle.attention(om, osw, b, bits(q[b, j]), idx[b, j].numpy(), int(qpos[b, j]), scale)
        _check_attn(out[b, j], ref)
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("D,H,K,window,scale_mul,use_ws", [(512, 64, 512, 128, 1.0, True),
                                                           (512, 64, 100, 128, 64.0, True),
                                                           (256, 17, 300, 200, 1.0, True),
                                                           (128, 8, 512, 64, 32.0, False),
                                                           (512, 64, 0, 128, 1.0, True)])
def test_attention_many_waves(D, H, K, window, scale_mul, use_ws):
    """200 query rows: more blocks than SMs, so the launch takes the
    pipelined form (64-key tiles in two buffers).  Large softmax scales make
    the reference max move between tiles (the in-TMEM rescale path); K = 100
    leaves a ragged last tile; no workspace gives one split per row."""
    B, T_q, n, cap = 50, 4, 900, 1024
    gm, gs, om, osw, _ = build_pair(B=B, cap=cap, D=D, dI=64, m=1, T=n, pos0=[0] * B, seed=D + K + 3, s_swa=0.5,
                                    window=window, W_cap=max(window, 128))
    g = gen(K + 5)
    q = torch.randn(B, T_q, H, D, generator=g).to(torch.bfloat16)
    qpos = np.stack([np.arange(n - T_q, n) for _ in range(B)]).astype(np.int32)
    qpos[1, 2] = 30   # fewer rows than the window
    if K > 0:
        idx = torch.stack([torch.stack([I.random_indices(int(qpos[b, j]) + 1, K, g, n_missing=(b + j) % 3)
                                        for j in range(T_q)]) for b in range(B)])
        idx_d = idx.cuda()
    else:
        idx, idx_d = None, None
    out = torch.empty(B, T_q, H, D, dtype=torch.bfloat16, device="cuda")
    ws = C.workspace(C.csa2_attn_workspace_size(B, T_q, H, D, K, window)) if use_ws else None
    scale = scale_mul / math.sqrt(D)
    C.csa2_sparse_attn_decode(gm, gs, q.cuda(), torch.from_numpy(qpos).cuda(), idx_d, scale, out, ws=ws)
    torch.cuda.synchronize()
    for b, j in [(0, 0), (1, 2), (B // 2, 1), (B - 1, T_q - 1)]:
        sel = idx[b, j].numpy() if K > 0 else np.zeros(0, np.int32)
        ref = oracle.attention(om, osw, b, bits(q[b, j]), sel, int(qpos[b, j]), scale)
        _check_attn(out[b, j], ref)
    assert C.csa2_device_status() == 0


@pytest.mark.parametrize("D,H,B,T_q,window,W_cap,use_ws", [(512, 64, 2, 1, 128, 128, True),
                                                           (512, 64, 8, 1, 128, 128, False),
                                                           (256, 17, 3, 4, 128, 200, True),
                                                           (128, 8, 1, 2, 64, 160, True)])
def test_window_only_attention(D, H, B, T_q, window, W_cap, use_ws):
    """K = 0: the SWA-only layers of the encoder (jaehun review, "새로운 접근법"
    and its flowchart: layers 1-2 use sliding-window attention only) -- a
    softmax over the window rows alone, no index array."""
    n = 700
    gm, gs, om, osw, _ = build_pair(B=B, cap=768, D=D, dI=64, m=1, T=n, pos0=[0] * B, seed=D + 7 * H, W_cap=W_cap,
                                    s_swa=0.5, window=window)
    g = gen(55)
    q = torch.randn(B, T_q, H, D, generator=g).to(torch.bfloat16)
    qpos = np.stack([np.arange(n - T_q, n) for _ in range(B)]).astype(np.int32)
    qpos[0, 0] = 40   # fewer rows than the window
    out = torch.empty(B, T_q, H, D, dtype=torch.bfloat16, device="cuda")
    ws = C.workspace(C.csa2_attn_workspace_size(B, T_q, H, D, 0, window)) if use_ws else None
    scale = 1 / math.sqrt(D)
    C.csa2_sparse_attn_decode(gm, gs, q.cuda(), torch.from_numpy(qpos).cuda(), None, scale, out, ws=ws)
    torch.cuda.synchronize()
    none = np.zeros(0, np.int32)
    for b in range(B):
        for j in range(T_q):
            ref = oracle.attention(om, osw, b, bits(q[b, j]), none, int(qpos[b, j]), scale)
            _check_attn(out[b, j], ref)
    assert C.csa2_device_status() == 0


def test_attention_out_of_range_index_is_masked_and_flagged():
    B, D, n, cap, K = 1, 128, 300, 384, 16
    gm, gs, om, osw, _ = build_pair(B=B, cap=cap, D=D, dI=64, m=1, T=n, pos0=[0], seed=41)
    g = gen(42)
    q = torch.randn(B, 1, 8, D, generator=g).to(torch.bfloat16)
    idx = torch.arange(K, dtype=torch.int32).view(1, 1, K) * 7
    idx[0, 0, 3] = cap + 5          # out of the cache: masked, flagged
    out = torch.empty(B, 1, 8, D, dtype=torch.bfloat16, device="cuda")
    C.csa2_sparse_attn_decode(gm, gs, q.cuda(), torch.tensor([[n - 1]], dtype=torch.int32).cuda(), idx.cuda(),
                              0.1, out)
    torch.cuda.synchronize()
    assert C.csa2_device_status() & C.DEV_INDEX_RANGE
    ref = oracle.attention(om, osw, 0, bits(q[0, 0]), idx[0, 0].numpy(), n - 1, 0.1)
    _check_attn(out[0, 0], ref)


# ------------------------------------------------------------------ whole steps


def _oracle_decode_chain(st, b, layer_q_idx, layer_w):
    """Oracle cache, scores, Top-K of one sequence of a runner.Step."""
    wl = st.wl
    om = oracle.MainCache(1, st.cap, wl.D, wl.dI, wl.m)
    oracle.append(om, bits(st._kv_ctx[b])[None], None, bits(st.w_ik), None, None, np.zeros(1, np.int32),
                  wl.total_tokens)
    t = wl.total_tokens - 1
    n_vis = oracle.n_visible(int(om.n_entries[0]), t, wl.m)
    sc = oracle.index_scores(om, 0, bits(layer_q_idx[b, 0]), layer_w[b, 0].cpu().numpy(), n_vis)
    return om, sc, t


def _band_ok(sel_gpu, sel_ref, scores, K):
    fin = scores[np.isfinite(scores)]
    kth = np.sort(fin)[-K] if fin.size >= K else -np.inf
    diff = set(sel_gpu.tolist()) ^ set(sel_ref.tolist())
    diff.discard(-1)
    return all(abs(scores[i] - kth) <= BAND * abs(kth) for i in diff), len(diff)


def test_tiny_step_end_to_end():
    from fp4_kv_cache_append_b200 import runner
    wl = I.WORKLOADS["tiny"]
    st = runner.Step(wl, seed=0)
    st.prefill()
    st.run()
    torch.cuda.synchronize()
    b = 0
    om, sc, t = _oracle_decode_chain(st, b, st.q_idx[0], st.w[0])
    for name in ("codes", "scales", "ik"):
        np.testing.assert_array_equal(getattr(st.main[0], name)[b].cpu().numpy(), getattr(om, name)[0])
    gsc = st.scores[b, :wl.entries].cpu().numpy()
    _check_scores(gsc, sc)
    top = oracle.topk(sc, wl.K)
    got = st.idx[b].cpu().numpy()
    ok, nd = _band_ok(got, top, sc, wl.K)
    assert ok, "Top-K differs outside the tie band"
    planted = I.planted_positions(wl, 0, b).numpy()
    assert set(planted.tolist()) <= set(got.tolist())
    pool = st.pool[b].cpu().numpy()
    assert set((got // 8).tolist()) <= set(pool.tolist())
    osw = oracle.SwaCache(1, st.W_cap, wl.D, window=wl.window)
    lo = I.window_lo(wl)
    oracle.append(None, None, None, None, osw, bits(st.win_rows[0][b])[None], np.array([lo], np.int32),
                  st.win_rows[0][b].shape[0])
    np.testing.assert_array_equal(st.swa[0][0].rows[b].cpu().numpy(), osw.rows[0])
    ref = oracle.attention(om, osw, 0, bits(st.q[0][b, 0]), got, t, st.scale)
    _check_attn(st.out[0][b, 0], ref)
