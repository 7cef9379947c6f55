"""csa2_topk_noalloc -- Top-K for callers that cannot allocate device memory
when they call the library (a plugin whose memory belongs to a host
framework, a serving path that must not allocate) -- gives the same result as
csa2_topk with a caller workspace, and the oracle's selection on the same
scores.  Both entry points are called through the C ABI, call after call with
different inputs; rows of more than 65,536 columns take the path that keeps
its scratch in the library's built-in array, so each of those calls runs on
the scratch contents the previous one left behind.  Runs alone in a fresh
process or after the rest of the suite (this file is collected last)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_append_b200 import csa2 as C

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20   # the built-in array's size (include/csa2.h, entry 6)


def _scores(rows, n, seed, levels=None):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((rows, n)).astype(np.float32)
    if levels:
        s = (np.round(s * levels) / levels).astype(np.float32)   # many exact ties
    s[:, rng.choice(n, n // 16, replace=False)] = -np.inf
    n_valid = np.array([n - 3 * r for r in range(rows)], np.int32)
    return s, n_valid


def _oracle_rows(s, n_valid, K, P):
    """The oracle's Top-K and block pool of each row over its valid columns."""
    idx = np.stack([oracle.topk(s[r, :n_valid[r]].astype(np.float64), K) for r in range(s.shape[0])])
    pool = np.stack([oracle.block_pool(s[r, :n_valid[r]].astype(np.float64), P) for r in range(s.shape[0])]) \
        if P else None
    return idx, pool


# (rows, n_cols, K, P_out, tie levels, seed); the first two fit the one-launch
# cluster path (no scratch), the rest use the built-in scratch, back to back
CASES = [(8, 65536, 512, 2048, None, 1), (5, 20000, 100, 256, 7, 2), (2, 100000, 512, 2048, 5, 3),
         (3, 150000, 256, 1024, 5, 4), (1, 300000, 512, 2048, None, 5), (2, 200000, 2048, 0, 3, 6)]


def test_topk_noalloc_matches_topk_and_oracle_call_after_call():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    scratch_calls = 0
    for rows, n, K, P, levels, seed in CASES:
        s_np, nv_np = _scores(rows, n, seed, levels)
        s, nv = torch.from_numpy(s_np).cuda(), torch.from_numpy(nv_np).cuda()
        need = C.csa2_topk_workspace_size(rows, n, K, P)
        assert need <= SCRATCH_BYTES
        scratch_calls += need > 0
        ref_i = torch.empty(rows, K, dtype=torch.int32, device="cuda")
        ref_p = torch.empty(rows, max(P, 1), dtype=torch.int32, device="cuda")
        ws = C.workspace(need)
        C.csa2_topk(s, n, K, ref_i, n_valid=nv, P_out=P, out_pool=ref_p if P else None, ws=ws)
        got_i = torch.full((rows, K), -7, dtype=torch.int32, device="cuda")
        got_p = torch.full((rows, max(P, 1)), -7, dtype=torch.int32, device="cuda")
        C.csa2_topk_noalloc(s, n, K, got_i, n_valid=nv, P_out=P, out_pool=got_p if P else None)
        torch.cuda.synchronize()
        # integer outputs of identical fp32 scores: the tolerance is exact equality
        assert torch.equal(got_i, ref_i)
        o_i, o_p = _oracle_rows(s_np, nv_np, K, P)
        np.testing.assert_array_equal(got_i.cpu().numpy(), o_i)
        if P:
            assert torch.equal(got_p, ref_p)
            np.testing.assert_array_equal(got_p.cpu().numpy(), o_p)
        assert C.csa2_device_status() == 0
    assert scratch_calls >= 3


def test_topk_noalloc_rejects_more_than_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rows, n, K = 64, 1 << 20, 512       # rows over 65,536 columns need scratch; these 256 MiB
    assert C.csa2_topk_workspace_size(rows, n, K, 0) > SCRATCH_BYTES
    s = torch.zeros(16, dtype=torch.float32, device="cuda")
    out = torch.zeros(rows, K, dtype=torch.int32, device="cuda")
    with pytest.raises(C.Csa2Error) as ei:
        st = C.lib().csa2_topk_noalloc(s.data_ptr(), rows, n, n, None, None, K, out.data_ptr(), 0, None,
                                       torch.cuda.current_stream().cuda_stream)
        C._check(st)
    assert ei.value.status == 5 and "scratch" in str(ei.value)
