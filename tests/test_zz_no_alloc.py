"""csa2_topk_noalloc -- Top-K for callers that cannot allocate device memory
when they call the library (a plugin whose memory belongs to a host
framework, a serving path that must not allocate) -- gives the same result as
csa2_topk with a caller workspace.  Both are called through the C ABI, twice
in a row with different inputs, so a call also runs on the scratch contents
the previous one left behind.  Runs alone in a fresh process or after the
rest of the suite (this file is collected last)."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_append_b200 import csa2 as C

pytestmark = pytest.mark.gpu


def _scores(rows, n, seed, levels=None):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((rows, n)).astype(np.float32)
    if levels:
        s = (np.round(s * levels) / levels).astype(np.float32)   # many exact ties
    s[:, rng.choice(n, n // 16, replace=False)] = -np.inf
    n_valid = np.array([n - 3 * r for r in range(rows)], np.int32)
    return torch.from_numpy(s).cuda(), torch.from_numpy(n_valid).cuda()


def test_topk_noalloc_matches_topk_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    cases = [(8, 65536, 512, 2048, None, 1), (5, 20000, 100, 256, 7, 2), (2, 100000, 512, 2048, 5, 3)]
    for rows, n, K, P, levels, seed in cases:
        s, nv = _scores(rows, n, seed, levels)
        ref_i = torch.empty(rows, K, dtype=torch.int32, device="cuda")
        ref_p = torch.empty(rows, P, dtype=torch.int32, device="cuda")
        ws = C.workspace(C.csa2_topk_workspace_size(rows, n, K, P))
        C.csa2_topk(s, n, K, ref_i, n_valid=nv, P_out=P, out_pool=ref_p, ws=ws)
        got_i = torch.full((rows, K), -7, dtype=torch.int32, device="cuda")
        got_p = torch.full((rows, P), -7, dtype=torch.int32, device="cuda")
        C.csa2_topk_noalloc(s, n, K, got_i, n_valid=nv, P_out=P, out_pool=got_p)
        torch.cuda.synchronize()
        # integer outputs: the tolerance is exact equality
        assert torch.equal(got_i, ref_i)
        assert torch.equal(got_p, ref_p)


def test_topk_noalloc_rejects_more_than_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rows, n, K = 64, 1 << 20, 512       # rows over 65,536 columns need scratch; these 256 MiB
    assert C.csa2_topk_workspace_size(rows, n, K, 0) > (4 << 20)
    s = torch.zeros(16, dtype=torch.float32, device="cuda")
    out = torch.zeros(rows, K, dtype=torch.int32, device="cuda")
    with pytest.raises(C.Csa2Error) as ei:
        C.lib()
        st = C.lib().csa2_topk_noalloc(s.data_ptr(), rows, n, n, None, None, K, out.data_ptr(), 0, None,
                                       torch.cuda.current_stream().cuda_stream)
        C._check(st)
    assert ei.value.status == 5 and "scratch" in str(ei.value)
