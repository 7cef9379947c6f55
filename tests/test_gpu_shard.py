"""The context-sharded decode step on one GPU: every rank's phases run in one
process (fp4_kv_cache_append_b200.shard.step_emulated: the all-gather is a
concatenation, the reduce a byte sum) with the CUDA kernels -- the fused scan +
selection per shard (csa2_index_topk with selected scores), the merge
(csa2_topk_merge), the copies of the selected entries (csa2_gather_entries)
and the owner's attention.  The result must equal, bit for bit, the unsharded
step on one cache holding the whole context: the selection is exact and the
attention sees the same entries in the same order."""
import math

import numpy as np
import pytest
import torch

from fp4_kv_cache_append_b200 import csa2 as C
from fp4_kv_cache_append_b200 import shard as S

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,n,world,K,P", [(2, 50000, 3, 512, 2048), (1, 9000, 2, 100, 64), (3, 4000, 4, 512, 256)])
def test_sharded_step_equals_unsharded(B, n, world, K, P):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    D, dI, H, H_I, W = 512, 128, 64, 64, 128
    g = torch.Generator().manual_seed(n + world)
    kv = torch.randn(B, n, D, generator=g).to(torch.bfloat16).cuda()
    Wik = (torch.randn(D, dI, generator=g) / math.sqrt(D)).to(torch.bfloat16).cuda()
    win = torch.randn(B, W, D, generator=g).to(torch.bfloat16).cuda()
    qi = torch.randn(B, 1, H_I, dI, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(B, 1, H_I, generator=g).cuda()
    q = torch.randn(B, 1, H, D, generator=g).to(torch.bfloat16).cuda()
    q_pos = torch.full((B, 1), n - 1, dtype=torch.int32).cuda()
    zero = torch.zeros(B, dtype=torch.int32).cuda()
    swa = C.SwaCache(B, W, D, window=W)
    C.csa2_append_quant(None, None, None, None, swa, win, torch.full((B,), n - W, dtype=torch.int32).cuda(), W)
    scale = 1 / math.sqrt(D)

    # unsharded
    cap = (n + 127) // 128 * 128
    full = C.MainCache(B, cap, D, dI, 1)
    C.csa2_append_quant(full, kv, None, Wik, None, None, zero, n)
    scores = torch.empty(B, cap, device="cuda")
    idx = torch.empty(B, K, dtype=torch.int32, device="cuda")
    pool = torch.empty(B, P, dtype=torch.int32, device="cuda")
    C.csa2_index_topk(full, qi, w, q_pos, scores, K, idx, P_out=P, out_pool=pool)
    ref = torch.empty(B, 1, H, D, dtype=torch.bfloat16, device="cuda")
    ws = C.workspace(C.csa2_attn_workspace_size(B, 1, H, D, K, W))
    C.csa2_sparse_attn_decode(full, swa, q, q_pos, idx.view(B, 1, K), scale, ref, ws=ws)

    # sharded
    ranks = []
    for lo, hi in S.shard_ranges(n, world):
        sh = C.MainCache(B, max(128, (hi - lo + 127) // 128 * 128), D, dI, 1)
        C.csa2_append_quant(sh, kv[:, lo:hi].contiguous(), None, Wik, None, None, zero, hi - lo)
        ranks.append(S.Rank(shard=sh, lo=lo))
    ranks[-1].swa, ranks[-1].q = swa, q
    out = torch.empty(B, 1, H, D, dtype=torch.bfloat16, device="cuda")
    m_idx, m_pool = S.step_emulated(ranks, S.CudaOps(K, P), qi, w, q_pos, scale, out)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    assert torch.equal(m_idx, idx)
    assert torch.equal(m_pool, pool)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
