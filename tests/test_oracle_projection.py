"""Pins for the oracle's CED decoder-KV projection (no GPU).

kv_t = H_t W_KV (jaehun review, "1) CED": the decoder's global KV is the final
encoder hidden state projected by each decoder layer's W_KV^l; the equation
itself was lost, so the plainest linear projection is the reading), the exact
sum rounded once to binary32; the projected token then becomes an FP4 entry
and its indexer key exactly as an appended token does.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from test_oracle_formats import _round_f32


def bf16_bits(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16).contiguous().view(torch.int16).numpy() \
        .view(np.uint16)


def bf16_vals(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_integer_grid_is_exact():
    """Small integers: every partial sum is an exact integer."""
    rng = np.random.default_rng(1)
    d, D = 512, 64
    H = rng.integers(-8, 9, size=d)
    W = rng.integers(-8, 9, size=(d, D))
    kv = oracle.project_kv(bf16_bits(H), bf16_bits(W))
    np.testing.assert_array_equal(kv, (H @ W).astype(np.float32))


def test_unit_row_selects_a_row_of_w():
    rng = np.random.default_rng(2)
    d, D = 256, 128
    W = bf16_bits(rng.standard_normal((d, D)))
    for i in (0, 17, d - 1):
        h = np.zeros(d)
        h[i] = 1.0
        np.testing.assert_array_equal(oracle.project_kv(bf16_bits(h), W), bf16_vals(W[i]).astype(np.float32))


@pytest.mark.parametrize("seed,d,D", [(3, 256, 16), (4, 1024, 8)])
def test_random_equals_exact_sum_rounded_once(seed, d, D):
    rng = np.random.default_rng(seed)
    H = bf16_bits(rng.standard_normal(d))
    W = bf16_bits(rng.standard_normal((d, D)) / math.sqrt(d))
    kv = oracle.project_kv(H, W)
    hv, wv = bf16_vals(H), bf16_vals(W)
    for c in range(D):
        exact = sum(Fraction(float(hv[i])) * Fraction(float(wv[i, c])) for i in range(d))
        assert float(kv[c]) == _round_f32(exact)


def test_cancellation_is_exact():
    """1 + 2^-30 - 1: a plain binary32 running sum gives 0; the exact value is 2^-30."""
    d, D = 3, 1
    H = bf16_bits([1.0, 2.0 ** -30, -1.0])
    W = bf16_bits([[1.0], [1.0], [1.0]])
    assert oracle.project_kv(H, W)[0] == np.float32(2.0 ** -30)


def test_projected_append_is_the_token_path():
    """An m = 1 cache filled by the projection holds, entry by entry, the FP4
    row and indexer key of the projected token, at positions pos0 + tau."""
    rng = np.random.default_rng(5)
    B, T, d, D, dI, cap = 2, 5, 128, 128, 64, 128
    H = bf16_bits(rng.standard_normal((B, T, d)))
    Wkv = bf16_bits(rng.standard_normal((d, D)) / math.sqrt(d))
    Wik = bf16_bits(rng.standard_normal((D, dI)) / math.sqrt(D))
    pos0 = np.array([0, 40], np.int32)
    om = oracle.MainCache(B, cap, D, dI, 1)
    oracle.append_project(om, H, Wkv, Wik, pos0, T)
    for b in range(B):
        assert om.n_entries[b] == pos0[b] + T
        for t in range(T):
            e = pos0[b] + t
            codes, scales = oracle.quant_fp4_row(oracle.project_kv(H[b, t], Wkv))
            ik, s = oracle.index_key(codes, scales, Wik)
            np.testing.assert_array_equal(om.codes[b, e], codes)
            np.testing.assert_array_equal(om.scales[b, e], scales)
            np.testing.assert_array_equal(om.ik[b, e], ik)
            assert om.ik_scale[b, e] == s
    assert not om.codes[0, T:].any() and not om.codes[1, :40].any()
