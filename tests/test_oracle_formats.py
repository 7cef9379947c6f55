"""Pins for the oracle's number formats and codecs (no GPU).

Each test checks the oracle against something other than itself: hand-worked
vectors in tests/golden (cited there), torch's own float8 E4M3 codec, exact
rational arithmetic, or closed-form properties of the definitions.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def bf16_exact(x):
    return float(torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).float()) == x or x == 0


# ---------------------------------------------------------------- E2M1 / E4M3


def test_e2m1_table():
    for line in read_golden("e2m1_table.txt"):
        code, val = line.split()
        v = oracle.e2m1_value(int(code))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))


def test_e4m3_decode_matches_torch_all_bytes():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for b in range(256):
        v = oracle.e4m3_value(b)
        if math.isnan(ref[b]):
            assert math.isnan(v), hex(b)
        else:
            assert v == ref[b], hex(b)


def test_e4m3_encode_hand_vectors():
    for line in read_golden("e4m3_encode.txt"):
        val, byte = line.split()
        got = int(oracle.e4m3_encode(np.float32(float(val))))
        assert got == int(byte, 16), (val, hex(got), byte)


def test_e4m3_encode_matches_torch_on_every_bf16_in_range():
    # torch rounds to nearest even and returns NaN (not saturation) above 464,
    # so the comparison covers |x| < 464; saturation is pinned by the hand vectors.
    allbits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    x = allbits[torch.isfinite(allbits) & (allbits.abs() < 464)]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x.numpy())
    np.testing.assert_array_equal(got, ref)


def test_e4m3_encode_midpoints_go_to_even():
    vals = [oracle.e4m3_value(c) for c in range(127)]
    mids = np.array([(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])], dtype=np.float64)
    assert np.all(mids.astype(np.float32) == mids)  # exact in binary32
    ref = torch.tensor(mids, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(mids.astype(np.float32))
    np.testing.assert_array_equal(got, ref)
    assert np.all(got % 2 == 0)


def test_e2m1_encode_hand_vectors():
    # scale 1: 0.25->0 0.75->2 1.25->2 1.75->4 2.5->4 3.5->6 5->6 6->7 7->7 -6->F
    cases = {0.25: 0x0, 0.75: 0x2, 1.25: 0x2, 1.75: 0x4, 2.5: 0x4, 3.5: 0x6, 5.0: 0x6,
             6.0: 0x7, 7.0: 0x7, -6.0: 0xF, -0.1: 0x8, 0.26: 0x1, 1e30: 0x7, 0.0: 0x0}
    for x, code in cases.items():
        assert int(oracle.e2m1_encode(np.float32(x))) == code, x


# ---------------------------------------------------------------- FP4 groups


def _golden_groups():
    lines = list(read_golden("fp4_groups.txt"))
    for i in range(0, len(lines), 3):
        g = [float(v) for v in lines[i].split(":")[1].split()]
        s = int(lines[i + 1].split(":")[1], 16)
        c = [int(v, 16) for v in lines[i + 2].split(":")[1].split()]
        yield g, s, c


@pytest.mark.parametrize("case", list(_golden_groups()))
def test_fp4_group_hand_vectors(case):
    g, s, c = case
    assert all(bf16_exact(v) for v in g)
    x = np.array(g, np.float32)
    x = np.copysign(x, np.array(g))  # keep -0
    codes, scales = oracle.quant_fp4_row(x)
    assert int(scales[0]) == s
    assert [int(v) for v in codes] == c


def test_fp4_grid_roundtrip_every_scale_and_code():
    """x = e2m1(c) * e4m3(s) with amax = 6 e4m3(s) quantises back to (s, c)."""
    for s in range(1, 127):
        sv = oracle.e4m3_value(s)
        x = np.array([oracle.e2m1_value(c) * sv for c in range(16)], np.float64)
        x[0] = 6 * sv  # amax
        x = x.astype(np.float32)
        assert np.all(x.astype(np.float64) == np.array([6 * sv] + [oracle.e2m1_value(c) * sv for c in range(1, 16)]))
        codes, scales = oracle.quant_fp4_row(x)
        assert scales[0] == s
        got = [(codes[i // 2] >> (4 * (i % 2))) & 0xF for i in range(16)]
        assert got[0] == 7
        for c in range(1, 16):
            if c == 8:   # -0: sign kept
                assert got[c] == 8
            else:
                assert got[c] == c, (s, c, got[c])


def test_fp4_dequant_is_product_of_decodes():
    tab = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    e2 = [0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6]
    for s in list(range(0, 127)) + list(range(128, 255)):
        codes = np.array([c | (c << 4) for c in range(8)] * 2, np.uint8)  # 16 bytes, 32 ch
        codes[8:] = np.array([(8 + c) | ((8 + c) << 4) for c in range(8)], np.uint8)
        scales = np.array([s, s], np.uint8)
        v = oracle.fp4_dequant_row(codes, scales, 32)
        for ch in range(32):
            code = (codes[ch // 2] >> (4 * (ch % 2))) & 0xF
            assert v[ch] == e2[code] * tab[s]


# ---------------------------------------------------------------- exp and the m=2 gate


def _ulp(x):
    return float(np.spacing(np.float32(x)))


def test_exp_neg_within_two_ulp_of_exp():
    xs = np.concatenate([np.linspace(-80, 0, 40001, dtype=np.float32),
                         -np.logspace(-8, 0, 2001).astype(np.float32)])
    for x in xs:
        got = oracle.exp_neg(float(x))
        ref = math.exp(float(x))
        assert abs(got - ref) <= 2 * _ulp(ref), (x, got, ref)


def test_exp_neg_special_values():
    assert oracle.exp_neg(0.0) == 1.0
    assert oracle.exp_neg(-80.5) == 0.0
    assert oracle.exp_neg(-math.inf) == 0.0
    assert abs(oracle.exp_neg(-math.log(2)) - 0.5) <= _ulp(0.5)


def _bf(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def test_pool_equal_gates_is_mean():
    g = torch.Generator().manual_seed(1)
    a = torch.randn(512, generator=g).to(torch.bfloat16)
    b = torch.randn(512, generator=g).to(torch.bfloat16)
    z = torch.randn(512, generator=g).to(torch.bfloat16)
    out = oracle.pool_pair(oracle_bits(a), oracle_bits(b), oracle_bits(z), oracle_bits(z))
    ref = (a.float() + b.float()) * 0.5   # fl(a/2 + b/2) == fl(a + b)/2
    np.testing.assert_array_equal(out, ref.numpy())


def test_pool_dominant_gate_selects_token():
    g = torch.Generator().manual_seed(2)
    a = torch.randn(64, generator=g).to(torch.bfloat16)
    b = torch.randn(64, generator=g).to(torch.bfloat16)
    za = torch.full((64,), 50.0).to(torch.bfloat16)
    zb = torch.full((64,), -50.0).to(torch.bfloat16)
    out = oracle.pool_pair(oracle_bits(a), oracle_bits(b), oracle_bits(za), oracle_bits(zb))
    np.testing.assert_array_equal(out, a.float().numpy())
    out = oracle.pool_pair(oracle_bits(a), oracle_bits(b), oracle_bits(zb), oracle_bits(za))
    np.testing.assert_array_equal(out, b.float().numpy())


def test_pool_is_symmetric_and_close_to_softmax():
    g = torch.Generator().manual_seed(3)
    a, b, za, zb = (torch.randn(4096, generator=g).mul(3).to(torch.bfloat16) for _ in range(4))
    out = oracle.pool_pair(*(oracle_bits(t) for t in (a, b, za, zb)))
    swp = oracle.pool_pair(*(oracle_bits(t) for t in (b, a, zb, za)))
    np.testing.assert_array_equal(out, swp)
    A, Bv, ZA, ZB = (t.double().numpy() for t in (a, b, za, zb))
    wa = 1.0 / (1.0 + np.exp(ZB - ZA))
    ref = wa * A + (1 - wa) * Bv
    err = np.abs(out - ref)
    bound = 4 * np.finfo(np.float32).eps * (np.abs(A) + np.abs(Bv)) + 1e-30
    assert np.all(err <= bound)


def oracle_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- FP8 rule, indexer key


def test_fp8_row_rule():
    g = torch.Generator().manual_seed(4)
    v = torch.randn(128, generator=g).numpy().astype(np.float32)
    codes, s = oracle.quant_fp8_row(v)
    assert s == np.float32(np.abs(v).max()) / np.float32(448)
    j = int(np.argmax(np.abs(v)))
    assert codes[j] & 0x7F == 0x7E
    dec = np.array([oracle.e4m3_value(int(c)) for c in codes]) * float(s)
    assert np.all(np.abs(dec - v) <= np.abs(v) * 2.0 ** -4 + float(s) * 2.0 ** -10)
    codes0, s0 = oracle.quant_fp8_row(np.zeros(16, np.float32))
    assert s0 == 0 and not codes0.any()


def _entry(x):
    codes, scales = oracle.quant_fp4_row(np.asarray(x, np.float32))
    return codes, scales


def test_index_key_integer_grid_is_exact():
    """Small integer entries and weights: every partial sum is exact, so the
    projection must equal the integer dot product."""
    rng = np.random.default_rng(5)
    D, dI = 64, 32
    x = np.zeros(D, np.float32)
    for g in range(D // 16):   # amax 6 -> scale 1 -> integer-valued entries in {0,1,2,3,4,6}
        x[16 * g:16 * g + 16] = rng.choice([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6], 16)
        x[16 * g] = 6
    codes, scales = _entry(x)
    xh = oracle.fp4_dequant_row(codes, scales, D)
    assert np.array_equal(xh, x)
    Wi = rng.integers(-8, 9, size=(D, dI)).astype(np.float32)
    W = oracle_bits(torch.tensor(Wi).to(torch.bfloat16))
    ik, s = oracle.index_key(codes, scales, W)
    k = (x.astype(np.int64) @ Wi.astype(np.int64)).astype(np.float32)
    ref_codes, ref_s = _fp8_by_hand(k)
    assert s == ref_s
    np.testing.assert_array_equal(ik, ref_codes)


def _fp8_by_hand(k):
    amax = np.float32(np.abs(k).max())
    s = amax / np.float32(448)
    ref = torch.tensor(k / s, dtype=torch.float32).clamp(-448, 448).to(torch.float8_e4m3fn)
    return ref.view(torch.uint8).numpy(), s


def test_index_key_within_error_bound_of_exact_sum():
    rng = np.random.default_rng(6)
    D, dI = 512, 16
    x = rng.standard_normal(D).astype(np.float32)
    x = torch.tensor(x).to(torch.bfloat16).float().numpy()
    codes, scales = _entry(x)
    xh = oracle.fp4_dequant_row(codes, scales, D)
    Wt = torch.tensor(rng.standard_normal((D, dI)) / math.sqrt(D), dtype=torch.float32).to(torch.bfloat16)
    W = oracle_bits(Wt)
    Wf = Wt.double().numpy()
    # reconstruct the binary32 projection the oracle quantised, from its codes:
    ik, s = oracle.index_key(codes, scales, W)
    exact = [sum(Fraction(float(xh[c])) * Fraction(float(Wf[c, i])) for c in range(D)) for i in range(dI)]
    absum = [sum(abs(float(xh[c]) * float(Wf[c, i])) for c in range(D)) for i in range(dI)]
    amax = max(abs(float(e)) for e in exact)
    # one chain of D fused multiply-adds: |error| <= gamma_D * sum |x_c W_ci|
    gamma = (D + 4) * 2.0 ** -24
    bound_amax = gamma * max(absum)
    assert abs(float(s) * 448 - amax) <= bound_amax + amax * 2 ** -23
    dec = np.array([oracle.e4m3_value(int(c)) for c in ik]) * float(s)
    for i in range(dI):
        assert abs(dec[i] - float(exact[i])) <= abs(float(exact[i])) * 2 ** -4 + float(s) * 2 ** -9 + gamma * absum[i] * 2


# ---------------------------------------------------------------- the projection's order
# The indexer key is one fused multiply-add chain per output, channels in
# ascending order from +0 (the plain left-to-right sum of k_i = sum_c x^_c W_ci).
# Every quantised key byte depends on that order, so it is pinned exactly.


def _round_f32(v: Fraction) -> float:
    """Exact rational -> nearest binary32, ties to even (IEEE 754 roundTiesToEven)."""
    if v == 0:
        return 0.0
    sign = -1.0 if v < 0 else 1.0
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+2)
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                           # subnormal quantum 2^-149
    q = Fraction(2) ** (e - 23)                # spacing of binary32 in [2^e, 2^(e+1))
    m = a / q
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = sign * float(fl * q)
    assert np.float32(r) == r
    return r


def _fmaf_exact(a: float, b: float, c: float) -> float:
    return _round_f32(Fraction(a) * Fraction(b) + Fraction(c))


def _ascending_chain(xh, Wf, i):
    acc = 0.0
    for c in range(len(xh)):
        acc = _fmaf_exact(float(xh[c]), float(Wf[c, i]), acc)
    return acc


def _blocked_pairwise(xh, Wf, i):
    """32-channel chains added pairwise: a plausible other order, used only to
    show that the fixtures below tell the orders apart."""
    parts = []
    for g in range(len(xh) // 32):
        acc = 0.0
        for c in range(32 * g, 32 * g + 32):
            acc = _fmaf_exact(float(xh[c]), float(Wf[c, i]), acc)
        parts.append(acc)
    while len(parts) > 1:
        nxt = [_round_f32(Fraction(parts[j]) + Fraction(parts[j + 1])) for j in range(0, len(parts) - 1, 2)]
        if len(parts) % 2:
            nxt.append(parts[-1])
        parts = nxt
    return parts[0]


def test_index_key_chain_order_hand_case():
    """Worked by hand.  Column 0: product 2^24 at channel 0, then 31 products
    of 1 at channels 32..62.  In one ascending chain every +1 meets an
    accumulator of 2^24, where binary32 has spacing 2: 2^24 + 1 is a tie and
    goes to the even 2^24, so k_0 = 2^24 exactly.  (Summing channels 32..63
    on their own first would give 31 and k_0 = 2^24 + 32.)  Column 1 starts
    from -2^24: -2^24 + j is exact for j < 2^24, so k_1 = -2^24 + 31."""
    D, dI = 64, 2
    codes = np.zeros(D // 2, np.uint8)
    scales = np.zeros(D // 16, np.uint8)
    scales[0] = 0x78            # E4M3 2^8
    codes[0] = 0x6              # channel 0: E2M1 code 6 = 4.0 -> x^ = 1024
    scales[2] = scales[3] = 0x38    # E4M3 1.0
    for c in range(32, 63):     # channels 32..62: E2M1 code 2 = 1.0
        codes[c // 2] |= 0x2 << (4 * (c & 1))
    xh = oracle.fp4_dequant_row(codes, scales, D)
    assert xh[0] == 1024 and xh[32:63].tolist() == [1.0] * 31 and xh[63] == 0
    Wf = np.zeros((D, dI), np.float32)
    Wf[0, 0], Wf[0, 1] = 2.0 ** 14, -(2.0 ** 14)
    Wf[32:63, :] = 1.0
    W = oracle_bits(torch.tensor(Wf).to(torch.bfloat16))
    k = oracle.project_key(codes, scales, W)
    assert k[0] == np.float32(2 ** 24)
    assert k[1] == np.float32(-(2 ** 24) + 31)
    assert _blocked_pairwise(xh, Wf.astype(np.float64), 0) == 2 ** 24 + 32   # the other order differs
    ik, s = oracle.index_key(codes, scales, W)
    assert s == np.float32(2 ** 24) / np.float32(448)


@pytest.mark.parametrize("seed,D,dI", [(11, 512, 16), (12, 256, 32), (13, 128, 32)])
def test_index_key_matches_exact_rounding_of_each_fma(seed, D, dI):
    """Random entries: every output equals the ascending chain evaluated with
    exact rationals, each step rounded once to binary32; on the same data the
    blocked pairwise order gives other bits for some outputs."""
    rng = np.random.default_rng(seed)
    x = torch.tensor(rng.standard_normal(D), dtype=torch.float32).to(torch.bfloat16).float().numpy()
    codes, scales = _entry(x)
    xh = oracle.fp4_dequant_row(codes, scales, D)
    Wt = torch.tensor(rng.standard_normal((D, dI)) / math.sqrt(D), dtype=torch.float32).to(torch.bfloat16)
    Wf = Wt.double().numpy()
    k = oracle.project_key(codes, scales, oracle_bits(Wt))
    ref = [_ascending_chain(xh, Wf, i) for i in range(dI)]
    assert [float(v) for v in k] == ref
    other = [_blocked_pairwise(xh, Wf, i) for i in range(dI)]
    assert other != ref
    ik, s = oracle.index_key(codes, scales, oracle_bits(Wt))
    codes_ref, s_ref = oracle.quant_fp8_row(np.array(ref, np.float32))
    assert s == s_ref and np.array_equal(ik, codes_ref)


def test_quant_query_follows_fp8_rule():
    g = torch.Generator().manual_seed(7)
    q = torch.randn(128, generator=g).to(torch.bfloat16)
    c1, s1 = oracle.quant_query(oracle_bits(q))
    c2, s2 = oracle.quant_fp8_row(q.float().numpy())
    assert s1 == s2 and np.array_equal(c1, c2)
    ref, rs = _fp8_by_hand(q.float().numpy())
    assert rs == s1 and np.array_equal(ref, c1)


def test_bf16_rounding_from_double():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -3.14159, 1e-40, 3.4e38, 0.0, -0.0])
    got = oracle.f64_to_bf16(vals)
    # 1+2^-8 is the tie between 1 and 1+2^-7 -> even (1.0)
    assert got[0] == 0x3F80 and got[1] == 0x3F80
    assert got[2] == 0x3F81          # 1 + 3*2^-9 -> 1 + 2^-7 = 0x3F81 (nearer)
    ref = torch.tensor(vals[3:5], dtype=torch.float64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert got[3] == ref[0] and got[4] == ref[1]
    assert got[6] == 0 and got[7] == 0x8000
