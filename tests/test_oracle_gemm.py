"""Pins of the oracle's row-wise scaled GEMM (CPU only): an exact-rational
triple loop on small shapes (including the whole tiny W8A8 linear, M=4 K=256
N=128, from its q4_0-grid weights and bf16 activations), exact integer sums
at the largest K the library accepts, one-hot rows, and the negation /
scale-doubling identities."""

from fractions import Fraction

import numpy as np

import oracle
from oracle import formats as F
from workloads import activations_bf16, q4_weights


def _triple_loop(x8, w8):
    dec = [Fraction(float(v)) if not np.isnan(v) else None for v in F.DEC_E4M3]
    M, K = x8.shape
    N = w8.shape[0]
    out = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        xr = [dec[int(c)] for c in x8[m]]
        for n in range(N):
            wr = w8[n]
            acc = Fraction(0)
            for k in range(K):
                acc += xr[k] * dec[int(wr[k])]
            out[m][n] = acc
    return out


def _finite_codes(rng, shape):
    pool = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], dtype=np.uint8)
    return rng.choice(pool, size=shape)


def test_exact_accumulation_small():
    rng = np.random.default_rng(1)
    x8 = _finite_codes(rng, (3, 80))
    w8 = _finite_codes(rng, (5, 80))
    ones_t = np.ones(3, np.float32)
    ones_c = np.ones(5, np.float32)
    y = oracle.rowwise_linear_ref(x8, ones_t, w8, ones_c)
    ref = _triple_loop(x8, w8)
    for m in range(3):
        for n in range(5):
            assert Fraction(float(y[m, n])) == ref[m][n]


def test_tiny_linear_end_to_end_against_exact_rationals():
    M, K, N = 4, 256, 128
    q4, d = q4_weights(N, K, seed=0)
    xb = activations_bf16(M, K, seed=0)
    w = oracle.repack_qat(q4, d)
    a = oracle.quant_act(xb)
    y = oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales)
    ref = _triple_loop(a.codes, w.codes[:16])
    for m in range(M):
        for n in range(16):
            exact = ref[m][n] * Fraction(float(a.scales[m])) * Fraction(float(w.scales[n]))
            assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def test_one_hot_rows_pick_single_weights():
    rng = np.random.default_rng(2)
    K, N = 64, 33
    w8 = _finite_codes(rng, (N, K))
    s_ch = rng.uniform(0.5, 2, N).astype(np.float32)
    x8 = np.zeros((K, K), dtype=np.uint8)
    x8[np.arange(K), np.arange(K)] = 0x38          # 1.0
    s_tok = np.full(K, 0.25, np.float32)
    y = oracle.rowwise_linear_ref(x8, s_tok, w8, s_ch)
    expect = F.dec_e4m3(w8).T * 0.25 * s_ch[None, :].astype(np.float64)
    assert np.array_equal(y, expect)


def test_negation_and_scale_doubling():
    rng = np.random.default_rng(3)
    x8 = _finite_codes(rng, (7, 96))
    w8 = _finite_codes(rng, (9, 96))
    st = rng.uniform(0.1, 1, 7).astype(np.float32)
    sc = rng.uniform(0.1, 1, 9).astype(np.float32)
    y = oracle.rowwise_linear_ref(x8, st, w8, sc)
    neg = x8 ^ np.uint8(0x80)
    assert np.array_equal(oracle.rowwise_linear_ref(neg, st, w8, sc), -y)
    assert np.array_equal(oracle.rowwise_linear_ref(x8, st, w8, sc * 2), 2 * y)


def test_tolerance_and_bf16_ulp():
    assert oracle.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert oracle.bf16_ulp(np.array([3.0]))[0] == 2.0 ** -6
    assert oracle.bf16_ulp(np.array([-0.75]))[0] == 2.0 ** -8
    assert oracle.bf16_ulp(np.array([0.0]))[0] == 2.0 ** -133
    y = np.array([[1.0]])
    ok, r = oracle.check_linear(np.array([[1.0 + 2.0 ** -7]]), y, np.array([[0.0]]))
    assert ok and r == 1.0
    ok, _ = oracle.check_linear(np.array([[1.0 + 2.0 ** -6]]), y, np.array([[0.0]]))
    assert not ok


def test_exact_at_the_largest_k():
    """K = 65536 (the library's limit): the fp64 product equals the exact sum,
    computed with Python integers in units of 2^-18 (E4M3 values are integer
    multiples of 2^-9), on rows that mix the largest products (+-448 * 448),
    the smallest (2^-9 * 2^-9) and random codes, so that a partial sum needs
    every one of fp64's 53 bits."""
    K = 65536
    rng = np.random.default_rng(7)
    units = [None if np.isnan(v) else int(round(float(v) * 512)) for v in F.DEC_E4M3]
    x8 = _finite_codes(rng, (3, K))
    w8 = _finite_codes(rng, (4, K))
    x8[0, :] = 0x7E                     # +448
    w8[0, : K // 2] = 0x7E              # +448 * 448 on half the terms ...
    w8[0, K // 2:] = 0x01               # ... then 2^-9 * 448 units
    x8[1, 1::2] = 0x01                  # 2^-9 on every other term
    w8[1, 0::2] = 0xFE                  # -448
    w8[1, 1::2] = 0x01                  # 2^-9: adds 2^-18 per odd term
    ones = np.ones(3, np.float32)
    got = oracle.rowwise_linear_ref(x8, ones, w8, np.ones(4, np.float32))
    for m in range(3):
        xu = [units[int(c)] for c in x8[m]]
        for n in range(4):
            exact = sum(a * units[int(b)] for a, b in zip(xu, w8[n]))     # units of 2^-18
            assert Fraction(float(got[m, n])) == Fraction(exact, 2 ** 18), (m, n)
