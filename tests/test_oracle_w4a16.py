"""Pins of the W4A16 oracle (CPU only): an exact-rational triple loop on
small shapes, one-hot activation rows, and the linearity identities."""

from fractions import Fraction

import numpy as np

from oracle import unpack_q4
from oracle import w4a16 as W
from workloads import activations_bf16, q4_weights


def _bits_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_exact_rational_triple_loop():
    M, N, K = 3, 5, 96
    q4, d = q4_weights(N, K, seed=1)
    xb = activations_bf16(M, K, seed=2, outlier_frac=0.05)
    y, a = W.w4a16_linear_ref(xb, q4, d, return_abs=True)
    q = unpack_q4(q4)
    x = _bits_to_f32(xb)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(x[m, k])) * Fraction(float(d[n, k // 32])) * int(q[n, k])
                        for k in range(K))
            mag = sum(abs(Fraction(float(x[m, k])) * Fraction(float(d[n, k // 32])) * int(q[n, k]))
                      for k in range(K))
            assert abs(Fraction(float(y[m, n])) - exact) <= mag * Fraction(K, 2 ** 52)
            assert abs(Fraction(float(a[m, n])) - mag) <= mag * Fraction(K, 2 ** 52)


def test_one_hot_rows_pick_single_weights():
    N, K = 7, 64
    q4, d = q4_weights(N, K, seed=3)
    q = unpack_q4(q4)
    xb = np.zeros((K, K), np.uint16)
    xb[np.arange(K), np.arange(K)] = 0x3F80          # bf16 1.0
    y = W.w4a16_linear_ref(xb, q4, d)
    for k in range(K):
        for n in range(N):
            assert y[k, n] == float(d[n, k // 32]) * int(q[n, k])


def test_negation_and_scale_doubling():
    M, N, K = 4, 6, 128
    q4, d = q4_weights(N, K, seed=4)
    xb = activations_bf16(M, K, seed=5)
    y = W.w4a16_linear_ref(xb, q4, d)
    assert np.array_equal(W.w4a16_linear_ref(xb ^ np.uint16(0x8000), q4, d), -y)
    assert np.array_equal(W.w4a16_linear_ref(xb, q4, (d * np.float32(2)).astype(np.float32)), 2 * y)


def test_unpacked_weights_round_once_from_the_qat_value():
    """bf16_RN(fp32(d q)) for every value, checked against exact rationals:
    the fp32 product is the nearest fp32 to d q, and the bf16 pattern the
    nearest bf16 to that (ties to the even significand)."""
    from fractions import Fraction as Fr

    q4, d = q4_weights(6, 64, seed=8)
    d[0, 0] = np.float32(1.00390625)        # 1 + 2^-8: q = +-1 is a bf16 tie (to even)
    bits = W.w4a16_unpacked_bits(q4, d)
    q = unpack_q4(q4)

    def rn(v: Fr, mant_bits: int) -> Fr:
        if v == 0:
            return Fr(0)
        sgn = 1 if v > 0 else -1
        a = abs(v)
        e = 0
        while a >= 2:
            a /= 2
            e += 1
        while a < 1:
            a *= 2
            e -= 1
        scaled = a * 2 ** (mant_bits - 1)
        fl = scaled.numerator // scaled.denominator
        rem = scaled - fl
        if rem > Fr(1, 2) or (rem == Fr(1, 2) and fl % 2 == 1):
            fl += 1
        return sgn * Fr(fl) / 2 ** (mant_bits - 1) * Fr(2) ** e

    got = (bits.astype(np.uint32) << 16).view(np.float32)
    for n in range(6):
        for k in range(64):
            exact = Fr(float(d[n, k // 32])) * int(q[n, k])
            assert Fr(float(got[n, k])) == rn(rn(exact, 24), 8), (n, k)
    q[0, :32] = 1
    tie = W.w4a16_unpacked_bits(_pack(q[:1]), d[:1])
    assert np.all(tie[0, :32] == 0x3F80)            # 1 + 2^-8 -> 1.0 (even)


def _pack(q):
    u = (q.astype(np.int16) & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
