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
