"""Pins of the int8 W8A8 oracle (CPU only): hand-worked ties, on-grid round
trips, the half-level error bound of 255 levels per row, an exact-rational
check of every code's rounding, exact integer GEMM sums, and hand-worked
epilogue roundings."""

from fractions import Fraction

import numpy as np

from oracle import int8 as I8
from oracle import qat_values
from workloads import activations_bf16, q4_weights


def test_half_integers_round_to_even():
    # amax 127 gives s = 1 exactly, so each code is the rounded value itself
    v = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 126.5, -127.0, 0.0]], np.float32)
    r = I8.quantize_rows_int8(v)
    assert r.scales.tolist() == [1.0]
    assert r.codes.tolist() == [[127, 2, 4, -2, 0, 0, 2, 126, -127, 0]]


def test_rows_on_the_integer_grid_round_trip():
    rng = np.random.default_rng(0)
    for p in (-20, -3, 0, 5):
        k = rng.integers(-127, 128, (4, 64))
        k[:, 7] = 127
        k[1, 9] = -127
        v = (k * 2.0 ** p).astype(np.float32)
        r = I8.quantize_rows_int8(v)
        assert np.all(r.scales == np.float32(2.0 ** p))
        assert np.array_equal(r.codes.astype(np.int64), k)


def test_zero_row_and_255_levels():
    r = I8.quantize_rows_int8(np.zeros((2, 32), np.float32))
    assert np.all(r.codes == 0) and np.all(r.scales == 0)
    rng = np.random.default_rng(1)
    r = I8.quantize_rows_int8(rng.standard_normal((64, 2048)).astype(np.float32))
    assert r.codes.min() >= -127 and r.codes.max() <= 127
    assert np.all(np.max(np.abs(r.codes.astype(np.int64)), axis=1) == 127)


def test_error_at_most_half_a_level_of_the_row_maximum():
    """255 levels per row: every value within s / 2 = amax / 254 of its code,
    up to the fp32 roundings of s (relative 2^-24) and of the quotient
    (|v / s| <= 128, so at most 2^-17 of a level): err <= s (1/2 + 2^-17)
    with s <= (amax / 127)(1 + 2^-24). The half-level bound is reached."""
    q4, d = q4_weights(256, 1024, seed=3)
    rows = [qat_values(q4, d),
            (activations_bf16(256, 1024, seed=4, outlier_frac=0.01).astype(np.uint32) << 16).view(np.float32)]
    worst = 0.0
    for v in rows:
        r = I8.quantize_rows_int8(v)
        err = np.abs(r.codes.astype(np.float64) * r.scales[:, None].astype(np.float64) - v.astype(np.float64))
        amax = np.max(np.abs(v.astype(np.float64)), axis=1)
        rel = np.max(err, axis=1) / amax
        assert np.all(rel <= (0.5 + 2 ** -17) * (1 + 2 ** -24) / 127)
        worst = max(worst, float(rel.max()))
    assert worst > (1 / 254) * 0.99


def _rn_fp32(q: Fraction) -> np.float32:
    """The fp32 value nearest the rational q (ties to the even significand),
    chosen among the fp32 neighbours of fp64(q) by exact comparison."""
    c = np.float32(float(q))
    cands = {c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(-np.inf))}
    best = None
    for x in cands:
        dist = abs(Fraction(float(x)) - q)
        key = (dist, int(np.array(x, np.float32).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, x)
    return best[1]


def test_every_code_against_exact_rationals():
    q4, d = q4_weights(12, 256, seed=5)
    v = np.concatenate([qat_values(q4, d),
                        (activations_bf16(12, 256, seed=6).astype(np.uint32) << 16).view(np.float32)])
    r = I8.quantize_rows_int8(v)
    for i in range(v.shape[0]):
        amax = max(abs(Fraction(float(x))) for x in v[i])
        s = _rn_fp32(amax / 127)
        assert s == r.scales[i]
        for j in range(v.shape[1]):
            qf = Fraction(float(_rn_fp32(Fraction(float(v[i, j])) / Fraction(float(s)))))
            fl = qf.numerator // qf.denominator
            frac = qf - fl
            code = fl + (1 if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and fl % 2 == 1) else 0)
            code = max(-127, min(127, code))
            assert code == int(r.codes[i, j]), (i, j)


def test_integer_gemm_exact_small_and_at_the_largest_k():
    rng = np.random.default_rng(7)
    x8 = rng.integers(-127, 128, (3, 50)).astype(np.int8)
    w8 = rng.integers(-127, 128, (4, 50)).astype(np.int8)
    acc = I8.int8_gemm_acc(x8, w8)
    for m in range(3):
        for n in range(4):
            assert acc[m, n] == sum(int(a) * int(b) for a, b in zip(x8[m], w8[n]))
    K = 65536
    x8 = np.full((2, K), 127, np.int8)
    w8 = np.full((2, K), 127, np.int8)
    x8[1, ::2] = -127
    w8[1, 1::3] = -127
    acc = I8.int8_gemm_acc(x8, w8)
    assert acc[0, 0] == 127 * 127 * K
    assert acc[1, 1] == sum(int(a) * int(b) for a, b in zip(x8[1], w8[1]))


def test_epilogue_roundings_by_hand():
    def y(acc, st, sc):
        # |acc| = n * 127 * 127 + 127 * q + r, one int8 product per column
        n, rem = divmod(abs(acc), 127 * 127)
        q, r = divmod(rem, 127)
        xs = [127] * n + [127, r]
        ws = [127] * n + [q, 1]
        x8 = np.array([xs], np.int8) * (1 if acc >= 0 else -1)
        w8 = np.array([ws], np.int8)
        assert I8.int8_gemm_acc(x8, w8)[0, 0] == acc
        return int(I8.int8_linear_ref(x8, np.float32([st]), w8, np.float32([sc]))[0, 0])

    assert y(3, 0.5, 0.25) == 0x3EC0               # 0.375
    assert y(-3, 0.5, 0.25) == 0xBEC0
    assert y(1, 1 + 2 ** -8, 1.0) == 0x3F80        # tie between 1 and 1 + 2^-7 -> 1 (even)
    assert y(1, 1 + 3 * 2 ** -8, 1.0) == 0x3F82    # tie -> 1 + 2^-6 (even)
    assert y(0, 5.0, 7.0) == 0x0000
    # the scales apply one after the other: (acc * s_tok) * s_ch, not
    # acc * (s_tok * s_ch), which rounds differently here
    st = float(np.array(1070077415, np.uint32).view(np.float32))
    sc = float(np.array(1071091490, np.uint32).view(np.float32))
    assert y(91996, st, sc) == 0x486C
    # fp32 rounding of the integer sum: 2^24 + 1 -> 2^24 (tie to even) before scaling
    x8 = np.full((1, 1041), 127, np.int8)
    w8 = np.full((1, 1041), 127, np.int8)
    x8[0, -1], w8[0, -1] = 8, 54                        # 1040 * 16129 + 432 = 16774592
    acc = int(I8.int8_gemm_acc(x8, w8)[0, 0])
    assert acc == 1040 * 16129 + 432
    got = int(I8.int8_linear_ref(x8, np.float32([1.0]), w8, np.float32([1.0]))[0, 0])
    exp_f32 = float(np.float32(float(acc)))
    assert exp_f32 == float(acc)                         # below 2^24: exact
    assert got == int(np.float32(exp_f32).view(np.uint32) + 0x7FFF + ((np.float32(exp_f32).view(np.uint32) >> 16) & 1)) >> 16
