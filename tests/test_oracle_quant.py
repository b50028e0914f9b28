"""Pins of the oracle's per-row quantizers (CPU only).

Against what the pages fix: the 31B model card's largest requant error,
3.57 % of the row maximum (= 16/448, half the top-binade E4M3 step), and the
E2B article's native-FNUZ verify output, max_rel_err 0.0333334 (about 8/240);
plus exact round trips of values already on the grid, the tie at 3/8 of the
row maximum, zero rows, an exact-rational brute force of the whole chain and
the FNUZ conversion's value-exactness.
"""

import json
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import formats as F
from oracle.quantize import requant_error_stats
from workloads import activations_bf16, q4_weights

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "verify_stats.json")))


def test_unpack_q4_nibble_order_and_sign():
    q4 = np.array([[0x8F, 0x70, 0x00, 0x19]], dtype=np.uint8)
    assert oracle.unpack_q4(q4).tolist() == [[-1, -8, 0, 7, 0, 0, -7, 1]]


def test_e4m3_error_bound_matches_card():
    pct = GOLDEN["e4m3_card_31b"]["largest_error_fraction_of_row_max_pct"]
    bound = 16.0 / 448.0
    assert round(100 * bound, 2) == pct
    q4, d = q4_weights(1024, 2048, seed=123)
    v = oracle.qat_values(q4, d)
    r = oracle.repack_qat(q4, d)
    st = requant_error_stats(v, r.codes, r.scales)
    # fp32 rounding: the scale moves the bound by 2^-24 relative, and the
    # rounded quotient can land on a midpoint it was half an fp32 ulp (2^-16
    # at 256..448) short of, adding up to 2^-16 / 16 = 2^-20 relative.
    assert st["max_rel_err"] <= bound * (1 + 2.0 ** -19)
    assert st["max_rel_err"] > 0.034        # the bound is approached, as on the card
    assert 0.005 < st["relative_rms_error"] < 0.05


def test_fnuz_error_bound_matches_e2b_verify():
    page = GOLDEN["e4m3fnuz_e2b"]["max_rel_err"]
    bound = 8.0 / 240.0
    assert abs(page - bound) / bound < 1e-5
    q4, d = q4_weights(1024, 2048, seed=321)
    v = oracle.qat_values(q4, d)
    r = oracle.quantize_rows_fnuz(v)
    st = requant_error_stats(v, r.codes, r.scales, dec=F.dec_e4m3fnuz)
    assert st["max_rel_err"] <= page
    assert st["max_rel_err"] > 0.032


def test_on_grid_rows_round_trip():
    rng = np.random.default_rng(5)
    finite = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], dtype=np.uint8)
    for p in (-20, -3, 0, 7):
        codes = rng.choice(finite, size=(64, 96))
        codes[:, 17] = rng.choice([0x7E, 0xFE], size=64)   # |e| = 448 in every row
        vals = F.dec_e4m3(codes) * 2.0 ** p
        r = oracle.quantize_rows(vals.astype(np.float32))
        assert np.all(r.scales == np.float32(2.0 ** p))
        expect = codes.copy()
        expect[expect == 0x80] = 0       # the encoder emits +0 only
        assert np.array_equal(r.codes, expect)


def test_tie_at_three_eighths_of_row_max_rounds_to_even():
    # QAT grid row: q = 8 sets the row max, q = 3 sits at 3/8 of it.
    d = np.array([[0.125]], dtype=np.float32)
    q = np.zeros((1, 32), dtype=np.int64)
    q[0, 0], q[0, 1] = -8, 3
    nib = (q & 0xF).astype(np.uint8)
    q4 = nib[:, 0::2] | (nib[:, 1::2] << 4)
    r = oracle.repack_qat(q4, d)
    s = np.float32(1.0) / np.float32(448.0)
    assert r.scales[0] == s
    quot = np.float32(0.375) / s
    assert quot == np.float32(168.0)          # exactly between 160 and 176
    assert F.dec_e4m3(r.codes[0, 1]) == 160.0  # even mantissa wins
    assert r.codes[0, 0] == 0xFE


def test_zero_and_nonfinite_rows():
    v = np.zeros((3, 64), dtype=np.float32)
    v[1, 5] = np.inf
    v[2, 7] = np.nan
    r = oracle.quantize_rows(v)
    assert r.scales[0] == 0 and np.all(r.codes[0] == 0)
    assert r.bad_rows.tolist() == [False, True, True]


def _fp32_rn(x: Fraction) -> Fraction:
    """Round a rational to the nearest fp32 value (ties to even), normal or
    subnormal; written from the IEEE 754 definition."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def _exact_chain(row_vals):
    """Scale and codes of one row from exact rationals and explicit RN steps."""
    v = [Fraction(float(x)) for x in row_vals]
    amax = max(abs(x) for x in v)
    s = _fp32_rn(amax / 448)
    mags = [Fraction(float(m)) for m in F.DEC_E4M3[:0x7F]]
    codes = []
    for x in v:
        if s == 0:
            codes.append(0)
            continue
        q = _fp32_rn(x / s)
        a = abs(q)
        if a >= 448:
            c = 0x7E
        else:
            c = min(range(127), key=lambda i: (abs(a - mags[i]), i % 2))
        codes.append(c | (0x80 if (q < 0 and c != 0) else 0))
    return s, codes


def test_whole_chain_against_exact_rationals():
    q4, d = q4_weights(6, 64, seed=9)
    v = oracle.qat_values(q4, d)
    # the QAT values are single fp32 products d*q
    qv = oracle.unpack_q4(q4)
    for n in range(6):
        for k in range(64):
            assert Fraction(float(v[n, k])) == _fp32_rn(Fraction(float(d[n, k // 32])) * int(qv[n, k]))
    r = oracle.repack_qat(q4, d)
    for n in range(6):
        s, codes = _exact_chain(v[n])
        assert Fraction(float(r.scales[n])) == s
        assert r.codes[n].tolist() == codes
    xb = activations_bf16(5, 96, seed=4, outlier_frac=0.05)
    ra = oracle.quant_act(xb)
    for m in range(5):
        vals = [struct.unpack("<f", struct.pack("<I", int(b) << 16))[0] for b in xb[m]]
        s, codes = _exact_chain(vals)
        assert Fraction(float(ra.scales[m])) == s
        assert ra.codes[m].tolist() == codes


def test_fnuz_copy_converts_back_bit_exactly():
    q4, d = q4_weights(256, 512, seed=2)
    r = oracle.repack_qat(q4, d)
    cn, sn = oracle.fnuz_copy_of_e4m3(r.codes, r.scales)
    # the FNUZ copy holds the same weights
    assert np.array_equal(F.dec_e4m3fnuz(cn) * sn[:, None].astype(np.float64),
                          F.dec_e4m3(r.codes) * r.scales[:, None].astype(np.float64))
    c = oracle.convert_fnuz_to_e4m3(cn, sn)
    assert np.array_equal(c.codes, r.codes) and np.array_equal(c.scales, r.scales)
    assert c.halved_rows.all() and not c.inexact_rows.any() and not c.nan_rows.any()


def test_native_fnuz_conversion_is_value_exact_or_flagged():
    q4, d = q4_weights(512, 256, seed=6)
    v = oracle.qat_values(q4, d)
    rn = oracle.quantize_rows_fnuz(v)
    c = oracle.convert_fnuz_to_e4m3(rn.codes, rn.scales)
    assert not c.halved_rows.all()            # native rows hold +-240
    lhs = F.dec_e4m3(c.codes) * c.scales[:, None].astype(np.float64)
    rhs = F.dec_e4m3fnuz(rn.codes) * rn.scales[:, None].astype(np.float64)
    ok = ~c.inexact_rows
    assert np.array_equal(lhs[ok], rhs[ok])
    # flagged rows hold a FNUZ code with exponent field <= 1 and an odd mantissa
    e = (rn.codes >> 3) & 0xF
    odd_low = np.any((e <= 1) & (rn.codes & 1).astype(bool) & (rn.codes != 0x80), axis=1)
    assert np.array_equal(c.inexact_rows, odd_low & ~c.halved_rows)


def test_fnuz_nan_code_is_flagged():
    codes = np.zeros((2, 32), dtype=np.uint8)
    codes[1, 3] = 0x80
    c = oracle.convert_fnuz_to_e4m3(codes, np.ones(2, np.float32))
    assert c.nan_rows.tolist() == [False, True]
