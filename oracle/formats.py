"""FP8 E4M3 and E4M3FNUZ: decode tables and round-to-nearest-even encoders.

Source: [E2B] tip "E4M3 还是 E4M3FNUZ，都能用" — both formats have 3 mantissa
bits; E4M3FNUZ tops out at 240 instead of 448 and has no negative zero.
[CARD] header paragraph — weights are FP8 E4M3.

Reading of the pages (they print no bit layouts): with a sign bit, a 4-bit
exponent field e and a 3-bit mantissa field m,

* E4M3 reaches 448 = 1.75 * 2^8 only with exponent bias 7 and the all-ones
  code S.1111.111 reserved (NaN), so e = 0 encodes subnormals m/8 * 2^-6 and
  e > 0 encodes (1 + m/8) * 2^(e-7).
* E4M3FNUZ reaches 240 = 1.875 * 2^7 only with bias 8 and e = 15 fully
  usable, so e = 0 encodes m/8 * 2^-7 and e > 0 encodes (1 + m/8) * 2^(e-8);
  "no negative zero" leaves 0x80 without a value, read here as its NaN.

Encoder reading: round to the nearest representable magnitude, ties to the
even code (the even mantissa), saturate magnitudes above the format maximum
to the maximum, NaN to the format's NaN code, and a zero result is always the
+0 code 0x00 (FNUZ has no -0, and the two formats must carry the same bytes,
[E2B] same tip: "同样权重").

Pinned by tests/test_oracle_formats.py: the tables against torch's own
float8_e4m3fn / float8_e4m3fnuz decoding (a library routine), the maxima
448/240 and the minimum subnormals, the FNUZ = E4M3 / 2 identity, and the
encoders against torch's RNE casts on every fp32 value below the overflow
threshold in a dense sweep, plus an exact-rational brute force.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3FNUZ_MAX = 240.0
E4M3_NAN = 0x7F
E4M3FNUZ_NAN = 0x80


def _build_e4m3_table() -> np.ndarray:
    t = np.empty(256, dtype=np.float64)
    for b in range(256):
        s = -1.0 if b & 0x80 else 1.0
        e = (b >> 3) & 0xF
        m = b & 0x7
        if e == 15 and m == 7:
            t[b] = np.nan
        elif e == 0:
            t[b] = s * (m / 8.0) * 2.0 ** -6
        else:
            t[b] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


def _build_e4m3fnuz_table() -> np.ndarray:
    t = np.empty(256, dtype=np.float64)
    for b in range(256):
        if b == 0x80:
            t[b] = np.nan
            continue
        s = -1.0 if b & 0x80 else 1.0
        e = (b >> 3) & 0xF
        m = b & 0x7
        if e == 0:
            t[b] = s * (m / 8.0) * 2.0 ** -7
        else:
            t[b] = s * (1.0 + m / 8.0) * 2.0 ** (e - 8)
    return t


DEC_E4M3 = _build_e4m3_table()
DEC_E4M3FNUZ = _build_e4m3fnuz_table()

# Non-negative finite magnitudes in code order (codes 0x00..0x7E for E4M3,
# 0x00..0x7F for FNUZ); both are strictly increasing with the code.
_MAG_E4M3 = DEC_E4M3[:0x7F].copy()
_MAG_E4M3FNUZ = DEC_E4M3FNUZ[:0x80].copy()


def dec_e4m3(codes) -> np.ndarray:
    """E4M3 bytes -> float64 values (NaN for 0x7F / 0xFF)."""
    return DEC_E4M3[np.asarray(codes, dtype=np.uint8)]


def dec_e4m3fnuz(codes) -> np.ndarray:
    """E4M3FNUZ bytes -> float64 values (NaN for 0x80)."""
    return DEC_E4M3FNUZ[np.asarray(codes, dtype=np.uint8)]


def _encode(x, mags: np.ndarray, nan_code: int) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    top = mags.size - 1
    # lo = index of the largest magnitude <= a (a >= 0 always finds one).
    lo = np.searchsorted(mags, np.minimum(a, mags[top]), side="right") - 1
    lo = np.clip(lo, 0, top)
    hi = np.minimum(lo + 1, top)
    d_lo = a - mags[lo]
    d_hi = mags[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi != lo) & ((hi & 1) == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= mags[top], top, code)          # saturate
    neg = (x < 0) & (code != 0)                          # zero is always +0
    out = (code | np.where(neg, 0x80, 0)).astype(np.uint8)
    out = np.where(np.isnan(x), np.uint8(nan_code), out).astype(np.uint8)
    return out


def enc_e4m3(x) -> np.ndarray:
    """Encode values (exact in float64) to E4M3 bytes, RNE + saturation."""
    return _encode(x, _MAG_E4M3, E4M3_NAN)


def enc_e4m3fnuz(x) -> np.ndarray:
    """Encode values (exact in float64) to E4M3FNUZ bytes, RNE + saturation."""
    return _encode(x, _MAG_E4M3FNUZ, E4M3FNUZ_NAN)


def bf16_rne_bits(v: np.ndarray) -> np.ndarray:
    """fp64 values -> bf16 bit patterns (uint16), round to nearest even: bf16
    keeps 8 significant bits, so the rounding quantum is 2^(e-8) for
    v = m 2^e (0.5 <= |m| < 1), and 2^-133 in the subnormal range. Values past
    the largest finite bf16 (after rounding) become Inf; NaN stays NaN."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        _, e = np.frexp(v)
        q = np.ldexp(1.0, np.maximum(e - 8, -133))
        r = np.where(np.isfinite(v), np.round(v / q) * q, v)   # numpy rounds half to even
        return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
