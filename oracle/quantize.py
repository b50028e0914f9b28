"""Per-row FP8 quantization: QAT repack, per-token activation quant, FNUZ.

Sources:

* [CARD] header paragraph: every Linear is FP8 E4M3 with one float32 scale
  per output channel, activations are quantized to FP8 per token at run time;
  section "QAT trained the weights onto a 4-bit grid with one scale per group
  of 32 values ... this build rounds the QAT weights again".
* [SIZES] table "Format / Linear layers / Built with": fp8 = E4M3 weights per
  channel, FP8 activations per token.
* [E2B] section "十种构建": the QAT release's weights already lie on a 4-bit
  grid, one shared scale per group of 32 values.
* [E2B] section "第一步：构建各种格式": the ``--fnuz`` build and its verify
  report (max_rel_err 0.0333..., relative_rms_error 0.0264...).
* [E2B] tip "E4M3 还是 E4M3FNUZ，都能用": FNUZ checkpoints are converted at
  load and then serve like the E4M3 build of the same weights.

Readings where the pages are silent (each listed in the design notes):

* Scale rule: ``s = amax / 448`` per row (amax/240 for a native FNUZ build);
  the pages' error figures 3.57 % = 16/448 and 0.0333 = 8/240 are exactly
  half the top-binade step of each format relative to the format maximum,
  which is what this rule gives.
* Arithmetic: all steps in fp32 with IEEE round-to-nearest and no fused
  multiply-add: ``w = fp32(d * q)``, ``s = fp32(amax / 448)``,
  ``code = RNE_E4M3(fp32(v / s))``. Division by ``s`` (not multiplication by
  a reciprocal) is the plainest reading of "scale = amax / 448".
* A row whose amax is 0 gets ``s = 0`` and all-zero codes.
* A row holding NaN or Inf is reported (``bad_rows``); its outputs are
  unspecified.
* q4 packing: element ``2j`` in the low nibble, ``2j+1`` in the high nibble,
  4-bit two's complement; group ``g = k // 32`` along K.
* FNUZ load conversion: a row with no +-240 code (and an exactly halvable
  scale) keeps its bytes and halves its scale; otherwise every value is
  re-encoded in E4M3 at the same scale, which is exact except for FNUZ codes
  with exponent field <= 1 and an odd mantissa (reported as inexact).
  Code 0x80 (FNUZ NaN) is reported.

Pinned by tests/test_oracle_quant.py: the per-row error bound 16/448
([CARD] verify table, 3.57 %) and 8/240 ([E2B] verify JSON), exact round
trip of values already on the grid, the tie case 3/8 of the row maximum,
zero rows, exact-rational brute force of the whole chain on small rows, and
the FNUZ conversion's exactness property checked value by value in fp64.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .formats import (
    E4M3_MAX,
    E4M3FNUZ_MAX,
    dec_e4m3,
    dec_e4m3fnuz,
    enc_e4m3,
    enc_e4m3fnuz,
)


@dataclass
class QuantResult:
    codes: np.ndarray       # uint8 [R, K]
    scales: np.ndarray      # float32 [R]
    bad_rows: np.ndarray    # bool [R]: amax not finite (outputs unspecified)


def quantize_rows(v: np.ndarray, fmt_max: float = E4M3_MAX, enc=enc_e4m3) -> QuantResult:
    """Quantize each row of fp32 values with one scale ``amax / fmt_max``."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    if v.ndim != 2:
        raise ValueError("expected [rows, K]")
    R, K = v.shape
    if K == 0:
        return QuantResult(np.zeros((R, 0), np.uint8), np.zeros(R, np.float32),
                           np.zeros(R, bool))
    amax = np.max(np.abs(v), axis=1)                       # exact; NaN propagates
    bad = ~np.isfinite(amax)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        s = (amax / np.float32(fmt_max)).astype(np.float32)      # fp32 RN division
        q = (v / s[:, None]).astype(np.float32)                  # fp32 RN division
    codes = enc(q.astype(np.float64))
    codes[s == 0] = 0
    return QuantResult(codes.astype(np.uint8), s, bad)


def quantize_rows_fnuz(v: np.ndarray) -> QuantResult:
    """A native E4M3FNUZ build of the same rows: scale ``amax / 240``."""
    return quantize_rows(v, E4M3FNUZ_MAX, enc_e4m3fnuz)


def unpack_q4(q4: np.ndarray) -> np.ndarray:
    """Packed int4 ``[N, K/2]`` bytes -> int8 ``[N, K]`` in [-8, 7]."""
    q4 = np.asarray(q4, dtype=np.uint8)
    lo = (q4 & 0x0F).astype(np.int8)
    hi = (q4 >> 4).astype(np.int8)
    q = np.empty((q4.shape[0], q4.shape[1] * 2), dtype=np.int8)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    q[q >= 8] -= 16
    return q


def qat_values(q4: np.ndarray, d: np.ndarray) -> np.ndarray:
    """The QAT weights ``w[n, k] = fp32(d[n, k // 32] * q[n, k])``."""
    q = unpack_q4(q4)
    d = np.asarray(d, dtype=np.float32)
    if d.shape[1] * 32 != q.shape[1]:
        raise ValueError("d must hold one scale per 32 values along K")
    return (np.repeat(d, 32, axis=1) * q.astype(np.float32)).astype(np.float32)


def repack_qat(q4: np.ndarray, d: np.ndarray) -> QuantResult:
    """QAT q4_0 grid -> per-output-channel E4M3 (one fp32 scale per row)."""
    return quantize_rows(qat_values(q4, d))


def quant_act(x_bf16_bits: np.ndarray) -> QuantResult:
    """Per-token activation quant of bf16 rows (given as uint16 patterns)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    v = (x.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return quantize_rows(v)


def fnuz_copy_of_e4m3(codes: np.ndarray, s: np.ndarray):
    """The E4M3FNUZ-stored copy of an E4M3 build of the same weights.

    Every E4M3 code this quantizer emits (never 0x80, 0x7F or 0xFF) means
    exactly half as much in FNUZ, so the same bytes with a doubled scale hold
    the same weights.
    """
    return np.array(codes, dtype=np.uint8, copy=True), (np.asarray(s, np.float32) * np.float32(2)).astype(np.float32)


@dataclass
class FnuzConversion:
    codes: np.ndarray       # uint8 [R, K] E4M3
    scales: np.ndarray      # float32 [R]
    nan_rows: np.ndarray    # bool [R]: a 0x80 code (FNUZ NaN) was present
    inexact_rows: np.ndarray  # bool [R]: some value is not representable
    bad_rows: np.ndarray    # bool [R]: the FNUZ scale is not finite
    halved_rows: np.ndarray  # bool [R]: bytes kept, scale halved


def convert_fnuz_to_e4m3(codes_nuz: np.ndarray, s_nuz: np.ndarray) -> FnuzConversion:
    codes_nuz = np.asarray(codes_nuz, dtype=np.uint8)
    s_nuz = np.asarray(s_nuz, dtype=np.float32)
    R = codes_nuz.shape[0]
    nan_rows = np.any(codes_nuz == 0x80, axis=1)
    has_max = np.any((codes_nuz & 0x7F) == 0x7F, axis=1)
    bad = ~np.isfinite(s_nuz)
    half = (s_nuz / np.float32(2)).astype(np.float32)
    with np.errstate(invalid="ignore", over="ignore"):
        halvable = (half * np.float32(2)).astype(np.float32) == s_nuz
    keep = ~has_max & halvable
    out = np.array(codes_nuz, copy=True)
    scales = np.where(keep, half, s_nuz).astype(np.float32)
    inexact = np.zeros(R, dtype=bool)
    re = ~keep
    if np.any(re):
        vals = dec_e4m3fnuz(codes_nuz[re])
        enc = enc_e4m3(np.nan_to_num(vals, nan=0.0))
        out[re] = enc
        with np.errstate(invalid="ignore"):
            inexact[re] = np.any(dec_e4m3(enc) != np.nan_to_num(vals, nan=0.0), axis=1)
    return FnuzConversion(out, scales, nan_rows, inexact, bad, keep)


def requant_error_stats(v: np.ndarray, codes: np.ndarray, s: np.ndarray, dec=dec_e4m3):
    """The verify statistics of [E2B] step 1 / [CARD] verify table.

    ``max_rel_err``: the largest ``|dec(code) * s - v|`` as a fraction of its
    row's largest ``|v|``; ``relative_rms_error``: ``sqrt(sum err^2 / sum v^2)``.
    """
    v = np.asarray(v, dtype=np.float64)
    deq = dec(codes) * np.asarray(s, dtype=np.float64)[:, None]
    err = np.abs(deq - v)
    amax = np.max(np.abs(v), axis=1)
    nz = amax > 0
    max_rel = float(np.max(np.max(err[nz], axis=1) / amax[nz])) if np.any(nz) else 0.0
    den = float(np.sum(v * v))
    rms = float(np.sqrt(np.sum(err * err) / den)) if den > 0 else 0.0
    return {"max_rel_err": max_rel, "relative_rms_error": rms, "values": int(v.size)}
