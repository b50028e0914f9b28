"""int8 W8A8: int8 weights per output channel, int8 activations per token.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources:

* [SIZES] section "The Sizes and the Builds", format table: w8a8 = int8
  weights per channel and int8 activations per token, built from the same QAT
  q4_0 release as the FP8 build.
* [E2B] section "它们离训练权重有多近？": the int8 build rounds every value to
  one of 255 levels per row.
* [E2B] section "第二步：测这张卡的矩阵乘法": the int8 GEMM of the E2B GEMM
  set at M = 64 (and PyTorch's int8 matmul refusing M < 17, a limit this
  path does not have).

Readings where the pages are silent (each listed in the design notes):

* 255 levels per row = the symmetric integers -127..127 with one fp32 scale
  ``s = fp32(amax / 127)`` per row (IEEE division).
* ``code = clamp(RNE(fp32(v / s)), -127, 127)``: IEEE fp32 division, then
  round half to even to an integer (the clamp never acts on finite rows,
  since |v| <= amax gives |v / s| <= 127 (1 + 2^-23); it only bounds the
  contract). A row with amax == 0 gets s = 0 and all-zero codes; a row with
  NaN or Inf is reported and its outputs are unspecified.
* Weight source values are the QAT values ``w = fp32(d * q)`` of the q4_0
  grid, as for the FP8 repack.
* GEMM: the int8 products are summed exactly (an integer, |acc| <= 127^2 K
  < 2^31 for K <= 65536), and the row-wise scales are applied in fp32 with
  one IEEE rounding per step:
  ``y = bf16_RN(fp32(fp32(fp32(acc) * s_tok) * s_ch))``. Every step is
  fixed, so the result is bit-exact, not a bound.

Pinned by tests/test_oracle_int8.py: hand-worked ties (half-integers go to
the even integer), exact round trips of rows already on the integer grid,
the per-row error bound of half a level (amax / 254, 255 levels per row),
an exact-rational check of every code's rounding, exact integer GEMM sums
against a triple loop at small K and K = 65536, and hand-worked epilogue
roundings.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_rne_bits
from .quantize import QuantResult, qat_values

INT8_LEVEL_MAX = 127


def quantize_rows_int8(v: np.ndarray) -> QuantResult:
    """Each row of fp32 values -> int8 codes (as int8) and one fp32 scale."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    if v.ndim != 2:
        raise ValueError("expected [rows, K]")
    R, K = v.shape
    amax = np.max(np.abs(v), axis=1) if K else np.zeros(R, np.float32)
    bad = ~np.isfinite(amax)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        s = (amax / np.float32(INT8_LEVEL_MAX)).astype(np.float32)   # fp32 RN division
        q = (v / s[:, None]).astype(np.float32)                      # fp32 RN division
        r = np.rint(q.astype(np.float64))                            # half to even
    r = np.clip(np.nan_to_num(r, nan=0.0), -INT8_LEVEL_MAX, INT8_LEVEL_MAX)
    codes = r.astype(np.int8)
    codes[s == 0] = 0
    return QuantResult(codes, s, bad)


def repack_qat_int8(q4: np.ndarray, d: np.ndarray) -> QuantResult:
    """QAT q4_0 grid -> per-output-channel int8 (one fp32 scale per row)."""
    return quantize_rows_int8(qat_values(q4, d))


def quant_act_int8(x_bf16_bits: np.ndarray) -> QuantResult:
    """Per-token int8 quantization of bf16 rows (given as uint16 patterns)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    v = (x.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return quantize_rows_int8(v)


def int8_gemm_acc(x8: np.ndarray, w8: np.ndarray) -> np.ndarray:
    """Exact integer sums acc[m, n] = sum_k x8[m, k] * w8[n, k] (int64).

    Computed as an fp64 matrix product (a library primitive): every product
    is an integer of magnitude <= 127^2 and every partial sum an integer of
    magnitude <= 127^2 K < 2^53 for K < 2^39, so fp64 holds each one exactly,
    in any order and blocking."""
    x = np.asarray(x8, dtype=np.int8).astype(np.float64)
    w = np.asarray(w8, dtype=np.int8).astype(np.float64)
    if x.shape[1] != w.shape[1]:
        raise ValueError("K mismatch")
    if x.shape[1] >= (1 << 39):
        raise ValueError("K too large for exact fp64 integer sums")
    return (x @ w.T).astype(np.int64)


def int8_linear_ref(x8, s_tok, w8, s_ch) -> np.ndarray:
    """y as bf16 bit patterns (uint16 [M, N]):
    bf16_RN(fp32(fp32(fp32(acc) * s_tok[m]) * s_ch[n]))."""
    acc = int8_gemm_acc(x8, w8)
    a32 = acc.astype(np.float64).astype(np.float32)   # exact int -> one RN to fp32
    st = np.asarray(s_tok, dtype=np.float32)[:, None]
    sc = np.asarray(s_ch, dtype=np.float32)[None, :]
    y32 = ((a32 * st).astype(np.float32) * sc).astype(np.float32)
    return bf16_rne_bits(y32.astype(np.float64))
