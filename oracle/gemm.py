"""Row-wise scaled FP8 GEMM: ``y[m, n] = (sum_k x8[m,k] * w8[n,k]) * s_tok[m] * s_ch[n]``.

Sources: [E2B] step 3 boot log and tip "E4M3 还是 E4M3FNUZ" — vLLM selects
RowWiseTorchFP8ScaledMMLinearKernel for the CompressedTensorsW8A8Fp8 scheme;
[CARD] "vLLM picked RowWiseTorchFP8ScaledMMLinearKernel"; [CARD] header
paragraph — per-output-channel fp32 weight scales, per-token activation
scales, bf16 other tensors. The output is bf16.

Exactness: every E4M3 value is an integer multiple of 2^-9 (the smallest
subnormal) below 448, so every product is an integer multiple of 2^-18 of
magnitude at most 448^2 < 2^18, i.e. fewer than 2^36 units of 2^-18. Every
partial sum of K such terms is again an integer number of units, fewer than
K * 2^36; for K < 2^17 that is below 2^53, so fp64 (53-bit significand) holds
every partial sum exactly, in any order. Hence the fp64 matrix product below
(a library primitive) is the exact integer-scaled dot product, whatever
blocking the library uses, for any K < 2^17; larger K is refused.

Acceptance bound (the contract for the GPU result, which accumulates in fp32
in an order this oracle does not fix):
``|y - y_ref| <= 4e-3 * s_tok * s_ch * sum_k |x8 * w8| + 1 ulp_bf16(y_ref)``.

Pinned by tests/test_oracle_gemm.py against an exact-rational triple loop on
small shapes, exact integer sums at K = 65536 with the largest products and
the smallest units mixed, one-hot rows, negation and scale-doubling
identities.
"""

from __future__ import annotations

import numpy as np

from .formats import dec_e4m3

GEMM_REL_TOL = 4e-3
_MAX_EXACT_K = 1 << 17


def _dec(codes) -> np.ndarray:
    v = dec_e4m3(codes)
    if np.isnan(v).any():
        raise ValueError("E4M3 NaN code in GEMM operand")
    return v


def rowwise_linear_ref(x8, s_tok, w8, s_ch, return_abs: bool = False):
    """Exact fp64 reference (the scale products in fp64)."""
    x8 = np.asarray(x8, dtype=np.uint8)
    w8 = np.asarray(w8, dtype=np.uint8)
    if x8.shape[1] != w8.shape[1]:
        raise ValueError("K mismatch")
    if x8.shape[1] >= _MAX_EXACT_K:
        raise ValueError("K too large for the exact fp64 accumulation argument")
    A = _dec(x8)
    B = _dec(w8)
    acc = A @ B.T
    st = np.asarray(s_tok, dtype=np.float64)[:, None]
    sc = np.asarray(s_ch, dtype=np.float64)[None, :]
    y = acc * st * sc
    if not return_abs:
        return y
    absacc = np.abs(A) @ np.abs(B).T
    return y, absacc * np.abs(st) * np.abs(sc)


def bf16_ulp(y: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |y| (subnormal spacing 2^-133 below 2^-126)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.exp2(e - 7.0), 2.0 ** -133)


def rowwise_linear_tolerance(y_ref: np.ndarray, abs_scaled: np.ndarray) -> np.ndarray:
    return GEMM_REL_TOL * abs_scaled + bf16_ulp(y_ref)


def check_linear(y_gpu: np.ndarray, y_ref: np.ndarray, abs_scaled: np.ndarray):
    """Compare a GPU output (float64 values of its bf16 results) with the
    reference. Returns ``(ok, worst_ratio)`` where ratio = err / tolerance."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    tol = rowwise_linear_tolerance(y_ref, abs_scaled)
    err = np.abs(y_gpu - y_ref)
    ratio = np.where(np.isfinite(err), err / tol, np.inf)
    worst = float(np.max(ratio)) if ratio.size else 0.0
    return bool(worst <= 1.0), worst
