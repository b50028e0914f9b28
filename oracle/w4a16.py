"""W4A16: int4 weights holding the QAT grid exactly, bf16 activations.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources:

* [SIZES] section "The Sizes and the Builds", format table: q4w4a16 = int4
  holding the QAT grid exactly, bf16 activations; section "The 4-Bit Builds
  Stay Slow at Every Size": the kernel unpacks the weights to bf16 before
  each multiply.
* [E2B] section "十种构建": the 4-bit repack restores each group's trained
  step and stores the values as int4 without rounding them again; "核心结论"
  item 2: it keeps the QAT grid exactly (90.0 % of values bit-identical).

The method's result is a plain definition: ``y[m, n] = sum_k x[m, k] *
d[n, k // 32] * q[n, k]`` over the exact QAT weights, rounded once to bf16.
This oracle evaluates that sum in fp64 (each product x * d * q is exact in
fp64 - 8 + 24 + 4 significant bits - and the K-term sum carries a relative
error below K * 2^-53, far under the acceptance bound).

Acceptance bound for a GPU result that, as the pages' kernel does, unpacks
the weights to bf16 before the multiply (each weight rounded once, relative
error <= 2^-9) and accumulates in fp32:
``|y - y_ref| <= 4e-3 * sum_k |x * w| + 1 ulp_bf16(y_ref)``, the same form
as the FP8 GEMM's bound.

The unpacked weight the GPU multiplies by is a plain definition too:
``bf16_RN(fp32(d * q))``, the QAT value (as the FP8 repack reads it) rounded
once to bf16 (``w4a16_unpacked_bits``); it is compared bit for bit.

Pinned by tests/test_oracle_w4a16.py: an exact-rational triple loop on small
shapes, one-hot activation rows (y = bf16 of one weight), the linearity
identities (negated x, doubled d), and the unpacked bf16 weights against
exact-rational rounding.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_rne_bits
from .quantize import qat_values, unpack_q4


def w4a16_weights(q4: np.ndarray, d: np.ndarray) -> np.ndarray:
    """The exact QAT weights d[n, k // 32] * q[n, k] in fp64."""
    q = unpack_q4(q4).astype(np.float64)
    d = np.asarray(d, dtype=np.float32).astype(np.float64)
    if d.shape[1] * 32 != q.shape[1]:
        raise ValueError("d must hold one scale per 32 values along K")
    return np.repeat(d, 32, axis=1) * q


def w4a16_linear_ref(x_bf16_bits, q4, d, return_abs: bool = False):
    """fp64 y = x . w^T over the exact QAT weights (and sum_k |x w| if asked)."""
    x = (np.asarray(x_bf16_bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    X = x.astype(np.float64)
    if not np.all(np.isfinite(X)):
        raise ValueError("non-finite activation")
    W = w4a16_weights(q4, d)
    y = X @ W.T
    if not return_abs:
        return y
    return y, np.abs(X) @ np.abs(W).T


def w4a16_unpacked_bits(q4: np.ndarray, d: np.ndarray) -> np.ndarray:
    """The bf16 weights the 4-bit build multiplies by: bf16_RN(fp32(d * q))
    as bit patterns (uint16 [N, K])."""
    return bf16_rne_bits(qat_values(q4, d).astype(np.float64))
