"""Mixture-of-experts layer around the row-wise FP8 GEMM.

Source: [SIZES] section "Step 1 - Build the Larger Repacks" (26B-A4B has 128
experts per layer; the fused banks experts.gate_up_proj / experts.down_proj
are split into one gate/up/down module per expert; the router stays bf16) and
section "Why the Mixture-of-Experts Model Sits Lower" (each token goes through
a few of the 128 experts; the fp8_w8a8 expert kernel for E=128, N=704).

Readings where the pages are silent (listed in the design notes):

* Routing is an input (seeded, uniform top-k); the tokens of one expert are
  taken in ascending (token, slot) order, i.e. a stable sort of the flattened
  token-major [T, k] expert ids by expert.
* Activations are quantized once per token (the scale is per token, so it
  does not depend on the expert); an expert's rows are gathered copies.
* The expert MLP is GeGLU with the tanh-approximated GELU:
  h = bf16(gelu_tanh(gate) * up), computed here in fp64 (relative accuracy
  near 1e-15 for every gate, the far negative tail included) and rounded once
  to bf16; h is quantized per row like any activation.
* The combine weights are uniform, 1/k, unless given (the router's), and the
  sum runs in slot order.
* The router (router.proj, bf16 in every build) is a bf16 linear: logits =
  bf16(x . Wr^T) with the products summed exactly here in fp64; its expert
  choice takes the top_k largest logits, ties to the lower expert index, and
  the renormalized softmax over the chosen logits as weights (the pages give
  no router weights).

Pinned by tests/test_oracle_moe.py: a hand-worked routing example, the
stable-order and counting invariants, gelu_tanh against torch's
approximate='tanh' GELU in fp64 (a library routine), against a 300-digit
decimal evaluation of 0.5 x (1 + tanh v) with tanh from its exponential
definition (relative error, the far negative tail included) and its
closed-form limits, the grouped GEMM against an exact-rational triple loop on a tiny
two-expert case and against the dense GEMM when every token picks the same
expert, and the combine against a direct per-token sum, an exact-rational
weighted sum and a hand-worked weighted case; the router GEMM against an
exact-rational triple loop, the top-k choice against a hand-worked example
with ties and the weights against the two-expert closed form (a logistic).
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_rne_bits
from .gemm import rowwise_linear_ref


def route_sort(topk_ids: np.ndarray, num_experts: int):
    """Group the (token, slot) pairs by expert.

    Returns ``perm`` (int32 [T*k]: the flat index token*k + slot of each row
    of the expert-sorted order), ``inv`` (its inverse) and ``offsets``
    (int32 [E+1]: expert e owns rows offsets[e]:offsets[e+1])."""
    ids = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    if ids.size and (ids.min() < 0 or ids.max() >= num_experts):
        raise ValueError("expert id out of range")
    perm = np.argsort(ids, kind="stable").astype(np.int32)
    counts = np.bincount(ids, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return perm, inv, offsets


def gather_rows(x8: np.ndarray, s_tok: np.ndarray, perm: np.ndarray, top_k: int):
    """Rows of the per-token quantized activations in expert-sorted order."""
    tok = np.asarray(perm, dtype=np.int64) // top_k
    return np.ascontiguousarray(np.asarray(x8)[tok]), np.asarray(s_tok, np.float32)[tok]


def grouped_linear_ref(x8s, s_rows, offsets, w8, s_ch, return_abs: bool = False):
    """Per-expert row-wise scaled GEMM: rows offsets[e]:offsets[e+1] of x8s
    against expert e's weight w8[e] ([N, K]) and scales s_ch[e] ([N])."""
    x8s = np.asarray(x8s, np.uint8)
    E = len(offsets) - 1
    N = np.asarray(w8).shape[1]
    y = np.zeros((x8s.shape[0], N), dtype=np.float64)
    a = np.zeros_like(y) if return_abs else None
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        res = rowwise_linear_ref(x8s[r0:r1], np.asarray(s_rows)[r0:r1], w8[e], s_ch[e],
                                 return_abs=return_abs)
        if return_abs:
            y[r0:r1], a[r0:r1] = res
        else:
            y[r0:r1] = res
    return (y, a) if return_abs else y


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """0.5 x (1 + tanh(v)), v = sqrt(2/pi) (x + 0.044715 x^3), in fp64.

    Evaluated through the identity 0.5 (1 + tanh v) = 1 / (1 + exp(-2v)):
    written as 1 + tanh(v), the sum cancels for v << 0 (tanh(v) rounds to -1
    in fp64 for x below about -7, leaving no correct digit), while the
    quotient keeps fp64's relative accuracy for every x (exp(-2v) overflows
    to inf only where the exact value is below 1e-300)."""
    x = np.asarray(x, dtype=np.float64)
    v = np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-2.0 * v))


def geglu_bf16(gate_up_bits: np.ndarray, inter: int) -> np.ndarray:
    """h = bf16(gelu_tanh(gate) * up) from a [M, 2*inter] bf16 (uint16 bits)
    matrix holding gate in the first half and up in the second."""
    g = np.asarray(gate_up_bits, dtype=np.uint16)
    vals = (g.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    gate, up = vals[:, :inter], vals[:, inter:2 * inter]
    return bf16_rne_bits(gelu_tanh(gate) * up)


def combine(y_rows: np.ndarray, inv: np.ndarray, tokens: int, top_k: int,
            weights: np.ndarray | None = None) -> np.ndarray:
    """out[t] = sum_j w[t, j] * y_rows[inv[t*k + j]] in fp64."""
    y_rows = np.asarray(y_rows, dtype=np.float64)
    w = np.full((tokens, top_k), 1.0 / top_k) if weights is None else np.asarray(weights, np.float64)
    idx = np.asarray(inv, dtype=np.int64).reshape(tokens, top_k)
    out = np.zeros((tokens, y_rows.shape[1]), dtype=np.float64)
    for j in range(top_k):
        out += w[:, j:j + 1] * y_rows[idx[:, j]]
    return out


def bf16_linear_ref(x_bits, w_bits, return_abs: bool = False):
    """y = x . w^T in fp64 from bf16 operands (uint16 patterns). Each product
    of two bf16 values is exact in fp64 (16 significant bits); the sum is
    fp64's, with relative error below K 2^-53. The contract for a GPU result
    accumulated in fp32 (any order): |y - y_ref| <= K 2^-24 sum|x w| + 1 bf16
    ulp (bf16_linear_tolerance)."""
    X = (np.asarray(x_bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    W = (np.asarray(w_bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    y = X @ W.T
    if not return_abs:
        return y
    return y, np.abs(X) @ np.abs(W).T


def bf16_linear_tolerance(y_ref, abs_sum, K):
    from .gemm import bf16_ulp
    return K * 2.0 ** -24 * np.asarray(abs_sum) + bf16_ulp(y_ref)


def topk_softmax(logits_bits, top_k: int):
    """Router choice: per token the top_k largest logits (bf16 patterns
    [T, E]), in descending order, ties to the lower expert index; weights =
    exp(l_j - l_max) / sum_i exp(l_i - l_max) over the chosen ones, in fp64.
    Returns (ids int32 [T, k], weights float64 [T, k])."""
    L = (np.asarray(logits_bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    T, E = L.shape
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx, -L), axis=1)[:, :top_k]     # key: -logit, then expert index
    ids = order.astype(np.int32)
    v = np.take_along_axis(L, order, axis=1)
    ex = np.exp(v - v[:, :1])
    return ids, ex / ex.sum(axis=1, keepdims=True)
