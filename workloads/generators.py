"""Seeded generators for the synthetic workloads.

Every tensor comes from its own numpy PCG64 substream, keyed by ``(seed, tag)``,
so that changing one tensor's shape never shifts another tensor's numbers.

Recipes (the pages' model shapes with synthetic values, since no checkpoint is
available):

* QAT q4_0 grid weights (Gemma 4 QAT release: 4-bit grid, one scale per group
  of 32 values along K). ``d = fp32(|N(0, 0.02)| / 8)`` per group and
  ``q`` uniform on the integers ``[-8, 7]``. ``q`` is packed two per byte:
  element ``2j`` in the low nibble and ``2j+1`` in the high nibble, as 4-bit
  two's complement.
* Activations: ``bf16(N(0, 1))`` per element. With ``outlier_frac > 0`` a
  seeded set of ``round(outlier_frac * K)`` distinct channels holds
  ``bf16(20 * N(0, 1))`` for every token (the same channels for all tokens).
* MoE routing: every token picks ``top_k`` distinct experts uniformly at
  random (argsort of uniform keys, which gives every ordered k-subset the same
  probability).
"""

from __future__ import annotations

import numpy as np

# Substream tags, one per generated tensor.
_TAG_D = 1
_TAG_Q = 2
_TAG_X = 3
_TAG_OUTLIER_CH = 4
_TAG_OUTLIER_X = 5
_TAG_ROUTE = 6


def _rng(seed: int, tag: int, *extra: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag), *[int(e) for e in extra]])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even) and return
    the 16-bit patterns as uint16. Inputs must be finite."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 patterns (uint16) to fp32 exactly."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def q4_weights(N: int, K: int, seed: int, rows: slice | None = None):
    """QAT q4_0-grid weights for an ``[N, K]`` linear.

    Returns ``(q4, d)``: ``q4`` uint8 ``[N, K/2]`` (packed int4) and ``d``
    float32 ``[N, K/32]``. With ``rows`` only that row range is generated; the
    values are the same as in the full matrix (generation is row-blocked).
    """
    if K % 32 != 0:
        raise ValueError("K must be a multiple of 32 (q4_0 groups)")
    r0, r1 = (0, N) if rows is None else (rows.start or 0, N if rows.stop is None else rows.stop)
    # Row blocks of 256 make row-sliced generation reproduce the full matrix.
    blk = 256
    q4 = np.empty((r1 - r0, K // 2), dtype=np.uint8)
    d = np.empty((r1 - r0, K // 32), dtype=np.float32)
    for b0 in range((r0 // blk) * blk, r1, blk):
        b1 = min(b0 + blk, N)
        gd = _rng(seed, _TAG_D, N, K, b0)
        gq = _rng(seed, _TAG_Q, N, K, b0)
        dz = gd.standard_normal((b1 - b0, K // 32))
        db = (np.abs(dz * 0.02) / 8.0).astype(np.float32)
        qb = gq.integers(-8, 8, size=(b1 - b0, K), dtype=np.int8)
        nib = (qb.astype(np.uint8) & np.uint8(0x0F))
        pb = nib[:, 0::2] | (nib[:, 1::2] << np.uint8(4))
        s0, s1 = max(b0, r0), min(b1, r1)
        q4[s0 - r0:s1 - r0] = pb[s0 - b0:s1 - b0]
        d[s0 - r0:s1 - r0] = db[s0 - b0:s1 - b0]
    return q4, d


def outlier_channels(K: int, seed: int, outlier_frac: float) -> np.ndarray:
    n = int(round(outlier_frac * K))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    g = _rng(seed, _TAG_OUTLIER_CH, K)
    return np.sort(g.choice(K, size=n, replace=False))


def activations_bf16(M: int, K: int, seed: int, outlier_frac: float = 0.0,
                     rows: slice | None = None) -> np.ndarray:
    """Activations ``[M, K]`` as bf16 bit patterns (uint16).

    With ``rows`` only that token range is generated, with the same values as
    in the full matrix (generation is blocked by 1024 tokens).
    """
    r0, r1 = (0, M) if rows is None else (rows.start or 0, M if rows.stop is None else rows.stop)
    ch = outlier_channels(K, seed, outlier_frac)
    out = np.empty((r1 - r0, K), dtype=np.uint16)
    blk = 1024
    for b0 in range((r0 // blk) * blk, r1, blk):
        b1 = min(b0 + blk, M)
        g = _rng(seed, _TAG_X, K, b0)
        xb = g.standard_normal((b1 - b0, K), dtype=np.float32)
        if ch.size:
            go = _rng(seed, _TAG_OUTLIER_X, K, b0)
            xb[:, ch] = (20.0 * go.standard_normal((b1 - b0, ch.size))).astype(np.float32)
        s0, s1 = max(b0, r0), min(b1, r1)
        out[s0 - r0:s1 - r0] = f32_to_bf16_bits(xb[s0 - b0:s1 - b0])
    return out


def moe_routing(tokens: int, experts: int, top_k: int, seed: int) -> np.ndarray:
    """``[tokens, top_k]`` int32 expert ids, distinct within each token."""
    g = _rng(seed, _TAG_ROUTE, tokens, experts, top_k)
    keys = g.random((tokens, experts))
    return np.argsort(keys, axis=1)[:, :top_k].astype(np.int32)
