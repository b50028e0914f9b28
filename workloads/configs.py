"""Workload shapes of the FP8 W8A8 linear path.

The shapes follow the pages' workloads: the Gemma 4 E2B per-token GEMM
microbenchmark at 1/8/64 rows (geoz.com.cn MI300X E2B article, step 2 table),
the serving grid of 1/8/64 requests by 128/1,024/8,192-token prompts (same
article, step 5; dev.to Gemma 4 sizes article, step 3), the 31B-class dense
layer and the 26B-A4B mixture-of-experts layer with 128 experts of
intermediate size 704 (dev.to article, "Why the Mixture-of-Experts Model Sits
Lower").
"""

from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class DecodeShapes:
    """One dense linear ``y[M, N] = x[M, K] . w[N, K]^T`` at several M."""

    name: str
    K: int
    N: int
    Ms: tuple
    seed: int
    outlier_frac: float
    fnuz_copy: bool = False
    repack: bool = False
    notes: str = ""


@dataclass(frozen=True)
class MoEShapes:
    name: str
    tokens: int
    hidden: int
    inter: int
    experts: int
    top_k: int
    seed: int
    outlier_frac: float
    notes: str = ""


CONFIGS = {
    "tiny": DecodeShapes(
        name="tiny", K=256, N=128, Ms=(4,), seed=0, outlier_frac=0.0,
        notes="tiny W8A8 linear, M=4 K=256 N=128, seed 0, no outlier channels"),
    "decode": DecodeShapes(
        name="decode", K=2048, N=8192, Ms=(1, 8, 64), seed=1, outlier_frac=0.01,
        notes="decode GEMM sweep, K=2048 N=8192, M in {1,8,64}, 1% outlier channels x20"),
    "prefill": DecodeShapes(
        name="prefill", K=4096, N=14336, Ms=(128, 1024, 8192), seed=2, outlier_frac=0.01,
        fnuz_copy=True,
        notes="prefill GEMM, K=4096 N=14336, M in {128,1024,8192}, with an E4M3FNUZ-stored copy"),
    "large": DecodeShapes(
        name="large", K=5376, N=21504, Ms=(1, 64, 65536), seed=3, outlier_frac=0.01,
        repack=True,
        notes="large dense layer K=5376 N=21504, M in {1,64,65536}, plus the standalone repack"),
    "moe": MoEShapes(
        name="moe", tokens=8192, hidden=2048, inter=704, experts=128, top_k=8, seed=4,
        outlier_frac=0.01,
        notes="MoE layer: 128 experts gate/up/down (hidden 2048, inter 704), 8192 tokens top-8"),
}


def workload(name: str):
    return CONFIGS[name]
