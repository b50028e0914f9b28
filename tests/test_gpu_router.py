"""GPU parity of the bf16 router: the bf16 GEMM (router.proj) within its
fp32-accumulation bound K 2^-24 sum|x w| + 1 bf16 ulp against the fp64
oracle, element by element; the top-k choice compared exactly with the
oracle's choice from the GPU's own logits (unique: ties go to the lower
expert index) and its softmax weights within 1e-6 relative."""

import numpy as np
import pytest
import torch

from oracle import moe
from tests.gpu_util import bf16_to_np_bits, bf16_values, f32, to_dev
from workloads import activations_bf16, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


def _bf16_normal(shape, seed, scale=1.0):
    return f32_to_bf16_bits((np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32))


@pytest.mark.parametrize("M,N,K", [(8192, 128, 2048), (1, 128, 2048), (64, 128, 2048), (300, 200, 520),
                                   (1000, 1000, 1024), (4, 8192, 2048), (129, 256, 64), (2048, 2304, 4096),
                                   (8, 384, 32768)])
def test_bf16_linear_within_bound(lib, M, N, K):
    xb = activations_bf16(M, K, seed=M + K, outlier_frac=0.01)
    wb = _bf16_normal((N, K), seed=N + K, scale=K ** -0.5)
    y = lib.bf16_linear(to_dev(xb), to_dev(wb))
    ref, a = moe.bf16_linear_ref(xb, wb, return_abs=True)
    tol = moe.bf16_linear_tolerance(ref, a, K)
    err = np.abs(bf16_values(y) - ref)
    assert np.all(err <= tol), float(np.max(err / tol))
    assert lib.device_status() == 0


@pytest.mark.parametrize("T,E,k", [(8192, 128, 8), (1, 128, 8), (333, 64, 4), (100, 1024, 16),
                                   (50, 8, 8), (77, 200, 2), (10, 256, 1)])
def test_topk_matches_oracle_on_gpu_logits(lib, T, E, k):
    logits = _bf16_normal((T, E), seed=T + E, scale=2.0)
    logits[: T // 4, :E // 2] = logits[: T // 4, E // 2: 2 * (E // 2)]   # many exact ties
    logits[T // 4: T // 2, ::3] = 0x0000                                 # +0 ...
    logits[T // 4: T // 2, 1::3] = 0x8000                                # ... and -0 tie by index
    ids, w = lib.moe_topk(to_dev(logits), k)
    rid, rw = moe.topk_softmax(logits, k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.all(np.abs(f32(w) - rw) <= 1e-6 * rw + 1e-30)
    assert lib.device_status() == 0


def test_router_chain_on_the_moe_workload(lib):
    """The MoE layer's router: x [8192, 2048] bf16 (the workload's activations)
    times a bf16 router [128, 2048], then top-8. The GEMM within its bound on
    every element; the top-k and weights from the GPU's logits exactly / to
    1e-6; every token's experts distinct."""
    T, H, E, k = 8192, 2048, 128, 8
    xb = activations_bf16(T, H, seed=4, outlier_frac=0.01)
    wr = _bf16_normal((E, H), seed=5, scale=H ** -0.5)
    logits = lib.bf16_linear(to_dev(xb), to_dev(wr))
    ref, a = moe.bf16_linear_ref(xb, wr, return_abs=True)
    assert np.all(np.abs(bf16_values(logits) - ref) <= moe.bf16_linear_tolerance(ref, a, H))
    ids, w = lib.moe_topk(logits, k)
    rid, rw = moe.topk_softmax(bf16_to_np_bits(logits), k)
    ids = ids.cpu().numpy()
    assert np.array_equal(ids, rid)
    assert np.all(np.abs(f32(w) - rw) <= 1e-6 * rw + 1e-30)
    assert all(len(set(r)) == k for r in ids)


def test_topk_flags_nonfinite_logits(lib):
    logits = _bf16_normal((16, 32), seed=3)
    logits[5, 7] = 0x7FC0          # NaN
    logits[9, 2] = 0x7F80          # +inf
    lib.moe_topk(to_dev(logits), 4)
    assert lib.device_status() & lib.DEV_NONFINITE
