"""GPU parity of the W4A16 build against the CPU oracle: the unpacked bf16
weights bf16(fp32(d q)) bit for bit, and the GEMM - with the weights unpacked
on chip (M <= 128) or into the workspace (longer M) - within
|y - y_exact| <= 4e-3 sum_k |x w| + 1 bf16 ulp of the exact sum over the QAT
weights, element by element."""

import numpy as np
import pytest
import torch

import oracle
from oracle import w4a16 as W
from tests.gpu_util import bf16_to_np_bits, bf16_values, to_dev
from workloads import activations_bf16, q4_weights

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(128, 256), (300, 2048), (8192, 2048), (21504, 5376), (7, 96)])
def test_unpacked_weights_bit_exact(lib, N, K):
    q4, d = q4_weights(N, K, seed=N + K)
    w = lib.w4a16_dequant(to_dev(q4), to_dev(d))
    assert np.array_equal(bf16_to_np_bits(w), W.w4a16_unpacked_bits(q4, d))


def _check(y, xb, q4, d, rows=None):
    xr = xb if rows is None else xb[rows]
    ref, a = W.w4a16_linear_ref(xr, q4, d, return_abs=True)
    got = bf16_values(y) if rows is None else bf16_values(y)[rows]
    ok, worst = oracle.check_linear(got, ref, a)
    assert ok, f"worst error / tolerance = {worst}"


W4_SHAPES = [
    # on-chip unpacking (M <= 128, K % 128 == 0): splits, variants, ragged N
    (1, 128, 256), (1, 8192, 2048), (8, 8192, 2048), (64, 8192, 2048), (16, 256, 4096),
    (17, 1000, 2048), (33, 130, 1024), (3, 21504, 5376), (64, 21504, 5376), (5, 520, 32768),
    (65, 1024, 2048), (128, 14336, 4096), (100, 21504, 5376),
    # workspace path: M > 128, or K % 128 != 0
    (129, 1024, 2048), (300, 4096, 4096), (1000, 1000, 2048), (4, 256, 96), (200, 1001, 224),
]


@pytest.mark.parametrize("M,N,K", W4_SHAPES)
def test_w4a16_linear_within_bound(lib, M, N, K):
    q4, d = q4_weights(N, K, seed=M + N + K)
    xb = activations_bf16(M, K, seed=M + 3, outlier_frac=0.01)
    y = lib.w4a16_linear(to_dev(xb), to_dev(q4), to_dev(d))
    _check(y, xb, q4, d)
    assert lib.device_status() == 0


def test_w4a16_workspace_is_required_and_sized(lib):
    assert lib.w4a16_workspace_bytes(128, 1024, 2048) == 0
    assert lib.w4a16_workspace_bytes(129, 1024, 2048) == 1024 * 2048 * 2
    assert lib.w4a16_workspace_bytes(8, 1024, 96) == 1024 * 96 * 2
    q4, d = q4_weights(256, 512, seed=1)
    x = to_dev(activations_bf16(200, 512, seed=1))
    y = torch.empty((200, 256), dtype=torch.bfloat16, device="cuda")
    small = torch.empty((256, 100), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.Fp8Error):
        lib.w4a16_linear(x, to_dev(q4), to_dev(d), y=y, ws=small)


@pytest.mark.parametrize("M", [1, 64, 8192])
def test_w4a16_prefill_layer_sampled(lib, M):
    """The prefill layer K=4096, N=14336 at M = 1, 64 and 8192 (the
    workspace path), on all rows (M <= 64) or 128 sampled rows."""
    N, K = 14336, 4096
    q4, d = q4_weights(N, K, seed=2)
    xb = activations_bf16(M, K, seed=2 + M, outlier_frac=0.01)
    y = lib.w4a16_linear(to_dev(xb), to_dev(q4), to_dev(d))
    rows = None if M <= 64 else np.random.default_rng(4).choice(M, 128, replace=False)
    _check(y, xb, q4, d, rows)


def test_w4a16_on_chip_equals_workspace_path(lib):
    """Both paths multiply by the same bf16 weights; with one token and no K
    split the decode kernel's fp32 sums may differ from the bf16 GEMM's only
    in accumulation order, so both stay within the bound of each other's
    exact reference (checked above) - and here, per element, within twice
    the bound of one another."""
    N, K, M = 2048, 1024, 16
    q4, d = q4_weights(N, K, seed=5)
    xb = activations_bf16(M, K, seed=6)
    y1 = bf16_values(lib.w4a16_linear(to_dev(xb), to_dev(q4), to_dev(d)))
    w = lib.w4a16_dequant(to_dev(q4), to_dev(d))
    y2 = bf16_values(lib.bf16_linear(to_dev(xb), w))
    ref, a = W.w4a16_linear_ref(xb, q4, d, return_abs=True)
    tol = oracle.rowwise_linear_tolerance(ref, a)
    assert np.all(np.abs(y1 - y2) <= 2 * tol)
