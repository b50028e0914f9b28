"""The no-allocation linear entry point, fp8_linear_bf16_noalloc.

Some callers cannot allocate device memory at all - for instance a plugin
that a host framework hands only fixed input and output buffers because the
framework owns all of device memory, or a latency-critical serving loop that
cannot take cudaMalloc's implicit device synchronization. For them the library
keeps the quantized activations in its own fixed device scratch array. These
tests call that entry point through the C ABI and check, on two calls in a row
with different inputs, that its output matches the regular fp8_linear_bf16
entry point's within the GEMM tolerance every test here uses (and, as the
kernels are the same, bit for bit); and that a problem too large for the
scratch array is refused before anything runs.
"""

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import bf16_to_np_bits, bf16_values, to_dev
from workloads import activations_bf16, q4_weights

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT_STATUS = 6  # FP8_ERR_SCRATCH_LIMIT


def _noalloc(lib, x, w8, s_ch, y):
    M, K = x.shape
    N = w8.shape[0]
    return lib.raw.fp8_linear_bf16_noalloc(x.data_ptr(), w8.data_ptr(), s_ch.data_ptr(), M, N, K,
                                           y.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,N,K", [(1, 8192, 2048), (64, 8192, 2048), (300, 1024, 4096)])
def test_noalloc_matches_regular_entry_point_on_two_calls(lib, M, N, K):
    q4, d = q4_weights(N, K, seed=31)
    w = oracle.repack_qat(q4, d)
    w8, s_ch = to_dev(w.codes), to_dev(w.scales)
    for seed in (41, 42):
        xb = activations_bf16(M, K, seed=seed, outlier_frac=0.01)
        x = to_dev(xb)
        y_regular = lib.linear(x, w8, s_ch)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(lib, x, w8, s_ch, y) == 0
        torch.cuda.synchronize()
        a = oracle.quant_act(xb)
        _, abs_scaled = oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales,
                                                  return_abs=True)
        ok, worst = oracle.check_linear(bf16_values(y), bf16_values(y_regular), abs_scaled)
        assert ok, f"worst error / tolerance = {worst}"
        assert np.array_equal(bf16_to_np_bits(y), bf16_to_np_bits(y_regular))
    assert lib.device_status() == 0


def test_noalloc_refuses_problems_beyond_its_scratch(lib):
    M, N, K = 1024, 256, 4096          # 4 MiB of codes + 4 KiB of scales: one block too many
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    w8 = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    s_ch = torch.ones((N,), dtype=torch.float32, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, x, w8, s_ch, y) == SCRATCH_LIMIT_STATUS
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())        # nothing was enqueued
