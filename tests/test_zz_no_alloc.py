"""The no-allocation linear entry point, fp8_linear_bf16_noalloc.

Some callers cannot allocate device memory at all - for instance a plugin
that a host framework hands only fixed input and output buffers because the
framework owns all of device memory, or a latency-critical serving loop that
cannot take cudaMalloc's implicit device synchronization. For them the library
keeps the quantized activations in its own fixed device scratch array. These
tests call that entry point through the C ABI and check, on two calls in a row
with different inputs, that its output is within the GEMM tolerance every test
here uses of the oracle's exact result and bit for bit the regular
fp8_linear_bf16 entry point's (the kernels are the same); that two calls
enqueued back to back on one stream with no host synchronization - the second
with fewer tokens, so its scales sit at another offset of the shared array -
each give their own correct result; and that a problem too large for the
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
        y_ref, abs_scaled = oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales,
                                                      return_abs=True)
        ok, worst = oracle.check_linear(bf16_values(y), y_ref, abs_scaled)
        assert ok, f"worst error / tolerance = {worst}"
        assert np.array_equal(bf16_to_np_bits(y), bf16_to_np_bits(y_regular))
    assert lib.device_status() == 0


@pytest.mark.parametrize("N,K,Ms", [(8192, 2048, (64, 8)), (1024, 2048, (1000, 300))])
def test_noalloc_back_to_back_on_one_stream(lib, N, K, Ms):
    """Two calls with different inputs enqueued on one stream with no host
    synchronization in between: the second call's quantizer may only rewrite
    the shared scratch once the first call's GEMM has read it. The second call
    has fewer tokens, so its per-token scales start at another offset of the
    array than the first call's; it goes through the Python wrapper."""
    q4, d = q4_weights(N, K, seed=33)
    w = oracle.repack_qat(q4, d)
    w8, s_ch = to_dev(w.codes), to_dev(w.scales)
    xbs = [activations_bf16(M, K, seed=60 + i, outlier_frac=0.01) for i, M in enumerate(Ms)]
    xs = [to_dev(xb) for xb in xbs]
    ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for M in Ms]
    torch.cuda.synchronize()
    assert _noalloc(lib, xs[0], w8, s_ch, ys[0]) == 0
    lib.linear_noalloc(xs[1], w8, s_ch, y=ys[1])
    torch.cuda.synchronize()
    for xb, y in zip(xbs, ys):
        a = oracle.quant_act(xb)
        y_ref, abs_scaled = oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales,
                                                      return_abs=True)
        ok, worst = oracle.check_linear(bf16_values(y), y_ref, abs_scaled)
        assert ok, f"worst error / tolerance = {worst}"
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
