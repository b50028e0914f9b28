"""The bounded in-kernel waits, exercised on the GPU without a fault: a test
hook lowers the wait limit to 2^16 cycles and makes CTA 0 of the decode GEMM
skip one pipeline step (no arrive, no copies, so nothing is outstanding on
the barrier it leaves empty). The call must return promptly, the device
status must read FP8_DEV_TIMEOUT, and a normal call afterwards must be
correct with a clean status."""

import time

import numpy as np
import pytest

import oracle
from tests.gpu_util import bf16_values, to_dev
from workloads import activations_bf16, q4_weights

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed):
    q4, d = q4_weights(N, K, seed=seed)
    w = oracle.repack_qat(q4, d)
    a = oracle.quant_act(activations_bf16(M, K, seed=seed + 1, outlier_frac=0.01))
    return a, w


# (M, N, K, dropped step): K split 8 ways over a cluster (2 tiles), then one
# CTA per 128 channels without a split (more tiles than SMs)
@pytest.mark.parametrize("M,N,K,step", [(1, 256, 8192, 2), (8, 21504, 5376, 0), (64, 512, 4096, 1)])
def test_a_dropped_stage_times_out_and_the_device_stays_usable(lib, M, N, K, step):
    a, w = _operands(M, N, K, seed=M + N)
    x8, st, w8, sc = (to_dev(a.codes), to_dev(a.scales), to_dev(w.codes), to_dev(w.scales))
    lib.device_status()
    lib.test_set_fault(1 << 16, step)
    try:
        t0 = time.perf_counter()
        lib.rowwise_linear(x8, st, w8, sc)
        status = lib.device_status()          # synchronizes
        elapsed = time.perf_counter() - t0
    finally:
        lib.test_set_fault(0, -1)
    assert status & lib.DEV_TIMEOUT
    # the other roles left at once: well under the default one-second limit
    assert elapsed < 0.5, elapsed
    y = lib.rowwise_linear(x8, st, w8, sc)
    y_ref, abs_s = oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales, return_abs=True)
    ok, worst = oracle.check_linear(bf16_values(y), y_ref, abs_s)
    assert ok, worst
    assert lib.device_status() == 0
