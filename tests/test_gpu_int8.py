"""GPU parity of the int8 W8A8 build against the CPU oracle, bit for bit:
per-token int8 quantization and the int8 QAT repack (codes and scales), and
the int8 GEMM (exact int32 sums, fp32 epilogue in a fixed order, one bf16
rounding), whose every output bit is fixed by the contract."""

import numpy as np
import pytest
import torch

from oracle import int8 as I8
from tests.gpu_util import bf16_to_np_bits, f32, same_bits_f32, to_dev
from workloads import activations_bf16, q4_weights

pytestmark = pytest.mark.gpu


def _i8(t):
    return t.cpu().numpy().astype(np.int8)


@pytest.mark.parametrize("M,K", [(1, 2048), (4, 256), (64, 5376), (300, 4096), (1000, 16),
                                 (1025, 2048), (4096, 704), (16384, 5376), (3000, 65536),
                                 (2049, 4096)])
def test_int8_quant_act_bit_exact(lib, M, K):
    xb = activations_bf16(M, K, seed=M + K, outlier_frac=0.01)
    ref = I8.quant_act_int8(xb)
    x8, st = lib.int8_quant_act(to_dev(xb))
    assert np.array_equal(_i8(x8), ref.codes) and same_bits_f32(f32(st), ref.scales)
    assert lib.device_status() == 0


def test_int8_quant_act_special_rows(lib):
    K = 512
    xb = activations_bf16(8, K, seed=9)
    xb[1] = 0                                   # zero row: s = 0, codes 0
    xb[2] = 0x8000                              # -0 row
    xb[3, :] = 0x3F80                           # all 1.0: codes 127
    xb[4, 5] = 0x7FC0                           # NaN: flagged
    xb[5, :] = 0x0001                           # smallest subnormal everywhere
    x8, st = lib.int8_quant_act(to_dev(xb))
    assert lib.device_status() & lib.DEV_NONFINITE
    ref = I8.quant_act_int8(xb)
    ok = np.ones(8, bool)
    ok[4] = False
    assert np.array_equal(_i8(x8)[ok], ref.codes[ok]) and same_bits_f32(f32(st)[ok], ref.scales[ok])
    assert np.all(_i8(x8)[3] == 127) and f32(st)[1] == 0


@pytest.mark.parametrize("N,K", [(128, 256), (300, 2048), (4096, 704), (21504, 5376), (8192, 96)])
def test_int8_repack_bit_exact(lib, N, K):
    q4, d = q4_weights(N, K, seed=N + K)
    ref = I8.repack_qat_int8(q4, d)
    w8, sc = lib.int8_repack_qat(to_dev(q4), to_dev(d))
    assert np.array_equal(_i8(w8), ref.codes) and same_bits_f32(f32(sc), ref.scales)
    assert lib.device_status() == 0


def _operands(M, N, K, seed):
    K32 = -(-K // 32) * 32
    q4, d = q4_weights(N, K32, seed=seed)
    w = I8.repack_qat_int8(q4, d)
    wc = np.ascontiguousarray(w.codes[:, :K])
    xb = activations_bf16(M, K, seed=seed + 1, outlier_frac=0.01)
    a = I8.quant_act_int8(xb)
    return xb, a, wc, w.scales


INT8_GEMM_SHAPES = [
    (1, 128, 16), (4, 128, 256), (3, 200, 48), (17, 1000, 272), (33, 130, 4096),
    (64, 8190, 512), (128, 520, 1040), (129, 520, 1040), (255, 256, 128),
    (1000, 1000, 2000), (2048, 2304, 4096), (300, 4096, 5376),
    (5, 6000, 1040), (3, 4000, 2096), (120, 19000, 512), (200, 1001, 256),
    (600, 1003, 4096), (700, 2056, 4096), (300, 520, 704), (1000, 1024, 416),
    (1, 8192, 2048), (8, 8192, 2048), (64, 8192, 2048),
    (1, 256, 65536), (16, 256, 65536), (300, 256, 65536),
    (2048, 2560, 1024), (2000, 2504, 1040),   # more pair tiles than pairs, ragged
]


@pytest.mark.parametrize("M,N,K", INT8_GEMM_SHAPES)
def test_int8_gemm_bit_exact(lib, M, N, K):
    xb, a, wc, sc = _operands(M, N, K, seed=M + 7 * N + K)
    y = lib.int8_rowwise_linear(to_dev(a.codes), to_dev(a.scales), to_dev(wc), to_dev(sc))
    ref = I8.int8_linear_ref(a.codes, a.scales, wc, sc)
    got = bf16_to_np_bits(y)
    bad = got != ref
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:4])
    assert lib.device_status() == 0


# Shapes on CTA pairs with a partial last wave (148 SMs: 74 pairs), split
# by k-blocks when a workspace is given: ragged N, shifted and zero-filled
# last k-blocks, every tile split, six waves and a partial seventh.
INT8_SPLIT_SHAPES = [(1024, 14336, 4096), (700, 20001, 4096), (768, 19000, 4160),
                     (1000, 12800, 4112), (400, 12000, 8192), (2048, 14336, 4096)]


@pytest.mark.parametrize("M,N,K", INT8_SPLIT_SHAPES)
def test_int8_split_bit_exact(lib, M, N, K):
    """int8_rowwise_linear_ws: the k-block split's int32 parts add exactly,
    so every output bit is still the oracle's (all rows up to M = 1024, 96
    sampled rows above), on two calls with the same workspace."""
    xb, a, wc, sc = _operands(M, N, K, seed=M + 3 * N + K)
    x8, st, w8, s8 = to_dev(a.codes), to_dev(a.scales), to_dev(wc), to_dev(sc)
    ws = lib.linear_workspace()
    y1 = lib.int8_rowwise_linear_ws(x8, st, w8, s8, ws)
    y2 = lib.int8_rowwise_linear_ws(x8, st, w8, s8, ws)
    assert lib.device_status() == 0
    rows = np.arange(M) if M <= 1024 else np.random.default_rng(M).choice(M, 96, replace=False)
    ref = I8.int8_linear_ref(a.codes[rows], a.scales[rows], wc, sc)
    got = bf16_to_np_bits(y1)[rows]
    bad = got != ref
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:4])
    assert np.array_equal(bf16_to_np_bits(y2), bf16_to_np_bits(y1))


@pytest.mark.parametrize("M", [1, 64, 8192])
def test_int8_full_layer_sampled(lib, M):
    """The prefill layer K=4096, N=14336 at M = 1 / 64 / 8192: weights from the
    GPU repack (checked bit-exact), the one-call linear from bf16, and every
    output bit of 256 sampled rows (all rows for M <= 64)."""
    N, K = 14336, 4096
    q4, d = q4_weights(N, K, seed=2)
    w8, sc = lib.int8_repack_qat(to_dev(q4), to_dev(d))
    wr = I8.repack_qat_int8(q4, d)
    assert np.array_equal(_i8(w8), wr.codes) and same_bits_f32(f32(sc), wr.scales)
    xb = activations_bf16(M, K, seed=2 + M, outlier_frac=0.01)
    y = lib.int8_linear(to_dev(xb), w8, sc)
    rows = np.arange(M) if M <= 64 else np.random.default_rng(3).choice(M, 256, replace=False)
    a = I8.quant_act_int8(xb[rows])
    ref = I8.int8_linear_ref(a.codes, a.scales, wr.codes, wr.scales)
    assert np.array_equal(bf16_to_np_bits(y)[rows], ref)
    assert lib.device_status() == 0


def test_int8_one_call_is_the_two_calls(lib):
    N, K = 2048, 1024
    q4, d = q4_weights(N, K, seed=11)
    w8, sc = lib.int8_repack_qat(to_dev(q4), to_dev(d))
    for M in (1, 16, 100, 600):
        x = to_dev(activations_bf16(M, K, seed=M))
        y1 = lib.int8_linear(x, w8, sc)
        x8, st = lib.int8_quant_act(x)
        y2 = lib.int8_rowwise_linear(x8, st, w8, sc)
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
