"""GPU parity of the row-wise scaled FP8 GEMM against the exact fp64 oracle:
|y - y_ref| <= 4e-3 * s_tok * s_ch * sum_k |x8*w8| + 1 bf16 ulp, element by
element (the whole output at moderate sizes, sampled rows at full size),
plus bit-exact identities the kernels must keep (determinism, the one-call
quantize+GEMM path, the FNUZ-converted weights, one-hot rows)."""

import numpy as np
import pytest
import torch

import oracle
from oracle import formats as F
from tests.gpu_util import bf16_to_np_bits, bf16_values, f32, same_bits_f32, to_dev, u8
from workloads import activations_bf16, q4_weights

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed, outl=0.01):
    """Oracle-quantized operands. For K that is not a whole number of q4_0
    groups the weight is the first K columns of a wider repacked weight (still
    a valid E4M3 weight with per-channel scales)."""
    K32 = -(-K // 32) * 32
    q4, d = q4_weights(N, K32, seed=seed)
    xb = activations_bf16(M, K, seed=seed, outlier_frac=outl)
    w = oracle.repack_qat(q4, d)
    if K32 != K:
        w = oracle.QuantResult(np.ascontiguousarray(w.codes[:, :K]), w.scales, w.bad_rows)
    a = oracle.quant_act(xb)
    return xb, a, w


def _check(y_gpu, a, w, rows=None):
    x8, st = (a.codes, a.scales) if rows is None else (a.codes[rows], a.scales[rows])
    y_ref, abs_s = oracle.rowwise_linear_ref(x8, st, w.codes, w.scales, return_abs=True)
    got = bf16_values(y_gpu) if rows is None else bf16_values(y_gpu)[rows]
    ok, worst = oracle.check_linear(got, y_ref, abs_s)
    assert ok, f"worst error / tolerance = {worst}"
    return worst


GEMM_SHAPES = [
    # (M, N, K): decode (swap-AB, split-K) and prefill (persistent) kernels,
    # ragged M / N / K tails, K shorter than one 128-byte stage.
    (4, 128, 256),
    (1, 128, 16),
    (3, 200, 48),
    (17, 1000, 272),
    (33, 130, 4096),
    (64, 8190, 512),
    (100, 384, 1024),
    (128, 520, 1040),
    (129, 520, 1040),
    (255, 256, 128),
    (1000, 1000, 2000),   # single-SM prefill at larger M (fewer waves than pairs would take)
    (2048, 2304, 4096),
    (300, 4096, 5376),
    (5, 6000, 1040),      # one CTA per SM, no split: the deep-ring decode variant
    (3, 4000, 2096),      # few tokens, narrow layer: K split 4 ways, ragged N and K
    (120, 19000, 512),    # more 128-channel tiles than SMs at M = 128
    (200, 1001, 256),     # single-SM prefill, N % 8 != 0: element stores
    (600, 1003, 4096),    # CTA pairs, N % 8 != 0
    (700, 2056, 4096),    # CTA pairs, ragged M and N: TMA-stored and fallback chunks
    # K % 128 in {32, 64, 96}: the last k-block is loaded at K - 128 and its
    # first 1-3 MMA k-steps are skipped (single-SM kernel, then CTA pairs)
    (300, 520, 704),
    (1000, 1024, 416),
    (600, 768, 224),
    (129, 256, 160),
    (1024, 2048, 4160),
    # more pair tiles than pairs, with a last partial wave of a few tiles
    (2048, 2560, 1024),
    (2000, 2504, 1040),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_within_bound(lib, M, N, K):
    xb, a, w = _operands(M, N, K, seed=M + N + K)
    y = lib.rowwise_linear(to_dev(a.codes), to_dev(a.scales), to_dev(w.codes), to_dev(w.scales))
    _check(y, a, w)
    assert lib.device_status() == 0


# The long reductions the C ABI accepts (K up to 65536): decode (swap-AB, K
# split over a cluster) and prefill (single SMs and CTA pairs), including a
# K that is not a multiple of 128 bytes.
LONG_K_SHAPES = [
    (1, 256, 8192),
    (16, 384, 16384),
    (1, 200, 65536),
    (16, 256, 65536),
    (300, 512, 8192),
    (1000, 256, 16384),
    (300, 256, 65536),
    (640, 264, 65536),
    (130, 256, 65520),
]


@pytest.mark.parametrize("M,N,K", LONG_K_SHAPES)
def test_long_k_within_bound(lib, M, N, K):
    xb, a, w = _operands(M, N, K, seed=M + N + K)
    y = lib.rowwise_linear(to_dev(a.codes), to_dev(a.scales), to_dev(w.codes), to_dev(w.scales))
    _check(y, a, w)
    assert lib.device_status() == 0


# Prefill shapes that run on CTA pairs whose tiles make a few waves with a
# partial last one (148 SMs: 74 pairs), so fp8_rowwise_linear_ws shares the
# last full wave and the partial one out by k-blocks: ragged N (N % 8 != 0),
# a shifted last k-block (K % 128 = 64), a zero-filled one (K % 128 = 16),
# every tile split (fewer than two waves), six waves and a partial seventh.
SPLIT_SHAPES = [
    (1024, 14336, 4096),
    (700, 20001, 4096),
    (768, 19000, 4160),
    (1000, 12800, 4112),
    (400, 12000, 8192),
    (2048, 14336, 4096),
]


@pytest.mark.parametrize("M,N,K", SPLIT_SHAPES)
def test_split_within_bound_and_reproducible(lib, M, N, K):
    """The k-block split (stream-K over the CTA pairs) stays within the
    row-wise GEMM bound, gives the same bits on a second call with the same
    workspace (whose flags every call leaves zero), and equals the plain call
    when the workspace is too small to split."""
    xb, a, w = _operands(M, N, K, seed=M + N + K + 7)
    x8, st, w8, sw = to_dev(a.codes), to_dev(a.scales), to_dev(w.codes), to_dev(w.scales)
    ws = lib.linear_workspace()
    y1 = lib.rowwise_linear_ws(x8, st, w8, sw, ws)
    y2 = lib.rowwise_linear_ws(x8, st, w8, sw, ws)
    assert lib.device_status() == 0
    rows = None if M * N * K <= 4e9 else np.unique(np.concatenate([
        np.arange(8), np.arange(M - 8, M), np.random.default_rng(M).choice(M, 48, replace=False)]))
    _check(y1, a, w, rows)
    assert np.array_equal(bf16_to_np_bits(y1), bf16_to_np_bits(y2))
    # the flags: what precedes the pairs' 256 KB parts
    nflag = int(lib.raw.fp8_linear_workspace_bytes()) % (2 * 128 * 256 * 4)
    assert not u8(ws)[:nflag].any()
    y0 = lib.rowwise_linear(x8, st, w8, sw)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    assert np.array_equal(bf16_to_np_bits(lib.rowwise_linear_ws(x8, st, w8, sw, small)), bf16_to_np_bits(y0))


def test_split_entry_edge_cases(lib):
    """fp8_rowwise_linear_ws: M = 0 and N = 0 do nothing, K = 0 gives zeros, a
    workspace that is not 16-byte aligned is refused, and a null workspace
    is the plain call (the same bits)."""
    raw, st_ = lib.raw, torch.cuda.current_stream().cuda_stream
    ws = lib.linear_workspace()
    nb = ws.numel()
    w8 = torch.zeros((256, 64), dtype=torch.uint8, device="cuda")
    s = torch.ones(256, dtype=torch.float32, device="cuda")
    x8 = torch.zeros((300, 64), dtype=torch.uint8, device="cuda")
    y = torch.full((300, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    assert raw.fp8_rowwise_linear_ws(x8.data_ptr(), s.data_ptr(), w8.data_ptr(), s.data_ptr(), 0, 256, 64,
                                     y.data_ptr(), ws.data_ptr(), nb, st_) == 0
    assert raw.fp8_rowwise_linear_ws(x8.data_ptr(), s.data_ptr(), w8.data_ptr(), s.data_ptr(), 300, 0, 64,
                                     y.data_ptr(), ws.data_ptr(), nb, st_) == 0
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
    assert raw.fp8_rowwise_linear_ws(x8.data_ptr(), s.data_ptr(), w8.data_ptr(), s.data_ptr(), 300, 256, 0,
                                     y.data_ptr(), ws.data_ptr(), nb, st_) == 0
    torch.cuda.synchronize()
    assert not bf16_to_np_bits(y).any()
    assert raw.fp8_rowwise_linear_ws(x8.data_ptr(), s.data_ptr(), w8.data_ptr(), s.data_ptr(), 300, 256, 64,
                                     y.data_ptr(), ws.data_ptr() + 8, nb - 8, st_) != 0
    xb, a, w = _operands(1024, 14336, 4096, seed=5)
    xd, sd, wd, swd = to_dev(a.codes), to_dev(a.scales), to_dev(w.codes), to_dev(w.scales)
    yn = torch.empty((1024, 14336), dtype=torch.bfloat16, device="cuda")
    assert raw.fp8_rowwise_linear_ws(xd.data_ptr(), sd.data_ptr(), wd.data_ptr(), swd.data_ptr(), 1024, 14336,
                                     4096, yn.data_ptr(), None, 0, st_) == 0
    y0 = lib.rowwise_linear(xd, sd, wd, swd)
    assert np.array_equal(bf16_to_np_bits(yn), bf16_to_np_bits(y0))
    assert lib.device_status() == 0


def test_k_beyond_the_limit_is_refused(lib):
    x8 = torch.zeros((1, 65552), dtype=torch.uint8, device="cuda")
    w8 = torch.zeros((128, 65552), dtype=torch.uint8, device="cuda")
    s = torch.ones(128, dtype=torch.float32, device="cuda")
    with pytest.raises(lib.Fp8Error):
        lib.rowwise_linear(x8, s[:1], w8, s)


@pytest.mark.parametrize("M", [1, 8, 64])
def test_decode_sweep_shapes(lib, M):
    """Decode GEMM sweep: K=2048, N=8192, activations with 1% outlier channels."""
    xb, a, w = _operands(M, 8192, 2048, seed=1)
    x8, s = lib.quant_act(to_dev(xb))
    assert np.array_equal(u8(x8), a.codes) and same_bits_f32(f32(s), a.scales)
    wd, sw = lib.repack_qat(*[to_dev(t) for t in q4_weights(8192, 2048, seed=1)])
    assert np.array_equal(u8(wd), w.codes) and same_bits_f32(f32(sw), w.scales)
    y = lib.rowwise_linear(x8, s, wd, sw)
    _check(y, a, w)


def test_deterministic_and_one_call_path(lib):
    for M, N, K in [(8, 4096, 2048), (64, 1024, 4096), (512, 2048, 1024)]:
        xb, a, w = _operands(M, N, K, seed=21)
        x8d, sd = to_dev(a.codes), to_dev(a.scales)
        wd, swd = to_dev(w.codes), to_dev(w.scales)
        y1 = bf16_to_np_bits(lib.rowwise_linear(x8d, sd, wd, swd))
        y2 = bf16_to_np_bits(lib.rowwise_linear(x8d, sd, wd, swd))
        assert np.array_equal(y1, y2)
        y3 = bf16_to_np_bits(lib.linear(to_dev(xb), wd, swd))
        assert np.array_equal(y1, y3)


def test_one_hot_rows_are_exact(lib):
    K, N = 256, 384
    rng = np.random.default_rng(4)
    w = oracle.repack_qat(*q4_weights(N, K, seed=4))
    M = 200
    ks = rng.integers(0, K, M)
    x8 = np.zeros((M, K), np.uint8)
    x8[np.arange(M), ks] = 0x38                       # 1.0
    st = np.full(M, 0.5, np.float32)
    y = bf16_values(lib.rowwise_linear(to_dev(x8), to_dev(st), to_dev(w.codes), to_dev(w.scales)))
    # a single product: the fp32 path is exact up to the final bf16 rounding
    prod = (F.dec_e4m3(w.codes[:, ks].T) * 0.5).astype(np.float32) * w.scales[None, :]
    expect = bf16_values(torch.from_numpy(prod.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(y, expect)


def test_negated_activations_negate_output(lib):
    M, N, K = 96, 512, 768
    xb, a, w = _operands(M, N, K, seed=8)
    args = (to_dev(w.codes), to_dev(w.scales))
    y = bf16_values(lib.rowwise_linear(to_dev(a.codes), to_dev(a.scales), *args))
    neg = np.where(a.codes != 0, a.codes ^ 0x80, 0).astype(np.uint8)
    yn = bf16_values(lib.rowwise_linear(to_dev(neg), to_dev(a.scales), *args))
    assert np.array_equal(yn, -y)


@pytest.fixture(scope="module")
def prefill_weights():
    q4, d = q4_weights(14336, 4096, seed=2)
    return q4, d, oracle.repack_qat(q4, d)


def test_prefill_with_fnuz_weights_matches_e4m3_path(lib, prefill_weights):
    """Prefill GEMM (K=4096, N=14336) from an E4M3FNUZ-stored copy of the
    weights, converted at load, gives the same bits as from the E4M3 repack."""
    q4, d, w = prefill_weights
    wd, sw = lib.repack_qat(to_dev(q4), to_dev(d))
    assert np.array_equal(u8(wd), w.codes) and same_bits_f32(f32(sw), w.scales)
    cn, sn = oracle.fnuz_copy_of_e4m3(w.codes, w.scales)
    wf, sf = lib.convert_fnuz(to_dev(cn), to_dev(sn))
    assert np.array_equal(u8(wf), w.codes) and same_bits_f32(f32(sf), w.scales)
    for M in (128, 1024):
        xb = activations_bf16(M, 4096, seed=2, outlier_frac=0.01)
        x8, s = lib.quant_act(to_dev(xb))
        y1 = bf16_to_np_bits(lib.rowwise_linear(x8, s, wd, sw))
        y2 = bf16_to_np_bits(lib.rowwise_linear(x8, s, wf, sf))
        assert np.array_equal(y1, y2)
    assert lib.device_status() == 0


@pytest.mark.parametrize("M", [128, 1024, 8192])
def test_prefill_shapes_sampled(lib, prefill_weights, M):
    """Prefill GEMM, K=4096, N=14336: every output of 64 sampled rows (all of
    them at M=128) against the oracle."""
    q4, d, w = prefill_weights
    xb = activations_bf16(M, 4096, seed=2, outlier_frac=0.01)
    x8, s = lib.quant_act(to_dev(xb))
    y = lib.rowwise_linear(x8, s, to_dev(w.codes), to_dev(w.scales))
    rows = np.arange(M) if M <= 128 else np.sort(np.random.default_rng(M).choice(M, 64, replace=False))
    a = oracle.quant_act(xb[rows])
    assert np.array_equal(u8(x8)[rows], a.codes)
    y_ref, abs_s = oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales, return_abs=True)
    ok, worst = oracle.check_linear(bf16_values(y)[rows], y_ref, abs_s)
    assert ok, worst


@pytest.mark.parametrize("M", [1, 64, 65536])
def test_large_layer_sampled(lib, M):
    """Large dense layer K=5376, N=21504 from the GPU repack of its q4_0 grid:
    512 sampled weight rows bit-exact against the oracle repack, and the
    outputs of sampled token rows on those channels within the bound, at the
    sizes the benchmark runs."""
    N, K = 21504, 5376
    q4, d = q4_weights(N, K, seed=3)
    wd, sw = lib.repack_qat(to_dev(q4), to_dev(d))
    cols = np.sort(np.random.default_rng(1).choice(N, 512, replace=False))
    w = oracle.repack_qat(q4[cols], d[cols])
    assert np.array_equal(u8(wd)[cols], w.codes) and same_bits_f32(f32(sw)[cols], w.scales)
    xb = activations_bf16(M, K, seed=3, outlier_frac=0.01)
    x8 = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    st = torch.empty((M,), dtype=torch.float32, device="cuda")
    y = lib.linear(to_dev(xb), wd, sw, x8=x8, s_tok=st)
    rows = np.arange(M) if M <= 64 else np.sort(np.random.default_rng(M).choice(M, 32, replace=False))
    a = oracle.quant_act(xb[rows])
    assert np.array_equal(u8(x8)[rows], a.codes) and same_bits_f32(f32(st)[rows], a.scales)
    y_ref, abs_s = oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales, return_abs=True)
    ok, worst = oracle.check_linear(bf16_values(y)[rows][:, cols], y_ref, abs_s)
    assert ok, worst
    assert lib.device_status() == 0


@pytest.mark.parametrize("M,N,K", [(1, 8192, 2048), (3, 8192, 2064), (8, 8192, 2048),
                                   (16, 6144, 1024), (1, 21504, 5376), (16, 8192, 2048),
                                   (4, 8192, 8176), (5, 8192, 8176), (4, 8192, 2048),
                                   (2, 6144, 4096), (1, 1024, 4096)])
def test_linear_from_bf16_is_bit_identical_to_two_calls(lib, M, N, K):
    """fp8_linear_bf16 on decode batches: its codes and scales equal the
    oracle's, and y equals fp8_quant_act followed by fp8_rowwise_linear bit
    for bit (one- and two-wave tile counts, a K tail, a narrow layer whose K
    is split)."""
    xb, a, w = _operands(M, N, K, seed=40 + M)
    wd, sd = to_dev(w.codes), to_dev(w.scales)
    x8 = torch.full((M, K), 0x7F, dtype=torch.uint8, device="cuda")
    st = torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
    y_fused = lib.linear(to_dev(xb), wd, sd, x8=x8, s_tok=st)
    assert np.array_equal(u8(x8), a.codes) and same_bits_f32(f32(st), a.scales)
    x8b, stb = lib.quant_act(to_dev(xb))
    y_two = lib.rowwise_linear(x8b, stb, wd, sd)
    assert np.array_equal(bf16_to_np_bits(y_fused), bf16_to_np_bits(y_two))
    _check(y_fused, a, w)
    assert lib.device_status() == 0


def test_bf16_weights_quantized_per_channel_online(lib):
    """bf16 weights quantized per output channel at load time (the vLLM
    fp8_per_channel path for bf16 checkpoints): fp8_quant_act over the
    weight rows gives one amax/448 scale per channel, bit-exact against the
    oracle, and the GEMM with those weights stays within the bound."""
    M, N, K = 37, 3000, 2048
    wb = activations_bf16(N, K, seed=41)                  # bf16 weight rows [N, K]
    xb = activations_bf16(M, K, seed=42, outlier_frac=0.01)
    w_ref = oracle.quant_act(wb)
    a = oracle.quant_act(xb)
    w8, s_ch = lib.quant_act(to_dev(wb))
    assert np.array_equal(u8(w8), w_ref.codes) and same_bits_f32(f32(s_ch), w_ref.scales)
    y = lib.linear(to_dev(xb), w8, s_ch)
    y_ref, abs_s = oracle.rowwise_linear_ref(a.codes, a.scales, w_ref.codes, w_ref.scales,
                                             return_abs=True)
    ok, worst = oracle.check_linear(bf16_values(y), y_ref, abs_s)
    assert ok, worst
    assert lib.device_status() == 0


@pytest.mark.parametrize("M,K,Ns", [(1, 2048, (8192, 8192, 8192)), (8, 2048, (4096, 1024, 1024)),
                                    (64, 5376, (21504, 21504)), (300, 1024, (1000, 520, 4096))])
def test_sibling_linears_quantize_once(lib, M, K, Ns):
    """q/k/v- or gate/up-like siblings of one activation: x quantized once into
    x8 / s_tok (bit-exact against the oracle), every output within the bound
    of the oracle's GEMM and bit-identical to fp8_linear_bf16 per weight."""
    xb = activations_bf16(M, K, seed=M + K, outlier_frac=0.01)
    a = oracle.quant_act(xb)
    ws, wds = [], []
    for i, N in enumerate(Ns):
        q4, d = q4_weights(N, K, seed=100 + i)
        w = oracle.repack_qat(q4, d)
        ws.append(w)
        wds.append((to_dev(w.codes), to_dev(w.scales)))
    x = to_dev(xb)
    x8 = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    st = torch.empty((M,), dtype=torch.float32, device="cuda")
    ys = lib.linear_siblings(x, wds, x8=x8, s_tok=st)
    assert np.array_equal(u8(x8), a.codes) and same_bits_f32(f32(st), a.scales)
    for y, w, (w8, sc) in zip(ys, ws, wds):
        _check(y, a, w)
        assert torch.equal(y.view(torch.int16), lib.linear(x, w8, sc).view(torch.int16))
    assert lib.device_status() == 0
