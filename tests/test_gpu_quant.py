"""GPU parity of the streaming quantizers against the CPU oracle: E4M3 codes
and fp32 scales must match bit for bit. Calls go through the C ABI (the
ctypes binding passes device pointers and sizes)."""

import numpy as np
import pytest
import torch

import oracle
from oracle import formats as F
from tests.gpu_util import f32, same_bits_f32, to_dev, u8
from workloads import activations_bf16, f32_to_bf16_bits, q4_weights

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ encoder
def _oracle_boundaries():
    """First positive fp32 bit pattern whose oracle code is c, for c = 1..126.

    The oracle encoder is monotone in the value, and fp32 bit patterns of
    non-negative values are ordered like the values, so every code owns one
    contiguous range of patterns; binary search finds each range's start."""
    def code_of(p):
        return int(F.enc_e4m3(np.array([p], dtype=np.uint32).view(np.float32).astype(np.float64))[0])

    bounds = []
    for c in range(1, 127):
        lo, hi = 0, 0x7F800000
        while lo < hi:
            mid = (lo + hi) // 2
            if code_of(mid) >= c:
                hi = mid
            else:
                lo = mid + 1
        bounds.append(lo)
    return np.array(bounds, dtype=np.int64)


def test_cast_matches_oracle_on_every_fp32_pattern(lib):
    bounds = torch.tensor(_oracle_boundaries(), device="cuda")
    chunk = 1 << 28
    bad = 0
    for start in range(0, 1 << 32, chunk):
        pat = torch.arange(start, start + chunk, device="cuda", dtype=torch.int64)
        x = pat.to(torch.int32).view(torch.float32) if start < (1 << 31) else \
            (pat - (1 << 32)).to(torch.int32).view(torch.float32)
        got = lib.cast_e4m3(x.contiguous()).to(torch.int64)
        mag_pat = pat & 0x7FFFFFFF
        code = torch.searchsorted(bounds, mag_pat, right=True)          # 0..126 by magnitude
        neg = (pat >> 31) & 1
        exp = torch.where((neg == 1) & (code != 0), code | 0x80, code)
        exp = torch.where(mag_pat > 0x7F800000, torch.full_like(exp, 0x7F), exp)  # NaN
        bad += int((got != exp).sum())
        del pat, x, got, mag_pat, code, neg, exp
    assert bad == 0


# ------------------------------------------------------------------ activation quant
ACT_SHAPES = [
    (4, 256, 0, 0.0),        # tiny W8A8 linear
    (1, 2048, 1, 0.01),      # decode rows
    (8, 2048, 1, 0.01),
    (64, 2048, 1, 0.01),
    (3, 48, 5, 0.0),
    (1025, 5376, 3, 0.01),   # warp-per-row path, row held in registers
    (2000, 16, 7, 0.0),
    (5, 9008, 8, 0.01),      # 1024-thread block per row, row held in registers
    (2, 21504, 11, 0.01),
    (1100, 6160, 9, 0.01),   # warp-per-row path, re-read from cache
    (7, 65536, 10, 0.01),
    (4097, 4096, 13, 0.01),  # warp pair per row (each warp stages half of it)
    (1500, 4608, 14, 0.01),
]


@pytest.mark.parametrize("M,K,seed,outl", ACT_SHAPES)
def test_quant_act_bit_exact(lib, M, K, seed, outl):
    xb = activations_bf16(M, K, seed=seed, outlier_frac=outl)
    ref = oracle.quant_act(xb)
    x8, s = lib.quant_act(to_dev(xb))
    assert np.array_equal(u8(x8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)
    assert lib.device_status() == 0


def test_quant_act_special_rows(lib):
    K = 512
    rows = np.zeros((9, K), dtype=np.float32)
    rng = np.random.default_rng(0)
    rows[1] = rng.standard_normal(K) * 1e-38        # subnormal bf16 values
    rows[2] = rng.standard_normal(K) * 1e37         # huge values
    rows[3] = 3.0                                    # constant row
    rows[4] = -rng.random(K)                          # negative amax
    rows[5, 100] = -5.0                               # single nonzero
    rows[6] = rng.standard_normal(K)
    rows[6, ::3] = 0.0
    rows[7] = rng.standard_normal(K) * 2.0 ** -120
    rows[8] = rng.standard_normal(K)
    xb = f32_to_bf16_bits(rows)
    ref = oracle.quant_act(xb)
    x8, s = lib.quant_act(to_dev(xb))
    assert np.array_equal(u8(x8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)
    assert lib.device_status() == 0


def test_quant_act_quotients_near_e4m3_midpoints(lib):
    """Rows whose values sit on or next to s * (E4M3 midpoint): the division
    must round exactly like IEEE fp32 division for the codes to match."""
    rng = np.random.default_rng(17)
    mags = F.DEC_E4M3[:0x7F]
    mids = (mags[:-1] + mags[1:]) / 2
    M, K = 4096, 512
    amax = (rng.uniform(0.5, 2.0, M) * 2.0 ** rng.integers(-60, 60, M)).astype(np.float32)
    amax = f32_to_bf16_bits(amax)
    amax_f = (amax.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mu = rng.choice(mids, size=(M, K)) * rng.choice([-1.0, 1.0], size=(M, K))
    v = (mu * amax_f[:, None] / 448.0).astype(np.float32)
    xb = f32_to_bf16_bits(v)
    xb += rng.integers(-1, 2, size=(M, K)).astype(np.uint16)   # +-1 bf16 ulp around it
    xb[:, 0] = amax                                               # the row maximum
    ref = oracle.quant_act(xb)
    x8, s = lib.quant_act(to_dev(xb))
    assert np.array_equal(u8(x8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)


def test_quant_act_large_full_compare(lib):
    M, K = 16384, 5376
    xb = activations_bf16(M, K, seed=3, outlier_frac=0.01)
    ref = oracle.quant_act(xb)
    x8, s = lib.quant_act(to_dev(xb))
    assert np.array_equal(u8(x8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)


def test_quant_act_pitched_input(lib):
    M, K, ldx = 37, 1024, 1040
    xb = activations_bf16(M, ldx, seed=12)
    ref = oracle.quant_act(xb[:, :K])
    xd = to_dev(xb)
    x8 = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    st = lib.raw.fp8_quant_act(xd.data_ptr(), M, K, ldx, x8.data_ptr(), s.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert np.array_equal(u8(x8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)


def test_quant_act_warp_pair_rows(lib):
    """Rows split over a warp pair (M > 1024, K = 4096): the row maximum only
    in the first or only in the second half, zero halves, a NaN in the
    second half (flagged), a pitched input - bytes and scales bit-exact."""
    M, K, ldx = 2048, 4096, 4160
    xb = activations_bf16(M, ldx, seed=15, outlier_frac=0.01)
    xb[1, :K // 2] = 0                        # first half zero
    xb[2, K // 2:K] = 0                       # second half zero
    xb[3, :K] = 0                             # zero row: s = 0, codes 0
    xb[4, K // 2 + 7] = 0x4780                # 65536 in the second half only
    xb[5, 3] = 0xC780                         # -65536 in the first half only
    xb[6, K - 1] = 0x7FC0                     # NaN in the second half
    ref = oracle.quant_act(xb[:, :K])
    x8 = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    lib.device_status()
    st = lib.raw.fp8_quant_act(to_dev(xb).data_ptr(), M, K, ldx, x8.data_ptr(), s.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert lib.device_status() & lib.DEV_NONFINITE
    ok = np.ones(M, bool)
    ok[6] = False
    assert np.array_equal(u8(x8)[ok], ref.codes[ok])
    assert same_bits_f32(f32(s)[ok], ref.scales[ok])
    assert f32(s)[3] == 0 and not u8(x8)[3].any()


def test_quant_act_nonfinite_rows_are_reported(lib):
    xb = activations_bf16(6, 256, seed=1)
    xb[2, 17] = 0x7FC0   # NaN
    xb[4, 3] = 0xFF80    # -Inf
    lib.quant_act(to_dev(xb))
    assert lib.device_status() & lib.DEV_NONFINITE
    ref = oracle.quant_act(xb)
    assert ref.bad_rows.tolist() == [False, False, True, False, True, False]
    # status was cleared by the read
    assert lib.device_status() == 0


# ------------------------------------------------------------------ repack
REPACK_SHAPES = [(128, 256, 0), (7, 32, 1), (1, 5376, 3), (300, 5376, 3), (3, 12800, 4),
                 (1000, 2048, 1), (4097, 4096, 2)]


@pytest.mark.parametrize("N,K,seed", REPACK_SHAPES)
def test_repack_bit_exact(lib, N, K, seed):
    q4, d = q4_weights(N, K, seed=seed)
    ref = oracle.repack_qat(q4, d)
    w8, s = lib.repack_qat(to_dev(q4), to_dev(d))
    assert np.array_equal(u8(w8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)
    assert lib.device_status() == 0


def test_repack_special_scales(lib):
    N, K = 6, 256
    q4, d = q4_weights(N, K, seed=5)
    d = d.copy()
    d[0] = 0.0                       # zero row -> s = 0, all-zero codes
    d[1] = -d[1]                     # negative group scales
    d[2] *= 1e30                     # large values
    d[3, 2] = 0.0                    # one zero group
    d[4] *= 2.0 ** -100              # tiny values
    ref = oracle.repack_qat(q4, d)
    w8, s = lib.repack_qat(to_dev(q4), to_dev(d))
    assert np.array_equal(u8(w8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)
    assert ref.scales[0] == 0 and not ref.codes[0].any()
    assert lib.device_status() == 0
    d[5, 1] = np.inf
    lib.repack_qat(to_dev(q4), to_dev(d))
    assert lib.device_status() & lib.DEV_NONFINITE


# ------------------------------------------------------------------ FNUZ
def test_fnuz_copy_converts_to_identical_e4m3(lib):
    q4, d = q4_weights(512, 4096, seed=2)
    ref = oracle.repack_qat(q4, d)
    cn, sn = oracle.fnuz_copy_of_e4m3(ref.codes, ref.scales)
    w8, s = lib.convert_fnuz(to_dev(cn), to_dev(sn))
    assert np.array_equal(u8(w8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)
    assert lib.device_status() == 0


def test_native_fnuz_conversion_matches_oracle(lib):
    q4, d = q4_weights(777, 1024, seed=6)
    rn = oracle.quantize_rows_fnuz(oracle.qat_values(q4, d))
    ref = oracle.convert_fnuz_to_e4m3(rn.codes, rn.scales)
    w8, s = lib.convert_fnuz(to_dev(rn.codes), to_dev(rn.scales))
    assert np.array_equal(u8(w8), ref.codes)
    assert same_bits_f32(f32(s), ref.scales)
    st = lib.device_status()
    assert bool(st & lib.DEV_INEXACT) == bool(ref.inexact_rows.any())
    assert not st & lib.DEV_NAN_CODE


def test_fnuz_staged_rows_in_place_and_special_rows(lib):
    """The row-staged conversion (N >= 4 x SMs): in place, K not a multiple of
    128, +-240 rows re-encoded, odd-subnormal and zero scales, 0x80 flagged."""
    N, K = 1200, 1040
    rng = np.random.default_rng(31)
    codes = rng.integers(0, 0x7F, size=(N, K)).astype(np.uint8)
    codes[rng.random((N, K)) < 0.5] |= 0x80                        # negative codes
    codes[codes == 0x80] = 0x00                                     # no NaN code yet
    codes[3, 17] = 0x7F                                             # +240
    codes[700, 1039] = 0x7F
    codes[11, 0] = 0xFF                                             # -240
    s = rng.uniform(0.01, 2.0, N).astype(np.float32)
    s[5] = np.float32(2.0 ** -149 * 5)                              # odd subnormal: not halved
    s[6] = 0.0
    ref = oracle.convert_fnuz_to_e4m3(codes, s)
    cd, sd = to_dev(codes), to_dev(s)
    lib.device_status()
    lib.convert_fnuz(cd, sd, w8=cd, s_ch=sd)
    assert np.array_equal(u8(cd), ref.codes)
    assert same_bits_f32(f32(sd), ref.scales)
    st = lib.device_status()
    assert bool(st & lib.DEV_INEXACT) == bool(ref.inexact_rows.any())
    assert not st & lib.DEV_NAN_CODE
    codes[900, 33] = 0x80
    lib.convert_fnuz(to_dev(codes), to_dev(s))
    assert lib.device_status() & lib.DEV_NAN_CODE


def test_fnuz_in_place_and_special_cases(lib):
    N, K = 5, 64
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 0x7F, size=(N, K)).astype(np.uint8)   # no 0x7F, no 0x80
    codes[1, 5] = 0x7F                                             # +240: re-encode path
    s = np.array([1.0, 0.5, 0.0, 2.0 ** -149 * 3, 7.25], dtype=np.float32)  # row 3: odd subnormal
    ref = oracle.convert_fnuz_to_e4m3(codes, s)
    cd, sd = to_dev(codes), to_dev(s)
    lib.convert_fnuz(cd, sd, w8=cd, s_ch=sd)
    assert np.array_equal(u8(cd), ref.codes)
    assert same_bits_f32(f32(sd), ref.scales)
    assert not ref.halved_rows[1] and not ref.halved_rows[3] and ref.halved_rows[0]
    lib.device_status()
    codes[4, 9] = 0x80
    lib.convert_fnuz(to_dev(codes), to_dev(s))
    assert lib.device_status() & lib.DEV_NAN_CODE
