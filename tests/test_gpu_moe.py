"""GPU parity of the mixture-of-experts layer against the CPU oracle.

Routing, gather and the per-row quantization of h are bit-exact; the grouped
GEMM is within the row-wise GEMM bound; GeGLU may differ from the fp64 oracle
by one bf16 rounding (fp32 arithmetic), so h is compared within one bf16 ulp -
for every bf16 gate value in [-16, 16] - and h8 bit-exactly against the
oracle's quantization of the GPU's own h; the combine is within its
fp32-summation bound. The layer tests run the whole GPU chain and check each
stage element by element against the oracle applied to that stage's GPU
inputs, so every comparison is with the oracle and none compounds.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import moe
from tests.gpu_util import bf16_to_np_bits, bf16_values, f32, same_bits_f32, to_dev, u8
from workloads import activations_bf16, f32_to_bf16_bits, moe_routing, q4_weights

pytestmark = pytest.mark.gpu


def _ids(T, E, k, seed):
    return moe_routing(T, E, k, seed=seed)


@pytest.mark.parametrize("T,E,k,seed", [(8192, 128, 8, 4), (1, 4, 2, 1), (100, 1, 1, 2),
                                        (300, 64, 4, 3), (5000, 1024, 2, 5),
                                        (20001, 96, 3, 8),    # n % 4 != 0, ragged last chunk
                                        # many experts at larger n, and a handful
                                        (4096, 512, 2, 9), (8192, 1024, 8, 11),
                                        (5000, 7, 1, 10)])
def test_route_matches_oracle(lib, T, E, k, seed):
    ids = _ids(T, E, k, seed)
    if T == 300:
        ids = (ids % 7) * 9      # many experts get no token
        ids = np.stack([np.unique(r) if len(np.unique(r)) == k else r for r in ids]).astype(np.int32)
    perm, inv, off = lib.moe_route(to_dev(ids.astype(np.int32)), E)
    rp, ri, ro = moe.route_sort(ids, E)
    assert np.array_equal(off.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)
    assert lib.device_status() == 0


@pytest.mark.parametrize("T", [16, 4096])
def test_route_flags_out_of_range_ids(lib, T):
    ids = np.zeros((T, 2), np.int32)
    ids[3, 1] = 9
    ids[T - 1, 0] = -1
    lib.moe_route(to_dev(ids), 4)
    assert lib.device_status() & lib.DEV_BAD_INDEX


def test_gather_bit_exact(lib):
    T, E, k, K = 777, 32, 4, 1024
    ids = _ids(T, E, k, 6)
    xb = activations_bf16(T, K, seed=6, outlier_frac=0.01)
    a = oracle.quant_act(xb)
    perm, inv, off = moe.route_sort(ids, E)
    xs, ss = moe.gather_rows(a.codes, a.scales, perm, k)
    g8, gs = lib.moe_gather(to_dev(a.codes), to_dev(a.scales), to_dev(perm), k)
    assert np.array_equal(u8(g8), xs) and same_bits_f32(f32(gs), ss)


def _expert_weights(E, N, K, seed):
    """Oracle-repacked per-expert weights [E, N, K] and scales [E, N]."""
    q4, d = q4_weights(E * N, K, seed=seed)
    w = oracle.repack_qat(q4, d)
    return w.codes.reshape(E, N, K), w.scales.reshape(E, N)


@pytest.mark.parametrize("T,E,k,N,K", [(300, 8, 2, 384, 512), (300, 8, 2, 512, 512),
                                       (1000, 16, 4, 1408, 256), (64, 128, 8, 256, 704),
                                       # K <= 768 keeps A resident over several column
                                       # tiles (5 here: units of unequal length); 800 does not
                                       (2000, 4, 2, 1280, 768), (2000, 4, 2, 1280, 800),
                                       (500, 3, 1, 520, 32)])
def test_grouped_gemm_within_bound(lib, T, E, k, N, K):
    ids = _ids(T, E, k, 7)
    xb = activations_bf16(T, K, seed=7, outlier_frac=0.01)
    a = oracle.quant_act(xb)
    perm, inv, off = moe.route_sort(ids, E)
    xs, ss = moe.gather_rows(a.codes, a.scales, perm, k)
    w8, sc = _expert_weights(E, N, K, seed=8)
    y = lib.grouped_linear(to_dev(xs), to_dev(ss), to_dev(off), to_dev(w8), to_dev(sc))
    y_ref, abs_s = moe.grouped_linear_ref(xs, ss, off, w8, sc, return_abs=True)
    ok, worst = oracle.check_linear(bf16_values(y), y_ref, abs_s)
    assert ok, worst
    assert lib.device_status() == 0


def test_moe_config_expert_gemms_sampled(lib):
    """The MoE layer's shapes: 8192 tokens, top-8 of 128 experts, hidden 2048,
    intermediate 704. Expert weights come from the GPU repack; 3 experts'
    weights are checked bit-exact against the oracle repack and their rows'
    gate/up (N=1408, K=2048) and down (N=2048, K=704) GEMMs against the oracle."""
    T, E, k, Hd, I = 8192, 128, 8, 2048, 704
    ids = _ids(T, E, k, 4)
    perm, inv, off = moe.route_sort(ids, E)
    xb = activations_bf16(T, Hd, seed=4, outlier_frac=0.01)
    a = oracle.quant_act(xb)
    xs, ss = moe.gather_rows(a.codes, a.scales, perm, k)
    picks = [0, 57, 127]
    for (N, K, seed, xrows, srows) in [(2 * I, Hd, 9, xs, ss), (Hd, I, 10, None, None)]:
        q4, d = q4_weights(E * N, K, seed=seed)
        wd, sd = lib.repack_qat(to_dev(q4), to_dev(d))
        if xrows is None:   # down projection input: oracle-quantized synthetic h rows
            hb = activations_bf16(T * k, K, seed=11)
            h = oracle.quant_act(hb)
            xrows, srows = h.codes, h.scales
        y = lib.grouped_linear(to_dev(xrows), to_dev(srows), to_dev(off), wd, sd)
        yv = bf16_values(y)
        for e in picks:
            rows = slice(e * N, (e + 1) * N)
            w = oracle.repack_qat(q4[rows], d[rows])
            assert np.array_equal(u8(wd)[rows], w.codes)
            r0, r1 = off[e], off[e + 1]
            y_ref, abs_s = oracle.rowwise_linear_ref(xrows[r0:r1], srows[r0:r1], w.codes, w.scales,
                                                     return_abs=True)
            ok, worst = oracle.check_linear(yv[r0:r1], y_ref, abs_s)
            assert ok, (N, e, worst)
    assert lib.device_status() == 0


def test_geglu_quant_against_oracle(lib):
    M, I = 4096, 704
    rng = np.random.default_rng(12)
    gu = f32_to_bf16_bits((rng.standard_normal((M, 2 * I)) * 0.7).astype(np.float32))
    h_ref = moe.geglu_bf16(gu, I)
    h_out = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    h8, s_h = lib.moe_geglu_quant(to_dev(gu), I, h_out=h_out)
    h_gpu = bf16_to_np_bits(h_out)
    _assert_h_within_one_ulp(h_gpu, h_ref)
    # the quantization of h: the oracle's, of the GPU's own h, bit for bit
    q = oracle.quant_act(h_gpu)
    assert np.array_equal(u8(h8), q.codes) and same_bits_f32(f32(s_h), q.scales)


def _bf16_vals(bits):
    with np.errstate(invalid="ignore"):     # NaN patterns stay NaN
        return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _assert_h_within_one_ulp(h_gpu_bits, h_ref_bits):
    ref_v, gpu_v = _bf16_vals(h_ref_bits), _bf16_vals(h_gpu_bits)
    bad = ~(np.abs(gpu_v - ref_v) <= oracle.bf16_ulp(ref_v))
    assert not bad.any(), (int(bad.sum()), gpu_v[bad][:4], ref_v[bad][:4])


# Every finite bf16 gate value in [-16, 16] (33,538 of them), each paired with
# these up values (bf16 numbers; |up| <= 2^40 is the range the GeGLU unit
# holds to one bf16 ulp for every gate).
_UPS = [1.0, -1.0, 0.71875, 448.0, -0.0029296875, 2.0 ** 20, -(2.0 ** 40), 2.0 ** -60]


def _gate_up_sweep():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = _bf16_vals(b)
    gates = b[np.isfinite(v) & (np.abs(v) <= 16)]
    ups = f32_to_bf16_bits(np.array(_UPS, np.float32))
    assert np.array_equal(_bf16_vals(ups), np.array(_UPS))
    g = np.tile(gates, len(ups))
    u = np.repeat(ups, len(gates))
    return g, u


def test_geglu_every_bf16_gate_through_geglu_quant(lib):
    """fp8_moe_geglu_quant on every bf16 gate in [-16, 16] (down to the
    subnormals and the far negative tail, where the exact GELU is 1e-37 ...
    1e-138) against the oracle's fp64 GeGLU, within one bf16 ulp."""
    g, u = _gate_up_sweep()
    I = 704
    M = -(-g.size // I)
    pad = M * I - g.size
    gate = np.concatenate([g, np.zeros(pad, np.uint16)]).reshape(M, I)
    up = np.concatenate([u, np.zeros(pad, np.uint16)]).reshape(M, I)
    gu = np.concatenate([gate, up], axis=1)
    h_out = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    h8, s_h = lib.moe_geglu_quant(to_dev(gu), I, h_out=h_out)
    h_gpu = bf16_to_np_bits(h_out)
    _assert_h_within_one_ulp(h_gpu, moe.geglu_bf16(gu, I))
    q = oracle.quant_act(h_gpu)
    assert np.array_equal(u8(h8), q.codes) and same_bits_f32(f32(s_h), q.scales)
    assert lib.device_status() == 0


def test_geglu_every_bf16_gate_through_the_fused_epilogue(lib):
    """fp8_grouped_linear_geglu on the same sweep. Each expert's gate and up
    rows hold E4M3 1.0 in column 0 and the rows of x8 hold 1.0 there too, so
    every accumulator is exactly 1 and gate = bf16(1 * 1 * s_gate) = s_gate,
    up = s_up: the channel scales carry the swept (gate, up) values into the
    epilogue, whose h is checked against the oracle's fp64 GeGLU."""
    g, u = _gate_up_sweep()
    I, K, rows_per_expert = 704, 32, 3
    E = -(-g.size // I)
    assert E <= 1024
    pad = E * I - g.size
    gate = _bf16_vals(np.concatenate([g, np.zeros(pad, np.uint16)])).astype(np.float32).reshape(E, I)
    up = _bf16_vals(np.concatenate([u, np.zeros(pad, np.uint16)])).astype(np.float32).reshape(E, I)
    w = np.zeros((E, 2 * I, K), np.uint8)
    w[:, :, 0] = 0x38                       # E4M3 1.0
    s = np.concatenate([gate, up], axis=1)  # [E, 2I]: gate rows, then up rows
    R = E * rows_per_expert
    x8 = np.zeros((R, K), np.uint8)
    x8[:, 0] = 0x38
    s_rows = np.ones(R, np.float32)
    off = (np.arange(E + 1) * rows_per_expert).astype(np.int32)
    w_il, s_il = lib.moe_interleave_gate_up(to_dev(w), to_dev(s), E, I)
    h = bf16_to_np_bits(lib.grouped_linear_geglu(to_dev(x8), to_dev(s_rows), to_dev(off),
                                                 w_il, s_il, I))
    gate_b = f32_to_bf16_bits(gate)
    up_b = f32_to_bf16_bits(up)
    gu = np.concatenate([np.repeat(gate_b, rows_per_expert, axis=0),
                         np.repeat(up_b, rows_per_expert, axis=0)], axis=1)
    _assert_h_within_one_ulp(h, moe.geglu_bf16(gu, I))
    assert lib.device_status() == 0


@pytest.mark.parametrize("T,E,k,H", [(2048, 128, 8, 2048), (333, 16, 1, 512), (100, 64, 16, 264)])
def test_combine_within_bound(lib, T, E, k, H):
    ids = _ids(T, E, k, 13)
    perm, inv, off = moe.route_sort(ids, E)
    rows = activations_bf16(T * k, H, seed=13)
    out = lib.moe_combine(to_dev(rows), to_dev(inv), T, k)
    vals = (rows.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = moe.combine(vals, inv, T, k)
    absum = moe.combine(np.abs(vals), inv, T, k)
    tol = 2 * k * 2.0 ** -24 * absum + oracle.bf16_ulp(ref)
    assert np.all(np.abs(bf16_values(out) - ref) <= tol)
    w = np.random.default_rng(1).uniform(0, 1, (T, k)).astype(np.float32)
    out_w = lib.moe_combine(to_dev(rows), to_dev(inv), T, k, weights=to_dev(w))
    ref_w = moe.combine(vals, inv, T, k, weights=w)
    abs_w = moe.combine(np.abs(vals), inv, T, k, weights=w)
    assert np.all(np.abs(bf16_values(out_w) - ref_w) <= 2 * k * 2.0 ** -24 * abs_w + oracle.bf16_ulp(ref_w))


def _check_moe_layer_stagewise(lib, T, E, k, Hd, I, seed, row_sample=None, expert_sample=None):
    """The whole layer on the GPU - route, quantize x, gather, gate/up GEMM
    (plain, and with the fused GeGLU epilogue), GeGLU + quantization of h,
    down GEMM, weighted combine - with every stage checked element by element
    against the oracle applied to that stage's GPU inputs: routing, x8,
    gather and h8 bit-exact; gate/up and down within the row-wise GEMM bound;
    h within one bf16 ulp of the fp64 GeGLU of the GPU's gate/up; the fused
    epilogue's h bit-identical to the unfused h; the combine within its fp32
    bound. row_sample(e, r0, r1) picks the rows of expert e the GEMM stages
    check (all rows when None); expert_sample the experts whose repacked
    weights are compared with the oracle's repack (all when None)."""
    ids = _ids(T, E, k, seed)
    xb = activations_bf16(T, Hd, seed=seed, outlier_frac=0.01)
    q4g, dg = q4_weights(E * 2 * I, Hd, seed=seed + 1)
    q4d, dd = q4_weights(E * Hd, I, seed=seed + 2)
    wts = np.random.default_rng(seed + 3).dirichlet(np.ones(k), T).astype(np.float32)
    # GPU chain
    wgu, sgu = lib.repack_qat(to_dev(q4g), to_dev(dg))
    wdn, sdn = lib.repack_qat(to_dev(q4d), to_dev(dd))
    p, iv, of = lib.moe_route(to_dev(ids), E)
    x8, st = lib.quant_act(to_dev(xb))
    g8, gs = lib.moe_gather(x8, st, p, k)
    y1 = lib.grouped_linear(g8, gs, of, wgu, sgu)
    h_gpu = torch.empty((T * k, I), dtype=torch.bfloat16, device="cuda")
    h8, sh = lib.moe_geglu_quant(y1, I, h_out=h_gpu)
    w_il, s_il = lib.moe_interleave_gate_up(wgu, sgu, E, I)
    h_fused = lib.grouped_linear_geglu(g8, gs, of, w_il, s_il, I)
    y2 = lib.grouped_linear(h8, sh, of, wdn, sdn)
    out = lib.moe_combine(y2, iv, T, k, weights=to_dev(wts))
    assert lib.device_status() == 0
    # routing, quantization, gather: exact
    rp, ri, ro = moe.route_sort(ids, E)
    assert np.array_equal(p.cpu().numpy(), rp) and np.array_equal(iv.cpu().numpy(), ri)
    assert np.array_equal(of.cpu().numpy(), ro)
    a = oracle.quant_act(xb)
    assert np.array_equal(u8(x8), a.codes) and same_bits_f32(f32(st), a.scales)
    xs, ss = moe.gather_rows(a.codes, a.scales, rp, k)
    assert np.array_equal(u8(g8), xs) and same_bits_f32(f32(gs), ss)
    # weights: the oracle's repack, bit for bit, on the sampled experts (the
    # GEMM stages below take the GPU's repacked weights as their inputs)
    wg8, wgs = u8(wgu).reshape(E, 2 * I, Hd), f32(sgu).reshape(E, 2 * I)
    wd8, wds = u8(wdn).reshape(E, Hd, I), f32(sdn).reshape(E, Hd)
    for e in (range(E) if expert_sample is None else expert_sample):
        wg = oracle.repack_qat(q4g[e * 2 * I:(e + 1) * 2 * I], dg[e * 2 * I:(e + 1) * 2 * I])
        wd = oracle.repack_qat(q4d[e * Hd:(e + 1) * Hd], dd[e * Hd:(e + 1) * Hd])
        assert np.array_equal(wg8[e], wg.codes) and same_bits_f32(wgs[e], wg.scales)
        assert np.array_equal(wd8[e], wd.codes) and same_bits_f32(wds[e], wd.scales)
    y1v, y2v = bf16_values(y1), bf16_values(y2)
    h8n, shn = u8(h8), f32(sh)
    for e in range(E):
        r0, r1 = int(ro[e]), int(ro[e + 1])
        if r1 == r0:
            continue
        rows = np.arange(r0, r1) if row_sample is None else row_sample(e, r0, r1)
        ref, abs_s = oracle.rowwise_linear_ref(xs[rows], ss[rows], wg8[e], wgs[e], return_abs=True)
        ok, worst = oracle.check_linear(y1v[rows], ref, abs_s)
        assert ok, ("gate/up", e, worst)
        ref, abs_s = oracle.rowwise_linear_ref(h8n[rows], shn[rows], wd8[e], wds[e], return_abs=True)
        ok, worst = oracle.check_linear(y2v[rows], ref, abs_s)
        assert ok, ("down", e, worst)
    # GeGLU of the GPU's own gate/up, and the quantization of the GPU's own h
    hb = bf16_to_np_bits(h_gpu)
    _assert_h_within_one_ulp(hb, moe.geglu_bf16(bf16_to_np_bits(y1), I))
    assert np.array_equal(bf16_to_np_bits(h_fused), hb)
    q = oracle.quant_act(hb)
    assert np.array_equal(h8n, q.codes) and same_bits_f32(shn, q.scales)
    # combine of the GPU's own down rows with the router weights
    ref = moe.combine(y2v, ri, T, k, weights=wts)
    absum = moe.combine(np.abs(y2v), ri, T, k, weights=wts)
    tol = 2 * k * 2.0 ** -24 * absum + oracle.bf16_ulp(ref)
    assert np.all(np.abs(bf16_values(out) - ref) <= tol)


def test_small_moe_layer_stage_by_stage(lib):
    _check_moe_layer_stagewise(lib, T=512, E=16, k=4, Hd=512, I=256, seed=14)


def test_moe_config_layer_stage_by_stage(lib):
    """The MoE workload itself (8192 tokens, top-8 of 128 experts, hidden 2048,
    intermediate 704), every expert's GEMMs checked on 12 of its rows: the
    first 4, the last 4 (a partial pair tile) and 4 drawn at random; the
    repack on 6 experts; every other stage on every row."""
    rng = np.random.default_rng(30)

    def sample(e, r0, r1):
        n = r1 - r0
        pick = set(range(min(4, n))) | set(range(max(0, n - 4), n))
        pick |= set(rng.choice(n, min(4, n), replace=False).tolist())
        return r0 + np.array(sorted(pick))

    _check_moe_layer_stagewise(lib, T=8192, E=128, k=8, Hd=2048, I=704, seed=4, row_sample=sample,
                               expert_sample=[0, 1, 57, 64, 126, 127])


def test_interleave_gate_up_layout(lib):
    """Row t*256 + s*128 + j of an expert is its gate (s=0) / up (s=1) row of
    feature t*128 + j; features past inter are zero rows with scale 0."""
    E, I, K = 3, 176, 96          # 2 feature tiles, the second one partial
    rng = np.random.default_rng(20)
    w = rng.integers(0, 0x7F, (E * 2 * I, K), dtype=np.uint8)
    s = rng.uniform(0.5, 2.0, E * 2 * I).astype(np.float32)
    w_il, s_il = lib.moe_interleave_gate_up(to_dev(w), to_dev(s), E, I)
    T = (I + 127) // 128
    ref_w = np.zeros((E * 256 * T, K), np.uint8)
    ref_s = np.zeros(E * 256 * T, np.float32)
    for e in range(E):
        for t in range(T):
            for sg in range(2):
                for j in range(128):
                    f = t * 128 + j
                    if f < I:
                        ref_w[e * 256 * T + t * 256 + sg * 128 + j] = w[e * 2 * I + sg * I + f]
                        ref_s[e * 256 * T + t * 256 + sg * 128 + j] = s[e * 2 * I + sg * I + f]
    assert np.array_equal(u8(w_il), ref_w) and same_bits_f32(f32(s_il), ref_s)


@pytest.mark.parametrize("T,E,k,I,K", [(8192, 128, 8, 704, 2048), (300, 8, 2, 176, 512),
                                       (64, 128, 8, 256, 704), (1000, 16, 4, 1408, 256),
                                       # last feature tile of 80 features (full width) and a
                                       # single tile of 64 (half width: N = 128 MMAs)
                                       (300, 8, 2, 720, 256), (200, 4, 2, 64, 256)])
def test_geglu_epilogue_bit_identical(lib, T, E, k, I, K):
    """fp8_grouped_linear_geglu gives bit for bit the h that the plain grouped
    GEMM followed by fp8_moe_geglu_quant gives, and fp8_quant_act of it the
    same codes and scales."""
    ids = _ids(T, E, k, 21)
    perm, inv, off = moe.route_sort(ids, E)
    xb = activations_bf16(T, K, seed=21, outlier_frac=0.01)
    a = oracle.quant_act(xb)
    xs, ss = moe.gather_rows(a.codes, a.scales, perm, k)
    q4, d = q4_weights(E * 2 * I, K, seed=22)
    wd, sd = lib.repack_qat(to_dev(q4), to_dev(d))
    xd, sxd, offd = to_dev(xs), to_dev(ss), to_dev(off)
    gu = lib.grouped_linear(xd, sxd, offd, wd, sd)
    h_ref = torch.empty((T * k, I), dtype=torch.bfloat16, device="cuda")
    h8_ref, sh_ref = lib.moe_geglu_quant(gu, I, h_out=h_ref)
    w_il, s_il = lib.moe_interleave_gate_up(wd, sd, E, I)
    h = lib.grouped_linear_geglu(xd, sxd, offd, w_il, s_il, I)
    assert np.array_equal(bf16_to_np_bits(h), bf16_to_np_bits(h_ref))
    h8, sh = lib.quant_act(h)
    assert np.array_equal(u8(h8), u8(h8_ref)) and same_bits_f32(f32(sh), f32(sh_ref))
    assert lib.device_status() == 0


def test_bad_device_indices_are_flagged_not_followed(lib):
    """Expert offsets outside [0, M] or running backwards, perm entries
    outside [0, rows) and inv entries outside [0, tokens*top_k) are device
    errors: flagged with FP8_DEV_BAD_INDEX and never used as addresses."""
    E, N, K, R = 4, 256, 128, 64
    rng = np.random.default_rng(50)
    xr = rng.integers(0, 0x7F, (R, K), dtype=np.uint8)
    sr = np.ones(R, np.float32)
    w8, sc = _expert_weights(E, N, K, seed=51)
    lib.device_status()
    y = torch.full((R, N), 7.0, dtype=torch.bfloat16, device="cuda")
    bad_off = np.array([0, 40, 20, 64, 64], np.int32)            # expert 1 runs backwards
    lib.grouped_linear(to_dev(xr), to_dev(sr), to_dev(bad_off), to_dev(w8), to_dev(sc), y)
    assert lib.device_status() & lib.DEV_BAD_INDEX
    big_off = np.array([0, 16, 32, 48, 10 ** 6], np.int32)       # past M_total
    lib.grouped_linear(to_dev(xr), to_dev(sr), to_dev(big_off), to_dev(w8), to_dev(sc), y)
    assert lib.device_status() & lib.DEV_BAD_INDEX
    # a valid expert next to the bad one is still computed
    yv = bf16_values(y)
    y_ref, abs_s = oracle.rowwise_linear_ref(xr[:16], sr[:16], w8[0], sc[0], return_abs=True)
    ok, worst = oracle.check_linear(yv[:16], y_ref, abs_s)
    assert ok, worst
    # gather: perm entries -1 and rows give zero rows
    T, k, Kx = 8, 2, 64
    x8 = rng.integers(1, 0x7F, (T, Kx), dtype=np.uint8)
    st = np.full(T, 2.0, np.float32)
    perm = np.arange(T * k, dtype=np.int32)
    perm[3], perm[5] = -1, T * k
    g8, gs = lib.moe_gather(to_dev(x8), to_dev(st), to_dev(perm), k)
    assert lib.device_status() & lib.DEV_BAD_INDEX
    g8, gs = u8(g8), f32(gs)
    assert not g8[3].any() and not g8[5].any() and gs[3] == 0 and gs[5] == 0
    assert np.array_equal(g8[4], x8[2]) and gs[4] == 2.0
    # combine: an inv entry past the rows contributes nothing
    H = 64
    rows = f32_to_bf16_bits(rng.standard_normal((T * k, H)).astype(np.float32))
    inv = np.arange(T * k, dtype=np.int32)
    inv[1] = 10 ** 6
    out = bf16_values(lib.moe_combine(to_dev(rows), to_dev(inv), T, k))
    assert lib.device_status() & lib.DEV_BAD_INDEX
    vals = (rows.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.allclose(out[0], 0.5 * vals[0], rtol=2 ** -7, atol=1e-30)   # slot 1 dropped
    assert np.allclose(out[1], 0.5 * (vals[2] + vals[3]), rtol=2 ** -7, atol=1e-6)
