"""Pins of the oracle's mixture-of-experts pieces (CPU only)."""

from decimal import Decimal, localcontext
from fractions import Fraction

import numpy as np
import torch

import oracle
from oracle import formats as F
from oracle import moe
from workloads import moe_routing


def test_route_sort_hand_worked_example():
    # 3 tokens, top-2, 4 experts
    ids = np.array([[2, 0], [0, 3], [2, 1]], dtype=np.int32)
    perm, inv, offsets = moe.route_sort(ids, 4)
    # expert 0: (t0,s1)=1, (t1,s0)=2; expert 1: (t2,s1)=5; expert 2: (t0,s0)=0, (t2,s0)=4; expert 3: (t1,s1)=3
    assert perm.tolist() == [1, 2, 5, 0, 4, 3]
    assert offsets.tolist() == [0, 2, 3, 5, 6]
    assert inv.tolist() == [3, 0, 1, 5, 4, 2]


def test_route_sort_invariants_on_the_moe_workload():
    T, E, k = 8192, 128, 8
    ids = moe_routing(T, E, k, seed=4)
    assert all(len(set(r)) == k for r in ids[:100])
    perm, inv, offsets = moe.route_sort(ids, E)
    assert offsets[-1] == T * k and np.all(np.diff(offsets) >= 0)
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    flat = ids.reshape(-1)
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)
    assert np.array_equal(perm[inv], np.arange(T * k))
    # uniform routing: every expert gets about T*k/E = 512 rows
    cnt = np.diff(offsets)
    assert 400 < cnt.min() and cnt.max() < 630


def test_gelu_tanh_against_torch_and_limits():
    x = np.linspace(-12, 12, 4001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.max(np.abs(moe.gelu_tanh(x) - ref)) < 1e-12
    assert moe.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(moe.gelu_tanh(np.array([30.0]))[0] - 30.0) < 1e-12
    assert abs(moe.gelu_tanh(np.array([-30.0]))[0]) < 1e-12


def _gelu_tanh_decimal(x: float) -> Decimal:
    """0.5 x (1 + tanh(v)), v = sqrt(2/pi) (x + 0.044715 x^3), in 300-digit
    decimal arithmetic, with tanh(v) = (e^v - e^-v) / (e^v + e^-v) from its
    exponential definition: at this precision 1 + tanh(v) keeps well over 100
    correct digits even where it is near 1e-138 (x = -16)."""
    with localcontext() as ctx:
        ctx.prec = 300
        pi = Decimal(0)
        # pi from Machin's formula, 4 (4 atan(1/5) - atan(1/239))
        def atan_inv(n):
            n = Decimal(n)
            term, total, k = 1 / n, 1 / n, 1
            while True:
                term = -term / (n * n)
                t = term / (2 * k + 1)
                if abs(t) < Decimal(10) ** -310:
                    return total
                total += t
                k += 1
        pi = 4 * (4 * atan_inv(5) - atan_inv(239))
        X = Decimal(x)
        v = (2 / pi).sqrt() * (X + Decimal("0.044715") * X ** 3)
        ep, em = v.exp(), (-v).exp()
        return Decimal("0.5") * X * (1 + (ep - em) / (ep + em))


def test_gelu_tanh_relative_accuracy_against_high_precision():
    """Relative error of the fp64 oracle below 1e-13 everywhere, the far
    negative tail (values down to 1e-138) included; a plain fp64 evaluation of
    0.5 x (1 + tanh v) has no correct digit below x = -7."""
    xs = np.concatenate([np.linspace(-16, 16, 321), [-7.0, -9.3, -10.0, -10.3, -12.5, -15.9921875,
                                                     1e-30, -1e-30, 2.0 ** -130, -2.0 ** -130]])
    got = moe.gelu_tanh(xs)
    for x, g in zip(xs, got):
        ref = _gelu_tanh_decimal(float(x))
        if x == 0:
            assert g == 0 and ref == 0
            continue
        rel = abs((Decimal(float(g)) - ref) / ref)
        assert rel < Decimal("1e-13"), (x, float(g), ref)


def test_geglu_rounds_once_to_bf16():
    rng = np.random.default_rng(0)
    g = rng.standard_normal((64, 2 * 16)).astype(np.float32)
    bits = (g.view(np.uint32) >> 16).astype(np.uint16)          # truncate to bf16 inputs
    h = moe.geglu_bf16(bits, 16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = moe.gelu_tanh(vals[:, :16]) * vals[:, 16:]
    back = (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # the nearest bf16: within half a bf16 ulp of the exact product
    assert np.all(np.abs(back - exact) <= 0.5 * oracle.bf16_ulp(exact) * (1 + 1e-12))
    ref = torch.from_numpy(exact).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(back, ref)


def test_grouped_linear_exact_on_tiny_two_expert_case():
    rng = np.random.default_rng(1)
    pool = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], dtype=np.uint8)
    T, k, E, N, K = 3, 2, 2, 4, 64
    ids = np.array([[0, 1], [1, 0], [1, 0]], dtype=np.int32)
    perm, inv, off = moe.route_sort(ids, E)
    x8 = rng.choice(pool, (T, K))
    st = rng.uniform(0.5, 2, T).astype(np.float32)
    w8 = rng.choice(pool, (E, N, K))
    sc = rng.uniform(0.5, 2, (E, N)).astype(np.float32)
    xs, ss = moe.gather_rows(x8, st, perm, k)
    y = moe.grouped_linear_ref(xs, ss, off, w8, sc)
    dec = [Fraction(float(v)) if not np.isnan(v) else None for v in F.DEC_E4M3]
    for i, p in enumerate(perm):
        t, s = divmod(int(p), k)
        e = ids[t, s]
        for n in range(N):
            acc = sum(dec[int(x8[t, kk])] * dec[int(w8[e, n, kk])] for kk in range(K))
            exact = acc * Fraction(float(st[t])) * Fraction(float(sc[e, n]))
            assert abs(Fraction(float(y[i, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def test_grouped_linear_with_one_expert_is_the_dense_gemm():
    rng = np.random.default_rng(2)
    pool = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], dtype=np.uint8)
    T, k, E, N, K = 10, 2, 3, 8, 96
    ids = np.ones((T, k), dtype=np.int32)
    ids[:, 1] = 2
    perm, inv, off = moe.route_sort(ids, E)
    x8 = rng.choice(pool, (T, K))
    st = rng.uniform(0.5, 2, T).astype(np.float32)
    w8 = rng.choice(pool, (E, N, K))
    sc = rng.uniform(0.5, 2, (E, N)).astype(np.float32)
    xs, ss = moe.gather_rows(x8, st, perm, k)
    y = moe.grouped_linear_ref(xs, ss, off, w8, sc)
    assert off.tolist() == [0, 0, T, 2 * T]
    assert np.array_equal(y[:T], oracle.rowwise_linear_ref(x8, st, w8[1], sc[1]))
    assert np.array_equal(y[T:], oracle.rowwise_linear_ref(x8, st, w8[2], sc[2]))


def test_combine_is_the_weighted_sum_of_a_tokens_rows():
    rng = np.random.default_rng(3)
    T, k, E, H = 5, 3, 4, 6
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    perm, inv, off = moe.route_sort(ids, E)
    y = rng.standard_normal((T * k, H))
    out = moe.combine(y, inv, T, k)
    for t in range(T):
        rows = [y[inv[t * k + j]] for j in range(k)]
        assert np.allclose(out[t], sum(rows) / k, rtol=0, atol=1e-15)
    v = rng.standard_normal((T, H))
    same = np.empty((T * k, H))
    for t in range(T):
        for j in range(k):
            same[inv[t * k + j]] = v[t]
    assert np.allclose(moe.combine(same, inv, T, k), v, rtol=0, atol=1e-15)


def test_combine_weighted_exact_rational():
    """With explicit weights the fp64 combine equals the exact-rational
    weighted sum of the token's rows, up to fp64 rounding of the k-term sum."""
    rng = np.random.default_rng(4)
    T, k, E, H = 6, 4, 9, 5
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    perm, inv, off = moe.route_sort(ids, E)
    y = rng.standard_normal((T * k, H)).astype(np.float32).astype(np.float64)
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    out = moe.combine(y, inv, T, k, weights=w)
    for t in range(T):
        for h in range(H):
            exact = sum(Fraction(float(w[t, j])) * Fraction(float(y[inv[t * k + j], h]))
                        for j in range(k))
            mag = sum(abs(Fraction(float(w[t, j])) * Fraction(float(y[inv[t * k + j], h])))
                      for j in range(k))
            assert abs(Fraction(float(out[t, h])) - exact) <= mag * Fraction(2 * k, 2 ** 53)


def test_combine_weighted_hand_worked():
    """Two tokens, top-2 over 3 experts, by hand:
    token 0 -> experts (2, 0) with weights (0.75, 0.25); token 1 -> (1, 2)
    with weights (0.5, 0.5). The expert-sorted rows are
    [t0s1 (e0), t1s0 (e1), t0s0 (e2), t1s1 (e2)]."""
    ids = np.array([[2, 0], [1, 2]], dtype=np.int32)
    perm, inv, off = moe.route_sort(ids, 3)
    assert perm.tolist() == [1, 2, 0, 3] and inv.tolist() == [2, 0, 1, 3]
    rows = np.array([[4.0, -8.0],     # t0 slot 1 (expert 0)
                     [2.0, 6.0],      # t1 slot 0 (expert 1)
                     [1.0, 2.0],      # t0 slot 0 (expert 2)
                     [-2.0, 10.0]])   # t1 slot 1 (expert 2)
    w = np.array([[0.75, 0.25], [0.5, 0.5]], dtype=np.float32)
    out = moe.combine(rows, inv, 2, 2, weights=w)
    # token 0: 0.75 * [1, 2] + 0.25 * [4, -8] = [1.75, -0.5]
    # token 1: 0.5 * [2, 6] + 0.5 * [-2, 10] = [0, 8]
    assert out.tolist() == [[1.75, -0.5], [0.0, 8.0]]


def test_router_gemm_exact_rational():
    rng = np.random.default_rng(10)
    M, N, K = 3, 4, 40
    xb = (rng.standard_normal((M, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    wb = (rng.standard_normal((N, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    y, a = moe.bf16_linear_ref(xb, wb, return_abs=True)
    xv = (xb.astype(np.uint32) << 16).view(np.float32)
    wv = (wb.astype(np.uint32) << 16).view(np.float32)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xv[m, k])) * Fraction(float(wv[n, k])) for k in range(K))
            mag = sum(abs(Fraction(float(xv[m, k])) * Fraction(float(wv[n, k]))) for k in range(K))
            assert abs(Fraction(float(y[m, n])) - exact) <= mag * Fraction(K, 2 ** 53)
            assert abs(Fraction(float(a[m, n])) - mag) <= mag * Fraction(K, 2 ** 53)


def _bf(vals):
    return (np.asarray(vals, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_topk_hand_worked_with_ties():
    # token 0: experts 1 and 4 tie at 3.0 (lower index first), then 2.0 at expert 0
    # token 1: all equal -> experts 0, 1, 2
    logits = _bf([[2.0, 3.0, -1.0, 0.5, 3.0, 1.0],
                  [0.25] * 6])
    ids, w = moe.topk_softmax(logits, 3)
    assert ids.tolist() == [[1, 4, 0], [0, 1, 2]]
    e = np.exp(-1.0)
    assert np.allclose(w[0], [1 / (2 + e), 1 / (2 + e), e / (2 + e)], rtol=1e-15, atol=0)
    assert np.allclose(w[1], [1 / 3] * 3, rtol=1e-15, atol=0)


def test_topk_weights_two_expert_logistic():
    """With top_k = 2 the weights are the logistic of the logit gap:
    w_0 = 1 / (1 + exp(-(a - b))), w_1 = 1 - w_0."""
    rng = np.random.default_rng(11)
    L = rng.standard_normal((500, 16)).astype(np.float32) * 3
    lb = _bf(L)
    ids, w = moe.topk_softmax(lb, 2)
    lv = (lb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(500):
        srt = sorted(range(16), key=lambda e: (-lv[t, e], e))
        assert ids[t].tolist() == srt[:2]
        a, b = lv[t, srt[0]], lv[t, srt[1]]
        assert abs(w[t, 0] - 1 / (1 + np.exp(-(a - b)))) <= 1e-15
        assert abs(w[t, 0] + w[t, 1] - 1) <= 1e-15
