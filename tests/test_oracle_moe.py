"""Pins of the oracle's mixture-of-experts pieces (CPU only)."""

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
