"""The work schedule of the stream-K split of the CTA-pair GEMM (the
PairItems iterator in gemm.cuh and the split choice in launch_pair), checked
on the CPU over many tile counts, pair counts and k-block counts.

The formulas are restated here from their definition (tiles dealt
round-robin, then the k-blocks of the last P + R tiles cut into P runs
[U p / P, U (p + 1) / P)); the test checks the properties the kernel relies
on: every k-block of every tile is computed exactly once, each run covers at
least one tile's k-blocks, a tile cut between pairs has exactly one part
(from the next pair, as that pair's first item) and one owner (whose last
item it is), so the owner's wait can only be on work that pair does first.
The same schedule is exercised on the GPU by the split parity tests, where
the int8 split is bit-exact.
"""

import itertools

import pytest

WHOLE, OWNED, PART = 0, 1, 2


def split_tiles(T, P):
    """The launch's choice: the last full wave and the partial one are split
    when there are between one and eight waves and the last one is partial."""
    if T > P and T % P != 0 and T < 8 * P:
        return P + T % P
    return 0


def items(p, P, T, sk, nkb):
    T_dp = T - sk
    U = sk * nkb
    u_lo = lambda q: (U * q) // P
    out = []
    dp = p
    while dp < T_dp:
        out.append((dp, 0, nkb, WHOLE))
        dp += P
    u, u_end = u_lo(p), u_lo(p + 1)
    while u < u_end:
        ts = u // nkb
        kb0 = u - ts * nkb
        kb1 = min(nkb, kb0 + (u_end - u))
        role = PART if kb0 > 0 else (WHOLE if kb1 == nkb else OWNED)
        out.append((T_dp + ts, kb0, kb1, role))
        u += kb1 - kb0
    return out, u_lo


def owner_contributors(p, P, T, sk, nkb, tile):
    """Pairs p+1 .. q_end-1, as the owner's epilogue finds them."""
    T_dp = T - sk
    U = sk * nkb
    u_lo = lambda q: (U * q) // P
    tile_end_u = (tile - T_dp + 1) * nkb
    q_end = p + 1
    while q_end < P and u_lo(q_end) < tile_end_u:
        q_end += 1
    return list(range(p + 1, q_end))


CASES = [(T, P, nkb)
         for P in (74, 73, 70, 64, 37, 8, 2)
         for T in sorted({P + 1, P + 2, 2 * P - 1, 3 * P + 2, 5 * P + P // 2, 8 * P - 1, 3 * P})
         for nkb in (1, 2, 3, 6, 32, 42, 64)]


@pytest.mark.parametrize("T,P,nkb", CASES)
def test_every_k_block_once_and_single_part_per_tile(T, P, nkb):
    sk = split_tiles(T, P)
    covered = {}
    per_pair = [items(p, P, T, sk, nkb)[0] for p in range(P)]
    for p, its in enumerate(per_pair):
        for (tile, kb0, kb1, role) in its:
            assert 0 <= tile < T and 0 <= kb0 < kb1 <= nkb
            for kb in range(kb0, kb1):
                assert (tile, kb) not in covered, (tile, kb)
                covered[(tile, kb)] = (p, role)
    assert len(covered) == T * nkb
    if sk == 0:
        assert all(role == WHOLE for its in per_pair for (*_, role) in its)
        return
    U = sk * nkb
    # each run holds at least one tile's k-blocks, so it cannot end inside
    # the tile it starts in
    assert all(U * (q + 1) // P - U * q // P >= nkb for q in range(P))
    for p, its in enumerate(per_pair):
        sk_items = [it for it in its if it[0] >= T - sk]
        for i, (tile, kb0, kb1, role) in enumerate(sk_items):
            if role == PART:
                assert i == 0, "a part is the pair's first split item"
            if role == OWNED:
                assert i == len(sk_items) - 1, "an owned piece is the pair's last item"
                contrib = owner_contributors(p, P, T, sk, nkb, tile)
                assert contrib == [p + 1]
                # the contributor's first split item is exactly the rest of the tile
                q_items = [it for it in per_pair[p + 1] if it[0] >= T - sk]
                assert q_items[0] == (tile, kb1, nkb, PART)


def test_split_choice():
    # few waves with a partial last one: split the last full wave and the rest
    assert split_tiles(224, 74) == 76          # prefill M = 1024: 3.03 waves
    assert split_tiles(448, 74) == 78          # 6.05 waves
    assert split_tiles(94, 74) == 94           # every tile split (1.27 waves)
    # whole waves, fewer tiles than pairs, or eight waves and more: no split
    assert split_tiles(222, 74) == 0
    assert split_tiles(60, 74) == 0
    assert split_tiles(74 * 8 + 3, 74) == 0    # M = 8192 layers and longer
    for T, P in itertools.product(range(1, 200), (74, 37)):
        sk = split_tiles(T, P)
        assert sk == 0 or (P < sk < 2 * P and sk <= T)
