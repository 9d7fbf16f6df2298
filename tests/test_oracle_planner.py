"""Pins for oracle.planner: a hand-worked example derived from the definition (not from
the oracle), plus cover / balance / ordering invariants over random lengths."""
import numpy as np
import pytest

from oracle import planner as OP


def _as_tuples(plan):
    return [(int(c), int(it["req"]), int(it["kv_head"]), int(it["tile_begin"]), int(it["tile_end"]))
            for c, it in zip(plan.item_cta, plan.items)]


def test_hand_worked_tiny_g8():
    """tiny: L = {17, 64, 200, 513}, tile 32, 2 kv heads, 8 CTAs.
    Tiles per kv head: nt = [1, 2, 7, 17]. T = 2 * 27 = 54 units, chunk = ceil(54/8) = 7.
    Segment unit ranges (r, kvh): (0,0) [0,1)  (0,1) [1,2)  (1,0) [2,4)  (1,1) [4,6)
    (2,0) [6,13)  (2,1) [13,20)  (3,0) [20,37)  (3,1) [37,54). Cutting at multiples of 7
    gives these (cta, r, kvh, tile_begin, tile_end):"""
    expect = [(0, 0, 0, 0, 1), (0, 0, 1, 0, 1), (0, 1, 0, 0, 2), (0, 1, 1, 0, 2), (0, 2, 0, 0, 1),
              (1, 2, 0, 1, 7), (1, 2, 1, 0, 1), (2, 2, 1, 1, 7), (2, 3, 0, 0, 1), (3, 3, 0, 1, 8),
              (4, 3, 0, 8, 15), (5, 3, 0, 15, 17), (5, 3, 1, 0, 5), (6, 3, 1, 5, 12), (7, 3, 1, 12, 17)]
    p = OP.plan_dynamic([17, 64, 200, 513], 2, 32, 8)
    assert p.n_units == 54 and p.chunk == 7
    assert _as_tuples(p) == expect
    # DIRECT exactly for the (r, kvh) with a single item: (0,*) and (1,*)
    direct = [bool(it["flags"] & OP.FLAG_DIRECT) for it in p.items]
    assert direct == [True] * 4 + [False] * 11
    assert p.cta_indptr.tolist() == [0, 5, 7, 9, 10, 11, 13, 14, 15]
    assert p.merge_indptr.tolist() == [0, 1, 2, 3, 4, 6, 8, 12, 15]
    assert p.merge_list.tolist() == [4, 5, 6, 7]


def test_tiny_g148_one_tile_per_cta():
    p = OP.plan_dynamic([17, 64, 200, 513], 2, 32, 148)
    assert p.chunk == 1 and len(p.items) == 54
    assert all(int(it["tile_end"]) - int(it["tile_begin"]) == 1 for it in p.items)
    assert p.cta_indptr[54:].tolist() == [54] * 95  # 94 idle CTAs + the end pointer


def _check_invariants(lens, Hkv, tl, G, p):
    nts = [OP.num_tiles(L, tl) for L in lens]
    seen = {}
    for c, it in zip(p.item_cta, p.items):
        r, g, tb, te = int(it["req"]), int(it["kv_head"]), int(it["tile_begin"]), int(it["tile_end"])
        assert 0 <= tb < te <= nts[r]
        for t in range(tb, te):
            assert (r, g, t) not in seen
            seen[(r, g, t)] = int(c)
    # exact cover
    assert len(seen) == sum(nts) * Hkv
    T = len(seen)
    chunk = -(-T // G) if T else 0
    # per-CTA load <= chunk, and CTAs own contiguous unit ranges in enumeration order
    load = np.zeros(G, dtype=np.int64)
    for c, it in zip(p.item_cta, p.items):
        load[int(c)] += int(it["tile_end"]) - int(it["tile_begin"])
    assert load.max(initial=0) <= chunk
    assert list(p.item_cta) == sorted(p.item_cta)
    # item count bound and index arrays
    assert len(p.items) <= G + len(lens) * Hkv - 1 or len(p.items) == 0
    assert p.cta_indptr[0] == 0 and p.cta_indptr[-1] == len(p.items)
    assert np.all(np.diff(p.cta_indptr) >= 0)
    segs = [int(it["req"]) * Hkv + int(it["kv_head"]) for it in p.items]
    assert segs == sorted(segs)
    for s in range(len(lens) * Hkv):
        i0, i1 = p.merge_indptr[s], p.merge_indptr[s + 1]
        assert all(segs[i] == s for i in range(i0, i1))
        direct = [bool(p.items[i]["flags"] & OP.FLAG_DIRECT) for i in range(i0, i1)]
        assert direct == ([True] if i1 - i0 == 1 else [False] * (i1 - i0))


@pytest.mark.parametrize("tl", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("G", [1, 7, 148, 296])
def test_exact_cover_random_lengths(tl, G):
    rng = np.random.default_rng(tl * 1000 + G)
    for _ in range(3):
        B = int(rng.integers(1, 40))
        lens = np.floor(np.power(2.0, rng.uniform(0, 14, B))).astype(int)
        lens[rng.random(B) < 0.1] = 0
        Hkv = int(rng.choice([1, 2, 8]))
        p = OP.plan_dynamic(lens, Hkv, tl, G)
        _check_invariants(lens, Hkv, tl, G, p)


def test_all_empty_requests():
    p = OP.plan_dynamic([0, 0, 0], 2, 32, 5)
    assert len(p.items) == 0 and p.n_units == 0
    assert p.cta_indptr.tolist() == [0] * 6
    assert p.merge_list.tolist() == list(range(6))  # every segment zero-filled by the merge


def test_static_split_plan():
    S = OP.static_splits(4, 2, 148)
    assert S == 37
    p = OP.plan_static([17, 64, 200, 513], 2, 32, 4)
    # (3, kvh): nt 17 -> per = 5 -> [0,5) [5,10) [10,15) [15,17)
    rows = [t for t in _as_tuples(p) if t[1] == 3 and t[2] == 0]
    assert [(a, b) for (_, _, _, a, b) in rows] == [(0, 5), (5, 10), (10, 15), (15, 17)]
    assert [c for (c, *_rest) in rows] == [24, 25, 26, 27]
    # (0, kvh): nt 1 -> only split 0 has work; splits 1..3 are empty CTAs
    rows0 = [t for t in _as_tuples(p) if t[1] == 0]
    assert [(c, a, b) for (c, _, _, a, b) in rows0] == [(0, 0, 1), (4, 0, 1)]
    assert len(p.cta_indptr) == 4 * 2 * 4 + 1
