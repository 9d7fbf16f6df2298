"""Pins for oracle.planner.plan_cost_split, the single-launch step's split with a fixed cost per
item start (host arithmetic only; tests/test_gpu_fused.py compares the kernel's own per-CTA
record with it byte for byte).

Definition (reading 21 of the path's spec). Units u enumerate (request, kv head, tile) as in the
planner. Unit u, a tile of the S-th segment with tiles (1-based), sits at cost position
W*u + c*S, with W = 16 per tile and c per item start. With total = W*T + c*(number of segments)
and chunk = W * ceil(total / (W*G)), CTA g owns the units whose positions fall in
[g*chunk, (g+1)*chunk).

Pinned here:
* a tiny example worked out by hand from the definition (values written in the test);
* with c = 0 the CTA ranges and items are the planner's (ceil(T / G) units per CTA), so the
  split reduces to reading 7, which the survey's hand-worked plan pins;
* for any c the ranges partition the units in order, every CTA's cost span is at most chunk,
  and no two pieces share a partial slot;
* the closed forms the kernel uses for a split segment (first and last owning CTA from the
  positions of its first and last tile; the first piece's slot 2*g1 or 2*g1 + 1) agree with the
  oracle's unit-by-unit owners.
"""
import numpy as np
import pytest

from oracle import planner as OP

W = OP.COST_PER_TILE


def _rows(split, g):
    return [tuple(int(v) for v in it) for it in split.items[g]]


def test_hand_worked_tiny_cost_38():
    # tiny: L = {17, 64, 200, 513}, tile 32 -> nt = {1, 2, 7, 17}; 2 kv heads -> 8 segments,
    # T = 54 units. G = 8, c = 38: total = 16*54 + 38*8 = 1168, chunk = 16*ceil(1168/128) = 160.
    # Position of unit u in segment S: 16u + 38S. For example segment 7 = (r 3, kvh 0) holds
    # units 20..36 at 586, 602, ..., 842: CTAs 3 (586..634), 4 (650..794) and 5 (810..842).
    s = OP.plan_cost_split((17, 64, 200, 513), 2, 32, 8, 38)
    assert s.chunk == 160 and s.n_units == 54
    assert s.unit_begin.tolist() == [0, 3, 9, 16, 24, 34, 41, 51]
    assert s.unit_end.tolist() == [3, 9, 16, 24, 34, 41, 51, 54]
    D, F, X = OP.FLAG_DIRECT, OP.FLAG_SECOND_SLOT, 0  # flags: direct, slot 2g + 1, slot 2g
    want = {  # (req, kv_head, flags, tile_begin, tile_end) per CTA, and the partial slots
        0: ([(0, 0, D, 0, 1), (0, 1, D, 0, 1), (1, 0, F, 0, 1)], [-1, -1, 1]),
        1: ([(1, 0, X, 1, 2), (1, 1, D, 0, 2), (2, 0, F, 0, 3)], [2, -1, 3]),
        2: ([(2, 0, X, 3, 7), (2, 1, F, 0, 3)], [4, 5]),
        3: ([(2, 1, X, 3, 7), (3, 0, F, 0, 4)], [6, 7]),
        4: ([(3, 0, X, 4, 14)], [8]),
        5: ([(3, 0, X, 14, 17), (3, 1, F, 0, 4)], [10, 11]),
        6: ([(3, 1, X, 4, 14)], [12]),
        7: ([(3, 1, X, 14, 17)], [14]),
    }
    for g, (items, slots) in want.items():
        assert _rows(s, g) == items, g
        assert s.slots[g] == slots, g


def _random_case(rng):
    B = int(rng.integers(1, 40))
    lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 64, 129, 300, 1000, 2049, 5000, 40000], size=B)]
    lens = [L if rng.random() < 0.7 else int(rng.integers(0, 9000)) for L in lens]
    return lens, int(rng.choice([1, 2, 4, 8])), int(rng.choice([16, 32, 64, 128])), \
        int(rng.choice([1, 3, 7, 37, 148, 296]))


def test_zero_cost_is_the_planners_split():
    rng = np.random.default_rng(0)
    for _ in range(300):
        lens, Hkv, tl, G = _random_case(rng)
        s = OP.plan_cost_split(lens, Hkv, tl, G, 0)
        plan = OP.plan_dynamic(lens, Hkv, tl, G)
        assert s.n_units == plan.n_units
        if s.n_units == 0:
            continue
        assert s.chunk == W * plan.chunk
        for g in range(G):
            assert s.unit_begin[g] == min(g * plan.chunk, plan.n_units)
            assert s.unit_end[g] == min((g + 1) * plan.chunk, plan.n_units)
            mine = s.items[g]
            ref = plan.items[plan.cta_indptr[g]:plan.cta_indptr[g + 1]]
            assert np.array_equal(mine[["req", "kv_head", "tile_begin", "tile_end"]],
                                  ref[["req", "kv_head", "tile_begin", "tile_end"]])
            assert np.array_equal(mine["flags"] & OP.FLAG_DIRECT, ref["flags"])


def _segments(lens, Hkv, tl):
    """(first unit, tile count, 1-based index) of every segment with tiles, in unit order."""
    out, u, S = [], 0, 0
    for L in lens:
        nt = OP.num_tiles(L, tl)
        if nt == 0:
            continue
        for _ in range(Hkv):
            S += 1
            out.append((u, nt, S))
            u += nt
    return out


def _kernel_closed_forms(seg, c, chunk):
    """The kernel's formulas for a segment: CTAs of its first and last tile, and the slot of its
    first piece (2 g1 unless the unit before the segment is also in g1)."""
    u0, nt, S = seg
    p_first = W * u0 + c * S
    g1, g2 = p_first // chunk, (p_first + W * (nt - 1)) // chunk
    starts = u0 == 0 or (W * (u0 - 1) + c * (S - 1)) // chunk != g1
    return g1, g2, (2 * g1 if starts else 2 * g1 + 1)


@pytest.mark.parametrize("c", [1, 16, 38, 76, 200, 1024])
def test_any_cost_partitions_and_closed_forms_hold(c):
    rng = np.random.default_rng(c)
    for _ in range(200):
        lens, Hkv, tl, G = _random_case(rng)
        s = OP.plan_cost_split(lens, Hkv, tl, G, c)
        T = s.n_units
        if T == 0:
            continue
        assert s.chunk >= W
        # contiguous runs that partition [0, T) in CTA order
        assert s.unit_begin[0] == 0 and s.unit_end[-1] == T
        assert np.all(s.unit_begin[1:] == s.unit_end[:-1]) and np.all(s.unit_end >= s.unit_begin)
        own = np.repeat(np.arange(G), s.unit_end - s.unit_begin)
        segs = _segments(lens, Hkv, tl)
        # positions of each CTA's units lie inside its chunk
        pos = np.empty(T, dtype=np.int64)
        for (u0, nt, S) in segs:
            pos[u0:u0 + nt] = W * np.arange(u0, u0 + nt) + c * S
        assert np.all(pos // s.chunk == own)
        slots = {}
        for g in range(G):
            for it, sl in zip(s.items[g], s.slots[g]):
                if sl >= 0:
                    assert sl not in slots, (sl, g, slots[sl])
                    slots[sl] = (g, tuple(it))
        for seg in segs:
            u0, nt, S = seg
            g1, g2, first_slot = _kernel_closed_forms(seg, c, s.chunk)
            assert sorted(set(own[u0:u0 + nt].tolist())) == list(range(g1, g2 + 1))
            if g1 == g2:
                continue  # one piece: a DIRECT item, no partial slot
            # the first piece's slot in the oracle, and the later pieces' slots 2g
            k = [i for i, it in enumerate(s.items[g1]) if it["req"] == lens_req(lens, Hkv, tl, S)[0]
                 and it["kv_head"] == lens_req(lens, Hkv, tl, S)[1]][0]
            assert s.slots[g1][k] == first_slot
            for g in range(g1 + 1, g2 + 1):
                assert s.slots[g][0] == 2 * g


def lens_req(lens, Hkv, tl, S):
    """(request, kv head) of the S-th segment with tiles (1-based)."""
    n = 0
    for r, L in enumerate(lens):
        if OP.num_tiles(L, tl) == 0:
            continue
        for kvh in range(Hkv):
            n += 1
            if n == S:
                return r, kvh
    raise IndexError(S)
