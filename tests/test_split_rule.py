"""The single-launch step's split with a fixed cost per item, written out from its definition
and checked on random batches (host arithmetic only; the kernel's outputs are checked on the
GPU by tests/test_gpu_fused.py::test_item_cost_split).

Definition. Units u enumerate (request, kv head, tile) as in the planner. Unit u, a tile of
the S-th segment with tiles (1-based), sits at cost position W*u + c*S, with W = 16 per tile
and c per item start. With total = W*T + c*(number of segments) and
chunk = W * ceil(total / (W*G)), CTA g owns the units whose positions fall in
[g*chunk, (g+1)*chunk).

Checked here:
* with c = 0 the CTA ranges are the oracle planner's (ceil(T / G) units per CTA);
* for any c the ranges partition the units, in order;
* the closed forms the kernel uses for a split segment (first and last owning CTA from the
  positions of its first and last tile; the first piece's partial slot 2*g1 or 2*g1 + 1)
  agree with a direct count of the owners, and partial slots are never shared.
"""
import numpy as np
import pytest

from oracle import planner as OP

W = 16


def segments(lens, Hkv, tl):
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
    return out, u


def owners(lens, Hkv, tl, G, c):
    """Owner CTA of every unit, by its cost position, and the chunk."""
    segs, T = segments(lens, Hkv, tl)
    total = W * T + c * len(segs)
    chunk = W * (-(-total // (W * G))) if T else 0
    own = np.empty(T, dtype=np.int64)
    for (u0, nt, S) in segs:
        for t in range(nt):
            own[u0 + t] = (W * (u0 + t) + c * S) // chunk
    return own, segs, chunk, T


def closed_forms(seg, c, chunk):
    u0, nt, S = seg
    p_first = W * u0 + c * S
    g1, g2 = p_first // chunk, (p_first + W * (nt - 1)) // chunk
    starts = u0 == 0 or (W * (u0 - 1) + c * (S - 1)) // chunk != g1
    return g1, g2, (2 * g1 if starts else 2 * g1 + 1)


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
        own, _, _, T = owners(lens, Hkv, tl, G, 0)
        plan = OP.plan_dynamic(lens, Hkv, tl, G)
        assert T == plan.n_units
        if T:
            assert np.array_equal(own, np.arange(T) // plan.chunk)


@pytest.mark.parametrize("c", [1, 16, 38, 76, 200, 1024])
def test_any_cost_partitions_and_closed_forms_hold(c):
    rng = np.random.default_rng(c)
    for _ in range(200):
        lens, Hkv, tl, G = _random_case(rng)
        own, segs, chunk, T = owners(lens, Hkv, tl, G, c)
        if T == 0:
            continue
        assert chunk >= W
        assert np.all(np.diff(own) >= 0) and own[0] >= 0 and own[-1] < G  # contiguous runs, all CTAs valid
        slots = {}
        for seg in segs:
            u0, nt, S = seg
            g1, g2, first_slot = closed_forms(seg, c, chunk)
            ctas = sorted(set(own[u0:u0 + nt].tolist()))
            assert ctas == list(range(g1, g2 + 1))  # every CTA in between owns a tile
            if g2 == g1 and (u0 == 0 or own[u0 - 1] != g1) and (u0 + nt == T or own[u0 + nt] != g1):
                continue  # the segment is a whole item of one CTA: no partial slot
            if len(ctas) == 1:
                continue  # one piece: written directly, no partial state
            # pieces: the first in CTA g1 (slot 2 g1 if the segment opens g1's run), then 2 g
            first_of_g1 = u0 == 0 or own[u0 - 1] != g1
            assert first_slot == (2 * g1 if first_of_g1 else 2 * g1 + 1)
            for g in range(g1 + 1, g2 + 1):
                assert own[u0 + np.argmax(own[u0:u0 + nt] == g) - 1] < g  # the piece opens g's run
            for s in [first_slot] + [2 * g for g in range(g1 + 1, g2 + 1)]:
                assert s not in slots, (s, seg, slots[s])
                slots[s] = seg
