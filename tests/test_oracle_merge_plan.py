"""Pin for oracle.merge.merge_plan_partials: a hand-worked plan of three items.

The survey's readings 8 and 9 (the pages describe no merge; an LSE merge is the plainest reading
of splitting one softmax): for every (request, kv head) whose plan has two or more items, the
output row of query head h = kvh * group + hh is O / L, with M = max_i m_i,
L = sum_i exp(m_i - M) l_i and O = sum_i exp(m_i - M) o_i over its items i (item k's state in
slot k). A (request, kv head) with exactly one item is written directly and is not merged; one
with no item (L_r = 0) is merged into zeros.

The plan: batch 2, kv_heads 2, group 2 (query heads 0..3), head_dim 2.
    segment 0 = (r 0, kvh 0): items 0 and 1   -> merged
    segment 1 = (r 0, kvh 1): item 2           -> skipped (written directly)
    segments 2, 3 = (r 1, kvh 0 / 1): no items -> zero rows for heads 0..3 of request 1
The expected rows below are worked out by hand from the formulas above.
"""
import math
from types import SimpleNamespace

import numpy as np
import pytest

from oracle import merge as OM


def _case():
    plan = SimpleNamespace(merge_indptr=np.array([0, 2, 3, 3, 3], dtype=np.int32))
    po = np.zeros((3, 2, 2))
    pml = np.zeros((3, 2, 2))
    # head hh = 0 of segment 0: m = (0, ln 3), l = (1, 2/3), o = ([1, 2], [2/3, 1/3]).
    #   M = ln 3, weights (1/3, 1): L = 1/3 + 2/3 = 1, O = [1/3 + 2/3, 2/3 + 1/3] = [1, 1].
    pml[0, 0] = (0.0, 1.0)
    pml[1, 0] = (math.log(3.0), 2.0 / 3.0)
    po[0, 0] = (1.0, 2.0)
    po[1, 0] = (2.0 / 3.0, 1.0 / 3.0)
    # head hh = 1 of segment 0: equal maxima m = (5, 5), l = (1, 3), o = ([4, 0], [0, 8]).
    #   weights (1, 1): L = 4, O = [4, 8], out = [1, 2].
    pml[0, 1] = (5.0, 1.0)
    pml[1, 1] = (5.0, 3.0)
    po[0, 1] = (4.0, 0.0)
    po[1, 1] = (0.0, 8.0)
    # item 2 (segment 1) holds a state that must not be merged into anything
    pml[2] = ((100.0, 7.0), (100.0, 7.0))
    po[2] = ((9.0, 9.0), (9.0, 9.0))
    return plan, po, pml


def test_hand_worked_three_item_plan():
    plan, po, pml = _case()
    out = OM.merge_plan_partials(plan, po, pml, batch=2, kv_heads=2, group=2)
    # heads of segment 0 are kvh 0's group: query heads 0 and 1; segment 1 (heads 2, 3 of
    # request 0) is skipped; request 1 has no items: heads 0..3 are zero rows
    assert set(out) == {(0, 0), (0, 1), (1, 0), (1, 1), (1, 2), (1, 3)}
    assert np.allclose(out[(0, 0)], [1.0, 1.0], rtol=0, atol=1e-15)
    assert np.allclose(out[(0, 1)], [1.0, 2.0], rtol=0, atol=1e-15)
    for h in range(4):
        assert np.array_equal(out[(1, h)], [0.0, 0.0])


@pytest.mark.parametrize("mistake", ["swap_heads", "no_rescale"])
def test_hand_worked_values_catch_planted_mistakes(mistake):
    """The same values with a planted mistake in the merged states give other rows: the pin
    distinguishes the head index inside the group and the exp(m_i - M) weights."""
    plan, po, pml = _case()
    if mistake == "swap_heads":  # reading head hh's state from the other head of the group
        po, pml = po[:, ::-1].copy(), pml[:, ::-1].copy()
    else:  # every part weighted as if its maximum were M
        pml[:, :, 0] = 0.0
    out = OM.merge_plan_partials(plan, po, pml, batch=2, kv_heads=2, group=2)
    assert not (np.allclose(out[(0, 0)], [1.0, 1.0]) and np.allclose(out[(0, 1)], [1.0, 2.0]))
