"""Regression pins: the oracle still reproduces the stored fixtures under tests/golden/
(written by tests/golden/make_golden.py, which calls only oracle/)."""
import os

import numpy as np

from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA
from oracle import planner as OP

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_plan(name):
    rows, extra = [], {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "n_units":
                extra["n_units"], extra["chunk"] = int(parts[1]), int(parts[3])
            elif parts[0] in ("cta_indptr", "merge_indptr", "merge_list"):
                extra[parts[0]] = [int(x) for x in parts[1:]]
            else:
                rows.append(tuple(int(x) for x in parts))
    return rows, extra


def test_tiny_plans():
    for G in (8, 148):
        rows, extra = _read_plan(f"tiny_plan_g{G}.txt")
        p = OP.plan_dynamic([17, 64, 200, 513], 2, 32, G)
        got = [(int(c), int(it["req"]), int(it["kv_head"]), int(it["flags"]), int(it["tile_begin"]),
                int(it["tile_end"])) for c, it in zip(p.item_cta, p.items)]
        assert got == rows
        assert (p.n_units, p.chunk) == (extra["n_units"], extra["chunk"])
        assert p.cta_indptr.tolist() == extra["cta_indptr"]
        assert p.merge_indptr.tolist() == extra["merge_indptr"]
        assert p.merge_list.tolist() == extra.get("merge_list", [])


def test_tiny_oracle_output():
    ref = np.zeros((4, 8, 64))
    with open(os.path.join(GOLDEN, "tiny_oracle_out.txt")) as f:
        for line in f:
            if line.startswith("#"):
                continue
            parts = line.split()
            ref[int(parts[0]), int(parts[1])] = [float(x) for x in parts[2:]]
    case = W.make_case(W.config_spec("tiny"))
    out = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    assert np.max(np.abs(out - ref)) <= 1e-15
