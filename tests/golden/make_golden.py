"""Writes the stored expected values under tests/golden/. It calls only ``oracle/`` and
the seeded input generator; nothing here comes from the CUDA path.

    python tests/golden/make_golden.py

* tiny_plan_g8.txt / tiny_plan_g148.txt: oracle planner output for the tiny workload
  (L = {17, 64, 200, 513}, 2 kv heads, tile 32) at 8 and 148 CTAs.
* tiny_oracle_out.txt: oracle attention output for the tiny workload, every value
  printed to 17 significant digits. It is a regression pin: a later change to the
  oracle's arithmetic must regenerate it and name its justification.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from load_balanced_split_step_b200 import workloads as W  # noqa: E402
from oracle import attention as OA  # noqa: E402
from oracle import planner as OP  # noqa: E402


def write_plan(path, G):
    p = OP.plan_dynamic([17, 64, 200, 513], 2, 32, G)
    with open(path, "w") as f:
        f.write(f"# oracle.planner.plan_dynamic(tiny lengths, kv_heads=2, tile_len=32, num_ctas={G})\n")
        f.write(f"n_units {p.n_units} chunk {p.chunk}\n")
        f.write("# cta req kv_head flags tile_begin tile_end\n")
        for c, it in zip(p.item_cta, p.items):
            f.write(f"{int(c)} {int(it['req'])} {int(it['kv_head'])} {int(it['flags'])} "
                    f"{int(it['tile_begin'])} {int(it['tile_end'])}\n")
        f.write("cta_indptr " + " ".join(str(int(x)) for x in p.cta_indptr) + "\n")
        f.write("merge_indptr " + " ".join(str(int(x)) for x in p.merge_indptr) + "\n")
        f.write("merge_list " + " ".join(str(int(x)) for x in p.merge_list) + "\n")


def write_out(path):
    case = W.make_case(W.config_spec("tiny"))
    out = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    with open(path, "w") as f:
        f.write("# oracle.attention.decode_attention on workloads.config_spec('tiny'), seed 0\n")
        f.write("# one line per (request, head): r h then D values\n")
        B, H, D = out.shape
        for r in range(B):
            for h in range(H):
                f.write(f"{r} {h} " + " ".join(f"{v:.17g}" for v in out[r, h]) + "\n")


if __name__ == "__main__":
    write_plan(os.path.join(HERE, "tiny_plan_g8.txt"), 8)
    write_plan(os.path.join(HERE, "tiny_plan_g148.txt"), 148)
    write_out(os.path.join(HERE, "tiny_oracle_out.txt"))
