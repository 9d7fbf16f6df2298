"""The seeded input generator: determinism, sampled subsets, and the workload recipes."""
import numpy as np
import torch

from load_balanced_split_step_b200 import workloads as W


def test_named_recipes():
    assert W.config_spec("tiny").seq_lens == (17, 64, 200, 513)
    ex = W.config_spec("extreme")
    assert ex.seq_lens[0] == 131072 and ex.seq_lens[1:] == (4096,) * 31
    hv = W.config_spec("heavy")
    assert len(hv.seq_lens) == 64 and min(hv.seq_lens) >= 512 and max(hv.seq_lens) < 65536
    assert hv.steps == 8
    f8 = W.config_spec("fp8")
    assert len(f8.seq_lens) == 256 and 1024 <= min(f8.seq_lens) and max(f8.seq_lens) <= 16384
    assert f8.kv_dtype == "e4m3" and f8.prologue
    assert W.config_spec("heavy").seq_lens == hv.seq_lens  # deterministic


def test_case_is_deterministic_and_layout_is_valid():
    spec = W.custom_spec((5, 40, 17), 8, 2, 64, 16, 32, steps=3, seed=9)
    a, b = W.make_case(spec), W.make_case(spec)
    assert torch.equal(a.k_pages, b.k_pages) and torch.equal(a.block_table, b.block_table)
    bt = a.block_table.numpy()
    used = bt[bt >= 0]
    assert len(set(used.tolist())) == len(used) == a.num_pages  # a permutation of the pool
    for r, L in enumerate((5, 40, 17)):
        assert (bt[r] >= 0).sum() == (L + 2 + 15) // 16 + 1


def test_sampled_subset_is_bit_identical():
    spec = W.custom_spec((30, 70, 12, 99), 8, 2, 64, 16, 32, seed=3)
    full = W.make_case(spec)
    sub = W.make_case(spec, requests=[3, 1])
    for i, r in enumerate([3, 1]):
        n = int(full.pages_per_req[r])
        fk = full.k_pages[full.block_table[r, :n].long()]
        sk = sub.k_pages[sub.block_table[i, :n].long()]
        assert torch.equal(fk, sk)
        assert torch.equal(full.q[r], sub.q[i])
    assert sub.num_pages == int(full.pages_per_req[3] + full.pages_per_req[1])


def test_e4m3_scales_are_amax_over_448():
    spec = W.custom_spec((20, 50), 8, 2, 64, 16, 32, kv_dtype="e4m3", seed=4)
    c = W.make_case(spec)
    vals = c.k_pages.view(torch.float8_e4m3fn).to(torch.float32)
    assert float(vals.abs().max()) == 448.0  # the amax element encodes to exactly 448
    assert c.k_scale.shape == (2,) and torch.all(c.k_scale > 0)
