"""Pins for oracle.attention.decode_lse, the natural-log log-sum-exp of each (request, query
head)'s scores, against things other than the function itself:

* torch.logsumexp in float64 on keys gathered token by token (a separate gather);
* closed forms: a single key gives its own score, L identical keys give score + ln L, and a
  request with no keys gives -inf;
* E4M3 caches: the same with keys decoded by torch's float8_e4m3fn and multiplied by the
  kv head's scale;
* a planted mistake (a score scale of 1 instead of 1/sqrt(D)) is caught.
"""
import math

import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA


def _loop_gather(pages, block_table, r, g, L):
    P = pages.shape[2]
    return torch.stack([pages[int(block_table[r, j // P]), g, j % P, :] for j in range(L)])


def _reference(case, scale=None):
    spec = case.spec
    B, Hq, Hkv, D = spec.batch, spec.num_heads, spec.kv_heads, spec.head_dim
    grp = Hq // Hkv
    s = 1.0 / math.sqrt(D) if scale is None else scale
    ref = np.full((B, Hq), -np.inf)
    for r in range(B):
        L = int(case.seq_lens[r])
        if L == 0:
            continue
        for g in range(Hkv):
            K = _loop_gather(case.k_pages, case.block_table, r, g, L)
            if spec.kv_dtype == "e4m3":
                K = K.view(torch.float8_e4m3fn).to(torch.float64) * float(case.k_scale[g])
            else:
                K = K.to(torch.float64)
            for h in range(g * grp, (g + 1) * grp):
                ref[r, h] = torch.logsumexp(s * (K @ case.q[r, h].to(torch.float64)), 0).item()
    return ref


@pytest.mark.parametrize("lens,Hq,Hkv,D,P,kv,seed", [
    ((0, 1, 17, 300), 8, 2, 64, 16, "bf16", 0),
    ((5, 64, 65, 1000), 16, 2, 128, 64, "bf16", 1),
    ((3, 129, 700), 8, 4, 128, 32, "e4m3", 2),
])
def test_matches_torch_logsumexp(lens, Hq, Hkv, D, P, kv, seed):
    case = W.make_case(W.custom_spec(lens, Hq, Hkv, D, P, 32, kv_dtype=kv, seed=seed))
    got = OA.decode_lse(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens, kv_dtype=kv,
                        k_scale=case.k_scale)
    ref = _reference(case)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    fin = np.isfinite(ref)
    assert np.max(np.abs(got[fin] - ref[fin])) <= 1e-12


def test_closed_forms():
    case = W.make_case(W.custom_spec((1, 9, 0), 4, 1, 64, 16, 32, seed=3))
    # request 1: nine copies of one key, so lse = score + ln 9
    k = case.k_pages
    p0 = int(case.block_table[1, 0])
    k[p0, 0, :9, :] = k[p0, 0, 0, :].clone()
    got = OA.decode_lse(case.q, k, case.v_pages, case.block_table, case.seq_lens)
    scale = 1.0 / math.sqrt(64)
    key0 = k[int(case.block_table[0, 0]), 0, 0].to(torch.float64)
    key1 = k[p0, 0, 0].to(torch.float64)
    for h in range(4):
        s0 = scale * float(key0 @ case.q[0, h].to(torch.float64))
        s1 = scale * float(key1 @ case.q[1, h].to(torch.float64))
        assert abs(got[0, h] - s0) <= 1e-12  # a single key: its own score
        assert abs(got[1, h] - (s1 + math.log(9))) <= 1e-12
    assert np.all(np.isneginf(got[2]))  # no keys


def test_planted_wrong_scale_is_caught():
    case = W.make_case(W.custom_spec((17, 300), 8, 2, 64, 16, 32, seed=4))
    got = OA.decode_lse(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens, sm_scale=1.0)
    ref = _reference(case)
    assert np.max(np.abs(got - ref)) > 1e-3
