"""Pins for oracle.attention.decode_attention_multi (several new tokens per request,
causal among themselves), against things other than the function itself:

* with one new token it equals decode_attention;
* torch's scaled_dot_product_attention in float64 with an explicit boolean mask
  (query t sees key j iff j <= L - T + t), on K/V gathered by a per-token loop;
* pure-Python loops with math.exp on tiny inputs;
* causality: changing the last cached token changes only the last query's output;
* the SDPA check is sensitive to the window: a mask shifted by one position, or no mask,
  gives a clearly different result.
"""
import math

import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA


def _case(lens, T, Hq=8, Hkv=2, D=64, P=16, seed=0):
    return W.make_case(W.custom_spec(lens, Hq, Hkv, D, P, 32, seed=seed, q_len=T))


def _loop_gather(pages, block_table, r, g, L):
    P = pages.shape[2]
    return torch.stack([pages[int(block_table[r, j // P]), g, j % P, :] for j in range(L)]).to(torch.float64)


def _sdpa(case, shift=0, causal=True):
    spec = case.spec
    B, T, Hq, Hkv, D = spec.batch, spec.q_len, spec.num_heads, spec.kv_heads, spec.head_dim
    grp = Hq // Hkv
    out = torch.zeros(B, T, Hq, D, dtype=torch.float64)
    for r in range(B):
        L = int(case.seq_lens[r])
        if L < T:
            continue
        K = torch.stack([_loop_gather(case.k_pages, case.block_table, r, g, L) for g in range(Hkv)])
        V = torch.stack([_loop_gather(case.v_pages, case.block_table, r, g, L) for g in range(Hkv)])
        K = K.repeat_interleave(grp, dim=0)  # [Hq, L, D]
        V = V.repeat_interleave(grp, dim=0)
        q = case.q[r].to(torch.float64).permute(1, 0, 2)  # [Hq, T, D]
        j = torch.arange(L).view(1, L)
        t = torch.arange(T).view(T, 1)
        mask = (j <= L - T + t + shift) if causal else torch.ones(T, L, dtype=torch.bool)
        o = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask)
        out[r] = o.permute(1, 0, 2)
    return out.numpy()


@pytest.mark.parametrize("lens,T,Hq,Hkv,D,P,seed", [
    ((5, 40, 129), 2, 8, 2, 64, 16, 0),
    ((3, 17, 300), 3, 16, 2, 128, 64, 1),
    ((4, 64, 65, 1000), 4, 8, 8, 64, 32, 2),
])
def test_matches_masked_sdpa_float64(lens, T, Hq, Hkv, D, P, seed):
    case = _case(lens, T, Hq, Hkv, D, P, seed)
    got = OA.decode_attention_multi(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    ref = _sdpa(case)
    assert np.max(np.abs(got - ref)) <= 1e-12
    # the comparison can tell the window apart
    assert np.max(np.abs(got - _sdpa(case, shift=-1))) > 1e-3
    assert np.max(np.abs(got - _sdpa(case, causal=False))) > 1e-3


def test_one_new_token_is_plain_decode():
    case = _case((1, 9, 200, 513), 1)
    q1 = case.q.unsqueeze(1)  # [B, 1, Hq, D]
    got = OA.decode_attention_multi(q1, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    ref = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    assert np.max(np.abs(got[:, 0] - ref)) <= 1e-15


def test_bruteforce_tiny():
    case = _case((3, 7, 12), 3, Hq=4, Hkv=2, D=8, P=4, seed=5)
    spec = case.spec
    T, Hq, Hkv, D, P = spec.q_len, spec.num_heads, spec.kv_heads, spec.head_dim, spec.page_size
    grp = Hq // Hkv
    q = case.q.to(torch.float64).tolist()
    kp = case.k_pages.to(torch.float64).tolist()
    vp = case.v_pages.to(torch.float64).tolist()
    bt = case.block_table.tolist()
    got = OA.decode_attention_multi(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    for r, L in enumerate(spec.seq_lens):
        for t in range(T):
            pos = L - T + t
            for h in range(Hq):
                g = h // grp
                keys = [kp[bt[r][j // P]][g][j % P] for j in range(pos + 1)]
                vals = [vp[bt[r][j // P]][g][j % P] for j in range(pos + 1)]
                s = [sum(q[r][t][h][d] * k[d] for d in range(D)) / math.sqrt(D) for k in keys]
                m = max(s)
                e = [math.exp(x - m) for x in s]
                z = sum(e)
                for d in range(D):
                    want = sum(e[j] * vals[j][d] for j in range(len(e))) / z
                    assert abs(got[r, t, h, d] - want) <= 1e-13


def test_causality_last_token_only_reaches_last_query():
    case = _case((50, 97), 3, seed=6)
    base = OA.decode_attention_multi(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    kp, vp = case.k_pages.clone(), case.v_pages.clone()
    P = case.spec.page_size
    for r, L in enumerate(case.spec.seq_lens):
        page = int(case.block_table[r, (L - 1) // P])
        kp[page, :, (L - 1) % P] = 3.0
        vp[page, :, (L - 1) % P] = -7.0
    got = OA.decode_attention_multi(case.q, kp, vp, case.block_table, case.seq_lens)
    assert np.array_equal(got[:, :2], base[:, :2])
    assert np.all(np.abs(got[:, 2] - base[:, 2]).max(axis=(1, 2)) > 1e-3)


def test_short_and_empty_requests_give_zeros():
    case = _case((0, 2, 10), 3, seed=7)
    got = OA.decode_attention_multi(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    assert not got[0].any() and not got[1].any() and got[2].any()
