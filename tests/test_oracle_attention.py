"""Pins for oracle.attention and oracle.merge, against things other than the oracle itself.

* torch's scaled_dot_product_attention in float64, on K/V gathered by an explicit
  per-token loop (library routine plus independent gather);
* pure-Python loops with math.exp on tiny inputs (brute force);
* closed forms: one key gives out = v, identical keys or q = 0 give out = mean(v);
* split invariance: any tiling merged by log-sum-exp equals the unsplit softmax;
* planted mistakes (wrong GQA map, wrong page index, missing scale), each caught by
  one of the above.
"""
import math

import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA
from oracle import fp8 as OF
from oracle import merge as OM


def _loop_gather(pages, block_table, r, g, L):
    P = pages.shape[2]
    rows = []
    for j in range(L):
        rows.append(pages[int(block_table[r, j // P]), g, j % P, :])
    return torch.stack(rows).to(torch.float64)


def _sdpa(case, scale=None):
    spec = case.spec
    B, Hq, Hkv, D = spec.batch, spec.num_heads, spec.kv_heads, spec.head_dim
    grp = Hq // Hkv
    out = torch.zeros(B, Hq, D, dtype=torch.float64)
    for r in range(B):
        L = int(case.seq_lens[r])
        K = torch.stack([_loop_gather(case.k_pages, case.block_table, r, g, L) for g in range(Hkv)])
        V = torch.stack([_loop_gather(case.v_pages, case.block_table, r, g, L) for g in range(Hkv)])
        K = K.repeat_interleave(grp, dim=0)  # [Hq, L, D]
        V = V.repeat_interleave(grp, dim=0)
        q = case.q[r].to(torch.float64).unsqueeze(1)  # [Hq, 1, D]
        o = torch.nn.functional.scaled_dot_product_attention(q, K, V, scale=scale)
        out[r] = o[:, 0, :]
    return out.numpy()


def _random_case(seed, lens, Hq=8, Hkv=2, D=64, P=16):
    return W.make_case(W.custom_spec(lens, Hq, Hkv, D, P, 32, seed=seed))


@pytest.mark.parametrize("seed,lens,Hq,Hkv,D,P", [
    (0, (17, 64, 200, 513), 8, 2, 64, 16),
    (1, (1, 2, 33), 8, 8, 64, 16),
    (2, (100, 5), 16, 2, 128, 64),
    (3, (300,), 4, 1, 32, 32),
])
def test_matches_torch_sdpa_float64(seed, lens, Hq, Hkv, D, P):
    case = _random_case(seed, lens, Hq, Hkv, D, P)
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    ref = _sdpa(case)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_tiny_config_matches_sdpa():
    case = W.make_case(W.config_spec("tiny"))
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    assert np.max(np.abs(got - _sdpa(case))) <= 1e-12


def _bruteforce(case):
    """Pure-Python two-pass softmax with math.exp; no numpy, no torch arithmetic."""
    spec = case.spec
    B, Hq, Hkv, D, P = spec.batch, spec.num_heads, spec.kv_heads, spec.head_dim, spec.page_size
    grp = Hq // Hkv
    q = case.q.to(torch.float64).tolist()
    kp = case.k_pages.to(torch.float64).tolist()
    vp = case.v_pages.to(torch.float64).tolist()
    bt = case.block_table.tolist()
    scale = 1.0 / math.sqrt(D)
    out = [[[0.0] * D for _ in range(Hq)] for _ in range(B)]
    for r in range(B):
        L = int(case.seq_lens[r])
        for h in range(Hq):
            g = h // grp
            s = []
            for j in range(L):
                k = kp[bt[r][j // P]][g][j % P]
                s.append(scale * sum(q[r][h][d] * k[d] for d in range(D)))
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            tot = sum(e)
            for d in range(D):
                out[r][h][d] = sum(e[j] * vp[bt[r][j // P]][g][j % P][d] for j in range(L)) / tot
    return np.array(out)


@pytest.mark.parametrize("seed,lens", [(5, (1, 7, 40)), (6, (16, 17)), (7, (33,))])
def test_matches_pure_python_bruteforce(seed, lens):
    case = _random_case(seed, lens, Hq=4, Hkv=2, D=16, P=8)
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    assert np.max(np.abs(got - _bruteforce(case))) <= 1e-13


def test_single_key_returns_v_exactly():
    case = _random_case(11, (1, 1, 1), Hq=8, Hkv=2, D=64, P=16)
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    for r in range(3):
        for h in range(8):
            v = case.v_pages[int(case.block_table[r, 0]), h // 4, 0].to(torch.float64).numpy()
            assert np.array_equal(got[r, h], v)


def test_identical_keys_and_zero_query_give_mean_v():
    case = _random_case(12, (37, 64), Hq=8, Hkv=2, D=64, P=16)
    k = case.k_pages.clone()
    k[:] = k[0, 0, 0]  # every key identical
    got = OA.decode_attention(case.q, k, case.v_pages, case.block_table, case.seq_lens)
    q0 = torch.zeros_like(case.q)
    got0 = OA.decode_attention(q0, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    for r, L in enumerate((37, 64)):
        for g in range(2):
            V = _loop_gather(case.v_pages, case.block_table, r, g, L).numpy()
            mean = V.mean(axis=0)
            for h in range(g * 4, g * 4 + 4):
                assert np.max(np.abs(got[r, h] - mean)) <= 1e-14
                assert np.max(np.abs(got0[r, h] - mean)) <= 1e-14


def test_empty_request_is_zero():
    case = _random_case(13, (0, 5), Hq=4, Hkv=1, D=32, P=16)
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    assert np.all(got[0] == 0.0)


@pytest.mark.parametrize("seed", range(6))
def test_split_invariance(seed):
    rng = np.random.default_rng(100 + seed)
    n, D = int(rng.integers(1, 400)), 64
    s = rng.normal(0, 3, n)
    v = rng.normal(0, 1, (n, D))
    p = np.exp(s - s.max())
    ref = (p / p.sum()) @ v
    for _ in range(5):
        k = int(rng.integers(0, min(n, 20)))
        cuts = [0] + sorted(rng.choice(np.arange(1, n), size=min(k, n - 1), replace=False).tolist()) + [n] if n > 1 else [0, n]
        assert np.max(np.abs(OM.attend_split(s, v, cuts) - ref)) <= 1e-12


def test_merge_of_disjoint_states_equals_joint_state():
    rng = np.random.default_rng(7)
    s = rng.normal(0, 5, 50)
    v = rng.normal(0, 1, (50, 8))
    a, b = OM.partial_state(s[:20], v[:20]), OM.partial_state(s[20:], v[20:])
    M, L, O = OM.merge_states([a[0], b[0]], [a[1], b[1]], [a[2], b[2]])
    m, l, o = OM.partial_state(s, v)
    assert M == m and abs(L - l) <= 1e-12 * l and np.max(np.abs(O - o)) <= 1e-12 * l


def test_e4m3_cache_equals_decoded_values_times_scale():
    """The oracle's E4M3 path equals the bf16/fp64 path run on torch-decoded values."""
    spec = W.custom_spec((40, 70), 8, 2, 64, 16, 32, kv_dtype="e4m3", seed=21)
    case = W.make_case(spec)
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens,
                              kv_dtype="e4m3", k_scale=case.k_scale, v_scale=case.v_scale)
    kd = case.k_pages.view(torch.float8_e4m3fn).to(torch.float64) * case.k_scale.double().view(1, 2, 1, 1)
    vd = case.v_pages.view(torch.float8_e4m3fn).to(torch.float64) * case.v_scale.double().view(1, 2, 1, 1)
    ref = OA.decode_attention(case.q, kd, vd, case.block_table, case.seq_lens)
    assert np.max(np.abs(got - ref)) <= 1e-13


# ---- planted mistakes: each pin must catch a plausible bug in the oracle ----

def _sdpa_gap(monkeypatch, patch):
    case = _random_case(31, (40, 90), Hq=8, Hkv=2, D=64, P=16)
    patch(monkeypatch)
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    return np.max(np.abs(got - _sdpa(case)))


def test_planted_wrong_page_index_is_caught(monkeypatch):
    def patch(mp):
        def bad(pages, bt, r, g, L):
            P = pages.shape[2]
            j = torch.arange(L)
            return pages[j // P, g, j % P, :]  # logical page used as physical: no block_table
        mp.setattr(OA, "_torch_gather", bad)
    assert _sdpa_gap(monkeypatch, patch) > 1e-3


def test_planted_wrong_gqa_map_is_caught(monkeypatch):
    orig = OA._torch_gather

    def patch(mp):
        mp.setattr(OA, "_torch_gather", lambda pages, bt, r, g, L: orig(pages, bt, r, 1 - g, L))
    assert _sdpa_gap(monkeypatch, patch) > 1e-3


def test_planted_missing_scale_is_caught():
    case = _random_case(32, (40, 90), Hq=8, Hkv=2, D=64, P=16)
    got = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens, sm_scale=1.0)
    assert np.max(np.abs(got - _sdpa(case))) > 1e-3
