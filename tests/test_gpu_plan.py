"""Device planner parity: the device plan equals the host twin and the oracle planner byte
for byte, for random lengths, the named workloads and each re-planned decode step."""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import planner as OP

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def _check_equal(got, ref, static=False):
    assert got["n_items"] == len(ref.items)
    assert got["items"].tobytes() == ref.items.tobytes()
    assert np.array_equal(got["cta_indptr"], ref.cta_indptr)
    assert np.array_equal(got["merge_indptr"], ref.merge_indptr)
    assert np.array_equal(got["merge_list"], ref.merge_list)
    assert got["n_units"] == ref.n_units
    if not static:
        assert got["chunk"] == ref.chunk


def _device_plan(B, lens, Hkv, tl, G, max_seq=0):
    t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = B.plan(t, Hkv * 8, Hkv, tl, G, max_seq, st)
    torch.cuda.synchronize()
    return p.to_numpy(), int(st.item())


def test_tiny_hand_example(B):
    got, st = _device_plan(B, [17, 64, 200, 513], 2, 32, 8)
    assert st == 0
    _check_equal(got, OP.plan_dynamic([17, 64, 200, 513], 2, 32, 8))


@pytest.mark.parametrize("tl", [16, 64, 128, 256])
@pytest.mark.parametrize("G", [1, 7, 148, 296, 1000])
def test_random_lengths(B, tl, G):
    rng = np.random.default_rng(tl * 31 + G)
    for _ in range(3):
        n = int(rng.integers(1, 400))
        lens = np.floor(np.power(2.0, rng.uniform(0, 15, n))).astype(int)
        lens[rng.random(n) < 0.05] = 0
        Hkv = int(rng.choice([1, 2, 8]))
        got, st = _device_plan(B, lens.tolist(), Hkv, tl, G)
        assert st == 0
        _check_equal(got, OP.plan_dynamic(lens, Hkv, tl, G))
        host, _ = B.plan_host(lens.astype(np.int32), Hkv * 8, Hkv, tl, G)
        h = host.to_numpy()
        assert h["items"].tobytes() == got["items"].tobytes()


def test_batch_larger_than_one_scan_block(B):
    rng = np.random.default_rng(5)
    lens = rng.integers(0, 300, 5000)
    for G in (148, 4096):
        got, st = _device_plan(B, lens.tolist(), 8, 64, G)
        assert st == 0
        _check_equal(got, OP.plan_dynamic(lens, 8, 64, G))


def test_named_workloads_every_step(B):
    for name in ("tiny", "uniform", "extreme", "heavy", "fp8"):
        spec = W.config_spec(name)
        for step in range(spec.steps):
            lens = [L + step for L in spec.seq_lens]
            got, st = _device_plan(B, lens, spec.kv_heads, spec.tile_len, 148)
            assert st == 0
            _check_equal(got, OP.plan_dynamic(lens, spec.kv_heads, spec.tile_len, 148))


def test_bad_lengths_are_flagged_and_dropped(B):
    lens = [10, -1, 40, 100000]
    got, st = _device_plan(B, lens, 2, 16, 5, max_seq=1000)
    assert st & B.DEV_STATUS["bad_seqlen"]
    _check_equal(got, OP.plan_dynamic([10, 0, 40, 0], 2, 16, 5))


def test_static_plan(B):
    for lens, Hkv, tl, S in (([17, 64, 200, 513], 2, 32, 4), ([131072] + [4096] * 31, 8, 128, 2),
                             ([1, 0, 5000, 33], 8, 64, 37)):
        t = torch.tensor(lens, dtype=torch.int32, device="cuda")
        p = B.plan_static(t, Hkv * 8, Hkv, tl, S)
        torch.cuda.synchronize()
        _check_equal(p.to_numpy(), OP.plan_static(lens, Hkv, tl, S), static=True)
