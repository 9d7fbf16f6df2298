"""The NHD (vLLM-style) cache layout and non-unit QK-norm weights, through the C ABI.

An NHD cache holds the same tokens as the HND cache it is permuted from. Attention on it
must match the fp64 oracle, which is given the HND original, and both step paths
(three launches and one launch) must agree with the HND run. The prologue must write the
new token into the NHD slot. With random (non-unit) norm weights, the RMSNorm-then-RoPE
order matters and is checked against the oracle."""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import fp8 as OF
from oracle import prologue as OR
from tests.helpers import assert_bf16_tol, errors, oracle_out, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def nhd(t):
    """HND [N, Hkv, P, D] -> NHD [N, P, Hkv, D] (same tokens)."""
    return t.permute(0, 2, 1, 3).contiguous()


@pytest.mark.parametrize("kv,Hq,Hkv,D,P,tl", [
    ("bf16", 8, 2, 64, 16, 32), ("bf16", 64, 8, 128, 64, 128), ("bf16", 16, 4, 128, 128, 128),
    ("e4m3", 64, 8, 128, 64, 128), ("e4m3", 16, 2, 128, 16, 32),
])
def test_nhd_attention_both_paths(B, kv, Hq, Hkv, D, P, tl):
    lens = (1, 17, 64, 65, 300, 1000, 2049)
    spec = W.custom_spec(lens, Hq, Hkv, D, P, tl, kv_dtype=kv, seed=61 + D + P)
    case = W.make_case(spec)
    ref = oracle_out(case)
    dc = to_device(case)
    kn, vn = nhd(dc["k_pages"]), nhd(dc["v_pages"])
    common = dict(kv_dtype=kv, k_scale=dc["k_scale"], v_scale=dc["v_scale"])
    hnd, _, _ = B.decode_step(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], Hq, Hkv, tl,
                              num_ctas=37, **common)
    split, _, st1 = B.decode_step(dc["q"], kn, vn, dc["block_table"], dc["seq_lens"], Hq, Hkv, tl, kv_layout="NHD",
                                  num_ctas=37, **common)
    # with no item cost the single launch cuts the tiles where the planner does: same sums
    fused0, st2, _ = B.decode_step_fused(dc["q"], kn, vn, dc["block_table"], dc["seq_lens"], Hq, Hkv, tl,
                                         kv_layout="NHD", num_ctas=37, item_cost=0, **common)
    fused, st3, _ = B.decode_step_fused(dc["q"], kn, vn, dc["block_table"], dc["seq_lens"], Hq, Hkv, tl,
                                        kv_layout="NHD", num_ctas=37, **common)
    torch.cuda.synchronize()
    assert int(st1.item()) == 0 and int(st2.item()) == 0 and int(st3.item()) == 0
    assert torch.equal(split, hnd)  # same boxes in shared memory: bit-identical
    assert torch.max(torch.abs(fused0 - hnd)).item() < 1e-5
    for o in (fused0, fused):
        if kv == "bf16":
            assert_bf16_tol(o, ref, what=f"nhd {kv}")
        else:
            assert errors(o, ref)[0] <= 5e-2


@pytest.mark.parametrize("kv,layout", [("bf16", "HND"), ("e4m3", "HND"), ("bf16", "NHD"), ("e4m3", "NHD")])
def test_prologue_layouts_and_nonunit_weights(B, kv, layout):
    lens = (1, 2, 64, 65, 1000, 16384)
    spec = W.custom_spec(lens, 16, 2, 128, 64, 128, kv_dtype=kv, prologue=True, seed=71)
    case = W.make_case(spec)
    rng = np.random.default_rng(5)
    qw = torch.from_numpy(rng.uniform(0.5, 1.5, 128).astype(np.float32))
    kw = torch.from_numpy(rng.uniform(0.5, 1.5, 128).astype(np.float32))
    dc = to_device(case)
    kp, vp = dc["k_pages"], dc["v_pages"]
    if layout == "NHD":
        kp, vp = nhd(kp), nhd(vp)
    q_out = B.prologue(dc["qkv"], qw.cuda(), kw.cuda(), kp, vp, dc["block_table"], dc["seq_lens"], 16, 2,
                       kv_dtype=kv, kv_layout=layout, k_scale=dc["k_scale"], v_scale=dc["v_scale"])
    torch.cuda.synchronize()
    if layout == "NHD":  # back to HND for the comparison
        kp, vp = kp.permute(0, 2, 1, 3), vp.permute(0, 2, 1, 3)
    k_host = case.k_pages.numpy().copy() if kv == "e4m3" else case.k_pages.view(torch.int16).numpy().view(np.uint16).copy()
    v_host = case.v_pages.numpy().copy() if kv == "e4m3" else case.v_pages.view(torch.int16).numpy().view(np.uint16).copy()
    q, k_new, v_new, writes = OR.decode_prologue(case.qkv, qw, kw, 1e-6, 1e6, case.seq_lens.numpy(),
                                                 case.block_table.numpy(), k_host, v_host, kv, case.k_scale,
                                                 case.v_scale, 16, 2)
    qg = q_out.float().cpu().numpy()
    ulp = np.spacing(np.abs(q).astype(np.float32)).astype(np.float64) * 65536.0
    assert np.all(np.abs(qg - q) <= ulp)
    gk, gv = kp.cpu(), vp.cpu()
    for (r, page, slot) in writes:
        for g in range(2):
            for dev_t, ref_val, ref_code in ((gk, k_new[r, g], k_host[page, g, slot]),
                                             (gv, v_new[r, g], v_host[page, g, slot])):
                row = dev_t[page, g, slot]
                if kv == "e4m3":
                    got = row.numpy()
                    near = OF.midpoint_distance(ref_val) <= 1e-5
                    assert not ((got != ref_code) & ~near).any()
                else:
                    got = row.float().numpy().astype(np.float64)
                    u = np.spacing(np.abs(ref_val).astype(np.float32)).astype(np.float64) * 65536.0
                    assert np.all(np.abs(got - ref_val) <= u)
