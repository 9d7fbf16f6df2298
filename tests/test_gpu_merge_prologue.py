"""Merge kernel and prologue kernel parity through the C ABI, and the large-batch FP8
workload (prologue -> plan -> attention -> merge) at full size on sampled requests."""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import fp8 as OF
from oracle import merge as OM
from oracle import planner as OP
from oracle import prologue as OR
from tests.helpers import errors, oracle_out, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


@pytest.mark.parametrize("lens,Hkv,grp,D,tl,G", [
    ([17, 64, 200, 513], 2, 4, 64, 32, 8),
    ([0, 4096, 131072, 5], 8, 8, 128, 128, 148),
    ([3000] * 40, 1, 2, 128, 64, 33),
])
def test_merge_kernel_vs_oracle(B, lens, Hkv, grp, D, tl, G):
    t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = B.plan(t, Hkv * grp, Hkv, tl, G)
    ref_plan = OP.plan_dynamic(lens, Hkv, tl, G)
    po, pml = W.random_partials(len(lens) * 7 + G, p.max_items, grp, D)
    out = torch.full((len(lens), Hkv * grp, D), float("nan"), device="cuda")
    B.merge(p, po.cuda(), pml.cuda(), out, Hkv * grp)
    torch.cuda.synchronize()
    ref = OM.merge_plan_partials(ref_plan, po.numpy(), pml.numpy(), len(lens), Hkv, grp)
    got = out.cpu().numpy()
    assert len(ref) > 0
    for (r, h), row in ref.items():
        scale = max(1.0, float(np.abs(row).max()))
        assert np.max(np.abs(got[r, h] - row)) <= 2e-6 * scale, (r, h)


def _prologue_case(lens, kv, D=128, Hq=16, Hkv=2, P=64, seed=0):
    spec = W.custom_spec(lens, Hq, Hkv, D, P, 128, kv_dtype=kv, prologue=True, seed=seed)
    return spec, W.make_case(spec)


@pytest.mark.parametrize("kv,D", [("e4m3", 128), ("bf16", 128), ("bf16", 64)])
def test_prologue_vs_oracle(B, kv, D):
    lens = (1, 2, 64, 65, 1000, 16384)
    spec, case = _prologue_case(lens, kv, D=D, seed=11)
    dc = to_device(case)
    q_out = B.prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                       dc["seq_lens"], spec.num_heads, spec.kv_heads, kv_dtype=kv, k_scale=dc["k_scale"],
                       v_scale=dc["v_scale"], eps=spec.rms_eps, rope_theta=spec.rope_theta)
    torch.cuda.synchronize()
    kp = case.k_pages.numpy().copy() if kv == "e4m3" else case.k_pages.view(torch.int16).numpy().view(np.uint16).copy()
    vp = case.v_pages.numpy().copy() if kv == "e4m3" else case.v_pages.view(torch.int16).numpy().view(np.uint16).copy()
    q, k_new, v_new, writes = OR.decode_prologue(
        case.qkv, case.q_norm_w, case.k_norm_w, spec.rms_eps, spec.rope_theta, case.seq_lens.numpy(),
        case.block_table.numpy(), kp, vp, kv, case.k_scale, case.v_scale, spec.num_heads, spec.kv_heads)
    # q: bf16 of a fp32 computation vs the fp64 value -> within one bf16 ulp
    qg = q_out.float().cpu().numpy()
    ulp = np.spacing(np.abs(q).astype(np.float32)).astype(np.float64) * 65536.0
    assert np.all(np.abs(qg - q) <= ulp), np.max(np.abs(qg - q) / ulp)
    # the new K/V slots
    gk = dc["k_pages"].cpu()
    gv = dc["v_pages"].cpu()
    for (r, page, slot) in writes:
        for g in range(spec.kv_heads):
            for src_dev, ref_val, ref_codes in ((gk, k_new[r, g], kp[page, g, slot]), (gv, v_new[r, g], vp[page, g, slot])):
                dev_row = src_dev[page, g, slot]
                if kv == "e4m3":
                    got = dev_row.numpy()
                    near = OF.midpoint_distance(ref_val) <= 1e-5  # reading: either neighbour is fine there
                    bad = (got != ref_codes) & ~near
                    assert not bad.any(), (r, g, np.nonzero(bad))
                    assert np.all(np.abs(got.astype(int) - ref_codes.astype(int)) <= 1)
                else:
                    got = dev_row.float().numpy().astype(np.float64)
                    u = np.spacing(np.abs(ref_val).astype(np.float32)).astype(np.float64) * 65536.0
                    assert np.all(np.abs(got - ref_val) <= u)
    # nothing else in the cache changed
    changed = torch.nonzero((gk.view(torch.uint8) != case.k_pages.view(torch.uint8)).any(-1))
    assert {(int(a), int(c)) for a, _, c in changed.tolist()} <= {(p, s) for _, p, s in writes}


def test_prologue_bad_length_flagged(B):
    spec, case = _prologue_case((5, 0, 7), "bf16", D=64, Hq=8, Hkv=2, P=16, seed=12)
    dc = to_device(case)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_out = B.prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                       dc["seq_lens"], 8, 2, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & B.DEV_STATUS["bad_seqlen"]
    assert torch.all(q_out[1] == 0)


def _fp8_step(B, spec, dc):
    q = B.prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                   dc["seq_lens"], spec.num_heads, spec.kv_heads, kv_dtype="e4m3", k_scale=dc["k_scale"],
                   v_scale=dc["v_scale"], eps=spec.rms_eps, rope_theta=spec.rope_theta)
    out, p, st = B.decode_step(q, dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], spec.num_heads,
                               spec.kv_heads, spec.tile_len, kv_dtype="e4m3", k_scale=dc["k_scale"],
                               v_scale=dc["v_scale"])
    torch.cuda.synchronize()
    return out, int(st.item())


def _fp8_oracle(spec, sub):
    kp, vp = sub.k_pages.numpy().copy(), sub.v_pages.numpy().copy()
    q, _, _, _ = OR.decode_prologue(sub.qkv, sub.q_norm_w, sub.k_norm_w, spec.rms_eps, spec.rope_theta,
                                    sub.seq_lens.numpy(), sub.block_table.numpy(), kp, vp, "e4m3", sub.k_scale,
                                    sub.v_scale, spec.num_heads, spec.kv_heads)
    from oracle import attention as OA
    return OA.decode_attention(q, kp, vp, sub.block_table, sub.seq_lens, kv_dtype="e4m3", k_scale=sub.k_scale,
                               v_scale=sub.v_scale)


def test_fp8_small_with_prologue(B):
    spec, case = _prologue_case((1, 2, 100, 1024, 5000), "e4m3", D=128, Hq=64, Hkv=8, seed=13)
    dc = to_device(case)
    out, st = _fp8_step(B, spec, dc)
    assert st == 0
    ref = _fp8_oracle(spec, case)
    mx, mean = errors(out, ref)
    assert mx <= 5e-2, mx


def test_fp8_full_size_workload(B):
    spec = W.config_spec("fp8")
    case = W.make_case(spec)
    dc = to_device(case)
    out, st = _fp8_step(B, spec, dc)
    assert st == 0
    lens = np.array(spec.seq_lens)
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 0, 128, 255})
    sub = W.make_case(spec, requests=rows)
    ref = _fp8_oracle(spec, sub)
    mx, mean = errors(out[rows], ref)
    assert mx <= 5e-2, mx
    assert torch.isfinite(out).all()
