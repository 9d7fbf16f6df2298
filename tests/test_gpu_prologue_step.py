"""The single-launch step with the decode prologue folded in (hpc_decode_step_prologue),
through the C ABI, against the fp64 oracle.

The oracle applies its own prologue (RMSNorm, NeoX RoPE, the new token's K/V encoded into its
copy of the cache), then exact attention. q is held as bf16 after the prologue (the kernel's
reading of the pages' silence on it), so a bf16 cache is compared with the oracle given
bf16(q); an E4M3 cache is compared with fp64 q under the E4M3 tolerance, as the two-kernel
path is. The cache the kernel leaves behind must hold the oracle's new token in every
written slot and be unchanged everywhere else."""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA
from oracle import fp8 as OF
from oracle import prologue as OR
from tests.helpers import assert_bf16_tol, errors, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def nhd(t):
    return t.permute(0, 2, 1, 3).contiguous()


def _host_bits(pages, kv):
    return pages.numpy().copy() if kv == "e4m3" else pages.view(torch.int16).numpy().view(np.uint16).copy()


def _as_pages(bits, kv):
    return bits if kv == "e4m3" else torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def _oracle(case, qw, kw, kv, Hq, Hkv):
    """Oracle prologue into host copies of the cache, then oracle attention."""
    kb, vb = _host_bits(case.k_pages, kv), _host_bits(case.v_pages, kv)
    q, k_new, v_new, writes = OR.decode_prologue(case.qkv, qw, kw, 1e-6, 1e6, case.seq_lens.numpy(),
                                                 case.block_table.numpy(), kb, vb, kv, case.k_scale, case.v_scale,
                                                 Hq, Hkv)
    if kv == "bf16":  # the kernel attends with q rounded to bf16
        q = torch.from_numpy(q).to(torch.bfloat16)
    ref = OA.decode_attention(q, _as_pages(kb, kv), _as_pages(vb, kv), case.block_table, case.seq_lens, kv_dtype=kv,
                              k_scale=case.k_scale, v_scale=case.v_scale)
    return ref, kb, vb, k_new, v_new, writes


def _check_cache(got_k, got_v, kb, vb, k_new, v_new, writes, kv, Hkv):
    """Written slots hold the oracle's new token (E4M3 codes exact except within 1e-5 of a
    rounding midpoint; bf16 within one ulp); every other byte equals the oracle's cache."""
    gk, gv = _host_bits(got_k, kv), _host_bits(got_v, kv)
    mask = np.zeros(gk.shape[:3], dtype=bool)
    for (r, page, slot) in writes:
        mask[page, :, slot] = True
        for g in range(Hkv):
            for got, ref_val, ref_code in ((gk[page, g, slot], k_new[r, g], kb[page, g, slot]),
                                           (gv[page, g, slot], v_new[r, g], vb[page, g, slot])):
                if kv == "e4m3":
                    near = OF.midpoint_distance(ref_val) <= 1e-5
                    assert not ((got != ref_code) & ~near).any()
                else:
                    gotf = torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).double().numpy()
                    u = np.spacing(np.abs(ref_val).astype(np.float32)).astype(np.float64) * 65536.0
                    assert np.all(np.abs(gotf - ref_val) <= u)
    assert np.array_equal(gk[~mask], kb[~mask]) and np.array_equal(gv[~mask], vb[~mask])


@pytest.mark.parametrize("kv,Hq,Hkv,D,P,tl,layout", [
    ("bf16", 8, 2, 64, 16, 32, "HND"), ("bf16", 64, 8, 128, 64, 128, "HND"), ("bf16", 16, 4, 128, 32, 64, "NHD"),
    ("e4m3", 64, 8, 128, 64, 128, "HND"), ("e4m3", 16, 2, 128, 16, 32, "NHD"), ("e4m3", 32, 8, 128, 128, 128, "HND"),
])
def test_step_with_prologue_matches_oracle(B, kv, Hq, Hkv, D, P, tl, layout):
    lens = (1, 2, 17, 64, 65, 300, 1000, 2049)
    spec = W.custom_spec(lens, Hq, Hkv, D, P, tl, kv_dtype=kv, prologue=True, seed=81 + D + P)
    case = W.make_case(spec)
    rng = np.random.default_rng(P + tl)
    qw = torch.from_numpy(rng.uniform(0.5, 1.5, D).astype(np.float32))
    kw = torch.from_numpy(rng.uniform(0.5, 1.5, D).astype(np.float32))
    ref, kb, vb, k_new, v_new, writes = _oracle(case, qw, kw, kv, Hq, Hkv)
    for G in (5, 148):
        dc = to_device(case)
        kp, vp = (nhd(dc["k_pages"]), nhd(dc["v_pages"])) if layout == "NHD" else (dc["k_pages"], dc["v_pages"])
        out, st, _ = B.decode_step_prologue(dc["qkv"], qw.cuda(), kw.cuda(), kp, vp, dc["block_table"],
                                            dc["seq_lens"], Hq, Hkv, tl, kv_dtype=kv, kv_layout=layout,
                                            k_scale=dc["k_scale"], v_scale=dc["v_scale"], num_ctas=G)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        if kv == "bf16":
            assert_bf16_tol(out, ref, what=f"prologue step {kv} {layout} G={G}")
        else:
            assert errors(out, ref)[0] <= 5e-2
        if layout == "NHD":
            kp, vp = kp.permute(0, 2, 1, 3), vp.permute(0, 2, 1, 3)
        _check_cache(kp.cpu(), vp.cpu(), kb, vb, k_new, v_new, writes, kv, Hkv)


def test_agrees_with_prologue_kernel_then_step(B):
    """Same inputs through hpc_decode_prologue + hpc_decode_step: both attend with bf16 q
    from the same formulas, so the outputs agree to the rounding of q's norm sum."""
    spec = W.custom_spec((1, 40, 513, 4000), 32, 4, 128, 64, 128, kv_dtype="e4m3", prologue=True, seed=82)
    case = W.make_case(spec)
    a, b = to_device(case), to_device(case)
    out1, st1, _ = B.decode_step_prologue(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["k_pages"], a["v_pages"],
                                          a["block_table"], a["seq_lens"], 32, 4, 128, kv_dtype="e4m3",
                                          k_scale=a["k_scale"], v_scale=a["v_scale"], num_ctas=37)
    q = B.prologue(b["qkv"], b["q_norm_w"], b["k_norm_w"], b["k_pages"], b["v_pages"], b["block_table"],
                   b["seq_lens"], 32, 4, kv_dtype="e4m3", k_scale=b["k_scale"], v_scale=b["v_scale"])
    out2, st2, _ = B.decode_step_fused(q, b["k_pages"], b["v_pages"], b["block_table"], b["seq_lens"], 32, 4, 128,
                                       kv_dtype="e4m3", k_scale=b["k_scale"], v_scale=b["v_scale"], num_ctas=37)
    torch.cuda.synchronize()
    assert int(st1.item()) == 0 and int(st2.item()) == 0
    assert torch.equal(a["k_pages"], b["k_pages"]) and torch.equal(a["v_pages"], b["v_pages"])
    assert torch.max(torch.abs(out1 - out2)).item() <= 2e-3


def test_empty_request_is_flagged_and_zero(B):
    spec = W.custom_spec((5, 0, 130), 16, 2, 128, 64, 128, kv_dtype="bf16", prologue=True, seed=83)
    case = W.make_case(spec)
    dc = to_device(case)
    out, st, _ = B.decode_step_prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"],
                                        dc["block_table"], dc["seq_lens"], 16, 2, 128, num_ctas=7)
    torch.cuda.synchronize()
    assert int(st.item()) & B.DEV_STATUS["bad_seqlen"]
    assert torch.count_nonzero(out[1]).item() == 0
    sub = W.make_case(spec, requests=[0, 2])  # the same two requests, bit for bit
    ref, *_ = _oracle(sub, sub.q_norm_w, sub.k_norm_w, "bf16", 16, 2)
    assert_bf16_tol(out[[0, 2]], ref, what="prologue step around an empty request")


def test_fp8_workload_full_size(B):
    """The large-batch E4M3 workload (256 requests, prologue with unit weights) in one launch,
    checked on sampled requests: their outputs and their new K codes in the cache."""
    spec = W.config_spec("fp8")
    case = W.make_case(spec)
    dc = to_device(case)
    out, st, ws = B.decode_step_prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"],
                                         dc["block_table"], dc["seq_lens"], spec.num_heads, spec.kv_heads,
                                         spec.tile_len, kv_dtype="e4m3", k_scale=dc["k_scale"],
                                         v_scale=dc["v_scale"], num_ctas=148)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    lens = np.array(spec.seq_lens)
    rows = sorted({0, int(np.argmax(lens)), int(np.argmin(lens)), 100, spec.batch - 1})
    sub = W.make_case(spec, requests=rows)
    kb, vb = sub.k_pages.numpy().copy(), sub.v_pages.numpy().copy()
    q, k_new, _, writes = OR.decode_prologue(sub.qkv, sub.q_norm_w, sub.k_norm_w, spec.rms_eps, spec.rope_theta,
                                             sub.seq_lens.numpy(), sub.block_table.numpy(), kb, vb, "e4m3",
                                             sub.k_scale, sub.v_scale, spec.num_heads, spec.kv_heads)
    ref = OA.decode_attention(q, kb, vb, sub.block_table, sub.seq_lens, kv_dtype="e4m3", k_scale=sub.k_scale,
                              v_scale=sub.v_scale)
    mx, _ = errors(out[rows], ref)
    assert mx <= 5e-2, mx
    # the sampled requests' new K codes, at their pages in the full cache
    gk = dc["k_pages"].cpu().numpy()
    bt = case.block_table.numpy()
    for i, r in enumerate(rows):
        pos = int(spec.seq_lens[r]) - 1
        page, slot = bt[r, pos // spec.page_size], pos % spec.page_size
        near = OF.midpoint_distance(k_new[i]) <= 1e-5
        assert not ((gk[page, :, slot] != OF.encode_array(k_new[i])) & ~near).any()
