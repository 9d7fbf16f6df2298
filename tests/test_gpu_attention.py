"""Attention parity through the C ABI against the fp64 oracle: small cases element by
element (several tiles, ragged tails, every supported shape), the named workloads at full
size on sampled requests, plus invariances (page permutation, run-to-run determinism,
plan choice) and edge cases (L = 1, L = 0, NaN in unused slots, bad page ids)."""

import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import fp8 as OF
from tests.helpers import assert_bf16_tol, errors, oracle_out, run_attention, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def _case(lens, Hq=8, Hkv=2, D=64, P=16, tl=32, seed=0, kv="bf16"):
    spec = W.custom_spec(lens, Hq, Hkv, D, P, tl, kv_dtype=kv, seed=seed)
    return spec, W.make_case(spec)


def test_tiny_workload(B):
    spec = W.config_spec("tiny")
    case = W.make_case(spec)
    dc = to_device(case)
    ref = oracle_out(case)
    for G in (1, 3, 8, 148, 296):  # 1 CTA: everything DIRECT in one CTA; 148: 1 tile per CTA
        out, p, st = run_attention(B, spec, dc, num_ctas=G)
        assert st == 0
        assert_bf16_tol(out, ref, what=f"tiny G={G}")


@pytest.mark.parametrize("Hq,Hkv,D,P,tl", [
    (8, 2, 64, 16, 32), (8, 1, 128, 64, 128), (16, 2, 128, 64, 64), (64, 8, 128, 64, 128),
    (4, 2, 64, 32, 16), (8, 4, 128, 16, 16), (8, 8, 64, 64, 256), (32, 8, 128, 128, 128),
    (16, 16, 64, 16, 48),
])
def test_shapes_ragged(B, Hq, Hkv, D, P, tl):
    if tl % P and P % tl:
        pytest.skip("tile/page combination not supported")
    lens = (1, 15, 16, 17, 63, 64, 65, 129, 300, 1000, 2049)
    spec, case = _case(lens, Hq, Hkv, D, P, tl, seed=Hq + D + P + tl)
    dc = to_device(case)
    ref = oracle_out(case)
    for G in (5, 148):
        out, _, st = run_attention(B, spec, dc, num_ctas=G)
        assert st == 0
        assert_bf16_tol(out, ref, what=f"{(Hq, Hkv, D, P, tl, G)}")


@pytest.mark.parametrize("consumer", ["mma.sync", "tcgen05"])
@pytest.mark.parametrize("Hq,Hkv,P,tl", [
    (8, 8, 16, 16), (16, 2, 16, 48), (16, 4, 32, 32), (32, 8, 32, 64), (8, 2, 64, 64), (64, 8, 64, 128),
    (32, 8, 128, 128), (16, 4, 128, 256),
])
def test_e4m3_shapes_ragged(B, Hq, Hkv, P, tl, consumer):
    """E4M3 cache over every stage size (mma.sync: 16, 32 and 64 tokens, one, two and four
    16-token blocks per consumer warp; tcgen05: 128-token stages of 16-, 32- and 64-token boxes)
    and every GQA group size, on both E4M3 kernels, three-launch and single-launch paths."""
    lens = (1, 15, 16, 17, 63, 64, 65, 129, 300, 1000, 2049)
    spec, case = _case(lens, Hq, Hkv, 128, P, tl, seed=Hq + P + tl, kv="e4m3")
    dc = to_device(case)
    ref = oracle_out(case)
    kernel = "tcgen05" if consumer == "tcgen05" else "mma"
    for G in (5, 148):
        out, _, st = run_attention(B, spec, dc, num_ctas=G, e4m3_kernel=kernel)
        assert st == 0
        mx, _ = errors(out, ref)
        assert mx <= 5e-2, (consumer, Hq, Hkv, P, tl, G, mx)
        out, st_t, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                                           dc["seq_lens"], Hq, Hkv, tl, kv_dtype="e4m3", k_scale=dc["k_scale"],
                                           v_scale=dc["v_scale"], num_ctas=G, e4m3_kernel=kernel)
        torch.cuda.synchronize()
        assert int(st_t.item()) == 0
        mx, _ = errors(out, ref)
        assert mx <= 5e-2, (consumer, "fused", Hq, Hkv, P, tl, G, mx)


@pytest.mark.parametrize("path", ["split", "fused"])
def test_e4m3_both_consumers(B, path):
    """An E4M3 cache runs on the mma.sync kernel by default; options.e4m3_kernel selects the
    tcgen05 kernel. Both must meet the E4M3 tolerance on the same ragged batch, on both step
    paths."""
    spec, case = _case((1, 2, 15, 16, 17, 127, 128, 129, 255, 256, 257, 4000), 32, 4, 128, 32, 64, seed=77,
                       kv="e4m3")
    dc = to_device(case)
    ref = oracle_out(case)
    outs = {}
    for consumer in ("tcgen05", "mma.sync"):
        kernel = "tcgen05" if consumer == "tcgen05" else "mma"
        if path == "split":
            out, _, st = run_attention(B, spec, dc, num_ctas=37, e4m3_kernel=kernel)
        else:
            out, st_t, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                                               dc["seq_lens"], 32, 4, 64, kv_dtype="e4m3", k_scale=dc["k_scale"],
                                               v_scale=dc["v_scale"], num_ctas=37, e4m3_kernel=kernel)
            torch.cuda.synchronize()
            st = int(st_t.item())
        assert st == 0
        mx, mean = errors(out, ref)
        assert mx <= 5e-2, (consumer, mx)
        outs[consumer] = out
    assert not torch.equal(outs["tcgen05"], outs["mma.sync"])  # two kernels really ran


def test_bf16_output_within_one_ulp(B):
    spec, case = _case((17, 200, 513, 1024), 16, 2, 128, 64, 128, seed=3)
    dc = to_device(case)
    ref = oracle_out(case)
    out, _, st = run_attention(B, spec, dc, num_ctas=7, out_dtype=torch.bfloat16)
    assert st == 0
    ref_b = torch.from_numpy(ref).to(torch.bfloat16).float().numpy()
    ulp = np.spacing(np.abs(ref_b).astype(np.float32)).astype(np.float64) * 65536.0  # bf16 spacing
    diff = np.abs(out.float().cpu().numpy() - ref_b)
    assert np.all(diff <= ulp + 2e-3)


def test_page_permutation_is_bit_identical(B):
    spec, case = _case((300, 1000, 77), 16, 2, 128, 64, 128, seed=4)
    dc = to_device(case)
    out1, _, _ = run_attention(B, spec, dc, num_ctas=11)
    # same logical K/V, different physical pages
    rng = np.random.default_rng(0)
    perm = torch.from_numpy(rng.permutation(case.num_pages)).long()
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(case.num_pages)
    bt2 = case.block_table.clone()
    ok = bt2 >= 0
    bt2[ok] = inv[bt2[ok].long()].int()
    dc2 = dict(dc)
    dc2["k_pages"] = case.k_pages[perm].cuda()
    dc2["v_pages"] = case.v_pages[perm].cuda()
    dc2["block_table"] = bt2.cuda()
    out2, _, _ = run_attention(B, spec, dc2, num_ctas=11)
    assert torch.equal(out1, out2)


def test_run_to_run_deterministic(B):
    spec, case = _case((5000, 40, 999), 64, 8, 128, 64, 128, seed=5)
    dc = to_device(case)
    outs = [run_attention(B, spec, dc, num_ctas=148)[0] for _ in range(3)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_single_key_returns_v(B):
    spec, case = _case((1, 1, 1), 8, 2, 128, 64, 128, seed=6)
    dc = to_device(case)
    out, _, st = run_attention(B, spec, dc, num_ctas=4)
    for r in range(3):
        for h in range(8):
            v = case.v_pages[int(case.block_table[r, 0]), h // 4, 0].float()
            assert torch.equal(out[r, h].cpu(), v)  # p = 1 exactly, bf16 v is exact in fp32


def test_empty_request_and_nan_slack(B):
    spec, case = _case((0, 33, 200), 8, 2, 64, 16, 32, seed=7)
    # poison every slot past L_r: masking must keep NaN out of the result
    for r, L in enumerate((0, 33, 200)):
        n = int(case.pages_per_req[r])
        for j in range(n):
            page = int(case.block_table[r, j])
            lo = max(0, L - j * 16)
            if lo < 16:
                case.k_pages[page, :, lo:] = float("nan")
                case.v_pages[page, :, lo:] = float("nan")
    dc = to_device(case)
    out = torch.full((3, 8, 64), 7.0, device="cuda")  # the zero rows must be written
    out, _, status = B.decode_step(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 8, 2,
                                   32, num_ctas=6, out=out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle_out(case)
    assert torch.all(out[0] == 0)
    assert torch.isfinite(out).all()
    assert_bf16_tol(out, ref, what="nan slack")


def _attention_without_pages(case, bt, kv):
    """fp64 attention of every (request, head) over the tokens whose block-table entry is a page
    of the pool: the kernels leave a bad page's tokens out of the softmax. Written from the
    oracle's pieces (its pinned single-part softmax state) on the tokens that remain."""
    from oracle import attention as OA
    from oracle import merge as OM
    spec = case.spec
    P, grp = spec.page_size, spec.group
    kp, vp = OA.to_f64(case.k_pages), OA.to_f64(case.v_pages)
    if kv == "e4m3":
        kp, vp = OF.decode_array(case.k_pages.numpy()), OF.decode_array(case.v_pages.numpy())
        kp = kp * case.k_scale.double().numpy()[None, :, None, None]
        vp = vp * case.v_scale.double().numpy()[None, :, None, None]
    q = OA.to_f64(case.q)
    out = np.zeros((spec.batch, spec.num_heads, spec.head_dim))
    for r, L in enumerate(spec.seq_lens):
        toks = [t for t in range(L) if 0 <= int(bt[r, t // P]) < case.num_pages]
        for g in range(spec.kv_heads):
            K = np.array([kp[int(bt[r, t // P]), g, t % P] for t in toks])
            V = np.array([vp[int(bt[r, t // P]), g, t % P] for t in toks])
            for h in range(g * grp, (g + 1) * grp):
                m, lsum, o = OM.partial_state(spec.sm_scale * (K @ q[r, h]), V)
                out[r, h] = o / lsum
    return out


@pytest.mark.parametrize("kv,kernel,tl", [("bf16", "mma", 32), ("bf16", "mma", 16), ("e4m3", "mma", 32),
                                          ("e4m3", "tcgen05", 32), ("e4m3", "tcgen05", 16)])
def test_bad_page_is_left_out_without_fault(B, kv, kernel, tl):
    """A block-table entry outside the pool is never handed to the copy engine: page 0 stands in,
    HPC_DEV_BAD_PAGE is set, and the page's tokens are left out of the request's softmax. The
    outputs then equal attention over the remaining tokens, for every request, on both paths.
    With 16-token tiles a split piece holds only a bad page (no live token) and must merge as
    nothing."""
    spec, case = _case((40, 100, 300), 8, 2, 128, 16, tl, seed=8, kv=kv)
    bt = case.block_table.clone()
    bt[1, 2] = case.num_pages + 5
    bt[0, 0] = -3
    bt[2, 5] = case.num_pages
    dc = to_device(case)
    dc["block_table"] = bt.cuda()
    ref = _attention_without_pages(case, bt.numpy(), kv)
    for G in (4, 148):
        out, _, st = run_attention(B, spec, dc, num_ctas=G, e4m3_kernel=kernel)
        fused, st_f, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                                             dc["seq_lens"], 8, 2, tl, kv_dtype=kv, k_scale=dc["k_scale"],
                                             v_scale=dc["v_scale"], num_ctas=G, e4m3_kernel=kernel)
        torch.cuda.synchronize()
        for o, s_ in ((out, st), (fused, int(st_f.item()))):
            assert s_ == B.DEV_STATUS["bad_page"]
            assert torch.isfinite(o).all()
            if kv == "bf16":
                assert_bf16_tol(o, ref, what=f"bad pages, G={G}")
            else:
                assert errors(o, ref)[0] <= 5e-2


def test_static_plan_matches_oracle(B):
    spec = W.config_spec("tiny")
    case = W.make_case(spec)
    dc = to_device(case)
    ref = oracle_out(case)
    for S in (1, 2, 4, 37):
        out, _, st = run_attention(B, spec, dc, static_splits=S)
        assert st == 0
        assert_bf16_tol(out, ref, what=f"static S={S}")


def test_e4m3_cache_small(B):
    spec, case = _case((1, 17, 64, 300, 1025), 64, 8, 128, 64, 128, seed=9, kv="e4m3")
    dc = to_device(case)
    ref = oracle_out(case)
    for G in (3, 148):
        out, _, st = run_attention(B, spec, dc, num_ctas=G)
        assert st == 0
        mx, mean = errors(out, ref)
        assert mx <= 5e-2, mx
    # The split moves only the running maxima against which p is rounded before the P.V
    # product. The mma.sync kernel rounds p to f16 (11 bits); the tcgen05 kernel sends p (scaled
    # by 2^8, so p <= 256) as an E4M3 high code plus an E4M3 residual code, off by at most
    # 2^-8 p + 2^-10 (the residual's subnormal spacing is 2^-9) against a normaliser l of at
    # least 256 (the maximum's own p). For the coarser of the two, one split's output is within
    # max|v| (2^-8 + L 2^-18) of the exact mix, and two splits within twice that.
    o1, _, _ = run_attention(B, spec, dc, num_ctas=1)
    o2, _, _ = run_attention(B, spec, dc, num_ctas=148)
    vmax = float(np.nanmax(np.abs(OF.decode_array(case.v_pages.numpy())) * case.v_scale.numpy()[None, :, None, None]))
    bound = 2 * vmax * (2.0**-8 + max(spec.seq_lens) * 2.0**-18)
    assert torch.max(torch.abs(o1 - o2)).item() <= bound


# ---------------------------------------------------------------- full-size workloads

def _sample_rows(spec, picks):
    return sorted(set(int(r) for r in picks if 0 <= r < spec.batch))


@pytest.mark.parametrize("name", ["uniform", "extreme"])
def test_full_size_bf16(B, name):
    spec = W.config_spec(name)
    case = W.make_case(spec)
    dc = to_device(case)
    out, p, st = run_attention(B, spec, dc)  # the launch configuration the bench times
    assert st == 0
    rows = _sample_rows(spec, [0, 1, spec.batch // 2, spec.batch - 1])
    sub = W.make_case(spec, requests=rows)
    ref = oracle_out(sub)
    assert_bf16_tol(out[rows], ref, what=name)
    assert torch.isfinite(out).all()


def test_full_size_heavy_eight_steps(B):
    spec = W.config_spec("heavy")
    case = W.make_case(spec)
    dc = to_device(case)
    lens = np.array(spec.seq_lens)
    rows = _sample_rows(spec, [int(np.argmax(lens)), int(np.argmin(lens)), 7, 33])
    sub = W.make_case(spec, requests=rows)
    seq = dc["seq_lens"].clone()
    for step in range(spec.steps):
        out, _, st = run_attention(B, spec, dc, seq_lens=seq)  # re-planned from the device lengths
        assert st == 0
        ref = oracle_out(sub, seq_lens=sub.seq_lens + step)
        assert_bf16_tol(out[rows], ref, what=f"heavy step {step}")
        seq += 1  # lengths grow on the device; nothing leaves the GPU between steps
