"""The single-launch step (hpc_decode_step: in-kernel planning, attention and ticket merge)
against the fp64 oracle, on the same cases as the three-launch path. Also checked: merge
tickets are left at zero, reuse of one workspace across steps (including the 8 re-planned
heavy-tailed steps), determinism, and zero rows for empty or invalid requests."""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from tests.helpers import assert_bf16_tol, errors, oracle_out, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def _fused(B, spec, dc, seq_lens=None, num_ctas=None, workspace=None, out_dtype=torch.float32, q=None,
           item_cost=None):
    out, st, ws = B.decode_step_fused(dc["q"] if q is None else q, dc["k_pages"], dc["v_pages"], dc["block_table"],
                                      dc["seq_lens"] if seq_lens is None else seq_lens, spec.num_heads,
                                      spec.kv_heads, spec.tile_len, kv_dtype=spec.kv_dtype, k_scale=dc["k_scale"],
                                      v_scale=dc["v_scale"], num_ctas=num_ctas, workspace=workspace,
                                      out_dtype=out_dtype, item_cost=item_cost)
    torch.cuda.synchronize()
    return out, int(st.item()), ws


def _tickets_zero(ws, batch, kv_heads):
    return bool(torch.all(ws[: batch * kv_heads * 4] == 0).item())


def test_tiny_every_cta_count(B):
    spec = W.config_spec("tiny")
    case = W.make_case(spec)
    dc = to_device(case)
    ref = oracle_out(case)
    for G in (1, 2, 3, 8, 54, 148, 296):
        out, st, ws = _fused(B, spec, dc, num_ctas=G)
        assert st == 0
        assert_bf16_tol(out, ref, what=f"fused tiny G={G}")
        assert _tickets_zero(ws, spec.batch, spec.kv_heads)


@pytest.mark.parametrize("Hq,Hkv,D,P,tl", [
    (8, 2, 64, 16, 32), (8, 1, 128, 64, 128), (16, 2, 128, 64, 64), (64, 8, 128, 64, 128),
    (4, 2, 64, 32, 16), (8, 4, 128, 16, 16), (8, 8, 64, 64, 256), (32, 8, 128, 128, 128),
])
def test_shapes_ragged(B, Hq, Hkv, D, P, tl):
    lens = (1, 15, 16, 17, 63, 64, 65, 129, 300, 1000, 2049)
    spec = W.custom_spec(lens, Hq, Hkv, D, P, tl, seed=Hq + D + P + tl + 1)
    case = W.make_case(spec)
    dc = to_device(case)
    ref = oracle_out(case)
    for G in (5, 37, 148):
        out, st, ws = _fused(B, spec, dc, num_ctas=G)
        assert st == 0
        assert_bf16_tol(out, ref, what=f"fused {(Hq, Hkv, D, P, tl, G)}")
        assert _tickets_zero(ws, spec.batch, spec.kv_heads)


@pytest.mark.parametrize("cost", [0, 16, 200, 1024])
def test_item_cost_split(B, cost):
    """The split of the single-launch step with a fixed cost per item (options.item_cost, in 1/16
    of a tile; 0 is the pages' split by tiles alone). Whatever the cost, every tile lands in
    exactly one CTA, every split segment's piece count and partial slots agree (the merge
    tickets end at zero) and the output equals the oracle, for CTA counts from 1 to 2 per SM."""
    lens = (1, 15, 16, 17, 63, 64, 65, 129, 300, 1000, 2049, 0, 5000)
    spec = W.custom_spec(lens, 16, 4, 128, 64, 64, seed=61)
    case = W.make_case(spec)
    dc = to_device(case)
    ref = oracle_out(case)
    for G in (1, 3, 8, 37, 148, 296):
        out, st, ws = _fused(B, spec, dc, num_ctas=G, item_cost=cost)
        assert st == 0
        assert_bf16_tol(out, ref, what=f"fused, item cost {cost}, G={G}")
        assert _tickets_zero(ws, spec.batch, spec.kv_heads)


@pytest.mark.parametrize("D,Bmax", [(128, 4095), (64, 2047)])
def test_largest_batch(B, D, Bmax):
    """The single launch keeps the per-request prefix (tile and segment counts packed in one
    int64) in shared memory. Its largest batch, 4095 requests at head_dim 128 and 2047 at 64,
    runs with short ragged lengths and empty requests, with and without the item cost, and
    matches the oracle on sampled requests. One request more is refused before launch."""
    rng = np.random.default_rng(D)
    lens = [int(x) for x in rng.integers(0, 80, size=Bmax)]
    spec = W.custom_spec(lens, 8, 2, D, 16, 32, seed=D + 7)
    case = W.make_case(spec)
    dc = to_device(case)
    empty = [i for i, L in enumerate(lens) if L == 0][:3]
    rows = sorted(set([0, 1, 2, Bmax // 2, Bmax - 2, Bmax - 1] + empty + [int(x) for x in rng.integers(0, Bmax, 6)]))
    ref = oracle_out(W.make_case(spec, requests=rows))
    for cost in (0, None):
        out, st, ws = _fused(B, spec, dc, item_cost=cost)
        assert st == 0
        assert_bf16_tol(out[rows], ref, what=f"largest batch {Bmax}, D {D}, cost {cost}")
        assert _tickets_zero(ws, spec.batch, spec.kv_heads)
    more = torch.cat([dc["seq_lens"], dc["seq_lens"][:1]])
    bt = torch.cat([dc["block_table"], dc["block_table"][:1]])
    q = torch.cat([dc["q"], dc["q"][:1]])
    with pytest.raises(B.HpcError, match="single-launch limit"):
        B.decode_step_fused(q, dc["k_pages"], dc["v_pages"], bt, more, 8, 2, 32)


def test_empty_and_invalid_requests(B):
    spec = W.custom_spec((0, 40, 5, 200), 8, 2, 64, 16, 32, seed=51)
    case = W.make_case(spec)
    dc = to_device(case)
    ref = oracle_out(case)
    out = torch.full((4, 8, 64), 3.0, device="cuda")
    out, st, ws = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 8, 2,
                                      32, num_ctas=7, out=out)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.all(out[0] == 0)
    assert_bf16_tol(out, ref, what="fused empty request")
    bad = dc["seq_lens"].clone()
    bad[2] = 10**6  # beyond the block table
    out2, st2, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], bad, 8, 2, 32,
                                       num_ctas=7)
    torch.cuda.synchronize()
    assert int(st2.item()) & B.DEV_STATUS["bad_seqlen"]
    assert torch.all(out2[2] == 0) and torch.isfinite(out2).all()


def test_matches_three_launch_path_and_is_deterministic(B):
    # with no item cost the single launch splits the tiles exactly as the planner does
    spec = W.custom_spec((5000, 40, 999, 131, 7777), 64, 8, 128, 64, 128, seed=52)
    case = W.make_case(spec)
    dc = to_device(case)
    split, _, _ = B.decode_step(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 64, 8,
                                128, num_ctas=148)
    outs, ws = [], None
    for _ in range(3):
        o, st, ws = _fused(B, spec, dc, num_ctas=148, workspace=ws, item_cost=0)
        assert st == 0
        outs.append(o.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    assert torch.max(torch.abs(outs[0] - split)).item() < 1e-5


def test_bf16_output(B):
    spec = W.custom_spec((17, 200, 513, 1024), 16, 2, 128, 64, 128, seed=53)
    case = W.make_case(spec)
    dc = to_device(case)
    ref = oracle_out(case)
    out, st, _ = _fused(B, spec, dc, num_ctas=7, out_dtype=torch.bfloat16)
    ref_b = torch.from_numpy(ref).to(torch.bfloat16).float().numpy()
    ulp = np.spacing(np.abs(ref_b).astype(np.float32)).astype(np.float64) * 65536.0
    assert np.all(np.abs(out.float().cpu().numpy() - ref_b) <= ulp + 2e-3)


@pytest.mark.parametrize("name", ["uniform", "extreme"])
def test_full_size(B, name):
    spec = W.config_spec(name)
    case = W.make_case(spec)
    dc = to_device(case)
    out, st, ws = _fused(B, spec, dc)
    assert st == 0
    rows = sorted({0, 1, spec.batch // 2, spec.batch - 1})
    ref = oracle_out(W.make_case(spec, requests=rows))
    assert_bf16_tol(out[rows], ref, what=f"fused {name}")
    assert _tickets_zero(ws, spec.batch, spec.kv_heads)


def test_heavy_eight_steps_one_workspace(B):
    spec = W.config_spec("heavy")
    case = W.make_case(spec)
    dc = to_device(case)
    lens = np.array(spec.seq_lens)
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 7, 33})
    sub = W.make_case(spec, requests=rows)
    seq = dc["seq_lens"].clone()
    ws = None
    for step in range(spec.steps):
        out, st, ws = _fused(B, spec, dc, seq_lens=seq, workspace=ws)
        assert st == 0
        ref = oracle_out(sub, seq_lens=sub.seq_lens + step)
        assert_bf16_tol(out[rows], ref, what=f"fused heavy step {step}")
        seq += 1


def test_fp8_with_prologue(B):
    from oracle import attention as OA
    from oracle import prologue as OR
    spec = W.custom_spec((1, 2, 100, 1024, 5000, 16384), 64, 8, 128, 64, 128, kv_dtype="e4m3", prologue=True,
                         seed=54)
    case = W.make_case(spec)
    dc = to_device(case)
    q = B.prologue(dc["qkv"], dc["q_norm_w"], dc["k_norm_w"], dc["k_pages"], dc["v_pages"], dc["block_table"],
                   dc["seq_lens"], 64, 8, kv_dtype="e4m3", k_scale=dc["k_scale"], v_scale=dc["v_scale"])
    out, st, _ = _fused(B, spec, dc, q=q, num_ctas=148)
    assert st == 0
    kp, vp = case.k_pages.numpy().copy(), case.v_pages.numpy().copy()
    qr, _, _, _ = OR.decode_prologue(case.qkv, case.q_norm_w, case.k_norm_w, 1e-6, 1e6, case.seq_lens.numpy(),
                                     case.block_table.numpy(), kp, vp, "e4m3", case.k_scale, case.v_scale, 64, 8)
    ref = OA.decode_attention(qr, kp, vp, case.block_table, case.seq_lens, kv_dtype="e4m3", k_scale=case.k_scale,
                              v_scale=case.v_scale)
    mx, _ = errors(out, ref)
    assert mx <= 5e-2, mx
