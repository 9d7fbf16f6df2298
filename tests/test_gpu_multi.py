"""Several new tokens per request (hpc_decode_step_multi) through the C ABI, against the
fp64 oracle's causal multi-token attention: every q_len from 1 to 4, bf16 and E4M3 caches,
every stage size, ragged lengths (including L = q_len and requests too short to hold q_len
tokens), several grid sizes, and a full-size heavy-tailed batch on sampled requests."""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA
from tests.helpers import assert_bf16_tol, errors, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def _q4(q):
    """q as [B, q_len, Hq, D] (a one-token case stores it as [B, Hq, D])."""
    return q if q.dim() == 4 else q.unsqueeze(1).contiguous()


def _oracle(case, rows=None):
    return OA.decode_attention_multi(_q4(case.q), case.k_pages, case.v_pages, case.block_table, case.seq_lens,
                                     kv_dtype=case.spec.kv_dtype, k_scale=case.k_scale, v_scale=case.v_scale,
                                     requests=rows)


def _run(B, spec, dc, G, **kw):
    out, st, ws = B.decode_step_multi(_q4(dc["q"]), dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                      spec.kv_heads, spec.tile_len, kv_dtype=spec.kv_dtype, k_scale=dc["k_scale"],
                                      v_scale=dc["v_scale"], num_ctas=G, **kw)
    torch.cuda.synchronize()
    return out, int(st.item()), ws


def _check(out, ref, kv, what):
    if kv == "bf16":
        assert_bf16_tol(out, ref, what=what)
    else:
        mx, _ = errors(out, ref)
        assert mx <= 5e-2, (what, mx)


@pytest.mark.parametrize("mk", ["default", "mma"])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("kv,Hq,Hkv,D,P,tl", [
    ("bf16", 8, 2, 64, 16, 32), ("bf16", 64, 8, 128, 64, 128), ("bf16", 16, 4, 128, 32, 32),
    ("e4m3", 64, 8, 128, 64, 128), ("e4m3", 16, 2, 128, 16, 48),
])
def test_matches_oracle(B, T, kv, Hq, Hkv, D, P, tl, mk):
    """The default kernel (tcgen05 for three or four tokens on a bf16 cache with head_dim 128)
    and the mma.sync consumers, against the oracle."""
    if tl % P and P % tl:
        pytest.skip("tile/page combination not supported")
    lens = (T, T + 1, 15, 16, 17, 64, 65, 129, 300, 1000, 2049)
    spec = W.custom_spec(lens, Hq, Hkv, D, P, tl, kv_dtype=kv, seed=90 + T + D + P, q_len=T)
    case = W.make_case(spec)
    dc = to_device(case)
    ref = _oracle(case)
    for G in (5, 148):
        out, st, _ = _run(B, spec, dc, G, multi_kernel=mk)
        assert st == 0
        _check(out, ref, kv, f"q_len {T} {kv} {(Hq, Hkv, D, P, tl)} G={G} {mk}")


def test_one_token_is_the_single_launch_step(B):
    spec = W.custom_spec((1, 17, 300, 2049), 16, 2, 128, 64, 128, seed=95)
    case = W.make_case(spec)
    dc = to_device(case)
    one, st1, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 16, 2,
                                      128, num_ctas=37)
    multi, st2, _ = B.decode_step_multi(dc["q"].unsqueeze(1).contiguous(), dc["k_pages"], dc["v_pages"],
                                        dc["block_table"], dc["seq_lens"], 2, 128, num_ctas=37)
    torch.cuda.synchronize()
    assert int(st1.item()) == 0 and int(st2.item()) == 0
    assert torch.equal(multi[:, 0], one)


def test_short_requests_are_flagged_and_zero(B):
    spec = W.custom_spec((0, 2, 3, 100), 16, 2, 128, 64, 128, seed=96, q_len=3)
    case = W.make_case(spec)
    dc = to_device(case)
    out, st, ws = _run(B, spec, dc, 7)
    assert st & B.DEV_STATUS["bad_seqlen"]
    assert torch.count_nonzero(out[:2]).item() == 0
    assert_bf16_tol(out[2:], _oracle(case)[2:], what="around short requests")
    # tickets left at zero: the same workspace serves the next call
    out2, _, _ = _run(B, spec, dc, 7, workspace=ws)
    assert torch.equal(out, out2)


def test_heavy_tailed_four_tokens_full_size(B):
    base = W.config_spec("heavy")
    spec = W.custom_spec(base.seq_lens, base.num_heads, base.kv_heads, base.head_dim, base.page_size, base.tile_len,
                         seed=0, q_len=4, name="heavy4")
    case = W.make_case(spec)
    dc = to_device(case)
    out, st, _ = _run(B, spec, dc, 148)
    assert st == 0
    lens = np.array(spec.seq_lens)
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 7, 33})
    sub = W.make_case(spec, requests=rows)
    ref = _oracle(sub)
    assert_bf16_tol(out[rows], ref, what="heavy-tailed, 4 new tokens")
    again, _, _ = _run(B, spec, dc, 148)
    assert torch.equal(out, again)  # run to run: bit-identical


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_nhd_layout_is_bit_identical(B, kv):
    """Several new tokens on the vLLM page layout: the same TMA boxes land in shared memory,
    so the output equals the HND run bit for bit."""
    spec = W.custom_spec((3, 40, 300, 2049), 32, 8, 128, 64, 128, kv_dtype=kv, seed=97, q_len=3)
    case = W.make_case(spec)
    dc = to_device(case)
    hnd, st1, _ = _run(B, spec, dc, 37)
    nhd = dict(dc)
    nhd["k_pages"] = dc["k_pages"].permute(0, 2, 1, 3).contiguous()
    nhd["v_pages"] = dc["v_pages"].permute(0, 2, 1, 3).contiguous()
    got, st2, _ = _run(B, spec, nhd, 37, kv_layout="NHD")
    assert st1 == 0 and st2 == 0
    assert torch.equal(got, hnd)
    _check(got, _oracle(case), kv, f"NHD q_len 3 {kv}")
