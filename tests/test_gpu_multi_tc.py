"""Several new tokens per request on the tcgen05 kernel (options.multi_kernel = HPC_MULTI_TCGEN05),
through the C ABI, against the fp64 oracle's causal multi-token attention: every q_len from 1 to
4, GQA groups of 8, 4 and 1, ragged lengths (including L = q_len, requests too short for q_len,
and empty ones), several grid sizes (up to twice the SM count), both page layouts, pages outside
the pool, the in-kernel split's record, and a full-size heavy-tailed batch with four new tokens on
sampled requests."""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA
from oracle import planner as OP
from tests.helpers import assert_bf16_tol, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def _q4(q):
    return q if q.dim() == 4 else q.unsqueeze(1).contiguous()


def _oracle(case, rows=None, seq_lens=None, block_table=None):
    return OA.decode_attention_multi(_q4(case.q), case.k_pages, case.v_pages,
                                     case.block_table if block_table is None else block_table,
                                     case.seq_lens if seq_lens is None else seq_lens, requests=rows)


def _run(B, spec, dc, G, kernel="tcgen05", **kw):
    out, st, ws = B.decode_step_multi(_q4(dc["q"]), dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                      spec.kv_heads, spec.tile_len, num_ctas=G, multi_kernel=kernel, **kw)
    torch.cuda.synchronize()
    return out, int(st.item()), ws


@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("Hq,Hkv,P,tl", [(64, 8, 64, 128), (16, 4, 32, 32), (8, 8, 16, 16), (32, 4, 64, 64)])
def test_matches_oracle(B, T, Hq, Hkv, P, tl):
    if T * (Hq // Hkv) > 32:
        pytest.skip("q_len x group above 32: the tcgen05 kernel does not take it")
    lens = (T, T + 1, 15, 16, 17, 64, 65, 127, 128, 129, 300, 1000, 2049)
    spec = W.custom_spec(lens, Hq, Hkv, 128, P, tl, seed=190 + T + P + tl, q_len=T)
    case = W.make_case(spec)
    dc = to_device(case)
    ref = _oracle(case)
    for G in (1, 5, 148, 296):  # 296: more CTAs than SMs (one CTA per SM is resident at a time)
        out, st, ws = _run(B, spec, dc, G)
        assert st == 0
        assert_bf16_tol(out, ref, what=f"tcgen05 q_len {T} {(Hq, Hkv, P, tl)} G={G}")
        assert bool(torch.all(ws[: spec.batch * spec.kv_heads * 4] == 0).item())  # merge tickets back at zero
    # the mma.sync kernel on the same batch: both meet the tolerance, and they agree closely
    other, st2, _ = _run(B, spec, dc, 148, kernel="mma")
    assert st2 == 0 and torch.max(torch.abs(other - out)).item() < 2e-3


def test_short_and_empty_requests(B):
    spec = W.custom_spec((0, 2, 3, 100, 4096), 64, 8, 128, 64, 128, seed=196, q_len=3)
    case = W.make_case(spec)
    dc = to_device(case)
    out, st, ws = _run(B, spec, dc, 7)
    assert st & B.DEV_STATUS["bad_seqlen"]
    assert torch.count_nonzero(out[:2]).item() == 0
    assert_bf16_tol(out[2:], _oracle(case)[2:], what="around short requests")
    out2, _, _ = _run(B, spec, dc, 7, workspace=ws)
    assert torch.equal(out, out2)  # tickets left at zero; the same workspace serves the next call


def test_repeated_runs_are_bit_identical(B):
    """Many short items and ragged last stages, so that item ends and the zeroing of dead V rows
    follow one another closely: every run gives the same bytes (the waits that order the softmax
    after the O products do not depend on timing)."""
    lens = tuple(int(x) for x in np.random.default_rng(198).integers(1, 700, size=48))
    spec = W.custom_spec(lens, 32, 8, 128, 64, 128, seed=198, q_len=4)
    case = W.make_case(spec)
    dc = to_device(case)
    first, st, ws = _run(B, spec, dc, 148)
    assert st == 0
    for _ in range(7):
        again, st2, _ = _run(B, spec, dc, 148, workspace=ws)
        assert st2 == 0
        assert torch.equal(again, first)
    assert_bf16_tol(first, _oracle(case), what="repeated runs")


def test_nhd_layout_is_bit_identical(B):
    spec = W.custom_spec((4, 40, 300, 2049), 32, 8, 128, 64, 128, seed=197, q_len=4)
    case = W.make_case(spec)
    dc = to_device(case)
    hnd, st1, _ = _run(B, spec, dc, 37)
    nhd = dict(dc)
    nhd["k_pages"] = dc["k_pages"].permute(0, 2, 1, 3).contiguous()
    nhd["v_pages"] = dc["v_pages"].permute(0, 2, 1, 3).contiguous()
    got, st2, _ = _run(B, spec, nhd, 37, kv_layout="NHD")
    assert st1 == 0 and st2 == 0
    assert torch.equal(got, hnd)
    assert_bf16_tol(got, _oracle(case), what="NHD q_len 4")


def test_bad_pages_are_left_out(B):
    """A page id outside the pool: page 0 stands in for the copy, HPC_DEV_BAD_PAGE is set, and
    that page's tokens are left out of every query token's softmax."""
    spec = W.custom_spec((40, 300, 700), 32, 4, 128, 16, 32, seed=198, q_len=2)
    case = W.make_case(spec)
    bt = case.block_table.clone()
    bt[1, 2] = case.num_pages + 3
    bt[2, 0] = -1
    dc = to_device(case)
    dc["block_table"] = bt.cuda()
    out, st, _ = _run(B, spec, dc, 5)
    assert st == B.DEV_STATUS["bad_page"] and torch.isfinite(out).all()
    # reference: fp64 causal attention of every query token over the keys that remain (written out
    # here on the kept tokens, from the definition the oracle follows)
    ref = np.zeros_like(out.cpu().numpy(), dtype=np.float64)
    q = case.q.double().numpy()
    P, grp = 16, 8
    for r, L in enumerate(spec.seq_lens):
        for g in range(spec.kv_heads):
            toks = [t for t in range(L) if 0 <= int(bt[r, t // P]) < case.num_pages]
            K = np.array([case.k_pages[int(bt[r, t // P]), g, t % P].double().numpy() for t in toks])
            V = np.array([case.v_pages[int(bt[r, t // P]), g, t % P].double().numpy() for t in toks])
            pos = np.array(toks)
            for tq in range(2):
                lim = L - 2 + tq
                sel = pos <= lim
                for h in range(g * grp, (g + 1) * grp):
                    s = (K[sel] @ q[r, tq, h]) / np.sqrt(128.0)
                    w = np.exp(s - s.max())
                    ref[r, tq, h] = (w / w.sum()) @ V[sel]
    assert_bf16_tol(out, ref, what="bad pages left out")


def test_record_matches_the_oracle_split(B):
    spec = W.config_spec("heavy")
    lens = list(spec.seq_lens)
    Bn, Hkv = len(lens), spec.kv_heads
    dev = torch.device("cuda")
    max_pages = -(-max(lens) // spec.page_size) + 1
    bt = torch.zeros((Bn, max_pages), dtype=torch.int32, device=dev)
    kp = torch.randn((1, Hkv, spec.page_size, 128), generator=torch.Generator().manual_seed(1)).bfloat16().to(dev)
    q = torch.randn((Bn, 4, spec.num_heads, 128), generator=torch.Generator().manual_seed(2)).bfloat16().to(dev)
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    G = torch.cuda.get_device_properties(0).multi_processor_count
    ri = Bn * Hkv + 1
    for cost in (0, None):
        rec = torch.full((B.record_bytes(G, ri),), 0xA5, dtype=torch.uint8, device=dev)
        _, st, _ = B.decode_step_multi(q, kp, kp, bt, seq, Hkv, spec.tile_len, num_ctas=G, item_cost=cost,
                                       record=rec, record_items=ri, multi_kernel="tcgen05")
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        heads, items = B.read_record(rec, G, ri)
        split = OP.plan_cost_split(lens, Hkv, spec.tile_len, G, int(heads[0]["item_cost"]))
        for g in range(G):
            assert (int(heads[g]["unit_begin"]), int(heads[g]["unit_end"])) == (int(split.unit_begin[g]),
                                                                                 int(split.unit_end[g]))
            assert int(heads[g]["n_items"]) == len(split.items[g])
            assert items[g].tobytes() == split.items[g].astype(B.ITEM_DTYPE).tobytes()


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
    assert_bf16_tol(out[rows], _oracle(sub), what="heavy-tailed, 4 new tokens, tcgen05")
    again, _, _ = _run(B, spec, dc, 148)
    assert torch.equal(out, again)  # run to run: bit-identical
