"""Log-sum-exp output, the log-sum-exp merge and request-sharded placement, through the
C ABI on one GPU.

* hpc_decode_step_lse writes the same output as hpc_decode_step, and lse matches the fp64
  oracle's log-sum-exp.
* hpc_merge_lse equals its definition (float64 torch) on random parts, -inf parts included.
* hpc_merge_lse_gather (parts found through an index) equals its definition; a single part is
  copied bit for bit. hpc_gather_rows is an exact row gather. Both flag indices out of range.
* A batch sharded over 2, 3 and 4 ranks gives the unsharded oracle result. The ranks run
  one after another in this process: each computes its parts, their (out, lse) are stacked
  as the all-gather would stack them, and split requests are merged. No kernel waits on
  another rank.
"""
import math

import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import shard as S
from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA
from tests.helpers import assert_bf16_tol, errors, oracle_out, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_lse_output(B, kv):
    spec = W.custom_spec((0, 1, 17, 300, 1000, 4097), 32, 4, 128, 64, 128, kv_dtype=kv, seed=31)
    case = W.make_case(spec)
    dc = to_device(case)
    kw = dict(kv_dtype=kv, k_scale=dc["k_scale"], v_scale=dc["v_scale"], num_ctas=37)
    out, lse, st, _ = B.decode_step_lse(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 32,
                                        4, 128, **kw)
    ref_out, _, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 32,
                                        4, 128, **kw)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(out, ref_out)
    ref = OA.decode_lse(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens, kv_dtype=kv,
                        k_scale=case.k_scale)
    got = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isneginf(got[0])) and np.all(np.isneginf(ref[0]))
    assert np.max(np.abs(got[1:] - ref[1:])) <= 1e-4


def test_merge_lse_definition(B):
    g = torch.Generator().manual_seed(5)
    parts, rows, D = 5, 70, 128
    outs = torch.randn(parts, rows, D, generator=g)
    lses = torch.randn(parts, rows, generator=g) * 4
    lses[1, :10] = -math.inf
    lses[:, 20] = -math.inf  # a row with no keys at all
    o, l = B.merge_lse(outs.cuda(), lses.cuda())
    torch.cuda.synchronize()
    ld = lses.double()
    M = ld.max(0).values
    Mf = torch.where(torch.isinf(M), torch.zeros_like(M), M)
    w = torch.exp(ld - Mf)
    L = Mf + torch.log(w.sum(0))
    ref = (torch.exp(ld - L)[..., None] * outs.double()).sum(0)
    ref[20] = 0.0
    assert torch.max(torch.abs(o.cpu().double() - ref)).item() <= 1e-5
    lc = l.cpu().double()
    assert torch.isneginf(lc[20]) and torch.max(torch.abs(lc[:20] - L[:20])).item() <= 1e-5


def test_merge_lse_gather_definition(B):
    g = torch.Generator().manual_seed(6)
    rows, Hq, D = 23, 8, 128
    outs = torch.randn(rows, Hq, D, generator=g)
    lses = torch.randn(rows, Hq, generator=g) * 4
    lses[3, :2] = -math.inf  # a part with no mass for two heads
    idx = torch.tensor([[-1, -1, -1, -1],   # no part: zeros, -inf
                        [7, -1, -1, -1],    # one part: copied exactly
                        [-1, 2, -1, 11],    # two parts, unused entries between
                        [3, 0, 22, 5],      # four parts
                        [3, -1, -1, -1]],   # one part whose lse is -inf for two heads
                       dtype=torch.int32)
    st = B.new_status("cuda")
    o, l = B.merge_lse_gather(outs.cuda(), lses.cuda(), idx.cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o, l = o.cpu().double(), l.cpu().double()
    for r in range(idx.shape[0]):
        parts = [int(i) for i in idx[r] if int(i) >= 0]
        if not parts:
            assert torch.all(o[r] == 0) and torch.all(torch.isneginf(l[r]))
            continue
        ld = lses[parts].double()
        L = torch.logsumexp(ld, 0)
        ref = (torch.exp(ld - L)[..., None] * outs[parts].double()).sum(0)
        ref = torch.where(torch.isneginf(L)[..., None], torch.zeros_like(ref), ref)
        assert torch.max(torch.abs(o[r] - ref)).item() <= 1e-5, r
        fin = torch.isfinite(L)
        assert torch.equal(torch.isneginf(l[r]), ~fin)
        assert torch.max(torch.abs(l[r][fin] - L[fin])).item() <= 1e-5
    assert torch.equal(o[1].float(), outs[7])  # a single part is a copy
    # an index past the parts is skipped and flagged
    bad = idx.clone()
    bad[2, 0] = 99
    st = B.new_status("cuda")
    o2, _ = B.merge_lse_gather(outs.cuda(), lses.cuda(), bad.cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == B.DEV_STATUS["bad_index"]
    assert torch.max(torch.abs(o2.cpu()[2].double() - o[2])).item() <= 1e-6


def test_gather_rows(B):
    g = torch.Generator().manual_seed(7)
    src = torch.randn(10, 8, 128, generator=g).bfloat16().cuda()
    index = torch.tensor([3, 0, 9, 3, 5], dtype=torch.int32, device="cuda")
    st = B.new_status("cuda")
    out = B.gather_rows(src, index, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.equal(out, src[index.long()])
    index[1] = 10  # outside the source: a zero row and the status bit
    out = B.gather_rows(src, index, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == B.DEV_STATUS["bad_index"]
    assert torch.all(out[1] == 0) and torch.equal(out[2:], src[index[2:].long()])


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
@pytest.mark.parametrize("world", [2, 3, 4])
def test_sharded_batch_equals_unsharded(B, world, kv):
    """Eight decode steps with lengths growing by 37 tokens per step (page boundaries crossed),
    each rank's parts run through the library and merged, every step against the oracle. The
    ranks are emulated one after the other on this GPU; each keeps its placement across steps
    and rebuilds its block-table view on the device."""
    steps_n, grow = 8, 37
    spec = W.custom_spec((9000, 64, 5, 130, 2047, 700), 32, 4, 128, 64, 128, kv_dtype=kv, seed=40 + world,
                         steps=steps_n * grow)
    case = W.make_case(spec)
    dc = to_device(case)
    compute = S.library_compute(32, 4, kv_dtype=kv, k_scale=dc["k_scale"], v_scale=dc["v_scale"], num_ctas=37)
    steps = [S.ShardedStep(spec.seq_lens, world, r, spec.page_size, 32, 128, compute=compute) for r in range(world)]
    assert sum(len(p) for p in steps[0].plan) > len(spec.seq_lens)  # the 9000-token request is split
    for i in range(steps_n):
        lens = [L + grow * i for L in spec.seq_lens]
        for st in steps:
            st.update(lens)
        local = [st.local(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], spec.tile_len) for st in steps]
        outs = torch.stack([o for o, _ in local])  # what the all-gather delivers to every rank
        lses = torch.stack([l for _, l in local])
        out = steps[0].assemble(outs, lses)
        torch.cuda.synchronize()
        ref = oracle_out(case, seq_lens=torch.tensor(lens, dtype=torch.int32))
        if kv == "bf16":
            assert_bf16_tol(out, ref, what=f"sharded over {world}, step {i}")
        else:
            assert errors(out, ref)[0] <= 5e-2
    assert all(st.replacements == steps[0].replacements for st in steps)  # the ranks agree


def test_gather_pages(B):
    bt = torch.arange(40, dtype=torch.int32).reshape(4, 10).cuda()
    req = torch.tensor([2, 0, 3], dtype=torch.int32, device="cuda")
    col0 = torch.tensor([3, 0, 9], dtype=torch.int32, device="cuda")
    st = B.new_status("cuda")
    out = B.gather_pages(bt, req, col0, status=st)
    torch.cuda.synchronize()
    want = torch.full((3, 10), -1, dtype=torch.int32)
    want[0, :7] = bt.cpu()[2, 3:]
    want[1] = bt.cpu()[0]
    want[2, :1] = bt.cpu()[3, 9:]
    assert int(st.item()) == 0 and torch.equal(out.cpu(), want)
    req[1] = 4  # outside the table: a row of -1 and the status bit
    out = B.gather_pages(bt, req, col0, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == B.DEV_STATUS["bad_index"] and torch.all(out[1] == -1)
    assert torch.equal(out.cpu()[0], want[0])
