"""Request-sharded placement of one decode batch (host side, CPU only).

* The planner covers every token of every request exactly once, with page-aligned parts,
  and balances tokens across ranks (LPT bound: no rank above the share plus one part).
* The oracle's log-sum-exp is pinned to torch.logsumexp in float64.
* Two ranks over gloo run the sharded step end to end over eight decode steps with growing
  lengths (update, local parts, one all-gather of (out, lse), merge of split requests), with
  the fp64 oracle standing in for the GPU kernel and the merge and block-table view written
  from their definitions; every step equals unsharded attention.
* ``ShardedStep.update`` keeps part starts while lengths grow and places the batch again when a
  request ends or starts or a rank's load drifts past its bound.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from load_balanced_split_step_b200 import shard as S
from load_balanced_split_step_b200 import workloads as W
from oracle import attention as OA

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("name", ["extreme", "heavy", "fp8", "uniform"])
def test_plan_covers_and_balances(world, name):
    spec = W.config_spec(name)
    P = spec.page_size
    plan = S.plan_shards(spec.seq_lens, world, P)
    seen = {}
    for parts in plan:
        for p in parts:
            assert p.tok0 % P == 0 and p.tok1 > p.tok0
            seen.setdefault(p.req, []).append((p.tok0, p.tok1))
    for r, L in enumerate(spec.seq_lens):
        rng = sorted(seen[r])
        assert rng[0][0] == 0 and rng[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(rng, rng[1:]))  # contiguous, disjoint
    load = S.tokens_per_rank(plan)
    share = -(-sum(spec.seq_lens) // world)
    biggest = max(p.tok1 - p.tok0 for parts in plan for p in parts)
    assert load.sum() == sum(spec.seq_lens)
    assert load.max() <= share + biggest  # LPT bound


def test_plan_splits_the_long_request():
    lens = [131072] + [4096] * 31
    plan = S.plan_shards(lens, 4, 64)
    owners = [k for k, parts in enumerate(plan) for p in parts if p.req == 0]
    assert len(set(owners)) >= 2
    load = S.tokens_per_rank(plan)
    assert load.max() - load.min() <= 4096  # within one short request


def test_oracle_lse_matches_torch_logsumexp():
    case = W.make_case(W.custom_spec((1, 17, 300), 16, 2, 64, 16, 32, seed=3))
    got = OA.decode_lse(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    P = case.spec.page_size
    for r, L in enumerate(case.spec.seq_lens):
        for h in range(16):
            g = h // 8
            K = torch.stack([case.k_pages[int(case.block_table[r, j // P]), g, j % P] for j in range(L)]).double()
            s = (K @ case.q[r, h].double()) / math.sqrt(64)
            assert abs(got[r, h] - torch.logsumexp(s, 0).item()) <= 1e-12


def _oracle_compute(case):
    def compute(q, k_pages, v_pages, bt, lens, tile_len, **kw):
        out = OA.decode_attention(q, k_pages, v_pages, bt, lens)
        lse = OA.decode_lse(q, k_pages, v_pages, bt, lens)
        return torch.from_numpy(out).float(), torch.from_numpy(lse).float()
    return compute


def _merge_by_definition(outs, lses, part_index):
    """For each request, its parts' rows: LSE = log sum_i exp(lse_i); out = sum_i exp(lse_i - LSE)
    out_i (float64). A request with no part gets zeros."""
    B, Hq, D = part_index.shape[0], outs.shape[1], outs.shape[2]
    out = torch.zeros((B, Hq, D), dtype=torch.float64)
    lse = torch.full((B, Hq), -math.inf, dtype=torch.float64)
    for r in range(B):
        rows = [int(i) for i in part_index[r] if int(i) >= 0]
        if not rows:
            continue
        l = lses[rows].double()
        L = torch.logsumexp(l, 0)
        out[r] = (torch.exp(l - L)[..., None] * outs[rows].double()).sum(0)
        lse[r] = L
    return out.float(), lse.float()


def _gather_rows(src, index):
    return src.index_select(0, index.long())


def _pages_view(block_table, req, col0):
    """The block-table view of a rank's parts, written out: row i is request req[i]'s table from
    column col0[i] on, -1 past its end."""
    n, width = req.numel(), block_table.shape[1]
    out = torch.full((n, width), -1, dtype=torch.int32)
    for i in range(n):
        row = block_table[int(req[i]), int(col0[i]):]
        out[i, :row.numel()] = row
    return out


STEPS = 8
LENS = (700, 64, 5, 2000, 33)


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = W.custom_spec(LENS, 16, 2, 64, 16, 32, seed=11, steps=STEPS)
        case = W.make_case(spec)
        st = S.ShardedStep(spec.seq_lens, world, rank, spec.page_size, 16, 64, compute=_oracle_compute(case),
                           merge=_merge_by_definition, gather=_gather_rows, pages=_pages_view)
        outs = []
        for i in range(STEPS):  # lengths grow by one token per decode step
            lens = [L + i for L in spec.seq_lens]
            out = st.step(case.q, case.k_pages, case.v_pages, case.block_table, spec.tile_len, seq_lens=lens)
            outs.append(out.numpy())
        q.put((rank, outs, [len(p) for p in st.plan]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_over_gloo_equal_unsharded():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spec = W.custom_spec(LENS, 16, 2, 64, 16, 32, seed=11, steps=STEPS)
    case = W.make_case(spec)
    for i in range(STEPS):
        lens = torch.tensor([L + i for L in spec.seq_lens], dtype=torch.int32)
        ref = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, lens)
        for rank, outs, nparts in res:
            assert sum(nparts) > len(spec.seq_lens)  # the 2000-token request was split
            assert np.max(np.abs(outs[i] - ref)) <= 1e-5, (rank, i)


def _covers(st, lens):
    seen = {}
    for parts in st.plan:
        for p in parts:
            assert p.tok0 % st.page_size == 0 and p.tok1 > p.tok0
            seen.setdefault(p.req, []).append((p.tok0, p.tok1))
    for r, L in enumerate(lens):
        if L == 0:
            assert r not in seen
            continue
        rng = sorted(seen[r])
        assert rng[0][0] == 0 and rng[-1][1] == L and all(a[1] == b[0] for a, b in zip(rng, rng[1:]))


def test_update_grows_tail_parts_and_replaces_on_drift():
    """Growing lengths keep every part's start and extend each request's tail part; the batch is
    placed again when a request ends or starts, or when a rank's load drifts past the bound.
    After every update each token is in exactly one page-aligned part."""
    lens = [131072] + [4096] * 31
    st = S.ShardedStep(lens, 4, 0, 64, 8, 64, compute=None, merge=lambda *a: None, gather=lambda *a: None,
                       pages=lambda *a: None)
    starts = {(p.req, p.tok0) for parts in st.plan for p in parts}
    for i in range(1, 9):  # eight decode steps, one token each: same parts, tails grown
        cur = [L + i for L in lens]
        assert st.update(cur) is False
        _covers(st, cur)
        assert {(p.req, p.tok0) for parts in st.plan for p in parts} == starts
    assert st.replacements == 0
    cur = [L + 8 for L in lens]
    cur[5] = 0  # a request ends
    assert st.update(cur) is True and st.replacements == 1
    _covers(st, cur)
    cur[5] = 300  # a new request starts
    assert st.update(cur) is True
    _covers(st, cur)
    # one short request growing far past the share: the rank that holds its tail drifts
    grown = list(cur)
    grown[7] += 60000
    assert st.update(grown) is True
    _covers(st, grown)
    load = S.tokens_per_rank(st.plan)
    assert load.max() <= (1 + st.drift) * -(-sum(grown) // 4) + 64 + max(p.tok1 - p.tok0 for ps in st.plan for p in ps)
