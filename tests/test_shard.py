"""Request-sharded placement of one decode batch (host side, CPU only).

* The planner covers every token of every request exactly once, with page-aligned parts,
  and balances tokens across ranks (LPT bound: no rank above the share plus one part).
* The oracle's log-sum-exp is pinned to torch.logsumexp in float64.
* Two ranks over gloo run the sharded step end to end (plan, local parts, one all-gather of
  (out, lse), merge of split requests), with the fp64 oracle standing in for the GPU kernel
  and the merge written from its definition; the result equals unsharded attention.
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


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = W.custom_spec((700, 64, 5, 2000, 33), 16, 2, 64, 16, 32, seed=11)
        case = W.make_case(spec)
        st = S.ShardedStep(spec.seq_lens, world, rank, spec.page_size, 16, 64, compute=_oracle_compute(case),
                           merge=_merge_by_definition, gather=_gather_rows)
        out = st.step(case.q, case.k_pages, case.v_pages, case.block_table, spec.tile_len)
        q.put((rank, out.numpy(), [len(p) for p in st.plan]))
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
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spec = W.custom_spec((700, 64, 5, 2000, 33), 16, 2, 64, 16, 32, seed=11)
    case = W.make_case(spec)
    ref = OA.decode_attention(case.q, case.k_pages, case.v_pages, case.block_table, case.seq_lens)
    for rank, out, nparts in res:
        assert sum(nparts) > len(spec.seq_lens)  # the 2000-token request was split
        assert np.max(np.abs(out - ref)) <= 1e-5
