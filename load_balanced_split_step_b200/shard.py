"""Request-sharded placement of one decode batch over several GPUs (host side).

Requests and kv heads are independent, so a decode batch shards by request with no
collective in the attention itself. A request longer than one GPU's share is cut into
page-aligned token ranges placed on different GPUs. Its parts are then combined by the
log-sum-exp merge (``hpc_merge_lse``): one exchange of num_heads * (head_dim + 1) floats
per part. The pages describe the split of a request's tiles across the processing units of
one GPU ("腾讯混元三算子杀入 SGLang" (AREX), Dynamic Attention paragraph). This module
applies the same idea one level up.

* ``plan_shards``: token-balanced placement. Parts are placed longest first onto the
  least-loaded rank (LPT greedy), after cutting every request longer than the share into
  nearly equal page-aligned ranges.
* ``rank_view``: the batch one rank runs. Each part becomes a request of its own, with its
  block-table row starting at the part's first page and its length set to the part's
  token count.
* ``ShardedStep``: runs a rank's parts through ``hpc_decode_step_lse``, exchanges (out, lse)
  with ``torch.distributed.all_gather_into_tensor`` and merges split requests with
  ``hpc_merge_lse``. Every rank ends with the whole batch's output.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Part:
    req: int
    tok0: int  # first token (a multiple of page_size)
    tok1: int  # one past the last token


def plan_shards(seq_lens, world: int, page_size: int) -> list[list[Part]]:
    """Parts per rank. Every token of every request is in exactly one part. A part starts on
    a page boundary. Requests with no tokens get no part."""
    lens = [int(x) for x in seq_lens]
    if world < 1 or page_size < 1:
        raise ValueError("world and page_size must be positive")
    total = sum(lens)
    share = max(page_size, -(-total // world))
    parts = []
    for r, L in enumerate(lens):
        if L <= 0:
            continue
        pieces = max(1, min(world, -(-L // share)))
        pages = -(-L // page_size)
        bounds = [min(L, (pages * k // pieces) * page_size) for k in range(pieces + 1)]
        bounds[-1] = L
        for k in range(pieces):
            if bounds[k + 1] > bounds[k]:
                parts.append(Part(r, bounds[k], bounds[k + 1]))
    # LPT: longest part first onto the least-loaded rank (ties: lower rank, earlier request)
    parts.sort(key=lambda p: (-(p.tok1 - p.tok0), p.req, p.tok0))
    load = [0] * world
    out: list[list[Part]] = [[] for _ in range(world)]
    for p in parts:
        r = min(range(world), key=lambda i: (load[i], i))
        out[r].append(p)
        load[r] += p.tok1 - p.tok0
    for lst in out:
        lst.sort(key=lambda p: (p.req, p.tok0))
    return out


def rank_view(parts: list[Part], block_table: torch.Tensor, page_size: int):
    """(block_table, seq_lens, requests) of the batch that runs one rank's parts."""
    n = len(parts)
    width = max([-(-(p.tok1 - p.tok0) // page_size) for p in parts] + [1])
    bt = torch.full((max(n, 1), width), -1, dtype=torch.int32, device=block_table.device)
    lens = torch.zeros(max(n, 1), dtype=torch.int32, device=block_table.device)
    for i, p in enumerate(parts):
        a, b = p.tok0 // page_size, -(-p.tok1 // page_size)
        bt[i, :b - a] = block_table[p.req, a:b]
        lens[i] = p.tok1 - p.tok0
    return bt, lens, [p.req for p in parts]


class ShardedStep:
    """One decode step of a batch sharded over ``world`` ranks.

    ``compute(q, k_pages, v_pages, block_table, seq_lens, tile_len) -> (out, lse)`` runs a
    rank's parts; on a GPU it is ``library_compute(...)`` (``hpc_decode_step_lse``). ``merge``
    combines the parts of a split request and defaults to ``hpc_merge_lse``. Tests without a
    GPU pass their own callbacks; the placement, exchange and assembly are the same code."""

    def __init__(self, seq_lens, world: int, rank: int, page_size: int, num_heads: int, head_dim: int,
                 compute, merge=None):
        self.plan = plan_shards(seq_lens, world, page_size)
        self.world, self.rank, self.page_size = world, rank, page_size
        self.batch = len(seq_lens)
        self.num_heads, self.head_dim = num_heads, head_dim
        self.compute = compute
        self.merge = merge if merge is not None else library_merge()
        self.max_parts = max(1, max(len(p) for p in self.plan))
        # where each request's parts land in the gathered buffer: (rank, slot)
        self.where: dict[int, list[tuple[int, int]]] = {}
        for rk, parts in enumerate(self.plan):
            for slot, p in enumerate(parts):
                self.where.setdefault(p.req, []).append((rk, slot))
        self.single = sorted(r for r, pl in self.where.items() if len(pl) == 1)
        self.split = sorted(r for r, pl in self.where.items() if len(pl) > 1)
        self.split_parts = max([len(self.where[r]) for r in self.split] + [1])
        self._view = None  # (block table pointer, device) -> this rank's view
        self._index = None

    def local(self, q, k_pages, v_pages, block_table, tile_len, **kw):
        """This rank's parts: (out [max_parts, Hq, D], lse [max_parts, Hq]), zero-padded."""
        parts = self.plan[self.rank]
        dev = q.device
        out = torch.zeros((self.max_parts, self.num_heads, self.head_dim), dtype=torch.float32, device=dev)
        lse = torch.full((self.max_parts, self.num_heads), -math.inf, dtype=torch.float32, device=dev)
        if parts:
            key = (block_table.data_ptr(), dev)
            if self._view is None or self._view[0] != key:  # built once per block table
                bt, lens, reqs = rank_view(parts, block_table, self.page_size)
                self._view = (key, bt, lens, torch.tensor(reqs, dtype=torch.long, device=dev))
            _, bt, lens, reqs = self._view
            o, l = self.compute(q.index_select(0, reqs).contiguous(), k_pages, v_pages, bt, lens, tile_len, **kw)
            out[:len(parts)] = o
            lse[:len(parts)] = l
        return out, lse

    def _indices(self, dev):
        if self._index is None or self._index[0] != dev:
            t = lambda v: torch.tensor(v, dtype=torch.long, device=dev)
            single = (t(self.single), t([self.where[r][0][0] for r in self.single]),
                      t([self.where[r][0][1] for r in self.single]))
            # split requests: [parts, n_split] grids of (rank, slot); missing parts are masked
            rk = [[self.where[r][i][0] if i < len(self.where[r]) else 0 for r in self.split]
                  for i in range(self.split_parts)]
            sl = [[self.where[r][i][1] if i < len(self.where[r]) else 0 for r in self.split]
                  for i in range(self.split_parts)]
            pad = [[i >= len(self.where[r]) for r in self.split] for i in range(self.split_parts)]
            split = (t(self.split), t(rk), t(sl), torch.tensor(pad, dtype=torch.bool, device=dev))
            self._index = (dev, single, split)
        return self._index[1], self._index[2]

    def assemble(self, outs, lses):
        """Whole-batch output from every rank's parts (outs [world, max_parts, Hq, D]): one
        gather for the requests in one part, one merge for all split requests."""
        dev = outs.device
        result = torch.zeros((self.batch, self.num_heads, self.head_dim), dtype=torch.float32, device=dev)
        (sreq, srank, sslot), (preq, prank, pslot, pad) = self._indices(dev)
        if len(self.single):
            result[sreq] = outs[srank, sslot]
        if len(self.split):
            o = outs[prank, pslot]                                        # [parts, n_split, Hq, D]
            l = lses[prank, pslot].masked_fill(pad[..., None], -math.inf)  # [parts, n_split, Hq]
            n = len(self.split)
            merged, _ = self.merge(o.reshape(self.split_parts, n * self.num_heads, self.head_dim).contiguous(),
                                   l.reshape(self.split_parts, n * self.num_heads).contiguous())
            result[preq] = merged.reshape(n, self.num_heads, self.head_dim)
        return result

    def step(self, q, k_pages, v_pages, block_table, tile_len, group=None, **kw):
        """Local parts, one all-gather of (out, lse), merge. ``group``: a torch.distributed
        process group (None with world 1)."""
        out, lse = self.local(q, k_pages, v_pages, block_table, tile_len, **kw)
        if self.world == 1:
            return self.assemble(out.unsqueeze(0), lse.unsqueeze(0))
        import torch.distributed as dist
        # concatenated along the first dimension (the form every backend accepts)
        outs = torch.empty((self.world * out.shape[0],) + tuple(out.shape[1:]), dtype=out.dtype, device=out.device)
        lses = torch.empty((self.world * lse.shape[0],) + tuple(lse.shape[1:]), dtype=lse.dtype, device=lse.device)
        dist.all_gather_into_tensor(outs, out.contiguous(), group=group)
        dist.all_gather_into_tensor(lses, lse.contiguous(), group=group)
        return self.assemble(outs.view((self.world,) + tuple(out.shape)), lses.view((self.world,) + tuple(lse.shape)))


def library_compute(num_heads, kv_heads, kv_dtype="bf16", k_scale=None, v_scale=None, num_ctas=None, status=None):
    """The library's single-launch step with log-sum-exp output, as a ``compute`` callback.
    Its workspace is kept between calls (the merge tickets stay zero); ``status`` collects the
    device status bits."""
    from . import binding as B
    ws = {}

    def compute(q, k_pages, v_pages, bt, lens, tile_len, **kw):
        key = (q.shape[0], q.device)
        out, lse, _, w = B.decode_step_lse(q, k_pages, v_pages, bt, lens, num_heads, kv_heads, tile_len,
                                           kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale, num_ctas=num_ctas,
                                           status=status, workspace=ws.get(key))
        ws[key] = w
        return out, lse
    return compute


def library_merge():
    from . import binding as B
    return lambda outs, lses: B.merge_lse(outs, lses)


def tokens_per_rank(plan) -> np.ndarray:
    return np.array([sum(p.tok1 - p.tok0 for p in parts) for parts in plan], dtype=np.int64)
