"""Request-sharded placement of one decode batch over several GPUs (host side).

Requests and kv heads are independent, so a decode batch shards by request with no
collective in the attention itself. A request longer than one GPU's share is cut into
page-aligned token ranges placed on different GPUs. Its parts are then combined by the
log-sum-exp merge (``hpc_merge_lse_gather``): one exchange of num_heads * (head_dim + 1) floats
per part. The pages describe the split of a request's tiles across the processing units of
one GPU ("腾讯混元三算子杀入 SGLang" (AREX), Dynamic Attention paragraph). This module
applies the same idea one level up.

* ``plan_shards``: token-balanced placement. Parts are placed longest first onto the
  least-loaded rank (LPT greedy), after cutting every request longer than the share into
  nearly equal page-aligned ranges.
* ``rank_view``: the batch one rank runs. Each part becomes a request of its own, with its
  block-table row starting at the part's first page and its length set to the part's
  token count.
* ``ShardedStep``: gathers the q rows of a rank's parts (``hpc_gather_rows``), runs the parts
  through ``hpc_decode_step_lse``, exchanges (out, lse) with
  ``torch.distributed.all_gather_into_tensor`` and forms every request's output from its parts
  with ``hpc_merge_lse_gather``. Every rank ends with the whole batch's output.
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

    ``compute(q, k_pages, v_pages, block_table, seq_lens, tile_len, out=, lse=) -> (out, lse)``
    runs a rank's parts; on a GPU it is ``library_compute(...)`` (``hpc_decode_step_lse``), which
    writes straight into the all-gather's send buffers. ``gather(src, index)`` collects the
    parts' q rows and defaults to ``hpc_gather_rows``. ``merge(outs, lses, part_index)``
    combines every request's parts from the gathered rows and defaults to
    ``hpc_merge_lse_gather``. Tests without a GPU pass their own callbacks; the placement,
    exchange and indexing are the same code."""

    def __init__(self, seq_lens, world: int, rank: int, page_size: int, num_heads: int, head_dim: int,
                 compute, merge=None, gather=None):
        self.plan = plan_shards(seq_lens, world, page_size)
        self.world, self.rank, self.page_size = world, rank, page_size
        self.batch = len(seq_lens)
        self.num_heads, self.head_dim = num_heads, head_dim
        self.compute = compute
        self.merge = merge if merge is not None else library_merge()
        self.gather = gather if gather is not None else library_gather()
        self.max_parts = max(1, max(len(p) for p in self.plan))
        # where each request's parts land in the gathered buffer: (rank, slot)
        self.where: dict[int, list[tuple[int, int]]] = {}
        for rk, parts in enumerate(self.plan):
            for slot, p in enumerate(parts):
                self.where.setdefault(p.req, []).append((rk, slot))
        self.split = sorted(r for r, pl in self.where.items() if len(pl) > 1)
        # part_index[r][k]: row rank * max_parts + slot of the gathered buffer, -1 when unused
        k = max([len(pl) for pl in self.where.values()] + [1])
        idx = np.full((self.batch, k), -1, dtype=np.int32)
        for r, pl in self.where.items():
            for i, (rk, slot) in enumerate(pl):
                idx[r, i] = rk * self.max_parts + slot
        self.part_index_host = idx
        self._dev = {}  # device -> (part_index, request index of this rank's parts)
        self._view = None  # (block table pointer, device) -> this rank's view

    def _device_tables(self, dev):
        if dev not in self._dev:
            reqs = [p.req for p in self.plan[self.rank]]
            self._dev[dev] = (torch.from_numpy(self.part_index_host).to(dev),
                              torch.tensor(reqs, dtype=torch.int32, device=dev))
        return self._dev[dev]

    def local(self, q, k_pages, v_pages, block_table, tile_len, **kw):
        """This rank's parts: (out [max_parts, Hq, D], lse [max_parts, Hq]). Rows past the
        rank's part count are left unwritten: no request's index points at them."""
        parts = self.plan[self.rank]
        dev = q.device
        out = torch.empty((self.max_parts, self.num_heads, self.head_dim), dtype=torch.float32, device=dev)
        lse = torch.empty((self.max_parts, self.num_heads), dtype=torch.float32, device=dev)
        if parts:
            n = len(parts)
            key = (block_table.data_ptr(), dev)
            if self._view is None or self._view[0] != key:  # built once per block table
                bt, lens, _ = rank_view(parts, block_table, self.page_size)
                self._view = (key, bt, lens)
            _, bt, lens = self._view
            _, reqs = self._device_tables(dev)
            o, l = self.compute(self.gather(q, reqs), k_pages, v_pages, bt, lens, tile_len, out=out[:n],
                                lse=lse[:n], **kw)
            if o.data_ptr() != out.data_ptr():  # a callback that returns its own tensors
                out[:n] = o
                lse[:n] = l
        return out, lse

    def assemble(self, outs, lses):
        """Whole-batch output from every rank's parts, outs [world, max_parts, Hq, D] (or the
        same rows flattened): one indexed log-sum-exp merge, which copies the requests that
        have a single part."""
        outs = outs.reshape(-1, self.num_heads, self.head_dim)
        lses = lses.reshape(-1, self.num_heads)
        part_index, _ = self._device_tables(outs.device)
        out, _ = self.merge(outs, lses, part_index)
        return out

    def step(self, q, k_pages, v_pages, block_table, tile_len, group=None, **kw):
        """Local parts, one all-gather of (out, lse), merge. ``group``: a torch.distributed
        process group (None with world 1)."""
        out, lse = self.local(q, k_pages, v_pages, block_table, tile_len, **kw)
        if self.world == 1:
            return self.assemble(out, lse)
        import torch.distributed as dist
        # concatenated along the first dimension (the form every backend accepts)
        outs = torch.empty((self.world * out.shape[0],) + tuple(out.shape[1:]), dtype=out.dtype, device=out.device)
        lses = torch.empty((self.world * lse.shape[0],) + tuple(lse.shape[1:]), dtype=lse.dtype, device=lse.device)
        dist.all_gather_into_tensor(outs, out, group=group)
        dist.all_gather_into_tensor(lses, lse, group=group)
        return self.assemble(outs, lses)


def library_compute(num_heads, kv_heads, kv_dtype="bf16", k_scale=None, v_scale=None, num_ctas=None, status=None):
    """The library's single-launch step with log-sum-exp output, as a ``compute`` callback.
    Its workspace is kept between calls (the merge tickets stay zero); ``status`` collects the
    device status bits."""
    from . import binding as B
    ws = {}

    def compute(q, k_pages, v_pages, bt, lens, tile_len, out=None, lse=None, **kw):
        key = (q.shape[0], q.device)
        out, lse, _, w = B.decode_step_lse(q, k_pages, v_pages, bt, lens, num_heads, kv_heads, tile_len,
                                           kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale, num_ctas=num_ctas,
                                           out=out, lse=lse, status=status, workspace=ws.get(key))
        ws[key] = w
        return out, lse
    return compute


def library_merge(status=None):
    """``hpc_merge_lse_gather`` as the ``merge`` callback."""
    from . import binding as B
    return lambda outs, lses, part_index: B.merge_lse_gather(outs, lses, part_index, status=status)


def library_gather(status=None):
    """``hpc_gather_rows`` as the ``gather`` callback."""
    from . import binding as B
    return lambda src, index: B.gather_rows(src, index, status=status)


def tokens_per_rank(plan) -> np.ndarray:
    return np.array([sum(p.tok1 - p.tok0 for p in parts) for parts in plan], dtype=np.int64)
