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
  token count (host form; on the device ``hpc_gather_pages`` builds the same rows).
* ``ShardedStep``: follows the lengths every step (``update``), builds the rank's block-table
  view on the device (``hpc_gather_pages``), gathers the q rows of its parts
  (``hpc_gather_rows``), runs the parts
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
    """One decode step of a batch sharded over ``world`` ranks, re-placed as lengths change.

    ``update(seq_lens)`` follows the batch from step to step, as the pages say the mapping is
    rebuilt while request lengths change during decode ("Tencent HPC llega a SGLang …",
    remio.ai, section "Por qué Tencent HPC importa …"). Every part keeps its page-aligned start
    and a request's last part grows to the new length. The placement is made again from
    scratch (``plan_shards``) when the batch changes (a request appears, ends or shrinks below
    a part boundary) or when the busiest rank's tokens drift more than ``drift`` above the
    ideal share. Every rank takes the same decision from the same lengths.

    Per step, the device tables of this rank (part lengths, and after a re-placement the parts'
    requests, first page columns and every request's part index) go up in one small
    host-to-device copy, and the rank's block-table view is rebuilt on the device
    (``pages``, default ``hpc_gather_pages``), so pages the caller appends are seen.

    ``compute(q, k_pages, v_pages, block_table, seq_lens, tile_len, out=, lse=) -> (out, lse)``
    runs a rank's parts; on a GPU it is ``library_compute(...)`` (``hpc_decode_step_lse``), which
    writes straight into the all-gather's send buffers. ``gather(src, index)`` collects the
    parts' q rows and defaults to ``hpc_gather_rows``. ``merge(outs, lses, part_index)``
    combines every request's parts from the gathered rows and defaults to
    ``hpc_merge_lse_gather``. Tests without a GPU pass their own callbacks; the placement,
    exchange and indexing are the same code."""

    def __init__(self, seq_lens, world: int, rank: int, page_size: int, num_heads: int, head_dim: int,
                 compute, merge=None, gather=None, pages=None, drift: float = 0.05):
        self.world, self.rank, self.page_size = world, rank, page_size
        self.num_heads, self.head_dim = num_heads, head_dim
        self.compute = compute
        self.merge = merge if merge is not None else library_merge()
        self.gather = gather if gather is not None else library_gather()
        self.pages = pages if pages is not None else library_pages()
        self.drift = drift
        self.replacements = 0
        self._place([int(x) for x in seq_lens])

    # ---- placement (host)
    def _place(self, lens):
        self.lens = list(lens)
        self.batch = len(lens)
        self.plan = plan_shards(lens, self.world, self.page_size)
        self.max_parts = max(1, max(len(p) for p in self.plan))
        # where each request's parts land in the gathered buffer: (rank, slot)
        self.where: dict[int, list[tuple[int, int]]] = {}
        for rk, parts in enumerate(self.plan):
            for slot, p in enumerate(parts):
                self.where.setdefault(p.req, []).append((rk, slot))
        for pl in self.where.values():  # in token order: the last entry is the request's tail part
            pl.sort(key=lambda w: self.plan[w[0]][w[1]].tok0)
        self.split = sorted(r for r, pl in self.where.items() if len(pl) > 1)
        # part_index[r][k]: row rank * max_parts + slot of the gathered buffer, -1 when unused
        k = max([len(pl) for pl in self.where.values()] + [1])
        idx = np.full((self.batch, k), -1, dtype=np.int32)
        for r, pl in self.where.items():
            for i, (rk, slot) in enumerate(pl):
                idx[r, i] = rk * self.max_parts + slot
        self.part_index_host = idx
        self._dev = {}  # device -> device tables of this placement
        self._stale = True

    def update(self, seq_lens) -> bool:
        """Follow this step's lengths. Returns True when the batch was placed again."""
        lens = [int(x) for x in seq_lens]
        replace = len(lens) != self.batch
        if not replace:
            for r, L in enumerate(lens):
                pl = self.where.get(r)
                if (L > 0) != (pl is not None):
                    replace = True  # a request started or ended
                    break
                if pl is not None:
                    last = self.plan[pl[-1][0]][pl[-1][1]]
                    if L <= last.tok0:
                        replace = True  # shrank below its last part's start
                        break
        if not replace:
            load = np.zeros(self.world, dtype=np.int64)
            for rk, parts in enumerate(self.plan):
                load[rk] = sum(p.tok1 - p.tok0 for p in parts)
            for r, pl in self.where.items():  # the tail parts grow to the new lengths
                rk, slot = pl[-1]
                load[rk] += lens[r] - self.plan[rk][slot].tok1
            share = -(-sum(lens) // self.world)
            replace = load.max() > (1.0 + self.drift) * share + self.page_size
        if replace:
            self._place(lens)
            self.replacements += 1
            return True
        # grow every request's last part to its new length
        for r, pl in self.where.items():
            rk, slot = pl[-1]
            p = self.plan[rk][slot]
            if p.tok1 != lens[r]:
                self.plan[rk][slot] = Part(p.req, p.tok0, lens[r])
        self.lens = lens
        self._stale = True
        return False

    # ---- device tables of this rank
    def _tables(self, dev):
        """(part_index [B, k], reqs [n], col0 [n], lens [n]) on dev, refreshed with one copy when
        the lengths or the placement changed since the last step."""
        parts = self.plan[self.rank]
        n = len(parts)
        B, k = self.part_index_host.shape
        t = self._dev.get(dev)
        if t is None:
            size = 3 * n + B * k
            pinned = dev.type == "cuda"
            host = [torch.empty(size, dtype=torch.int32, pin_memory=pinned) for _ in range(2 if pinned else 1)]
            t = {"dev": torch.empty(size, dtype=torch.int32, device=dev), "host": host, "turn": 0,
                 "events": [None] * len(host), "n": n, "shape": (B, k)}
            self._dev[dev] = t
            self._stale = True
        if self._stale:
            i = t["turn"]
            if t["events"][i] is not None:
                t["events"][i].synchronize()  # the copy that last read this host buffer is done
            h = t["host"][i].numpy()
            h[:n] = [p.tok1 - p.tok0 for p in parts]
            h[n:2 * n] = [p.req for p in parts]
            h[2 * n:3 * n] = [p.tok0 // self.page_size for p in parts]
            h[3 * n:] = self.part_index_host.reshape(-1)
            t["dev"].copy_(t["host"][i], non_blocking=True)
            if dev.type == "cuda":
                ev = torch.cuda.Event()
                ev.record()
                t["events"][i] = ev
            t["turn"] = (i + 1) % len(t["host"])
            self._stale = False
        d = t["dev"]
        return d[3 * n:].view(B, k), d[n:2 * n], d[2 * n:3 * n], d[:n]

    def local(self, q, k_pages, v_pages, block_table, tile_len, **kw):
        """This rank's parts: (out [max_parts, Hq, D], lse [max_parts, Hq]). Rows past the
        rank's part count are left unwritten: no request's index points at them."""
        parts = self.plan[self.rank]
        dev = q.device
        out = torch.empty((self.max_parts, self.num_heads, self.head_dim), dtype=torch.float32, device=dev)
        lse = torch.empty((self.max_parts, self.num_heads), dtype=torch.float32, device=dev)
        _, reqs, col0, lens = self._tables(dev)
        if parts:
            n = len(parts)
            bt = self.pages(block_table, reqs, col0)
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
        part_index = self._tables(outs.device)[0]
        out, _ = self.merge(outs, lses, part_index)
        return out

    def step(self, q, k_pages, v_pages, block_table, tile_len, group=None, seq_lens=None, **kw):
        """This step's lengths (``update``), local parts, one all-gather of (out, lse), merge.
        ``group``: a torch.distributed process group (None with world 1). ``seq_lens``: host
        lengths of this step, or None to keep the last ones."""
        if seq_lens is not None:
            self.update(seq_lens)
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


def library_pages(status=None):
    """``hpc_gather_pages`` as the ``pages`` callback: the rank's block-table view, as wide as the
    caller's table."""
    from . import binding as B
    return lambda block_table, req, col0: B.gather_pages(block_table, req, col0, status=status)


def library_gather(status=None):
    """``hpc_gather_rows`` as the ``gather`` callback."""
    from . import binding as B
    return lambda src, index: B.gather_rows(src, index, status=status)


def tokens_per_rank(plan) -> np.ndarray:
    return np.array([sum(p.tok1 - p.tok0 for p in parts) for parts in plan], dtype=np.int64)
