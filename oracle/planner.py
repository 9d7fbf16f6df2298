"""Per-step tile planner, unit by unit (test infrastructure; see ``oracle/__init__``).

What the pages say:

* "Tencent HPC llega a SGLang …" (remio.ai, section "Por qué Tencent HPC importa para
  el serving de modelos en línea"): the KV-cache work is cut into smaller tiles and
  assigned by current load. The mapping is rebuilt as request lengths change during
  decode. A scheduler splits requests into uniform tiles and spreads them over CTAs.
* "腾讯混元三算子杀入 SGLang" (AREX, section "Router GEMM：精度不丢，速度翻三倍", the
  Dynamic Attention paragraph): a persistent kernel assigns tiles every decode step by
  the actual KV length.

The pages do not fix the partition. The reading, step by step:

1. Request r has nt_r = ceil(L_r / tile_len) tiles per kv head. A partial last tile
   costs one unit, like any other ("uniform tiles").
2. Units are enumerated request-major, then kv head, then tile.
3. With T units and G CTAs, chunk = ceil(T / G). CTA g takes units
   [g*chunk, min((g+1)*chunk, T)). Trailing CTAs may get nothing.
4. Each CTA's run of units is cut into work items at (request, kv head) boundaries.
   An item is (request, kv_head, tile_begin, tile_end). Item k writes partial slot k.
5. An item that covers all of its (request, kv head) is DIRECT: it writes the final
   output itself. Every other (request, kv head) is merged from its items, which are
   contiguous in the list.

The static split-k plan (the baseline the pages compare against, same source, section
"Por qué …": a static split idles units or launches empty chunks for short requests)
cuts each (request, kv head) into S equal contiguous tile ranges, one CTA each.

Outputs use the byte layout of the device plan: the item record is
(req int32, kv_head int16, flags int16, tile_begin int32, tile_end int32).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

ITEM_DTYPE = np.dtype([("req", "<i4"), ("kv_head", "<i2"), ("flags", "<i2"),
                       ("tile_begin", "<i4"), ("tile_end", "<i4")])
FLAG_DIRECT = 1


@dataclass
class Plan:
    items: np.ndarray  # ITEM_DTYPE [n_items]
    item_cta: np.ndarray  # int [n_items]: the CTA that owns each item
    cta_indptr: np.ndarray  # int32 [G + 1]
    merge_indptr: np.ndarray  # int32 [B*Hkv + 1]
    merge_list: np.ndarray  # int32: segments (r*Hkv + kvh) whose item count != 1
    n_units: int
    chunk: int
    num_ctas: int


def num_tiles(L: int, tile_len: int) -> int:
    return (L + tile_len - 1) // tile_len if L > 0 else 0


def _finish(items_rows, item_cta, B, Hkv, G, n_units, chunk) -> Plan:
    n = len(items_rows)
    items = np.zeros(n, dtype=ITEM_DTYPE)
    for k, (r, kvh, tb, te, direct) in enumerate(items_rows):
        items[k] = (r, kvh, FLAG_DIRECT if direct else 0, tb, te)
    item_cta = np.asarray(item_cta, dtype=np.int64)
    # items were appended in unit order, so owners and segments are non-decreasing and
    # "number of items with owner < g" is a sorted-array count
    assert np.all(np.diff(item_cta) >= 0)
    # cta_indptr[g] = index of the first item owned by a CTA >= g
    cta_indptr = np.searchsorted(item_cta, np.arange(G + 1), side="left").astype(np.int32)
    seg = items["req"].astype(np.int64) * Hkv + items["kv_head"].astype(np.int64)
    assert np.all(np.diff(seg) >= 0)
    merge_indptr = np.searchsorted(seg, np.arange(B * Hkv + 1), side="left").astype(np.int32)
    counts = np.diff(merge_indptr)
    merge_list = np.array([s for s in range(B * Hkv) if counts[s] != 1], dtype=np.int32)
    return Plan(items, item_cta, cta_indptr, merge_indptr, merge_list, n_units, chunk, G)


def plan_dynamic(seq_lens, kv_heads: int, tile_len: int, num_ctas: int) -> Plan:
    """The load-balanced plan, following steps 1-5 of the module docstring literally."""
    lens = [int(x) for x in seq_lens]
    B, G = len(lens), int(num_ctas)
    units = []  # (r, kvh, tile) in enumeration order
    for r, L in enumerate(lens):
        for kvh in range(kv_heads):
            for t in range(num_tiles(L, tile_len)):
                units.append((r, kvh, t))
    T = len(units)
    chunk = -(-T // G) if T > 0 else 0
    rows, owner = [], []  # rows: [r, kvh, tile_begin, tile_end, direct]
    for u, (r, kvh, t) in enumerate(units):
        cta = u // chunk
        if rows and owner[-1] == cta and rows[-1][0] == r and rows[-1][1] == kvh:
            rows[-1][3] = t + 1  # extend the current item by one tile
        else:
            rows.append([r, kvh, t, t + 1, False])
            owner.append(cta)
    for row in rows:
        r, kvh, tb, te, _ = row
        row[4] = (tb == 0 and te == num_tiles(lens[r], tile_len))
    return _finish(rows, owner, B, kv_heads, G, T, chunk)


def plan_static(seq_lens, kv_heads: int, tile_len: int, splits: int) -> Plan:
    """Static split-k: CTA (r*Hkv + kvh)*S + j takes tiles
    [j*ceil(nt/S), min((j+1)*ceil(nt/S), nt)) of (r, kvh). It may be empty."""
    lens = [int(x) for x in seq_lens]
    B, S = len(lens), int(splits)
    G = B * kv_heads * S
    rows, owner = [], []
    T = 0
    for r, L in enumerate(lens):
        nt = num_tiles(L, tile_len)
        T += nt * kv_heads
        per = -(-nt // S) if nt > 0 else 0
        for kvh in range(kv_heads):
            for j in range(S):
                tb, te = j * per, min((j + 1) * per, nt)
                if tb < te:
                    rows.append([r, kvh, tb, te, tb == 0 and te == nt])
                    owner.append((r * kv_heads + kvh) * S + j)
    return _finish(rows, owner, B, kv_heads, G, T, 0)


def static_splits(batch: int, kv_heads: int, num_sms: int) -> int:
    """S = max(1, ceil(2 * num_SMs / (B * Hkv))): enough CTAs for two waves."""
    return max(1, -(-2 * num_sms // (batch * kv_heads)))


# ---------------------------------------------------------------------------------------------
# The single-launch step's split: tiles plus a fixed cost per item start.
#
# Reading 21 of the path's spec. The pages balance CTAs by "current load" (remio.ai, section
# "Por qué Tencent HPC importa …") and leave the measure of load open; reading 7 takes tile
# counts. The single-launch step counts each item start as a fixed number of tile-equivalents
# as well. Step by step:
#
# 1. Units and segments as in plan_dynamic: units u = 0..T-1 enumerate request -> kv head ->
#    tile; a segment is one (request, kv head) with tiles, numbered S = 1, 2, ... in unit order.
# 2. Every tile costs W = 16 and every segment start adds c = item_cost. Unit u, a tile of
#    segment S, sits at cost position W*u + c*S.
# 3. total = W*T + c*(number of segments); chunk = W * ceil(total / (W*G)), in cost units.
# 4. Unit u belongs to CTA floor(position(u) / chunk). Positions grow with u, so every CTA owns
#    one contiguous run of units (possibly empty).
# 5. A CTA's run is cut into items at segment boundaries. An item covering its whole segment is
#    DIRECT. Any other item writes a partial state: slot 2g if it is CTA g's first item, else
#    slot 2g + 1 (a split segment can only be the first or the last item of its CTA's run).
# With c = 0 the owners are u // ceil(T/G), the units of plan_dynamic.
# ---------------------------------------------------------------------------------------------

COST_PER_TILE = 16
FLAG_SECOND_SLOT = 2  # item record flag: the partial slot is 2g + 1 (else 2g)


@dataclass
class CostSplit:
    unit_begin: np.ndarray  # int64 [G]: first unit of each CTA's run
    unit_end: np.ndarray  # int64 [G]: one past its last unit
    items: list  # per CTA: ITEM_DTYPE array of its items, in order (flags DIRECT / SECOND_SLOT)
    slots: list  # per CTA: partial slot of each item, -1 for a DIRECT item
    chunk: int  # cost units per CTA
    n_units: int
    item_cost: int


def plan_cost_split(seq_lens, kv_heads: int, tile_len: int, num_ctas: int, item_cost: int) -> CostSplit:
    """Steps 1-5 above, unit by unit. seq_lens are the lengths that get tiles (0 for none)."""
    lens = [int(x) for x in seq_lens]
    G, W, c = int(num_ctas), COST_PER_TILE, int(item_cost)
    units = []  # (r, kvh, tile, S)
    S = 0
    for r, L in enumerate(lens):
        nt = num_tiles(L, tile_len)
        for kvh in range(kv_heads):
            if nt == 0:
                continue
            S += 1
            for t in range(nt):
                units.append((r, kvh, t, S))
    T = len(units)
    total = W * T + c * S
    chunk = W * (-(-total // (W * G))) if T > 0 else 0
    owner = [(W * u + c * s) // chunk for u, (_, _, _, s) in enumerate(units)]
    begin = np.full(G, T, dtype=np.int64)
    end = np.full(G, T, dtype=np.int64)
    rows = [[] for _ in range(G)]  # [r, kvh, tb, te]
    for u, (r, kvh, t, _) in enumerate(units):
        g = owner[u]
        if not rows[g]:
            begin[g] = u
        end[g] = u + 1
        last = rows[g][-1] if rows[g] else None
        if last is not None and last[0] == r and last[1] == kvh:
            last[3] = t + 1
        else:
            rows[g].append([r, kvh, t, t + 1])
    # CTAs with no units sit where the next owner starts: [T, T) at the end, or an empty run
    # at the first unit after the previous CTA's run
    for g in range(G - 1, -1, -1):
        if not rows[g]:
            begin[g] = end[g] = begin[g + 1] if g + 1 < G else T
    items, slots = [], []
    for g in range(G):
        arr = np.zeros(len(rows[g]), dtype=ITEM_DTYPE)
        sl = []
        for k, (r, kvh, tb, te) in enumerate(rows[g]):
            direct = tb == 0 and te == num_tiles(lens[r], tile_len)
            flags = FLAG_DIRECT if direct else (FLAG_SECOND_SLOT if k > 0 else 0)
            arr[k] = (r, kvh, flags, tb, te)
            sl.append(-1 if direct else 2 * g + (1 if k > 0 else 0))
        items.append(arr)
        slots.append(sl)
    return CostSplit(begin, end, items, slots, chunk, T, c)
