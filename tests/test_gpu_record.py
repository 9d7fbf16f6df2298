"""The single-launch step's own split, byte for byte against the oracle's cost split.

hpc_decode_step derives each CTA's work in the kernel (the planner's closed form, with a fixed
cost per item start: reading 21 of the path's spec, oracle.planner.plan_cost_split). Asked
through options.record, every CTA writes its unit run, the split's chunk and item cost, its item
count and its items in the order it ran them, with the partial slot of every split item. This
test compares that buffer byte for byte with the record written out from the oracle, for all
five named workloads, every re-planned step of the heavy-tailed batch, several new tokens per
request, and item costs 0 (the pages' rule), the default and 1024.

The split depends on the lengths and shapes alone. So that full-size workloads need no
multi-gigabyte cache, every block-table entry points at page 0 of a one-page cache: the kernel
streams the same page for every tile, and all of its loads stay in the pool.
"""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import planner as OP

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def _expected_record(B, split, record_items):
    """The record buffer as the header documents it, written from the oracle's split; entries
    past a CTA's item count keep the sentinel the buffer was filled with."""
    G = len(split.items)
    stride = B.RECORD_DTYPE.itemsize + record_items * B.ITEM_DTYPE.itemsize
    buf = np.full(G * stride, SENTINEL, dtype=np.uint8)
    for g in range(G):
        h = np.zeros(1, dtype=B.RECORD_DTYPE)
        h[0] = (split.unit_begin[g], split.unit_end[g], split.chunk, split.item_cost, len(split.items[g]))
        base = g * stride
        buf[base:base + B.RECORD_DTYPE.itemsize] = h.view(np.uint8)
        items = split.items[g][:record_items]
        raw = items.astype(B.ITEM_DTYPE).view(np.uint8)
        buf[base + B.RECORD_DTYPE.itemsize:base + B.RECORD_DTYPE.itemsize + raw.size] = raw
    return buf


def _default_cost(tile_len, head_dim, kv_dtype, q_len, group):
    """The documented default: the time of one item start as KV bytes streamed meanwhile, 152 KB
    with one new token; with several, 224 KB on the tcgen05 kernel (the default for three or four
    tokens on a bf16 cache with head_dim 128 and q_len * group <= 32) and 320 KB on the mma.sync
    consumers; in 1/16 of a tile of this shape, rounded."""
    tile_bytes = tile_len * head_dim * 2 * (1 if kv_dtype == "e4m3" else 2)
    tcm = q_len >= 3 and kv_dtype == "bf16" and head_dim == 128 and q_len * group <= 32
    item_bytes = (152 if q_len == 1 else (224 if tcm else 320)) * 1024
    return min(1024, (16 * item_bytes + tile_bytes // 2) // tile_bytes)


def _run(B, lens, Hq, Hkv, D, P, tl, kv, G, cost, q_len=1, seed=0, e4m3_kernel="mma"):
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(seed)
    Bn = len(lens)
    max_pages = max(1, -(-max(lens) // P)) + 1
    bt = torch.zeros((Bn, max_pages), dtype=torch.int32, device=dev)
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    if kv == "e4m3":
        kp = torch.randint(0, 0x7E, (1, Hkv, P, D), dtype=torch.uint8, generator=gen).to(dev)
        vp = torch.randint(0, 0x7E, (1, Hkv, P, D), dtype=torch.uint8, generator=gen).to(dev)
        ks = torch.full((Hkv,), 0.01, device=dev)
        vs = torch.full((Hkv,), 0.01, device=dev)
    else:
        kp = torch.randn((1, Hkv, P, D), generator=gen).to(torch.bfloat16).to(dev)
        vp = torch.randn((1, Hkv, P, D), generator=gen).to(torch.bfloat16).to(dev)
        ks = vs = None
    record_items = Bn * Hkv + 1
    rec = torch.full((B.record_bytes(G, record_items),), SENTINEL, dtype=torch.uint8, device=dev)
    if q_len == 1:
        q = torch.randn((Bn, Hq, D), generator=gen).to(torch.bfloat16).to(dev)
        _, st, _ = B.decode_step_fused(q, kp, vp, bt, seq, Hq, Hkv, tl, kv_dtype=kv, k_scale=ks, v_scale=vs,
                                       num_ctas=G, item_cost=cost, record=rec, record_items=record_items,
                                       e4m3_kernel=e4m3_kernel)
    else:
        q = torch.randn((Bn, q_len, Hq, D), generator=gen).to(torch.bfloat16).to(dev)
        _, st, _ = B.decode_step_multi(q, kp, vp, bt, seq, Hkv, tl, kv_dtype=kv, k_scale=ks, v_scale=vs,
                                       num_ctas=G, item_cost=cost, record=rec, record_items=record_items)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    used = int(B.read_record(rec, G, record_items)[0]["item_cost"][0])
    want_cost = _default_cost(tl, D, kv, q_len, Hq // Hkv) if cost is None else cost
    assert used == want_cost
    split = OP.plan_cost_split(lens, Hkv, tl, G, used)
    assert rec.cpu().numpy().tobytes() == _expected_record(B, split, record_items).tobytes()
    return split


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("cost", [0, None, 1024])
@pytest.mark.parametrize("name", ["tiny", "uniform", "extreme", "fp8"])
def test_record_named_workloads(B, name, cost):
    spec = W.config_spec(name)
    for G in (_sms(), 2 * _sms(), 7):
        _run(B, list(spec.seq_lens), spec.num_heads, spec.kv_heads, spec.head_dim, spec.page_size, spec.tile_len,
             spec.kv_dtype, G, cost)


@pytest.mark.parametrize("cost", [0, None])
def test_record_tcgen05_kernel(B, cost):
    """The tcgen05 E4M3 kernel walks the same split and writes the same record."""
    spec = W.config_spec("fp8")
    _run(B, list(spec.seq_lens), spec.num_heads, spec.kv_heads, spec.head_dim, spec.page_size, spec.tile_len,
         "e4m3", _sms(), cost, e4m3_kernel="tcgen05")


@pytest.mark.parametrize("cost", [0, None, 1024])
def test_record_every_heavy_tailed_step(B, cost):
    spec = W.config_spec("heavy")
    for step in range(spec.steps):
        lens = [L + step for L in spec.seq_lens]
        _run(B, lens, spec.num_heads, spec.kv_heads, spec.head_dim, spec.page_size, spec.tile_len, spec.kv_dtype,
             _sms(), cost)


@pytest.mark.parametrize("q_len", [2, 4])
def test_record_several_new_tokens(B, q_len):
    spec = W.config_spec("heavy")
    for cost in (0, None):
        _run(B, list(spec.seq_lens), spec.num_heads, spec.kv_heads, spec.head_dim, spec.page_size, spec.tile_len,
             "bf16", _sms(), cost, q_len=q_len)


def test_record_ragged_and_empty(B):
    rng = np.random.default_rng(5)
    for _ in range(6):
        lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 300, 2049, 5000], size=int(rng.integers(1, 60)))]
        for G in (1, 3, 37, 148):
            for cost in (0, 38, 1024):
                _run(B, lens, 16, 4, 128, 64, 64, "bf16", G, cost)


def test_record_items_beyond_capacity_are_counted(B):
    """A record with fewer item entries than a CTA runs keeps the first ones and the full count."""
    dev = torch.device("cuda")
    lens = [17] * 40
    bt = torch.zeros((40, 2), dtype=torch.int32, device=dev)
    kp = torch.zeros((1, 2, 16, 64), dtype=torch.bfloat16, device=dev)
    q = torch.zeros((40, 8, 64), dtype=torch.bfloat16, device=dev)
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    rec = torch.full((B.record_bytes(1, 3),), SENTINEL, dtype=torch.uint8, device=dev)
    B.decode_step_fused(q, kp, kp, bt, seq, 8, 2, 32, num_ctas=1, item_cost=0, record=rec, record_items=3)
    torch.cuda.synchronize()
    heads, items = B.read_record(rec, 1, 3)
    split = OP.plan_cost_split(lens, 2, 32, 1, 0)
    assert int(heads[0]["n_items"]) == 80 and len(items[0]) == 3
    assert items[0].tobytes() == split.items[0][:3].astype(B.ITEM_DTYPE).tobytes()
