"""The per-CTA trace of the HPC_TRACE build (libhpcdecode_trace.so).

North-star evidence for load balance is the busy time and the idle tail of every CTA. The
library built with HPC_TRACE stamps, per CTA, %globaltimer at entry, when its plan is ready,
when its first stage is consumed, when its consumers finish their last item and when its
producer is done, with its item and stage counts and SM id (include/hpc_decode.h,
hpc_step_options). The default build has none of this code and refuses a trace buffer.

Checked: the stamps are in order; the item count of every CTA equals the oracle's cost split
(single launch) or the device plan (three launches); the stage count equals the pipeline chunks
of those items; SM ids are valid; and the traced step's output matches the oracle.
"""
import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import planner as OP
from tests.helpers import assert_bf16_tol, oracle_out, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture
def BT():
    """The binding switched to the trace build for one test, and back to the default build after it."""
    from load_balanced_split_step_b200 import binding, build
    lib = build.build_trace()
    binding.use_library(lib)
    assert binding.build_flags() & binding.BUILD_TRACE
    yield binding
    binding.use_library()


def _chunks(items, lens, tl, P):
    C = min(tl, P, 64)
    n = 0
    for it in items:
        L = lens[int(it["req"])]
        t0, t1 = int(it["tile_begin"]) * tl, min(int(it["tile_end"]) * tl, L)
        n += -(-(t1 - t0) // C)
    return n


def _check_stamps(tr, n_items, n_stages, sms):
    for g in range(tr.shape[0]):
        t = tr[g]
        assert t[0] > 0 and t[0] <= t[1] <= t[4], (g, t)
        assert int(t[5]) == n_items[g] and int(t[6]) == n_stages[g], (g, t, n_items[g], n_stages[g])
        assert 0 <= int(t[7]) < sms
        if n_items[g]:
            assert t[1] <= t[2] <= t[3], (g, t)
        else:
            assert t[2] == 0 and t[3] == 0


@pytest.mark.parametrize("cost", [0, None])
def test_trace_single_launch(BT, cost):
    spec = W.custom_spec((1, 17, 300, 1000, 2049, 0, 5000, 64, 129), 16, 4, 128, 64, 64, seed=91)
    case = W.make_case(spec)
    dc = to_device(case)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for G in (5, sms):
        trace = torch.zeros((G, BT.TRACE_WORDS), dtype=torch.int64, device="cuda")
        ri = spec.batch * spec.kv_heads + 1
        rec = torch.zeros(BT.record_bytes(G, ri), dtype=torch.uint8, device="cuda")
        out, st, _ = BT.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                          16, 4, 64, num_ctas=G, item_cost=cost, trace=trace, record=rec,
                                          record_items=ri)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert_bf16_tol(out, oracle_out(case), what="traced step")
        used = int(BT.read_record(rec, G, ri)[0]["item_cost"][0])
        split = OP.plan_cost_split(spec.seq_lens, 4, 64, G, used)
        n_items = [len(split.items[g]) for g in range(G)]
        n_stages = [_chunks(split.items[g], spec.seq_lens, 64, 64) for g in range(G)]
        _check_stamps(trace.cpu().numpy(), n_items, n_stages, sms)


def test_trace_three_launch(BT):
    spec = W.config_spec("tiny")
    case = W.make_case(spec)
    dc = to_device(case)
    G = 8
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = BT.plan(dc["seq_lens"], 8, 2, 32, G, 0, st)
    trace = torch.zeros((G, BT.TRACE_WORDS), dtype=torch.int64, device="cuda")
    out, po, pml = BT.attention(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], p,
                                status=st, trace=trace)
    BT.merge(p, po, pml, out, 8, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_bf16_tol(out, oracle_out(case), what="traced three-launch step")
    ref = OP.plan_dynamic(spec.seq_lens, 2, 32, G)
    n_items = [int(ref.cta_indptr[g + 1] - ref.cta_indptr[g]) for g in range(G)]
    n_stages = [_chunks(ref.items[ref.cta_indptr[g]:ref.cta_indptr[g + 1]], spec.seq_lens, 32, 16) for g in range(G)]
    _check_stamps(trace.cpu().numpy(), n_items, n_stages, torch.cuda.get_device_properties(0).multi_processor_count)


def test_default_build_refuses_a_trace_buffer():
    from load_balanced_split_step_b200 import binding as B
    assert not (B.build_flags() & B.BUILD_TRACE)
    spec = W.config_spec("tiny")
    dc = to_device(W.make_case(spec))
    trace = torch.zeros((8, B.TRACE_WORDS), dtype=torch.int64, device="cuda")
    with pytest.raises(B.HpcError, match="HPC_TRACE"):
        B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 8, 2, 32,
                            num_ctas=8, trace=trace)


def test_trace_several_tokens_tcgen05(BT):
    """Four new tokens per request on the tcgen05 kernel (the default for three or four): the
    same stamps, with the stage count in its 128-token stages."""
    spec = W.custom_spec((4, 17, 300, 1000, 2049, 5000, 64, 129), 32, 4, 128, 64, 128, seed=93, q_len=4)
    case = W.make_case(spec)
    dc = to_device(case)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    q = dc["q"] if dc["q"].dim() == 4 else dc["q"].unsqueeze(1).contiguous()
    for G in (5, sms):
        trace = torch.zeros((G, BT.TRACE_WORDS), dtype=torch.int64, device="cuda")
        ri = spec.batch * spec.kv_heads + 1
        rec = torch.zeros(BT.record_bytes(G, ri), dtype=torch.uint8, device="cuda")
        out, st, _ = BT.decode_step_multi(q, dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                          spec.kv_heads, spec.tile_len, num_ctas=G, trace=trace, record=rec,
                                          record_items=ri)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        used = int(BT.read_record(rec, G, ri)[0]["item_cost"][0])
        split = OP.plan_cost_split(spec.seq_lens, spec.kv_heads, spec.tile_len, G, used)
        n_items = [len(split.items[g]) for g in range(G)]
        n_stages = [_chunks_of(split.items[g], spec.seq_lens, spec.tile_len, 128) for g in range(G)]
        _check_stamps(trace.cpu().numpy(), n_items, n_stages, sms)


def _chunks_of(items, lens, tl, C):
    n = 0
    for it in items:
        L = lens[int(it["req"])]
        t0, t1 = int(it["tile_begin"]) * tl, min(int(it["tile_end"]) * tl, L)
        n += -(-(t1 - t0) // C)
    return n
