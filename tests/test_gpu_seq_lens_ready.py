"""The seq_lens_ready option through the C ABI. With it, the single-launch kernels read seq_lens
and plan their split before they wait for the previous kernel on the stream, which the caller
promises does not write seq_lens. Checked: the same output bytes and the same record of the
split as without it, on the one-token kernel (bf16; E4M3 on both E4M3 kernels), on both kernels
for several new tokens, on the log-sum-exp step and with the prologue folded in (there also the
same cache bytes); and steps launched back to back, each on lengths written before the first
launch, against the fp64 oracle."""
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from tests.helpers import assert_bf16_tol, oracle_out, to_device

pytestmark = pytest.mark.gpu

LENS = (1, 17, 128, 129, 700, 4096, 33, 2500, 64, 1000)
G = 148


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


@pytest.mark.parametrize("kv_dtype,e4m3_kernel", [("bf16", "mma"), ("e4m3", "mma"), ("e4m3", "tcgen05")])
def test_one_token_same_bytes_and_split(B, kv_dtype, e4m3_kernel):
    spec = W.custom_spec(LENS, 64, 8, 128, 64, 128, kv_dtype=kv_dtype, seed=301)
    case = W.make_case(spec)
    dc = to_device(case)
    outs, recs = [], []
    for ready in (False, True):
        rec = torch.zeros(B.record_bytes(G, 8), dtype=torch.uint8, device="cuda")
        out, st, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                         64, 8, 128, kv_dtype=kv_dtype, k_scale=dc["k_scale"], v_scale=dc["v_scale"],
                                         num_ctas=G, e4m3_kernel=e4m3_kernel, record=rec, record_items=8,
                                         seq_lens_ready=ready)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs.append(out.clone())
        recs.append(rec.clone())
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(recs[0], recs[1])
    if kv_dtype == "bf16":
        assert_bf16_tol(outs[1], oracle_out(case), what="seq_lens_ready")


@pytest.mark.parametrize("kernel", ["tcgen05", "mma"])
def test_several_tokens_same_bytes(B, kernel):
    lens = tuple(max(L, 4) for L in LENS)  # every request holds its 4 new tokens
    spec = W.custom_spec(lens, 32, 8, 128, 64, 128, seed=302, q_len=4)
    case = W.make_case(spec)
    dc = to_device(case)
    outs = []
    for ready in (False, True):
        q = dc["q"] if dc["q"].dim() == 4 else dc["q"].unsqueeze(1).contiguous()
        out, st, _ = B.decode_step_multi(q, dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 8,
                                         128, num_ctas=G, multi_kernel=kernel, seq_lens_ready=ready)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1])


def test_lse_step_same_bytes(B):
    spec = W.custom_spec(LENS, 64, 8, 128, 64, 128, seed=303)
    case = W.make_case(spec)
    dc = to_device(case)
    got = []
    for ready in (False, True):
        out, lse, st, _ = B.decode_step_lse(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                            64, 8, 128, num_ctas=G, seq_lens_ready=ready)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        got.append((out.clone(), lse.clone()))
    assert torch.equal(got[0][0], got[1][0]) and torch.equal(got[0][1], got[1][1])


def test_back_to_back_steps(B):
    """Four steps launched without a synchronisation between them, each on its own lengths
    (L + step, written to the device before the first launch), one workspace: every kernel
    plans while the previous step's kernel is still running."""
    steps = 4
    spec = W.custom_spec(LENS, 64, 8, 128, 64, 128, seed=304, steps=steps)
    case = W.make_case(spec)
    dc = to_device(case)
    lens = [dc["seq_lens"] + s for s in range(steps)]
    status = B.new_status(torch.device("cuda"))
    torch.cuda.synchronize()
    outs, ws = [], None
    for s in range(steps):
        out, _, ws = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], lens[s], 64, 8,
                                         128, num_ctas=G, workspace=ws, status=status, seq_lens_ready=True)
        outs.append(out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for s in range(steps):
        ref = oracle_out(case, seq_lens=case.seq_lens + s)
        assert_bf16_tol(outs[s], ref, what=f"back-to-back step {s}")
    assert bool(torch.all(ws[: len(LENS) * 8 * 4] == 0).item())  # merge tickets left at zero


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_folded_prologue_same_bytes(B, kv_dtype):
    """The single launch with the prologue folded in: the same output, cache bytes and split
    record with and without the option (each run on its own copy of the cache, since the step
    writes the new token into it)."""
    spec = W.custom_spec(LENS, 64, 8, 128, 64, 128, kv_dtype=kv_dtype, prologue=True, seed=305)
    case = W.make_case(spec)
    got = []
    for ready in (False, True):
        d = to_device(case)
        rec = torch.zeros(B.record_bytes(G, 8), dtype=torch.uint8, device="cuda")
        out, st, _ = B.decode_step_prologue(d["qkv"], d["q_norm_w"], d["k_norm_w"], d["k_pages"], d["v_pages"],
                                            d["block_table"], d["seq_lens"], 64, 8, 128, kv_dtype=kv_dtype,
                                            k_scale=d["k_scale"], v_scale=d["v_scale"], num_ctas=G, record=rec,
                                            record_items=8, seq_lens_ready=ready)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        got.append((out.clone(), d["k_pages"].clone(), d["v_pages"].clone(), rec.clone()))
    for a, b in zip(got[0], got[1]):
        assert torch.equal(a, b)
