"""The give-up path of the library's bounded waits, made to run out without faulting the GPU.

Every pipeline wait in the kernels is the same time-limited mbarrier wait. hpc_wait_selftest
runs it on a barrier phase that nothing completes, with a short limit: the wait must give
up after about that limit, the status word must carry HPC_DEV_TIMEOUT, and the context must
stay usable (a decode step right after it matches the fp64 oracle with a clean status). A
phase that does complete must pass at once and leave the status clear."""
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from tests.helpers import assert_bf16_tol, oracle_out, to_device

pytestmark = pytest.mark.gpu

HPC_DEV_TIMEOUT = 0x8


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def test_completed_phase_passes_at_once(B):
    st, waited = B.wait_selftest(1_000_000_000, True, "cuda")
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert 0 <= int(waited.item()) < 1_000_000  # well under a millisecond


@pytest.mark.parametrize("limit_ms", [1, 20])
def test_wait_gives_up_after_its_limit(B, limit_ms):
    limit = limit_ms * 1_000_000
    st, waited = B.wait_selftest(limit, False, "cuda")
    torch.cuda.synchronize()
    assert int(st.item()) == HPC_DEV_TIMEOUT
    w = int(waited.item())
    assert limit <= w < limit + 50_000_000, w  # gives up once past the limit, not much later


def test_status_bits_accumulate_until_cleared(B):
    st = B.new_status("cuda")
    st.fill_(0x2)  # a bit left by an earlier call stays set: the word is OR-ed, never overwritten
    B.wait_selftest(1_000_000, False, "cuda", status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0x2 | HPC_DEV_TIMEOUT


def test_context_usable_after_a_timeout(B):
    B.wait_selftest(2_000_000, False, "cuda")
    spec = W.custom_spec((1, 17, 200, 513, 2049), 16, 2, 128, 64, 64, seed=5)
    case = W.make_case(spec)
    dc = to_device(case)
    out, st, _ = B.decode_step_fused(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                     spec.num_heads, spec.kv_heads, spec.tile_len)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_bf16_tol(out, oracle_out(case), what="step after a timed-out wait")
