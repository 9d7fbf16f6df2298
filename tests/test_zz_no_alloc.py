"""hpc_decode_step_noalloc: the decode step for callers that cannot allocate device memory.

Such callers include code running under CUDA graph capture, serving loops that reserve all
device memory up front, and plugins whose host framework owns the allocator. For them the
library keeps the plan workspace and the partial softmax states in its own static device
array. These tests call that entry point through the C ABI twice in a row, on two
different batches, so the second call runs on scratch left dirty by the first. Each
result is checked against the regular entry points (caller-owned buffers) within the
parity tolerance. They also check that an oversized shape is refused before any launch.
The file is named to be collected last, and passes both alone and after the others.
"""
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from tests.helpers import BF16_TOL, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from load_balanced_split_step_b200 import binding
    return binding


def _both(B, spec, dc, num_ctas):
    ref, _, st_ref = B.decode_step(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                   spec.num_heads, spec.kv_heads, spec.tile_len, kv_dtype=spec.kv_dtype,
                                   k_scale=dc["k_scale"], v_scale=dc["v_scale"], num_ctas=num_ctas)
    got, st = B.decode_step_noalloc(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"],
                                    spec.num_heads, spec.kv_heads, spec.tile_len, kv_dtype=spec.kv_dtype,
                                    k_scale=dc["k_scale"], v_scale=dc["v_scale"], num_ctas=num_ctas)
    torch.cuda.synchronize()
    return ref, got, int(st_ref.item()), int(st.item())


def test_noalloc_matches_regular_entry_points_twice(B):
    # first call: a mixed batch with splits; second call: a different, smaller batch on dirty scratch
    a = W.custom_spec((131, 4096, 17, 9000, 1, 640), 64, 8, 128, 64, 128, seed=41)
    b = W.custom_spec((33, 200, 513), 8, 2, 64, 16, 32, seed=42)
    for spec, G in ((a, 148), (b, 8)):
        dc = to_device(W.make_case(spec))
        ref, got, st_ref, st = _both(B, spec, dc, G)
        assert st == 0 and st_ref == 0
        d = (got - ref).abs()
        assert torch.isfinite(got).all()
        assert d.max().item() <= BF16_TOL["max"] and d.mean().item() <= BF16_TOL["mean"]


def test_noalloc_refuses_shapes_beyond_the_scratch(B):
    spec = W.custom_spec((16,), 8, 2, 64, 16, 32, seed=43)
    dc = to_device(W.make_case(spec))
    # 8 q heads x 64 dims x 4 B per item: a huge CTA count needs more than 16 MiB of partials
    with pytest.raises(B.HpcError, match="scratch"):
        B.decode_step_noalloc(dc["q"], dc["k_pages"], dc["v_pages"], dc["block_table"], dc["seq_lens"], 8, 2, 32,
                              num_ctas=1 << 18)
