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


def test_noalloc_binding_checks_mismatched_buffers(B):
    """The binding runs the same checks as the other entry points before calling the library: a
    cache head_dim different from q's, V pages shaped unlike K pages, tensors on another device,
    an output of the wrong dtype or shape, and missing E4M3 scales each raise HpcError."""
    spec = W.custom_spec((40, 100), 8, 2, 128, 16, 32, seed=44)
    dc = to_device(W.make_case(spec))
    args = dict(q=dc["q"], k_pages=dc["k_pages"], v_pages=dc["v_pages"], block_table=dc["block_table"],
                seq_lens=dc["seq_lens"], num_heads=8, kv_heads=2, tile_len=32)

    def call(**over):
        a = dict(args)
        extra = {k: over.pop(k) for k in list(over) if k in ("out", "kv_dtype", "k_scale", "v_scale")}
        a.update(over)
        return B.decode_step_noalloc(a["q"], a["k_pages"], a["v_pages"], a["block_table"], a["seq_lens"],
                                     a["num_heads"], a["kv_heads"], a["tile_len"], num_ctas=8, **extra)

    half = dc["k_pages"][..., :64].contiguous()  # a head_dim 64 cache under head_dim 128 queries
    cases = {
        "head_dim": dict(k_pages=half, v_pages=half),
        "v shape": dict(v_pages=dc["v_pages"][:-1].contiguous()),
        "device": dict(k_pages=dc["k_pages"].cpu()),
        "out dtype": dict(out=torch.empty((2, 8, 128), dtype=torch.float16, device="cuda")),
        "out shape": dict(out=torch.empty((2, 8, 64), dtype=torch.float32, device="cuda")),
        "out device": dict(out=torch.empty((2, 8, 128), dtype=torch.float32)),
        "e4m3 scales": dict(kv_dtype="e4m3", k_pages=dc["k_pages"].view(torch.uint8)[..., :128].contiguous(),
                            v_pages=dc["v_pages"].view(torch.uint8)[..., :128].contiguous()),
        "kv heads": dict(kv_heads=4, num_heads=8),
    }
    for what, over in cases.items():
        with pytest.raises(B.HpcError):
            call(**over)
        assert what  # every case raised


def test_noalloc_rejected_call_launches_nothing(B):
    """Every host check runs before the first of the three launches. A call with a bad length
    (which the planner kernel would flag in the status word) and a shape the attention refuses
    (head_dim 96, page size 48) returns an error, and the status word and the output stay
    untouched: no kernel ran."""
    spec = W.custom_spec((40, 100), 8, 2, 64, 16, 32, seed=45)
    dc = to_device(W.make_case(spec))
    bad_lens = dc["seq_lens"].clone()
    bad_lens[0] = -5
    for D, P in ((96, 16), (64, 48)):
        kp = torch.zeros((4, 2, P, D), dtype=torch.bfloat16, device="cuda")
        q = torch.zeros((2, 8, D), dtype=torch.bfloat16, device="cuda")
        out = torch.full((2, 8, D), 7.0, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        with pytest.raises(B.HpcError):
            B.decode_step_noalloc(q, kp, kp, dc["block_table"], bad_lens, 8, 2, 32, num_ctas=8, out=out, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and torch.all(out == 7.0)
