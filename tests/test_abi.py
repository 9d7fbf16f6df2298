"""CPU checks of the C-ABI library: it loads and exports every symbol include/hpc_decode.h
declares; host-detected argument errors return codes before any CUDA work; the host
planner twin equals the oracle planner byte for byte. No GPU compute is called here."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hpc_decode.h")


@pytest.fixture(scope="module")
def B():
    build.build()
    from load_balanced_split_step_b200 import binding
    return binding


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hpc_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("hpc_decode_plan", "hpc_decode_attention", "hpc_merge_states", "hpc_decode_prologue",
              "hpc_plan_cpu", "hpc_decode_plan_static", "hpc_decode_step", "hpc_decode_step_prologue",
              "hpc_decode_step_multi", "hpc_decode_step_lse", "hpc_merge_lse", "hpc_merge_lse_gather",
              "hpc_gather_rows", "hpc_wait_selftest"):
        assert n in names


def test_library_exports_every_declared_symbol(B):
    lib = ctypes.CDLL(B.library_path())
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert set(declared_symbols()) <= set(B.EXPORTS)


def test_abi_version_and_strings(B):
    assert B._lib.hpc_abi_version() == 9
    assert B.status_string(0) == "ok"
    assert B.status_string(6) == "buffer too small"


def test_host_argument_errors_return_codes(B):
    P = B.CPlan()
    i32 = ctypes.c_int32
    # null pointers -> HPC_ERR_ARG before any CUDA call
    rc = B._lib.hpc_decode_attention(None, None, None, 0, 0, None, None, 1, 16, 8, 2, 64, None, 1, None,
                                     ctypes.byref(P), 0.1, None, None, None, 1, None, None, None)
    assert rc == B.HPC_ERR_ARG
    assert "null" in B._lib.hpc_last_error().decode()
    rc = B._lib.hpc_merge_states(None, None, ctypes.byref(P), 8, 64, None, 1, None, None)
    assert rc == B.HPC_ERR_ARG
    # the single-launch step with the folded prologue: null qkv / norm weights, bad theta
    i32 = ctypes.c_int32
    rc = B._lib.hpc_decode_step_prologue(None, None, None, 1e-6, 1e6, None, None, 0, 0, None, None, 1, 16, 8, 2, 64,
                                         None, 1, None, 1, 32, 4, 0.1, None, 0, None, 1, None, None, None)
    assert rc == B.HPC_ERR_ARG
    w = ctypes.c_void_p(16)  # never dereferenced: the argument checks fail first
    rc = B._lib.hpc_decode_step_prologue(w, w, w, 1e-6, -1.0, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, 1,
                                         32, 4, 0.1, w, 0, w, 1, None, w, None)
    assert rc == B.HPC_ERR_ARG and "rope_theta" in B._lib.hpc_last_error().decode()
    # several new tokens: q_len outside 1..4 and zero-size workspace queries
    rc = B._lib.hpc_decode_step_multi(w, 5, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, 1, 32, 4, 0.1, w, 1 << 20,
                                      w, 1, None, w, None)
    assert rc == B.HPC_ERR_SHAPE and "q_len" in B._lib.hpc_last_error().decode()
    assert B._lib.hpc_decode_step_multi_workspace_bytes(4, 0, 8, 2, 64, 148) == 0
    assert (B._lib.hpc_decode_step_multi_workspace_bytes(4, 1, 8, 2, 64, 148)
            == B._lib.hpc_decode_step_workspace_bytes(4, 8, 2, 64, 148))
    # log-sum-exp step and merge: null outputs, bad sizes
    rc = B._lib.hpc_decode_step_lse(w, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, 1, 32, 4, 0.1, w, 1 << 20, w,
                                    1, None, None, w, None)
    assert rc == B.HPC_ERR_ARG
    assert B._lib.hpc_merge_lse(None, None, 2, 10, 64, None, None, None) == B.HPC_ERR_ARG
    assert B._lib.hpc_merge_lse(w, w, 0, 10, 64, w, None, None) == B.HPC_ERR_ARG
    assert B._lib.hpc_merge_lse(w, w, 2, 0, 64, w, None, None) == B.HPC_OK  # nothing to do
    # indexed merge and row gather: nulls, sizes, alignment
    assert B._lib.hpc_merge_lse_gather(None, w, 4, w, 2, 3, 8, 64, w, None, None, None) == B.HPC_ERR_ARG
    assert B._lib.hpc_merge_lse_gather(w, w, 4, w, 0, 3, 8, 64, w, None, None, None) == B.HPC_ERR_ARG
    assert B._lib.hpc_merge_lse_gather(w, w, 4, w, 2, 0, 8, 64, w, None, None, None) == B.HPC_OK  # nothing to do
    assert B._lib.hpc_gather_rows(w, 4, 256, None, 2, w, None, None) == B.HPC_ERR_ARG
    assert B._lib.hpc_gather_rows(w, 4, 200, w, 2, w, None, None) == B.HPC_ERR_SHAPE
    assert B._lib.hpc_gather_rows(ctypes.c_void_p(24), 4, 256, w, 2, w, None, None) == B.HPC_ERR_ALIGN
    assert B._lib.hpc_gather_rows(w, 4, 256, w, 0, w, None, None) == B.HPC_OK
    # wait diagnostic: null status, limit outside 1 .. 2 s
    assert B._lib.hpc_wait_selftest(1000, 0, None, None, None) == B.HPC_ERR_ARG
    assert B._lib.hpc_wait_selftest(0, 0, w, None, None) == B.HPC_ERR_ARG
    assert B._lib.hpc_wait_selftest(3_000_000_000, 0, w, None, None) == B.HPC_ERR_ARG
    assert "limit_ns" in B._lib.hpc_last_error().decode()
    # bad tile_len on the host planner
    lens = torch.tensor([5, 7], dtype=torch.int32)
    with pytest.raises(B.HpcError, match="tile_len"):
        B.plan_host(lens, 8, 2, 24, 4)
    with pytest.raises(B.HpcError, match="num_heads"):
        B.plan_host(lens, 7, 2, 32, 4)
    assert B._lib.hpc_plan_workspace_bytes(0, 2, 4) == 0


def test_options_are_checked_before_any_launch(B):
    """Per-call options (ABI 9): out-of-range values, options that belong to the single-launch
    step passed to the three-launch attention, and a trace buffer in a build without HPC_TRACE
    all return HPC_ERR_ARG before any CUDA call (the pointers are never dereferenced)."""
    w = ctypes.c_void_p(256)
    P = B.CPlan()
    P.kv_heads, P.num_ctas, P.tile_len = 2, 4, 32

    def step(opt):
        return B._lib.hpc_decode_step(w, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, 1, 32, 4, 0.1, w, 1 << 20,
                                      w, 1, None if opt is None else ctypes.byref(opt), w, None)

    def attention(opt):
        return B._lib.hpc_decode_attention(w, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, ctypes.byref(P), 0.1,
                                           w, w, w, 1, ctypes.byref(opt), w, None)

    for kw, what in ((dict(item_cost=-2), "item_cost"), (dict(item_cost=B.ITEM_COST_MAX + 1), "item_cost"),
                     (dict(e4m3_kernel="tcgen05"), None)):
        o = B.options(**kw)
        if what is None:
            o.e4m3_kernel = 7
            what = "e4m3_kernel"
        assert step(o) == B.HPC_ERR_ARG and what in B._lib.hpc_last_error().decode()
    o = B.options(item_cost=0)
    assert attention(o) == B.HPC_ERR_ARG and "single-launch" in B._lib.hpc_last_error().decode()
    o = B.options(seq_lens_ready=True)
    assert o.seq_lens_ready == 1
    assert attention(o) == B.HPC_ERR_ARG and "single-launch" in B._lib.hpc_last_error().decode()
    o.seq_lens_ready = 2
    assert step(o) == B.HPC_ERR_ARG and "seq_lens_ready" in B._lib.hpc_last_error().decode()
    assert B.options(seq_lens_ready=False) is None
    o = B.COptions(B.ITEM_COST_DEFAULT, 0, None, 0, 0, 4096)
    assert not (B.build_flags() & B.BUILD_TRACE)
    assert step(o) == B.HPC_ERR_ARG and "HPC_TRACE" in B._lib.hpc_last_error().decode()
    assert attention(o) == B.HPC_ERR_ARG
    o = B.COptions(B.ITEM_COST_DEFAULT, 0, 24, 4, 0, None)  # a record buffer that is not 16-byte aligned
    assert step(o) == B.HPC_ERR_ARG and "record" in B._lib.hpc_last_error().decode()
    assert B._lib.hpc_step_record_bytes(148, 4) == 148 * (32 + 4 * 16)
    assert B._lib.hpc_step_record_bytes(0, 4) == 0


def test_noalloc_size_checks_come_first(B):
    """The entry point without caller scratch rejects bad sizes, a token count beyond int32
    (computed in 64 bits) and shapes too big for its array before any CUDA call."""
    w = ctypes.c_void_p(256)

    def call(num_pages=8, page_size=16, num_heads=8, kv_heads=2, head_dim=64, max_pages=4, batch=3, tile_len=32,
             num_ctas=4):
        return B._lib.hpc_decode_step_noalloc(w, w, w, 0, None, None, num_pages, page_size, num_heads, kv_heads,
                                              head_dim, w, max_pages, w, batch, tile_len, num_ctas, 0.1, w, 1, w, None)

    assert call(batch=0) == B.HPC_ERR_ARG
    assert call(num_heads=7) == B.HPC_ERR_SHAPE
    assert call(max_pages=1 << 20, page_size=1 << 12) == B.HPC_ERR_SHAPE  # 2^32 tokens: no int32 wrap
    assert "INT32_MAX" in B._lib.hpc_last_error().decode()
    assert call(max_pages=0) == B.HPC_ERR_SHAPE
    assert call(batch=100000, kv_heads=8, num_heads=64, head_dim=128) == B.HPC_ERR_CAPACITY


def test_launch_info(B):
    info = B.launch_info(128, "bf16", 64, 128)
    assert info["threads"] == 288 and 2 <= info["stages"] <= 8 and info["smem_bytes"] <= 232448
    info8 = B.launch_info(128, "e4m3", 64, 128)
    assert info8["stages"] >= info["stages"]
    with pytest.raises(B.HpcError):
        B.launch_info(128, "bf16", 256, 256, ctas_per_sm=4)


def _oracle_plan(lens, Hkv, tl, G):
    from oracle import planner as OP
    return OP.plan_dynamic(lens, Hkv, tl, G)


def _compare(B, lens, Hkv, tl, G, max_seq=0):
    p, st = B.plan_host(np.asarray(lens, dtype=np.int32), Hkv * 4, Hkv, tl, G, max_seq)
    got = p.to_numpy()
    valid = [L if (L >= 0 and (max_seq <= 0 or L <= max_seq)) else 0 for L in lens]
    ref = _oracle_plan(valid, Hkv, tl, G)
    assert got["n_items"] == len(ref.items)
    assert got["items"].tobytes() == ref.items.astype(B.ITEM_DTYPE).tobytes()
    assert np.array_equal(got["cta_indptr"], ref.cta_indptr)
    assert np.array_equal(got["merge_indptr"], ref.merge_indptr)
    assert np.array_equal(got["merge_list"], ref.merge_list)
    assert got["n_units"] == ref.n_units and got["chunk"] == ref.chunk
    return st


def test_host_planner_hand_example(B):
    _compare(B, [17, 64, 200, 513], 2, 32, 8)
    _compare(B, [17, 64, 200, 513], 2, 32, 148)


@pytest.mark.parametrize("tl", [16, 32, 128, 256])
@pytest.mark.parametrize("G", [1, 7, 148, 296])
def test_host_planner_equals_oracle(B, tl, G):
    rng = np.random.default_rng(tl + 7 * G)
    for _ in range(4):
        n = int(rng.integers(1, 60))
        lens = np.floor(np.power(2.0, rng.uniform(0, 15, n))).astype(int)
        lens[rng.random(n) < 0.1] = 0
        _compare(B, lens.tolist(), int(rng.choice([1, 2, 8])), tl, G)


def test_host_planner_flags_bad_lengths(B):
    st = _compare(B, [10, -3, 50, 9999], 2, 16, 5, max_seq=100)
    assert st & B.DEV_STATUS["bad_seqlen"]
    assert _compare(B, [10, 20], 2, 16, 5, max_seq=100) == 0


def test_host_planner_full_size_workloads(B):
    from load_balanced_split_step_b200 import workloads as W
    for name in ("uniform", "extreme", "heavy", "fp8"):
        spec = W.config_spec(name)
        for step in range(spec.steps):
            lens = [L + step for L in spec.seq_lens]
            _compare(B, lens, spec.kv_heads, spec.tile_len, 148)
