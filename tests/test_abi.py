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
    assert B._lib.hpc_abi_version() == 7
    assert B.status_string(0) == "ok"
    assert B.status_string(6) == "buffer too small"


def test_host_argument_errors_return_codes(B):
    P = B.CPlan()
    i32 = ctypes.c_int32
    # null pointers -> HPC_ERR_ARG before any CUDA call
    rc = B._lib.hpc_decode_attention(None, None, None, 0, 0, None, None, 1, 16, 8, 2, 64, None, 1, None,
                                     ctypes.byref(P), 0.1, None, None, None, 1, None, None)
    assert rc == B.HPC_ERR_ARG
    assert "null" in B._lib.hpc_last_error().decode()
    rc = B._lib.hpc_merge_states(None, None, ctypes.byref(P), 8, 64, None, 1, None, None)
    assert rc == B.HPC_ERR_ARG
    # the single-launch step with the folded prologue: null qkv / norm weights, bad theta
    i32 = ctypes.c_int32
    rc = B._lib.hpc_decode_step_prologue(None, None, None, 1e-6, 1e6, None, None, 0, 0, None, None, 1, 16, 8, 2, 64,
                                         None, 1, None, 1, 32, 4, 0.1, None, 0, None, 1, None, None)
    assert rc == B.HPC_ERR_ARG
    w = ctypes.c_void_p(16)  # never dereferenced: the argument checks fail first
    rc = B._lib.hpc_decode_step_prologue(w, w, w, 1e-6, -1.0, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, 1,
                                         32, 4, 0.1, w, 0, w, 1, w, None)
    assert rc == B.HPC_ERR_ARG and "rope_theta" in B._lib.hpc_last_error().decode()
    # several new tokens: q_len outside 1..4 and zero-size workspace queries
    rc = B._lib.hpc_decode_step_multi(w, 5, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, 1, 32, 4, 0.1, w, 1 << 20,
                                      w, 1, w, None)
    assert rc == B.HPC_ERR_SHAPE and "q_len" in B._lib.hpc_last_error().decode()
    assert B._lib.hpc_decode_step_multi_workspace_bytes(4, 0, 8, 2, 64, 148) == 0
    assert (B._lib.hpc_decode_step_multi_workspace_bytes(4, 1, 8, 2, 64, 148)
            == B._lib.hpc_decode_step_workspace_bytes(4, 8, 2, 64, 148))
    # log-sum-exp step and merge: null outputs, bad sizes
    rc = B._lib.hpc_decode_step_lse(w, w, w, 0, 0, None, None, 1, 16, 8, 2, 64, w, 1, w, 1, 32, 4, 0.1, w, 1 << 20, w,
                                    1, None, w, None)
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
