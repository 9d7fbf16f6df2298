"""Helpers shared by the GPU parity tests: move a seeded case to the device, run the
library's decode step through the C ABI, and run the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

from load_balanced_split_step_b200 import workloads as W

BF16_TOL = {"max": 2e-3, "mean": 2e-4}  # bf16 KV vs the fp64 oracle (task tolerance)
FP8_TOL = {"max": 5e-2}  # E4M3 KV vs the fp64 oracle


def to_device(case: W.DecodeCase, dev="cuda") -> dict:
    d = {
        "seq_lens": case.seq_lens.to(dev),
        "block_table": case.block_table.to(dev),
        "k_pages": case.k_pages.to(dev),
        "v_pages": case.v_pages.to(dev),
    }
    for name in ("q", "qkv", "k_scale", "v_scale", "q_norm_w", "k_norm_w"):
        t = getattr(case, name)
        d[name] = None if t is None else t.to(dev)
    return d


def run_attention(B, spec, dc, seq_lens=None, num_ctas=None, out_dtype=torch.float32, static_splits=None,
                  q=None, tile_len=None, e4m3_kernel="mma"):
    """plan -> attention -> merge through the binding. Returns (out, plan, status int)."""
    seq = dc["seq_lens"] if seq_lens is None else seq_lens
    out, p, st = B.decode_step(dc["q"] if q is None else q, dc["k_pages"], dc["v_pages"], dc["block_table"], seq,
                               spec.num_heads, spec.kv_heads, tile_len or spec.tile_len, kv_dtype=spec.kv_dtype,
                               k_scale=dc["k_scale"], v_scale=dc["v_scale"], num_ctas=num_ctas,
                               out_dtype=out_dtype, static_splits=static_splits, e4m3_kernel=e4m3_kernel)
    torch.cuda.synchronize()
    return out, p, int(st.item())


def oracle_out(case: W.DecodeCase, seq_lens=None, requests=None, q=None):
    from oracle import attention as OA
    lens = case.seq_lens if seq_lens is None else seq_lens
    return OA.decode_attention(case.q if q is None else q, case.k_pages, case.v_pages, case.block_table, lens,
                               kv_dtype=case.spec.kv_dtype, k_scale=case.k_scale, v_scale=case.v_scale,
                               requests=requests)


def errors(got: torch.Tensor, ref: np.ndarray, rows=None):
    g = got.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        g, ref = g[rows], ref[rows]
    d = np.abs(g - ref)
    return float(d.max()), float(d.mean())


def assert_bf16_tol(got, ref, rows=None, what=""):
    mx, mean = errors(got, ref, rows)
    assert mx <= BF16_TOL["max"] and mean <= BF16_TOL["mean"], f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean
