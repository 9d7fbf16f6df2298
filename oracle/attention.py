"""Exact paged decode attention in fp64 (test infrastructure; see ``oracle/__init__``).

What the method computes. For every request r and query head h, the output is
softmax(scale * q K^T) V over all L_r cached tokens of r. That is the quantity the
load-balanced split-KV kernel reaches by tiles and merges. Sources:

* "vLLM × HPC-Ops: High-Performance Attention and MoE Backends from Tencent Hunyuan"
  (8sync News summary): split-KV decode attention with a per-step load-balanced
  scheduler;
* "腾讯混元三算子杀入 SGLang" (AREX, section "Router GEMM：精度不丢，速度翻三倍", the
  Dynamic Attention paragraph): each decode step, tiles are assigned by the actual KV
  length.

Splitting the KV sequence and merging partial softmax states by log-sum-exp is exact in
real arithmetic, so this oracle is the unsplit definition written out.

Readings where the pages are silent:

* GQA head map: query head h reads kv head floor(h / (Hq / Hkv)), in contiguous
  groups.
* scale = 1 / sqrt(head_dim) unless given.
* The cache is paged HND: token j of request r, kv head g, is
  ``pages[block_table[r, j // P], g, j % P, :]``.
* An E4M3 cache holds codes; the value is decode(code) * scale[g].
* A request with L_r = 0 attends over nothing; its output is defined as 0.

Pins (tests/test_oracle_attention.py, tests/test_oracle_multi.py): torch SDPA in fp64,
pure-Python loops on tiny inputs, closed forms (a single key returns v; identical keys or
q = 0 give the mean of v; no keys give 0), split invariance, and planted mistakes (a wrong
page index, GQA map or scale) that the pins catch. The pages print no worked numerical
example, so the pins tie the oracle to the definition itself.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import fp8


def to_f64(x) -> np.ndarray:
    """bf16 / fp32 tensor -> float64 numpy (exact widening)."""
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def gather_tokens(pages: np.ndarray, block_table: np.ndarray, r: int, kv_head: int, L: int):
    """Rows 0..L-1 of request r for one kv head, in logical token order: token j is
    ``pages[block_table[r, j // P], kv_head, j % P, :]``."""
    P = pages.shape[2]
    j = np.arange(L)
    return pages[block_table[r, j // P], kv_head, j % P, :]


def _kv_values(pages, kv_dtype: str, scale, block_table, r, g, L) -> np.ndarray:
    rows = gather_tokens(pages, block_table, r, g, L)
    if kv_dtype == "e4m3":
        return fp8.decode_array(rows) * float(scale[g])
    return rows.astype(np.float64)


def decode_attention(q, k_pages, v_pages, block_table, seq_lens, sm_scale=None,
                     kv_dtype="bf16", k_scale=None, v_scale=None, requests=None):
    """out[r, h, :] = sum_j softmax_j(sm_scale * q[r,h] . k_j) v_j for each request r
    (or only ``requests``) and query head h. Returns float64 [B, Hq, D]; rows for
    requests not asked for stay 0.

    q: [B, Hq, D] (bf16 tensor or float array). k_pages / v_pages: [num_pages, Hkv, P, D]
    bf16 tensors, or uint8 E4M3 codes when kv_dtype == "e4m3". block_table:
    int [B, max_pages]. seq_lens: int [B].
    """
    qf = to_f64(q)
    B, Hq, D = qf.shape
    if kv_dtype == "e4m3":
        kp = np.asarray(k_pages.cpu().numpy() if isinstance(k_pages, torch.Tensor) else k_pages, dtype=np.uint8)
        vp = np.asarray(v_pages.cpu().numpy() if isinstance(v_pages, torch.Tensor) else v_pages, dtype=np.uint8)
        ks, vs = to_f64(k_scale), to_f64(v_scale)
    else:
        kp, vp = k_pages, v_pages
        ks = vs = None
    Hkv = kp.shape[1]
    grp = Hq // Hkv
    bt = np.asarray(block_table.cpu().numpy() if isinstance(block_table, torch.Tensor) else block_table, dtype=np.int64)
    lens = np.asarray(seq_lens.cpu().numpy() if isinstance(seq_lens, torch.Tensor) else seq_lens, dtype=np.int64)
    scale = (1.0 / math.sqrt(D)) if sm_scale is None else float(sm_scale)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for r in (range(B) if requests is None else requests):
        L = int(lens[r])
        if L == 0:
            continue
        for g in range(Hkv):
            if kv_dtype == "e4m3":
                K = _kv_values(kp, kv_dtype, ks, bt, r, g, L)
                V = _kv_values(vp, kv_dtype, vs, bt, r, g, L)
            else:
                K = to_f64(_torch_gather(kp, bt, r, g, L))
                V = to_f64(_torch_gather(vp, bt, r, g, L))
            for h in range(g * grp, (g + 1) * grp):
                s = scale * (K @ qf[r, h])  # [L] scores
                p = np.exp(s - s.max())
                p = p / p.sum()
                out[r, h] = p @ V
    return out


def _torch_gather(pages: torch.Tensor, bt: np.ndarray, r: int, g: int, L: int) -> torch.Tensor:
    """``gather_tokens`` for a torch page pool (keeps bf16 until the exact widening)."""
    P = pages.shape[2]
    j = torch.arange(L)
    phys = torch.from_numpy(bt[r])[j // P]
    return pages[phys, g, j % P, :]


def decode_attention_multi(q, k_pages, v_pages, block_table, seq_lens, sm_scale=None,
                           kv_dtype="bf16", k_scale=None, v_scale=None, requests=None):
    """Several new tokens per request, attending causally (speculative verification, or a
    chunked extend of the decode batch).

    q: [B, T, Hq, D]. The T query tokens of request r are the last T of its L_r cached
    tokens: query token t sits at position L_r - T + t and attends to positions
    0 .. L_r - T + t, itself included. Returns float64 [B, T, Hq, D]:

        out[r, t, h, :] = sum_{j <= L_r - T + t} softmax_j(sm_scale * q[r,t,h] . k_j) v_j

    Readings where the pages are silent (they report the backend's effect on time to first
    token, not its prefill kernel): all requests of a step share T; L_r = 0 gives zeros, and a
    request with 0 < L_r < T has no valid query position and also gives zeros. The rest
    follows decode_attention (GQA map, page layout, E4M3 decoding, scale).
    """
    qf = to_f64(q)
    B, T, Hq, D = qf.shape
    if kv_dtype == "e4m3":
        kp = np.asarray(k_pages.cpu().numpy() if isinstance(k_pages, torch.Tensor) else k_pages, dtype=np.uint8)
        vp = np.asarray(v_pages.cpu().numpy() if isinstance(v_pages, torch.Tensor) else v_pages, dtype=np.uint8)
        ks, vs = to_f64(k_scale), to_f64(v_scale)
    else:
        kp, vp = k_pages, v_pages
        ks = vs = None
    Hkv = kp.shape[1]
    grp = Hq // Hkv
    bt = np.asarray(block_table.cpu().numpy() if isinstance(block_table, torch.Tensor) else block_table, dtype=np.int64)
    lens = np.asarray(seq_lens.cpu().numpy() if isinstance(seq_lens, torch.Tensor) else seq_lens, dtype=np.int64)
    scale = (1.0 / math.sqrt(D)) if sm_scale is None else float(sm_scale)
    out = np.zeros((B, T, Hq, D), dtype=np.float64)
    for r in (range(B) if requests is None else requests):
        L = int(lens[r])
        if L < T:
            continue
        for g in range(Hkv):
            if kv_dtype == "e4m3":
                K = _kv_values(kp, kv_dtype, ks, bt, r, g, L)
                V = _kv_values(vp, kv_dtype, vs, bt, r, g, L)
            else:
                K = to_f64(_torch_gather(kp, bt, r, g, L))
                V = to_f64(_torch_gather(vp, bt, r, g, L))
            for t in range(T):
                n = L - T + t + 1  # tokens that query t may see
                for h in range(g * grp, (g + 1) * grp):
                    s = scale * (K[:n] @ qf[r, t, h])
                    p = np.exp(s - s.max())
                    p = p / p.sum()
                    out[r, t, h] = p @ V[:n]
    return out


def decode_lse(q, k_pages, v_pages, block_table, seq_lens, sm_scale=None, kv_dtype="bf16", k_scale=None,
               requests=None):
    """Log-sum-exp of each request and query head's scores, in natural log:

        lse[r, h] = log sum_{j < L_r} exp(sm_scale * q[r,h] . k_j)    (-inf when L_r = 0),

    the weight that combines outputs computed over disjoint parts of the keys: with parts i,
    LSE = log sum_i exp(lse_i) and out = sum_i exp(lse_i - LSE) out_i. Returns float64 [B, Hq].
    """
    qf = to_f64(q)
    B, Hq, D = qf.shape
    if kv_dtype == "e4m3":
        kp = np.asarray(k_pages.cpu().numpy() if isinstance(k_pages, torch.Tensor) else k_pages, dtype=np.uint8)
        ks = to_f64(k_scale)
    else:
        kp, ks = k_pages, None
    Hkv = kp.shape[1]
    grp = Hq // Hkv
    bt = np.asarray(block_table.cpu().numpy() if isinstance(block_table, torch.Tensor) else block_table, dtype=np.int64)
    lens = np.asarray(seq_lens.cpu().numpy() if isinstance(seq_lens, torch.Tensor) else seq_lens, dtype=np.int64)
    scale = (1.0 / math.sqrt(D)) if sm_scale is None else float(sm_scale)
    out = np.full((B, Hq), -np.inf)
    for r in (range(B) if requests is None else requests):
        L = int(lens[r])
        if L == 0:
            continue
        for g in range(Hkv):
            K = _kv_values(kp, kv_dtype, ks, bt, r, g, L) if kv_dtype == "e4m3" else \
                to_f64(_torch_gather(kp, bt, r, g, L))
            for h in range(g * grp, (g + 1) * grp):
                s = scale * (K @ qf[r, h])
                m = s.max()
                out[r, h] = m + math.log(np.exp(s - m).sum())
    return out
