"""Fused decode prologue in fp64: QK-RMSNorm, RoPE and the KV-page write of the new token
(test infrastructure; see ``oracle/__init__``).

"vLLM × HPC-Ops: High-Performance Attention and MoE Backends from Tencent Hunyuan" (8sync
News summary) names a fused RoPE + QK-Norm + KV-write prologue in front of the
attention backend. It says nothing more. The readings:

* Norm: RMSNorm per head, x * w / sqrt(mean(x^2) + eps), on q heads (weight q_norm_w)
  and the new k heads (weight k_norm_w). V is not normalised.
* Order: RMSNorm first, then RoPE. With unit weights the order does not matter,
  because RoPE rotates coordinate pairs and so preserves the mean square.
* RoPE: NeoX rotate-half over pairs (i, i + D/2), i < D/2.
  inv_freq_i = theta^(-2i/D), angle = pos * inv_freq_i, and pos = L_r - 1 (seq_lens
  includes the new token).
* KV write: the new k and v go to page block_table[r, pos // P], slot pos % P, of
  kv head g. For an E4M3 cache the stored code is e4m3(x / scale[g]) (RNE, saturating).
* The normalised, rotated q is the attention query. This oracle keeps it in fp64.
"""
from __future__ import annotations

import numpy as np

from . import fp8
from .attention import to_f64


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    return x * np.asarray(w, dtype=np.float64) / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope_angles(pos: int, head_dim: int, theta: float) -> np.ndarray:
    i = np.arange(head_dim // 2, dtype=np.float64)
    return float(pos) * np.power(float(theta), -2.0 * i / head_dim)


def rope_neox(x: np.ndarray, pos: int, theta: float) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    ang = rope_angles(pos, D, theta)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def decode_prologue(qkv, q_norm_w, k_norm_w, eps, theta, seq_lens, block_table,
                    k_pages, v_pages, kv_dtype, k_scale, v_scale, num_heads, kv_heads):
    """Returns (q [B, Hq, D] float64, k_new [B, Hkv, D], v_new [B, Hkv, D], writes).

    k_new / v_new are the values to store before encoding: k after norm and RoPE, v
    as is, both divided by the per-head scale for an E4M3 cache. ``writes`` lists
    (r, page, slot). The page arrays (numpy, modified in place) receive the encoded
    new token: bf16 caches get the RNE bf16 of the value as uint16 bits; E4M3 caches
    get the code.
    """
    x = to_f64(qkv)
    B, _, D = x.shape
    Hq, Hkv = num_heads, kv_heads
    qn, kn = to_f64(q_norm_w), to_f64(k_norm_w)
    lens = np.asarray(seq_lens, dtype=np.int64)
    bt = np.asarray(block_table, dtype=np.int64)
    P = k_pages.shape[2]
    q = np.zeros((B, Hq, D))
    k_new = np.zeros((B, Hkv, D))
    v_new = np.zeros((B, Hkv, D))
    writes = []
    for r in range(B):
        pos = int(lens[r]) - 1
        for h in range(Hq):
            q[r, h] = rope_neox(rms_norm(x[r, h], qn, eps), pos, theta)
        for g in range(Hkv):
            k = rope_neox(rms_norm(x[r, Hq + g], kn, eps), pos, theta)
            v = x[r, Hq + Hkv + g]
            if kv_dtype == "e4m3":
                k = k / float(to_f64(k_scale)[g])
                v = v / float(to_f64(v_scale)[g])
            k_new[r, g], v_new[r, g] = k, v
        page, slot = int(bt[r, pos // P]), pos % P
        writes.append((r, page, slot))
        for g in range(Hkv):
            if kv_dtype == "e4m3":
                k_pages[page, g, slot, :] = fp8.encode_array(k_new[r, g])
                v_pages[page, g, slot, :] = fp8.encode_array(v_new[r, g])
            else:
                k_pages[page, g, slot, :] = bf16_bits(k_new[r, g])
                v_pages[page, g, slot, :] = bf16_bits(v_new[r, g])
    return q, k_new, v_new, writes


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even) and return the 16-bit
    patterns. bf16 is the top half of an IEEE binary32, so the value is rounded
    to 8 significant bits. This rounds the float64 directly (one rounding), not
    through float32."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    for idx, v in np.ndenumerate(x):
        out[idx] = _bf16_one(float(v))
    return out


def _bf16_one(v: float) -> int:
    if np.isnan(v):
        return 0x7FC0
    sign = 0x8000 if np.signbit(v) else 0
    a = abs(v)
    if a == 0.0:
        return sign
    # candidates: the two bf16 values bracketing a (found from the float32 grid)
    f32 = np.float32(a)
    bits = int(np.array(f32, dtype=np.float32).view(np.uint32))
    lo_bits = bits & 0xFFFF0000
    cands = [lo_bits - 0x10000 if lo_bits >= 0x10000 else lo_bits, lo_bits, lo_bits + 0x10000]
    best, best_d = None, None
    for cb in cands:
        val = float(np.array(cb, dtype=np.uint32).view(np.float32))
        d = abs(val - a)
        if best_d is None or d < best_d or (d == best_d and ((cb >> 16) & 1) == 0):
            best, best_d = cb, d
    return sign | (best >> 16)
