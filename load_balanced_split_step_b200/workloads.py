"""Seeded synthetic decode batches: the inputs both the CUDA path and the CPU oracle consume.

This module draws random numbers and lays them out as a paged KV cache. It contains none
of the attention, planning, merge, normalisation or rotary arithmetic.

Workloads follow the mixed-length decode scenario that "vLLM × HPC-Ops: High-Performance
Attention and MoE Backends from Tencent Hunyuan" (8sync News summary) quotes: one
1x128K request batched with 31x4K ones. They also follow the note in "Tencent HPC llega a
SGLang y desafía a los kernels de inferencia predeterminados" (remio.ai, section "Por qué
Tencent HPC importa para el serving de modelos en línea") that request lengths in one
continuous batch differ widely.

Stream layout. Every draw comes from numpy's PCG64 under one ``SeedSequence(seed)``
tree, so a single request's cache can be regenerated without the rest:

* child 0: request lengths (only for workloads whose lengths are drawn);
* child 1: the physical page permutation;
* child 2: q, shape [B, Hq, D];
* child 3: qkv (prologue input), shape [B, Hq + 2 Hkv, D];
* child 4 is spawned into B streams, one per request. Stream r draws request r's K
  pages, then its V pages, each float32 N(0, 1) of shape [pages_r, Hkv, P, D].

Values are rounded to bf16 (RNE) by torch. For an FP8 (OCP E4M3) cache, each kv head
gets scale = amax / 448, with amax taken over that head's float32 draws in the whole
cache. The stored code is ``e4m3(clamp(x / scale, +-448))`` via torch's float8_e4m3fn
conversion.

Cache layout (HND): ``k_pages[num_pages, Hkv, P, D]``. ``block_table[r, j]`` is the
physical page that holds request r's tokens ``[j*P, (j+1)*P)``. Physical pages are a
random permutation of the pool. Each request has ``ceil((L_r + steps - 1) / P) + 1``
pages: enough for every decode step, plus one slack page. Table entries past that
count are -1.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class DecodeSpec:
    """Shape of one decode batch. ``seq_lens`` count valid KV tokens including the token
    being decoded (for a prologue workload that token sits at position L_r - 1)."""

    name: str
    seq_lens: tuple
    num_heads: int
    kv_heads: int
    head_dim: int
    page_size: int
    tile_len: int
    kv_dtype: str = "bf16"  # "bf16" or "e4m3"
    steps: int = 1  # decode steps; step i uses seq_lens + i
    prologue: bool = False
    q_len: int = 1  # new tokens per request (the last q_len of the L_r cached tokens)
    rope_theta: float = 1e6
    rms_eps: float = 1e-6
    seed: int = 0

    @property
    def batch(self) -> int:
        return len(self.seq_lens)

    @property
    def group(self) -> int:
        return self.num_heads // self.kv_heads

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def kv_tokens(self, step: int = 0) -> int:
        return int(sum(self.seq_lens)) + step * self.batch


def _children(seed: int):
    return np.random.SeedSequence(seed).spawn(5)


# Named workloads.  The length recipes:
#   heavy-tailed:  L = floor(512 * 128**u), u ~ U[0, 1)  (log-uniform in [512, 65536))
#   large-batch:   L integer uniform in [1024, 16384]
CONFIG_NAMES = ("tiny", "uniform", "extreme", "heavy", "fp8")


def config_spec(name: str, seed: int = 0) -> DecodeSpec:
    if name == "tiny":
        return DecodeSpec("tiny", (17, 64, 200, 513), 8, 2, 64, 16, 32, seed=seed)
    if name == "uniform":
        return DecodeSpec("uniform", (4096,) * 32, 64, 8, 128, 64, 128, seed=seed)
    if name == "extreme":
        return DecodeSpec("extreme", (131072,) + (4096,) * 31, 64, 8, 128, 64, 128, seed=seed)
    if name == "heavy":
        rng = np.random.Generator(np.random.PCG64(_children(seed)[0]))
        u = rng.random(64)
        lens = tuple(int(x) for x in np.floor(512.0 * np.power(128.0, u)))
        return DecodeSpec("heavy", lens, 64, 8, 128, 64, 128, steps=8, seed=seed)
    if name == "fp8":
        rng = np.random.Generator(np.random.PCG64(_children(seed)[0]))
        lens = tuple(int(x) for x in rng.integers(1024, 16384, size=256, endpoint=True))
        return DecodeSpec("fp8", lens, 64, 8, 128, 64, 128, kv_dtype="e4m3", prologue=True, seed=seed)
    raise KeyError(f"unknown workload {name!r}; known: {CONFIG_NAMES}")


def custom_spec(seq_lens, num_heads=8, kv_heads=2, head_dim=64, page_size=16, tile_len=32,
                kv_dtype="bf16", steps=1, prologue=False, seed=0, name="custom", q_len=1) -> DecodeSpec:
    return DecodeSpec(name, tuple(int(x) for x in seq_lens), num_heads, kv_heads, head_dim,
                      page_size, tile_len, kv_dtype=kv_dtype, steps=steps, prologue=prologue,
                      seed=seed, q_len=q_len)


@dataclass
class DecodeCase:
    """Host (CPU) tensors of one synthetic decode batch."""

    spec: DecodeSpec
    seq_lens: torch.Tensor  # int32 [B], step-0 lengths
    block_table: torch.Tensor  # int32 [B, max_pages]
    pages_per_req: np.ndarray  # int64 [B]
    k_pages: torch.Tensor  # bf16 or uint8 (E4M3 codes) [num_pages, Hkv, P, D]
    v_pages: torch.Tensor
    q: torch.Tensor | None  # bf16 [B, Hq, D] (None for prologue workloads)
    qkv: torch.Tensor | None  # bf16 [B, Hq + 2 Hkv, D] (prologue workloads)
    k_scale: torch.Tensor | None = None  # fp32 [Hkv] (E4M3 cache)
    v_scale: torch.Tensor | None = None
    q_norm_w: torch.Tensor | None = None  # fp32 [D]
    k_norm_w: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)

    @property
    def num_pages(self) -> int:
        return int(self.k_pages.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])

    def seq_lens_at(self, step: int) -> torch.Tensor:
        return self.seq_lens + int(step)


def _pages_needed(spec: DecodeSpec) -> np.ndarray:
    P = spec.page_size
    cap = np.asarray(spec.seq_lens, dtype=np.int64) + (spec.steps - 1)
    return (cap + P - 1) // P + 1


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _draw_request(stream, shape):
    rng = np.random.Generator(np.random.PCG64(stream))
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    return k, v


def make_case(spec: DecodeSpec, requests=None) -> DecodeCase:
    """Build the batch described by ``spec``.

    ``requests``: optional subset of request indices. When given, the case holds only
    those requests (in that order) and a pool of only their pages. Their contents are
    bit-identical to the same requests of the full batch. This gives bounded samples
    of large workloads without drawing the whole cache.
    """
    B, Hq, Hkv, D, P = spec.batch, spec.num_heads, spec.kv_heads, spec.head_dim, spec.page_size
    assert Hq % Hkv == 0
    ch = _children(spec.seed)
    req_streams = ch[4].spawn(B)
    pages_full = _pages_needed(spec)
    rng = np.random.Generator(np.random.PCG64(ch[1]))
    num_pages_full = int(pages_full.sum())
    perm = rng.permutation(num_pages_full).astype(np.int64)
    offs = np.concatenate([[0], np.cumsum(pages_full)])

    sel = list(range(B)) if requests is None else [int(r) for r in requests]
    pages_sel = pages_full[sel]
    max_pages = int(pages_full.max()) if B else 1
    if requests is None:
        phys = [perm[offs[r]:offs[r + 1]] for r in sel]
        num_pages = num_pages_full
    else:
        # compact pool: keep the relative order of the selected requests' physical pages
        chosen = np.concatenate([perm[offs[r]:offs[r + 1]] for r in sel]) if sel else np.zeros(0, np.int64)
        order = np.argsort(chosen, kind="stable")
        remap = np.empty_like(order)
        remap[order] = np.arange(len(chosen))
        phys, o = [], 0
        for n in pages_sel:
            phys.append(remap[o:o + n])
            o += n
        num_pages = len(chosen)

    block_table = np.full((len(sel), max_pages), -1, dtype=np.int32)
    for i, pp in enumerate(phys):
        block_table[i, :len(pp)] = pp

    shape_of = lambda r: (int(pages_full[r]), Hkv, P, D)
    fp8 = spec.kv_dtype == "e4m3"
    if spec.kv_dtype not in ("bf16", "e4m3"):
        raise ValueError(spec.kv_dtype)

    k_scale = v_scale = None
    if fp8:
        # pass 1: per-kv-head amax over the whole cache (all requests, not only ``sel``)
        def amax(r):
            k, v = _draw_request(req_streams[r], shape_of(r))
            return np.abs(k).max(axis=(0, 2, 3)), np.abs(v).max(axis=(0, 2, 3))
        with ThreadPoolExecutor(_threads()) as ex:
            res = list(ex.map(amax, range(B)))
        ka = np.max(np.stack([a for a, _ in res]), axis=0)
        va = np.max(np.stack([b for _, b in res]), axis=0)
        k_scale = torch.from_numpy((ka / E4M3_MAX).astype(np.float32))
        v_scale = torch.from_numpy((va / E4M3_MAX).astype(np.float32))

    store_dtype = torch.uint8 if fp8 else torch.bfloat16
    k_pages = torch.empty((num_pages, Hkv, P, D), dtype=store_dtype)
    v_pages = torch.empty((num_pages, Hkv, P, D), dtype=store_dtype)

    def fill(i):
        r = sel[i]
        k, v = _draw_request(req_streams[r], shape_of(r))
        idx = torch.from_numpy(np.asarray(phys[i], dtype=np.int64))
        kt, vt = torch.from_numpy(k), torch.from_numpy(v)
        if fp8:
            kt = (kt / k_scale.view(1, Hkv, 1, 1)).clamp(-E4M3_MAX, E4M3_MAX)
            vt = (vt / v_scale.view(1, Hkv, 1, 1)).clamp(-E4M3_MAX, E4M3_MAX)
            kt = kt.to(torch.float8_e4m3fn).view(torch.uint8)
            vt = vt.to(torch.float8_e4m3fn).view(torch.uint8)
        else:
            kt, vt = kt.to(torch.bfloat16), vt.to(torch.bfloat16)
        k_pages[idx] = kt
        v_pages[idx] = vt

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(len(sel))))

    q = qkv = None
    rq = np.random.Generator(np.random.PCG64(ch[2]))
    if spec.q_len == 1:
        qa = rq.standard_normal((B, Hq, D), dtype=np.float32)[sel]
    else:  # [B, q_len, Hq, D]
        qa = rq.standard_normal((B, spec.q_len, Hq, D), dtype=np.float32)[sel]
    rqkv = np.random.Generator(np.random.PCG64(ch[3]))
    qkva = rqkv.standard_normal((B, Hq + 2 * Hkv, D), dtype=np.float32)[sel]
    if spec.prologue:
        qkv = torch.from_numpy(np.ascontiguousarray(qkva)).to(torch.bfloat16)
    else:
        q = torch.from_numpy(np.ascontiguousarray(qa)).to(torch.bfloat16)

    seq = torch.tensor([spec.seq_lens[r] for r in sel], dtype=torch.int32)
    ones = torch.ones(D, dtype=torch.float32)
    sub_spec = spec if requests is None else replace(
        spec, seq_lens=tuple(spec.seq_lens[r] for r in sel), name=spec.name + "[sample]")
    return DecodeCase(sub_spec, seq, torch.from_numpy(block_table), pages_sel.astype(np.int64),
                      k_pages, v_pages, q, qkv, k_scale, v_scale, ones.clone(), ones.clone(),
                      extra={"requests": sel})


def extract_requests(case: DecodeCase, requests) -> DecodeCase:
    """A case holding only ``requests`` of an existing case (copied pages, compact pool)."""
    rows = [int(r) for r in requests]
    bt = case.block_table[rows]
    used = bt[bt >= 0].long()
    remap = torch.full((case.num_pages,), -1, dtype=torch.int32)
    remap[used] = torch.arange(len(used), dtype=torch.int32)
    bt2 = torch.where(bt >= 0, remap[bt.clamp(min=0).long()], bt)
    sel = lambda t: None if t is None else t[rows].clone()
    return DecodeCase(replace(case.spec, seq_lens=tuple(case.spec.seq_lens[r] for r in rows),
                              name=case.spec.name + "[sample]"),
                      case.seq_lens[rows].clone(), bt2.contiguous(), case.pages_per_req[rows],
                      case.k_pages[used].clone(), case.v_pages[used].clone(), sel(case.q), sel(case.qkv),
                      case.k_scale, case.v_scale, case.q_norm_w, case.k_norm_w, extra={"requests": rows})


def random_partials(seed: int, n_items: int, group: int, head_dim: int):
    """Random partial softmax states (m, l, o) for merge tests: m ~ N(0, 4),
    l ~ U[0.5, 50), o ~ N(0, 1) * l.  Returns float32 tensors o [n, grp, D], ml [n, grp, 2]."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    m = rng.normal(0.0, 2.0, size=(n_items, group)).astype(np.float32)
    l = rng.uniform(0.5, 50.0, size=(n_items, group)).astype(np.float32)
    o = (rng.standard_normal((n_items, group, head_dim)).astype(np.float32) * l[..., None])
    ml = np.stack([m, l], axis=-1).astype(np.float32)
    return torch.from_numpy(np.ascontiguousarray(o)), torch.from_numpy(np.ascontiguousarray(ml))


def algorithmic_bytes(spec: DecodeSpec, step: int = 0, out_bytes: int = 4) -> int:
    """Bytes that must move for one decode step: each valid KV element once, q once, the
    output once (plus, for a prologue workload, the qkv read and the new K/V write)."""
    kv_elem = 1 if spec.kv_dtype == "e4m3" else 2
    tokens = spec.kv_tokens(step)
    b = tokens * spec.kv_heads * spec.head_dim * 2 * kv_elem
    b += spec.batch * spec.q_len * spec.num_heads * spec.head_dim * 2  # q (bf16)
    b += spec.batch * spec.q_len * spec.num_heads * spec.head_dim * out_bytes
    if spec.prologue:
        b += spec.batch * (spec.num_heads + 2 * spec.kv_heads) * spec.head_dim * 2
        b += spec.batch * spec.num_heads * spec.head_dim * 2  # q' written (bf16)
        b += 2 * spec.batch * spec.kv_heads * spec.head_dim * kv_elem
    return int(b)
