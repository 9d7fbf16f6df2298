"""Partial softmax states and their log-sum-exp merge, fp64 (test infrastructure).

Splitting one request across CTAs (the uniform tiles of "Tencent HPC llega a SGLang …",
remio.ai, section "Por qué Tencent HPC importa para el serving de modelos en línea")
means each CTA sees only part of the softmax. Each part reports its state:

    m = max_j s_j,   l = sum_j exp(s_j - m),   o = sum_j exp(s_j - m) v_j

over its tokens j, with s_j = scale * q . k_j in natural-log units. The states combine
exactly:

    M = max_i m_i,   L = sum_i exp(m_i - M) l_i,   O = sum_i exp(m_i - M) o_i,

and the output is O / L. The pages do not state the merge. It is the plainest reading
of splitting one softmax, and it is the operation named for the merge kernel.
"""
from __future__ import annotations

import numpy as np


def partial_state(s: np.ndarray, v: np.ndarray):
    """State (m, l, o) of one part: s [n] scaled scores, v [n, D] values; n >= 1."""
    s = np.asarray(s, dtype=np.float64)
    m = s.max()
    w = np.exp(s - m)
    return m, w.sum(), w @ np.asarray(v, dtype=np.float64)


def merge_states(ms, ls, os_):
    """Merge parts i = 0..n-1: ms [n], ls [n], os_ [n, D] -> (M, L, O)."""
    ms = np.asarray(ms, dtype=np.float64)
    ls = np.asarray(ls, dtype=np.float64)
    os_ = np.asarray(os_, dtype=np.float64)
    M = ms.max()
    a = np.exp(ms - M)
    return M, (a * ls).sum(), (a[:, None] * os_).sum(axis=0)


def attend_split(s: np.ndarray, v: np.ndarray, cuts) -> np.ndarray:
    """Output of one head computed as parts [cuts[i], cuts[i+1]) and merged."""
    parts = [partial_state(s[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
    M, L, O = merge_states([p[0] for p in parts], [p[1] for p in parts], [p[2] for p in parts])
    return O / L


def merge_plan_partials(plan, partial_o, partial_ml, batch: int, kv_heads: int, group: int):
    """Reference for the merge step of a whole plan: for every (request, kv head) with
    two or more items, merge its items' partial states (item k's state sits in slot k)
    and return {(r, h): output row}. A (request, kv head) with no item maps to zeros."""
    po = np.asarray(partial_o, dtype=np.float64)
    pml = np.asarray(partial_ml, dtype=np.float64)
    out = {}
    for s in range(batch * kv_heads):
        i0, i1 = int(plan.merge_indptr[s]), int(plan.merge_indptr[s + 1])
        if i1 - i0 == 1:
            continue
        r, kvh = divmod(s, kv_heads)
        for hh in range(group):
            h = kvh * group + hh
            if i1 == i0:
                out[(r, h)] = np.zeros(po.shape[-1])
                continue
            M, L, O = merge_states(pml[i0:i1, hh, 0], pml[i0:i1, hh, 1], po[i0:i1, hh, :])
            out[(r, h)] = O / L
    return out
