"""OCP 8-bit floating point, E4M3 variant (test infrastructure; see ``oracle/__init__``).

The format: 1 sign bit, 4 exponent bits (bias 7) and 3 mantissa bits. There are no
infinities. Exponent field 1111 with mantissa 111 is NaN. The largest finite magnitude
is 1.75 * 2^8 = 448 (code 0x7E). Exponent field 0000 encodes subnormals m/8 * 2^-6,
down to 2^-9 (code 0x01).

Cache precision as a variable, and Hy3-FP8, come from "Tencent HPC llega a SGLang …"
(remio.ai, section "Lo que la afirmación de un 48,8 % de TPOT no demuestra") and
"腾讯混元三算子杀入 SGLang" (AREX, opening paragraphs). The pages do not fix the FP8
variant. The reading here is OCP E4M3 with round-to-nearest-even, where finite values
beyond 448 saturate to +-448.
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_to_float(code: int) -> float:
    """Value of one E4M3 code, straight from the field definitions."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return math.nan
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** (-6)
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


# value of every code (NaN for 0x7F / 0xFF)
E4M3_VALUES = np.array([e4m3_to_float(c) for c in range(256)], dtype=np.float64)
# the finite non-negative codes 0x00..0x7E in increasing order of value
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = E4M3_VALUES[:0x7F]


def float_to_e4m3(x: float) -> int:
    """Nearest E4M3 code to x. Ties go to the code with an even mantissa (RNE).
    |x| >= 448 (and +-inf) saturates to +-448; NaN maps to 0x7F."""
    if math.isnan(x):
        return E4M3_NAN
    sign = 0x80 if (x < 0 or (x == 0 and math.copysign(1.0, x) < 0)) else 0
    a = abs(x)
    if a >= E4M3_MAX:
        return sign | 0x7E
    d = np.abs(_POS_VALUES - a)
    best = d.min()
    cands = _POS_CODES[d == best]
    if len(cands) == 1:
        code = int(cands[0])
    else:  # exact midpoint between two neighbours: keep the even mantissa
        code = int([c for c in cands if (c & 1) == 0][0])
    return sign | code


def encode_array(x: np.ndarray) -> np.ndarray:
    """Element-wise ``float_to_e4m3`` over an array (uint8 result)."""
    flat = np.asarray(x, dtype=np.float64).reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    step = 1 << 15
    for s in range(0, flat.size, step):
        v = flat[s:s + step]
        a = np.abs(v)
        d = np.abs(_POS_VALUES[None, :] - a[:, None])  # distance to every finite code
        best = d.min(axis=1, keepdims=True)
        is_best = d == best
        n_best = is_best.sum(axis=1)
        first = np.argmax(is_best, axis=1)
        # two equally near codes: keep the one with an even mantissa
        even = np.where(is_best & ((_POS_CODES[None, :] & 1) == 0), 1, 0).argmax(axis=1)
        code = np.where(n_best > 1, even, first)
        code = np.where(a >= E4M3_MAX, 0x7E, code)
        neg = np.signbit(v)
        code = code | np.where(neg, 0x80, 0)
        code = np.where(np.isnan(v), E4M3_NAN, code)
        out[s:s + step] = code.astype(np.uint8)
    return out.reshape(np.shape(x))


def decode_array(codes: np.ndarray) -> np.ndarray:
    """Element-wise code -> float64 value."""
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8).astype(np.int64)]


def midpoint_distance(x: np.ndarray) -> np.ndarray:
    """Relative distance of |x| from the nearest rounding midpoint between two adjacent
    finite E4M3 values. Tests use it to accept either neighbour when another
    precision could legitimately round the other way."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    mids = (_POS_VALUES[:-1] + _POS_VALUES[1:]) / 2.0
    idx = np.clip(np.searchsorted(mids, a), 1, len(mids) - 1)
    dist = np.minimum(np.abs(a - mids[idx - 1]), np.abs(a - mids[idx]))
    return dist / np.maximum(a, 2.0 ** -10)
