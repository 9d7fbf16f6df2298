"""Pins for oracle.prologue: closed forms of RMSNorm and RoPE, a complex-number form of
the rotation, angle recovery by atan2, the write location, and bf16 rounding against
torch."""
import math

import numpy as np
import pytest
import torch

from load_balanced_split_step_b200 import workloads as W
from oracle import fp8 as OF
from oracle import prologue as OR


def test_rope_position_zero_is_identity():
    x = np.random.default_rng(0).normal(size=(3, 128))
    assert np.array_equal(OR.rope_neox(x, 0, 1e6), x)


def test_rope_preserves_norm_and_matches_complex_rotation():
    rng = np.random.default_rng(1)
    x = rng.normal(size=128)
    for pos in (1, 17, 16383, 131071):
        y = OR.rope_neox(x, pos, 1e6)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-12 * np.linalg.norm(x)
        z = (x[:64] + 1j * x[64:]) * np.exp(1j * pos * 1e6 ** (-np.arange(64) / 64.0))
        assert np.max(np.abs(y - np.concatenate([z.real, z.imag]))) <= 1e-12


def test_rope_angle_by_atan2():
    rng = np.random.default_rng(2)
    x = rng.normal(size=64)
    pos, theta = 777, 1e4
    y = OR.rope_neox(x, pos, theta)
    for i in range(32):
        got = math.atan2(y[i + 32], y[i]) - math.atan2(x[i + 32], x[i])
        want = pos * theta ** (-2.0 * i / 64)
        d = (got - want + math.pi) % (2 * math.pi) - math.pi
        assert abs(d) <= 1e-9


def test_rmsnorm_closed_form():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(5, 128)) * 3.0
    eps = 1e-6
    y = OR.rms_norm(x, np.ones(128), eps)
    ms = np.mean(x * x, axis=-1)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0 / np.sqrt(1.0 + eps / ms), rtol=0, atol=1e-14)
    w = rng.normal(size=128)
    assert np.allclose(OR.rms_norm(x, w, eps), y * w, rtol=0, atol=1e-13)


def test_prologue_writes_new_token_slot():
    spec = W.custom_spec((5, 16, 33), 8, 2, 64, 16, 32, kv_dtype="e4m3", prologue=True, seed=4)
    case = W.make_case(spec)
    kp = case.k_pages.numpy().copy()
    vp = case.v_pages.numpy().copy()
    q, k_new, v_new, writes = OR.decode_prologue(
        case.qkv, case.q_norm_w, case.k_norm_w, 1e-6, 1e6, case.seq_lens.numpy(),
        case.block_table.numpy(), kp, vp, "e4m3", case.k_scale, case.v_scale, 8, 2)
    for (r, page, slot), L in zip(writes, (5, 16, 33)):
        assert page == int(case.block_table[r, (L - 1) // 16]) and slot == (L - 1) % 16
        for g in range(2):
            assert np.array_equal(kp[page, g, slot], OF.encode_array(k_new[r, g]))
    changed = np.argwhere(np.any(kp != case.k_pages.numpy(), axis=-1))
    assert {(int(a), int(c)) for a, _, c in changed} <= {(p, s) for _, p, s in writes}
    # q after the prologue: unit-norm-per-rms rows rotated -> rms stays 1/sqrt(1 + eps/ms)
    x = case.qkv.to(torch.float64).numpy()
    for r, L in enumerate((5, 16, 33)):
        ref = OR.rope_neox(OR.rms_norm(x[r, :8], np.ones(64), 1e-6), L - 1, 1e6)
        assert np.max(np.abs(q[r] - ref)) == 0.0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-3, 1000), rng.normal(0, 1e4, 1000)])
    x32 = x.astype(np.float32).astype(np.float64)  # exactly representable in fp32
    mine = OR.bf16_bits(x32)
    ref = torch.from_numpy(x32.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


# ---- the K/V write, decoded and compared with an independent computation ------------------
#
# Readings 13-15 of the path's spec (and "vLLM × HPC-Ops" summary: RoPE + QK-Norm + KV-write):
# the stored K is rope(rmsnorm(k)) and the stored V is the raw v, each divided by its kv head's
# scale and rounded to the nearest E4M3 value. Decoding a stored code and multiplying by the
# scale must therefore land within half an E4M3 step (times the scale) of the value computed
# here, which shares no code with the oracle: the rotation is written as a complex product and
# the norm from its definition. The checker must reject pages written with planted mistakes:
# k multiplied by the scale instead of divided, RoPE applied to V, RMSNorm applied to V.

def _e4m3_half_step(x):
    """Half the spacing of the E4M3 grid at |x| (|x| <= 448), from the format: 3 mantissa bits,
    normal numbers from 2^-6 (spacing 2^(e-3) in [2^e, 2^(e+1))), subnormals spaced 2^-9."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 0.5 * np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))


def _independent_new_token(qkv, q_norm_w, k_norm_w, eps, theta, seq_lens, Hq, Hkv):
    """(k, v) of every request's new token: k = rope(rmsnorm(k)) via a complex rotation, v raw."""
    x = qkv.to(torch.float64).numpy()
    D = x.shape[-1]
    wk = k_norm_w.to(torch.float64).numpy()
    ks, vs = [], []
    for r, L in enumerate(seq_lens):
        pos = int(L) - 1
        kr, vr = [], []
        for g in range(Hkv):
            k = x[r, Hq + g]
            k = k / math.sqrt(float(np.dot(k, k)) / D + eps) * wk
            z = (k[:D // 2] + 1j * k[D // 2:]) * np.exp(1j * pos * theta ** (-np.arange(D // 2) * 2.0 / D))
            kr.append(np.concatenate([z.real, z.imag]))
            vr.append(x[r, Hq + Hkv + g])
        ks.append(kr)
        vs.append(vr)
    return np.array(ks), np.array(vs)


def _kv_write_errors(kp, vp, case, k_ref, v_ref, Hkv):
    """Largest |decoded - expected| / allowed over the written K and V slots (<= 1 passes)."""
    P = kp.shape[2]
    ks = case.k_scale.to(torch.float64).numpy()
    vs = case.v_scale.to(torch.float64).numpy()
    worst = 0.0
    for r, L in enumerate(case.seq_lens.tolist()):
        pos = L - 1
        page, slot = int(case.block_table[r, pos // P]), pos % P
        for g in range(Hkv):
            for pages, ref, sc in ((kp, k_ref, ks), (vp, v_ref, vs)):
                got = OF.E4M3_VALUES[pages[page, g, slot].astype(np.int64)] * sc[g]
                want = np.clip(ref[r, g] / sc[g], -448.0, 448.0)
                allowed = _e4m3_half_step(want) * sc[g] * (1 + 1e-9)
                worst = max(worst, float(np.max(np.abs(got - want * sc[g]) / allowed)))
    return worst


def _e4m3_case(weights):
    spec = W.custom_spec((5, 16, 33, 70), 16, 2, 128, 16, 32, kv_dtype="e4m3", prologue=True, seed=9)
    case = W.make_case(spec)
    if weights:
        rng = np.random.default_rng(11)
        case.q_norm_w = torch.from_numpy(rng.uniform(0.5, 1.5, 128).astype(np.float32))
        case.k_norm_w = torch.from_numpy(rng.uniform(0.5, 1.5, 128).astype(np.float32))
    return spec, case


def _run_oracle(case, qkv=None, k_scale=None):
    kp, vp = case.k_pages.numpy().copy(), case.v_pages.numpy().copy()
    OR.decode_prologue(case.qkv if qkv is None else qkv, case.q_norm_w, case.k_norm_w, 1e-6, 1e6,
                       case.seq_lens.numpy(), case.block_table.numpy(), kp, vp, "e4m3",
                       case.k_scale if k_scale is None else k_scale, case.v_scale, 16, 2)
    return kp, vp


@pytest.mark.parametrize("weights", [False, True])
def test_e4m3_kv_write_decodes_to_independent_values(weights):
    _, case = _e4m3_case(weights)
    k_ref, v_ref = _independent_new_token(case.qkv, case.q_norm_w, case.k_norm_w, 1e-6, 1e6,
                                          case.seq_lens.tolist(), 16, 2)
    kp, vp = _run_oracle(case)
    assert _kv_write_errors(kp, vp, case, k_ref, v_ref, 2) <= 1.0


def test_e4m3_kv_write_checker_catches_planted_mistakes():
    _, case = _e4m3_case(False)
    k_ref, v_ref = _independent_new_token(case.qkv, case.q_norm_w, case.k_norm_w, 1e-6, 1e6,
                                          case.seq_lens.tolist(), 16, 2)
    # k * k_scale instead of k / k_scale: the oracle given 1 / k_scale writes exactly that
    kp, vp = _run_oracle(case, k_scale=1.0 / case.k_scale)
    assert _kv_write_errors(kp, vp, case, k_ref, v_ref, 2) > 1.0
    # RoPE (or RMSNorm) applied to V as well: the oracle given a rotated / normalised v writes that
    x = case.qkv.to(torch.float64).numpy().copy()
    L = case.seq_lens.tolist()
    for mistake in ("rope", "norm"):
        y = x.copy()
        for r in range(len(L)):
            for g in range(2):
                v = x[r, 18 + g]
                y[r, 18 + g] = OR.rope_neox(v, L[r] - 1, 1e6) if mistake == "rope" else OR.rms_norm(v, np.ones(128),
                                                                                                   1e-6)
        kp, vp = _run_oracle(case, qkv=torch.from_numpy(y))
        assert _kv_write_errors(kp, vp, case, k_ref, v_ref, 2) > 1.0, mistake


def test_bf16_kv_write_is_the_rounded_independent_value():
    spec = W.custom_spec((3, 40, 77), 8, 2, 64, 16, 32, prologue=True, seed=12)
    case = W.make_case(spec)
    kp = case.k_pages.view(torch.int16).numpy().view(np.uint16).copy()
    vp = case.v_pages.view(torch.int16).numpy().view(np.uint16).copy()
    OR.decode_prologue(case.qkv, case.q_norm_w, case.k_norm_w, 1e-6, 1e6, case.seq_lens.numpy(),
                       case.block_table.numpy(), kp, vp, "bf16", None, None, 8, 2)
    k_ref, v_ref = _independent_new_token(case.qkv, case.q_norm_w, case.k_norm_w, 1e-6, 1e6,
                                          case.seq_lens.tolist(), 8, 2)
    for r, L in enumerate(case.seq_lens.tolist()):
        page, slot = int(case.block_table[r, (L - 1) // 16]), (L - 1) % 16
        for g in range(2):
            got_k = torch.from_numpy(kp[page, g, slot].view(np.int16)).view(torch.bfloat16).double().numpy()
            got_v = torch.from_numpy(vp[page, g, slot].view(np.int16)).view(torch.bfloat16).double().numpy()
            # bf16 keeps 8 significant bits: within half a unit in the last place, 2^(e - 8) for
            # |x| in [2^e, 2^(e+1))
            half_ulp = 2.0 ** (np.floor(np.log2(np.abs(k_ref[r, g]))) - 8)
            assert np.all(np.abs(got_k - k_ref[r, g]) <= half_ulp)
            assert np.array_equal(got_v, v_ref[r, g])  # v is bf16 already: stored exactly
