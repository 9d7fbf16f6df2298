"""Pins for oracle.prologue: closed forms of RMSNorm and RoPE, a complex-number form of
the rotation, angle recovery by atan2, the write location, and bf16 rounding against
torch."""
import math

import numpy as np
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
