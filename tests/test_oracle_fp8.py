"""Pins for oracle.fp8: values fixed by the OCP OFP8 v1.0 E4M3 definition, and torch's
float8_e4m3fn conversion as an independent library routine."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8 as OF


@pytest.mark.parametrize("x,code", [
    (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (-448.0, 0xFE), (500.0, 0x7E), (math.inf, 0x7E),
    (2.0 ** -9, 0x01), (2.0 ** -6, 0x08), (0.0, 0x00), (-0.0, 0x80), (1.0625, 0x38),  # tie -> even
    (1.1875, 0x3A),  # tie between 0x39 (1.125) and 0x3A (1.25) -> even mantissa 0x3A
    (2.0 ** -10, 0x00),  # tie between 0 and the smallest subnormal -> 0
    (3 * 2.0 ** -10, 0x02),  # tie between 0x01 and 0x02 -> 0x02
    (240.0, 0x77), (256.0, 0x78),
])
def test_spec_values(x, code):
    assert OF.float_to_e4m3(x) == code
    assert OF.encode_array(np.array([x]))[0] == code


def test_nan():
    assert OF.float_to_e4m3(math.nan) == 0x7F
    assert math.isnan(OF.e4m3_to_float(0x7F)) and math.isnan(OF.e4m3_to_float(0xFF))


def test_decode_table_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = OF.E4M3_VALUES
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])
    assert np.nanmax(mine) == 448.0 and OF.e4m3_to_float(0x01) == 2.0 ** -9


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 50, 20000), rng.normal(0, 0.01, 5000),
                        rng.uniform(-447, 447, 5000)]).astype(np.float32).astype(np.float64)
    mine = OF.encode_array(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


def test_roundtrip_is_nearest_brute_force():
    rng = np.random.default_rng(1)
    finite = OF.E4M3_VALUES[~np.isnan(OF.E4M3_VALUES)]
    for x in rng.uniform(-460, 460, 3000):
        y = OF.e4m3_to_float(OF.float_to_e4m3(x))
        if abs(x) >= 448:
            assert y == math.copysign(448.0, x)
        else:
            assert abs(y - x) <= np.min(np.abs(finite - x)) + 0.0


def test_scalar_and_array_agree():
    rng = np.random.default_rng(2)
    x = rng.normal(0, 100, 2000)
    assert np.array_equal(OF.encode_array(x), np.array([OF.float_to_e4m3(v) for v in x], dtype=np.uint8))
