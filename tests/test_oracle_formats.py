"""Pins for the oracle's number formats: bf16 and OCP e4m3 against the format
definitions and against torch's own casts (an independent library routine)."""
import numpy as np
import pytest
import torch

from oracle import mla_oracle as O


def test_bf16_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3e-39, -7e-40]])
    x32 = x.astype(np.float32)  # torch casts from fp32; compare on fp32 inputs
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.to_bf16(x32.astype(np.float64)), ref)


def test_f16_matches_torch_cast():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 4, 20000),
                        [0.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2.0 ** -24, 2.0 ** -14, 3e-8]])
    x = x[np.abs(x) < 65504.0]
    ref = torch.from_numpy(x).to(torch.float16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.to_f16(x), ref)


def test_generic_rounding_at_fp32_matches_ieee_cast():
    # the same rounding routine at fp32's parameters (24-bit significand,
    # emin -126, gradual underflow) against the IEEE float32 conversion,
    # over normal and subnormal binades
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-44, 38, 20000),
                        [0.0, 1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 2.0 ** -149, 1.5 * 2.0 ** -149, 2.0 ** -126]])
    np.testing.assert_array_equal(O.round_to_format(x, 24, -126), x.astype(np.float32).astype(np.float64))


def test_bf16_ties_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even significand (1.0)
    assert O.to_bf16(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3*2^-8 lies halfway between 1+2^-7 and 1+2^-6: goes to 1+2^-6 (even)
    assert O.to_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x39, 1.125), (0x3F, 1.875), (0x40, 2.0), (0x7E, 448.0),
    (0xB8, -1.0), (0xFE, -448.0), (0x80, -0.0)])
def test_e4m3_decode_spec_values(code, value):
    assert O.e4m3_decode(np.uint8(code)) == value


def test_e4m3_nan_codes():
    assert np.isnan(O.e4m3_decode(np.uint8(0x7F)))
    assert np.isnan(O.e4m3_decode(np.uint8(0xFF)))


def test_e4m3_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(50000) * 2.0 ** rng.integers(-12, 9, 50000),
                        rng.uniform(-448, 448, 5000),
                        # exact midpoints between neighbouring codes (ties to even)
                        (O._E4M3_POS[1:] + O._E4M3_POS[:-1]) / 2,
                        -(O._E4M3_POS[1:] + O._E4M3_POS[:-1]) / 2])
    x32 = x.astype(np.float32)
    x32 = x32[np.abs(x32) <= 448]  # torch's cast does not saturate; saturation is pinned below
    ref = torch.from_numpy(x32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x32.astype(np.float64)), ref)


def test_e4m3_saturates():
    np.testing.assert_array_equal(O.e4m3_encode(np.array([449.0, 1e9, -500.0])),
                                  np.array([0x7E, 0x7E, 0xFE], dtype=np.uint8))


def test_e4m3_ties():
    # 1.0625 is halfway between 1.0 (m=0) and 1.125 (m=1) -> 1.0 ; 1.1875 -> 1.25 (m=2)
    assert O.e4m3_encode(1.0625) == 0x38
    assert O.e4m3_encode(1.1875) == 0x3A


def test_fp8_tile_quantiser_properties():
    rng = np.random.default_rng(2)
    c = rng.standard_normal((64, 512)) * 3
    c[5, 128:256] = 0.0  # an all-zero tile
    codes, scales = O.fp8_quantise_latent(c)
    assert codes.shape == (64, 512) and scales.shape == (64, 4) and scales.dtype == np.float32
    assert scales[5, 1] == 1.0 and np.all(codes[5, 128:256] == 0)
    # the element of largest magnitude of each tile maps to +-448 exactly
    t = c.astype(np.float32).reshape(64, 4, 128)
    arg = np.abs(t).argmax(-1)
    top = np.take_along_axis(codes.reshape(64, 4, 128), arg[..., None], -1)[..., 0]
    nz = np.abs(t).max(-1) > 0
    assert np.all(np.isin(top[nz], [0x7E, 0xFE]))
    # relative error of normal values within half an e4m3 ulp (2^-4)
    deq = O.fp8_dequantise_latent(codes, scales)
    q = np.abs(c.astype(np.float32).reshape(64, 4, 128) / scales[..., None]).reshape(64, 512)
    normal = q >= 2.0 ** -6
    rel = np.abs(deq - c.astype(np.float32))[normal] / np.abs(c.astype(np.float32))[normal]
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)
