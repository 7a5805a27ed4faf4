"""Pins for the oracle's number-format codecs against independent library codecs.

ml_dtypes and torch implement the OCP E4M3 / E2M1 / E8M0 and bf16 formats on
their own; every code is decoded and compared, and the encoders are compared on
random values, all representable values and all midpoints (ties).
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F


def test_e4m3_decode_every_code_matches_libraries():
    codes = np.arange(256, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    tor = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.E4M3_TABLE
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan) and np.array_equal(np.isnan(tor), nan)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], lib[~nan])
    assert np.array_equal(ours[~nan], tor[~nan])
    # sign of zero
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_decode_rejects_nan_codes():
    with pytest.raises(ValueError):
        F.decode_e4m3([0x10, 0x7F])
    with pytest.raises(ValueError):
        F.decode_e4m3([0xFF])


def test_e2m1_decode_every_code_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(F.E2M1_TABLE, lib)
    assert np.array_equal(np.signbit(F.E2M1_TABLE), np.signbit(lib))


def test_e2m1_packing_low_nibble_is_even_element():
    # codes 1 (0.5) and 7 (6.0): byte 0x71 -> [0.5, 6.0]; 0x17 -> [6.0, 0.5]
    assert F.unpack_e2m1(np.array([0x71, 0x17], dtype=np.uint8)).tolist() == [0.5, 6.0, 6.0, 0.5]
    rng = np.random.default_rng(5)
    elems = rng.integers(0, 16, size=(3, 64), dtype=np.uint8)
    packed = (elems[:, 0::2] | (elems[:, 1::2] << 4)).astype(np.uint8)
    ref = elems.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(F.unpack_e2m1(packed), ref)


def test_ue8m0_decode_every_code_matches_ml_dtypes():
    codes = np.arange(255, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert np.array_equal(F.decode_ue8m0(codes), lib)
    assert F.decode_ue8m0([127])[0] == 1.0
    with pytest.raises(ValueError):
        F.decode_ue8m0([255])


def test_mxfp4_dequant_applies_block_scale_per_32():
    packed = np.full((1, 32), 0x22, dtype=np.uint8)        # every element 1.0
    scales = np.array([[127, 128]], dtype=np.uint8)         # 1, 2
    v = F.dequant_mxfp4(packed, scales)
    assert v.shape == (1, 64)
    assert np.all(v[0, :32] == 1.0) and np.all(v[0, 32:] == 2.0)


def _e4m3_ml(values):
    return np.asarray(values, dtype=np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def test_e4m3_encode_matches_ml_dtypes_on_grid_midpoints_and_random():
    pos = F.E4M3_TABLE[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2            # exact in fp32: ties
    rng = np.random.default_rng(0)
    rnd = np.concatenate([rng.normal(0, 1, 20000) * s for s in (1e-3, 0.1, 1, 30, 200)])
    rnd = rnd[np.abs(rnd) < 448].astype(np.float32).astype(np.float64)
    vals = np.concatenate([pos, mids, -pos, -mids, rnd, [0.0, -0.0, 1e-30, -1e-30, 2.0 ** -10, 3 * 2.0 ** -11]])
    got = F.encode_e4m3(vals)
    exp = _e4m3_ml(vals)
    bad = np.nonzero(got != exp)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], exp[bad[:5]])
    # the same against torch's cast
    tor = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, tor)


def test_e4m3_encode_saturates_and_keeps_zero_sign():
    assert F.encode_e4m3([448.0, 449.0, 464.0, 500.0, 1e30]).tolist() == [0x7E] * 5
    assert F.encode_e4m3([-448.0, -1e9]).tolist() == [0xFE, 0xFE]
    assert F.encode_e4m3([-0.0, -1e-12, 0.0]).tolist() == [0x80, 0x80, 0x00]
    # tie between 0 and the smallest subnormal goes to the even code (zero)
    assert F.encode_e4m3([2.0 ** -10]).tolist() == [0x00]


def test_bf16_encode_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 1, 50000), rng.normal(0, 1e-38, 1000), [0.0, -0.0, 1.0, -3.5]])
    v = v.astype(np.float32)
    # exact midpoints between neighbouring bf16 values (ties)
    b = rng.integers(0, 0x7F00, 2000, dtype=np.uint32) << 16
    mids = (b | 0x8000).view(np.float32)
    v = np.concatenate([v, mids, -mids])
    got = F.f64_to_bf16(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    assert np.array_equal(F.bf16_to_f64(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_encode_rounds_once_from_float64():
    # 1 + 2^-8 + 2^-30 lies above the midpoint of 1 and 1 + 2^-7: one rounding
    # gives 1 + 2^-7 (0x3F81); rounding through fp32 first would give 1.0.
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert F.f64_to_bf16([v]).tolist() == [0x3F81]
    assert F.f64_to_bf16([1.0 + 2.0 ** -8]).tolist() == [0x3F80]       # tie -> even
    assert F.f64_to_bf16([1.0 + 3 * 2.0 ** -8]).tolist() == [0x3F82]   # tie -> even (up)


@pytest.mark.parametrize("q", [-20, -7, -1, 0, 3, 40])
def test_pow2_exponent_closed_forms(q):
    s = 2.0 ** q
    assert F.pow2_exponent([448 * s])[0] == q                     # exactly at the bound
    assert F.pow2_exponent([448 * s * (1 + 2.0 ** -52)])[0] == q + 1
    assert F.pow2_exponent([448 * s * (1 - 2.0 ** -53)])[0] == q
    assert F.pow2_exponent([224 * s])[0] == q - 1
    assert F.pow2_exponent([224 * s * (1 + 2.0 ** -52)])[0] == q


def test_pow2_exponent_invariant_and_special_cases():
    rng = np.random.default_rng(2)
    a = np.abs(rng.normal(0, 1, 10000)) * 10.0 ** rng.uniform(-20, 20, 10000)
    p = F.pow2_exponent(a)
    r = a / np.ldexp(1.0, p)
    assert np.all(r <= 448) and np.all(r > 224)
    assert F.pow2_exponent([0.0])[0] == 0
    assert F.pow2_exponent([2.0 ** -140])[0] == -126               # clamp keeps 2^p normal
    assert math.isfinite(np.ldexp(1.0, F.pow2_exponent([3e38])[0]))
