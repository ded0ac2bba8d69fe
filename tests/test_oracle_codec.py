"""Pins of the oracle's E4M3 codec and UE8M0 exponent (CPU only).

The codec is judged by things outside the oracle: the OCP landmark table
(tests/golden/e4m3_landmarks.txt), torch's own float8_e4m3fn conversion (a
library routine) on every in-range bf16 value and on the grid's midpoints, and
the closed-form properties of round-to-nearest-even with saturation.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore")


def _decode_all(oracle):
    return np.array([oracle.e4m3_decode(c) for c in range(256)], np.float64)


def test_landmarks_from_ocp_table(oracle_lib):
    for code, val in read_golden("e4m3_landmarks.txt"):
        got = oracle_lib.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got), code
        else:
            assert got == float(val), (code, got, val)


def test_decode_matches_torch_float8_for_all_codes(oracle_lib):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = _decode_all(oracle_lib)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ref[~nan], ours[~nan])
    # exactly two NaN codes, no infinities, symmetric grid
    assert nan.sum() == 2 and not np.isinf(ours).any()
    assert np.array_equal(ours[1:127], -ours[129:255])


def _encode_many(oracle, xs):
    return np.array([oracle.e4m3_encode(float(x)) for x in xs], np.uint8)


def _torch_encode(xs):
    t = torch.tensor(np.asarray(xs, np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_encode_matches_torch_on_every_in_range_bf16(oracle_lib):
    bits = np.arange(65536, dtype=np.uint32) << 16
    vals = bits.view(np.float32)
    ok = np.isfinite(vals) & (np.abs(vals) <= 448.0)
    vals = vals[ok]
    assert np.array_equal(_encode_many(oracle_lib, vals), _torch_encode(vals))


def test_encode_rounds_midpoints_to_even(oracle_lib):
    grid = _decode_all(oracle_lib)
    pos = np.sort(np.unique(grid[(grid >= 0) & np.isfinite(grid)]))
    mids = (pos[:-1] + pos[1:]) / 2.0  # exact in fp32 (4 significant bits + 1)
    for lo, hi, m in zip(pos[:-1], pos[1:], mids):
        m32 = np.float32(m)
        assert float(m32) == m
        c = oracle_lib.e4m3_encode(float(m32))
        # tie -> the neighbour with the even mantissa (even code)
        lo_c, hi_c = oracle_lib.e4m3_encode(lo), oracle_lib.e4m3_encode(hi)
        assert c == (lo_c if lo_c % 2 == 0 else hi_c), (lo, hi, c)
        below = np.nextafter(m32, np.float32(0))
        above = np.nextafter(m32, np.float32(1e9))
        assert oracle_lib.e4m3_encode(float(below)) == lo_c
        assert oracle_lib.e4m3_encode(float(above)) == hi_c
        # the same decisions as torch's conversion
        assert np.array_equal(_encode_many(oracle_lib, [m32, below, above, -m32, -below, -above]),
                              _torch_encode([m32, below, above, -m32, -below, -above]))


def test_encode_saturates_and_keeps_sign_of_zero(oracle_lib):
    for v in (448.0, 449.0, 463.99, 464.0, 480.0, 1e6, 3.0e38, float("inf")):
        assert oracle_lib.e4m3_encode(v) == 0x7E
        assert oracle_lib.e4m3_encode(-v) == 0xFE
    assert oracle_lib.e4m3_encode(0.0) == 0x00
    assert oracle_lib.e4m3_encode(-0.0) == 0x80
    # below half the smallest subnormal -> zero; exactly half -> even (zero)
    assert oracle_lib.e4m3_encode(2.0 ** -10) == 0x00
    assert oracle_lib.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 0x01
    assert oracle_lib.e4m3_encode(1e-30) == 0x00


def test_encode_random_fp32_matches_torch(oracle_lib):
    rng = np.random.default_rng(123)
    mag = np.exp2(rng.uniform(-14, np.log2(448.0), 200000)).astype(np.float32)
    xs = mag * rng.choice([-1, 1], mag.size).astype(np.float32)
    assert np.array_equal(_encode_many(oracle_lib, xs), _torch_encode(xs))


def test_ue8m0_exponent_is_least_power_covering_amax(oracle_lib):
    rng = np.random.default_rng(5)
    vals = np.concatenate([
        np.float32(448.0) * np.exp2(np.arange(-30, 30)).astype(np.float32),       # exact powers
        np.nextafter(np.float32(448.0) * np.exp2(np.arange(-30, 30)).astype(np.float32), np.float32(1e30)),
        np.exp2(rng.uniform(-120, 120, 5000)).astype(np.float32),
    ])
    for a in vals:
        e = oracle_lib.ue8m0_exponent(float(a))
        # closed form: 448 * 2^(e-1) < amax <= 448 * 2^e (exact in float64),
        # except at the clamp e = -127 where only the upper bound holds
        assert math.ldexp(448.0, e) >= float(a), (a, e)
        assert e == -127 or float(a) > math.ldexp(448.0, e - 1), (a, e)
    assert oracle_lib.ue8m0_exponent(0.0) == 0
    assert oracle_lib.ue8m0_exponent(448.0) == 0
    assert oracle_lib.ue8m0_exponent(1.0) == -8
    # clamp at the bottom of the exponent range
    assert oracle_lib.ue8m0_exponent(1e-40) == -127
