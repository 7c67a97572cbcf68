"""Pins for the 4-bit weight oracle (oracle/fp4.py): the E2M1 and E4M3 element formats
from their bit layouts, rounding ties worked out by hand, a library cast, exhaustive
round trips, and closed forms of the block scales.  CPU only.
"""
import math

import numpy as np
import pytest
import torch

from oracle import fp4 as Q

# the eight E2M1 magnitudes by code 0..7, from the layout: e = 0 subnormal m/2, else
# 2^(e-1) (1 + m/2)
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decodes_every_code():
    for c in range(16):
        v = Q.e2m1_decode(c)
        mag = E2M1_TABLE[c & 7]
        assert abs(v) == mag
        assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)


def test_e2m1_round_trip_of_every_code():
    for c in range(16):
        assert Q.e2m1_encode(Q.e2m1_decode(c)) == c


@pytest.mark.parametrize("v,expect", [
    (0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),   # ties to even m
    (0.26, 0.5), (0.74, 0.5), (1.26, 1.5), (2.51, 3.0), (4.99, 4.0), (5.01, 6.0),
    (6.0, 6.0), (6.9, 6.0), (100.0, 6.0),                                                      # saturation
    (-0.75, -1.0), (-5.0, -4.0), (-7.0, -6.0), (-0.1, -0.0),
])
def test_e2m1_rounding_hand_cases(v, expect):
    got = Q.e2m1_decode(Q.e2m1_encode(v))
    assert got == expect and math.copysign(1.0, got) == math.copysign(1.0, expect)


def test_e2m1_rounds_to_a_nearest_value_and_is_monotone():
    xs = np.linspace(-7.5, 7.5, 6001)
    r = Q.e2m1_round(xs)
    assert (np.diff(r) >= 0).all()
    grid = np.array(sorted(set(E2M1_TABLE + [-v for v in E2M1_TABLE])))
    inside = np.abs(xs) <= 6.0
    nearest = np.abs(grid[None, :] - xs[inside][:, None]).min(axis=1)
    assert np.allclose(np.abs(r[inside] - xs[inside]), nearest, rtol=0, atol=1e-15)


def test_e4m3_matches_the_library_cast_in_range():
    rng = np.random.default_rng(3)
    xs = np.concatenate([
        rng.uniform(-460.0, 460.0, 4000), rng.normal(0, 1e-2, 2000), rng.normal(0, 1e-3, 2000),
        np.ldexp(1.0, np.arange(-12, 9)).astype(np.float64),                  # powers of two, subnormal to 256
        (np.arange(1, 64) * 2.0 ** -10),                                        # subnormal ties and grid
        np.array([448.0, 463.9, -463.9, 1.0625, 1.1875, 0.0]),
    ])
    lib = torch.from_numpy(xs.astype(np.float32)).to(torch.float8_e4m3fn).float().double().numpy()
    ours = np.array([Q.e4m3_round(float(np.float32(x))) for x in xs])
    assert np.array_equal(ours, lib)


def test_e4m3_layout_values_and_saturation():
    assert Q.e4m3_round(448.0) == 448.0                       # exponent 15, mantissa 6 (7 is NaN)
    assert Q.e4m3_round(1e6) == 448.0 and Q.e4m3_round(-1e6) == -448.0
    assert Q.e4m3_round(2.0 ** -9) == 2.0 ** -9               # smallest subnormal
    assert Q.e4m3_round(2.0 ** -10) == 0.0                    # tie with 0: even
    assert Q.e4m3_round(3 * 2.0 ** -10) == 2.0 ** -8          # tie between 1 and 2 subnormal steps: even (2)
    assert Q.e4m3_round(1.0 + 2.0 ** -4) == 1.0               # tie: even mantissa
    assert Q.e4m3_round(1.0 + 3 * 2.0 ** -4) == 1.25


# ---------------------------------------------------------------- MXFP4
def test_mxfp4_scale_closed_forms():
    blk = np.zeros(32)
    for amax, E in [(6.0, 0), (12.0, 1), (7.0, 0), (4.0, 0), (3.99, -1), (1.0, -2), (0.75, -3), (2.0 ** -100, -102)]:
        blk[:] = 0
        blk[5] = amax
        e, codes = Q.mxfp4_block(blk)
        assert e == E, (amax, e)
    assert Q.mxfp4_block(np.zeros(32))[0] == -127
    e, codes = Q.mxfp4_block(np.full(32, 7.0))                 # 7 / 2^0 = 7 saturates to 6
    assert e == 0 and all(Q.e2m1_decode(c) == 6.0 for c in codes)


def test_mxfp4_is_invariant_under_powers_of_two():
    rng = np.random.default_rng(1)
    W = rng.normal(0, 0.02, (8, 64))
    E0, c0 = Q.mxfp4_quantize(W)
    for j in (-5, 3, 20):
        E1, c1 = Q.mxfp4_quantize(W * 2.0 ** j)
        assert np.array_equal(c0, c1) and np.array_equal(E1, E0 + j)
    np.testing.assert_array_equal(Q.mxfp4_dequantize(E0, c0) * 8.0, Q.mxfp4_dequantize(E0 + 3, c0))


def test_mxfp4_error_bound_and_hand_block():
    rng = np.random.default_rng(2)
    W = rng.normal(0, 0.02, (16, 128))
    E, c = Q.mxfp4_quantize(W)
    D = Q.mxfp4_dequantize(E, c)
    X = np.repeat(np.ldexp(1.0, E), 32, axis=1)
    # elements within [-6X, 6X] are off by at most half the widest E2M1 gap (1 X);
    # the saturated ones (|w| in (6X, 8X)) by at most 2X
    err = np.abs(W - D)
    assert (err <= np.where(np.abs(W) <= 6 * X, 1.0, 2.0) * X + 1e-18).all()
    blk = np.array([0.3, -0.7, 1.1, 2.6, -3.4, 5.2, 0.0, 2.2] + [0.0] * 24)
    e, codes = Q.mxfp4_block(blk)                              # amax 5.2 -> E = floor(log2 5.2) - 2 = 0
    assert e == 0
    assert [Q.e2m1_decode(x) for x in codes[:8]] == [0.5, -0.5, 1.0, 3.0, -3.0, 6.0, 0.0, 2.0]


# ---------------------------------------------------------------- NVFP4
def test_nvfp4_scales_closed_forms():
    W = np.zeros((2, 32))
    W[0, 3] = 6.0 * 448.0 * 0.01                               # the tensor amax -> block scale 448
    W[1, 20] = 0.01 * 6.0                                      # block amax 0.06 -> s_b = 0.06/6/0.01 = 1
    s_t, s_b, codes = Q.nvfp4_quantize(W)
    assert float(np.float32(s_t)) == s_t                       # the tensor scale is an fp32 value
    assert s_t == pytest.approx(0.01, rel=1e-7)
    assert s_b[0, 0] == 448.0 and s_b[1, 1] == 1.0
    assert s_b[0, 1] == 0.0 and s_b[1, 0] == 0.0               # all-zero blocks
    D = Q.nvfp4_dequantize(s_t, s_b, codes)
    np.testing.assert_allclose(D, W, rtol=1e-7, atol=0)        # the amax elements: 6 x s_b x s_t, s_t in fp32
    assert Q.nvfp4_quantize(np.zeros((1, 16)))[0] == 1.0


def test_nvfp4_is_invariant_under_powers_of_two_and_bounded():
    rng = np.random.default_rng(4)
    W = rng.normal(0, 0.02, (8, 64))
    s_t, s_b, c = Q.nvfp4_quantize(W)
    s_t2, s_b2, c2 = Q.nvfp4_quantize(W * 2.0 ** -7)
    assert np.array_equal(c, c2) and np.array_equal(s_b, s_b2) and s_t2 == s_t * 2.0 ** -7
    D = Q.nvfp4_dequantize(s_t, s_b, c)
    scale = np.repeat(s_b, 16, axis=1) * s_t
    # s_b is amax/6/s_t rounded in E4M3 (relative error <= 2^-4), so |w| / scale <= 6 (1 + 2^-4) / (1 - 2^-4):
    # at most one E2M1 half gap (1 x scale) plus the part above 6 that saturates
    lim = 6.0 * (1 + 2.0 ** -4) / (1 - 2.0 ** -4)
    assert (np.abs(W) / scale <= lim + 1e-12).all()
    assert (np.abs(W - D) <= scale * (1.0 + (lim - 6.0)) + 1e-18).all()


def test_fake_quantize_formats():
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, (4, 64))
    for fmt in ("mxfp4", "nvfp4"):
        D = Q.fake_quantize(W, fmt)
        assert D.shape == W.shape
        assert np.abs(D - W).max() < 0.5 * np.abs(W).max()
        assert np.array_equal(Q.fake_quantize(D, fmt), D) if fmt == "mxfp4" else True   # MX: idempotent
    with pytest.raises(ValueError):
        Q.fake_quantize(W, "fp8")


def test_e4m3_decode_matches_the_library_float8_on_every_byte():
    import torch
    b = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    ours = np.array([Q.e4m3_decode(int(v)) for v in b])
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan) and int(nan.sum()) == 2          # 0x7f and 0xff
    assert np.array_equal(ours[~nan], lib[~nan])


def test_e4m3_decode_hand_values():
    assert Q.e4m3_decode(0x7E) == 448.0                      # e = 15, m = 6: the largest finite
    assert Q.e4m3_decode(0x38) == 1.0                        # e = 7, m = 0
    assert Q.e4m3_decode(0x01) == 2.0 ** -9                  # the smallest subnormal
    assert Q.e4m3_decode(0x08) == 2.0 ** -6                  # the smallest normal
    assert Q.e4m3_decode(0xB8) == -1.0


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_decode_packed_equals_the_scalar_dequantizers(fmt):
    rng = np.random.default_rng(11)
    W = rng.normal(0, 0.02, (7, 64)) * np.logspace(-3, 3, 7)[:, None]
    if fmt == "mxfp4":
        E, codes = Q.mxfp4_quantize(W)
        want = Q.mxfp4_dequantize(E, codes)
        got = Q.decode_packed(Q.pack_codes(codes), (E + 127).astype(np.uint8), fmt)
    else:
        s_t, s_b, codes = Q.nvfp4_quantize(W)
        want = Q.nvfp4_dequantize(s_t, s_b, codes)
        import torch
        sb_bytes = torch.from_numpy(s_b.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = Q.decode_packed(Q.pack_codes(codes), sb_bytes, fmt, s_t)
    assert np.array_equal(got, want)


def test_decode_packed_hand_example():
    # one MXFP4 row of 64: byte 0x72 = elements (code 2 = 1.0, code 7 = 6.0); scales 2^0, 2^-3
    codes = np.full((1, 32), 0x72, np.uint8)
    scales = np.array([[127, 124]], np.uint8)
    W = Q.decode_packed(codes, scales, "mxfp4")
    assert list(W[0, :4]) == [1.0, 6.0, 1.0, 6.0] and list(W[0, 32:34]) == [0.125, 0.75]
    # sign nibble: 0xA9 = elements (code 9 = -0.5, code 10 = -1.0), NVFP4 scale 0x38 = 1, tensor scale 2
    W = Q.decode_packed(np.full((1, 8), 0xA9, np.uint8), np.full((1, 1), 0x38, np.uint8), "nvfp4", 2.0)
    assert list(W[0, :2]) == [-1.0, -2.0]
