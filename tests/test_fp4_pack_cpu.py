"""The library's host-side FP4 weight packer (moe_quantize_fp4_host /
moe_dequantize_fp4_host) against the FP4 oracle: codes and scales bit for bit,
dequantized values bit for bit after fp32 rounding, the E4M3 scale bytes against the
library float8 type, and the host validation.  CPU only (no device memory is touched).
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import fp4 as Q


@pytest.fixture(scope="module")
def M():
    from routing_dispatch_expert_moe_b200 import build
    build.build()
    from routing_dispatch_expert_moe_b200 import moe
    moe.lib()
    return moe


def _nibbles(codes):
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = codes & 15
    out[:, 1::2] = codes >> 4
    return out


def _weights(kind, rows, K, seed):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        return rng.normal(0, 0.02, (rows, K))
    if kind == "outliers":
        W = rng.normal(0, 0.02, (rows, K))
        W[rng.random((rows, K)) < 0.01] *= 300.0
        return W
    if kind == "zero_rows":
        W = rng.normal(0, 1.0, (rows, K))
        W[::3] = 0.0
        W[:, :16] = 0.0
        return W
    if kind == "wide_range":                    # magnitudes from 1e-30 to 1e30 across rows
        return rng.normal(0, 1.0, (rows, K)) * np.logspace(-30, 30, rows)[:, None]
    if kind == "ties":                          # exact E2M1 midpoints after scaling
        base = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.75, -2.5, -5.0, 0.0, 6.0, 4.0, 3.0, 0.5])
        W = np.tile(base, (rows, K // 16)) * np.ldexp(1.0, rng.integers(-8, 8, (rows, 1)))
        return W
    raise ValueError(kind)


KINDS = ["normal", "outliers", "zero_rows", "wide_range", "ties"]


@pytest.mark.parametrize("kind", KINDS)
def test_mxfp4_pack_matches_the_oracle(M, kind):
    W = _weights(kind, 24, 128, 1).astype(np.float32)
    codes, scales, ts = M.moe_quantize_fp4_host(W, "mxfp4", threads=3)
    E, oc = Q.mxfp4_quantize(W)
    assert ts is None
    assert np.array_equal(scales.astype(np.int32) - 127, E)
    assert np.array_equal(_nibbles(codes), oc)
    D = M.moe_dequantize_fp4_host(codes, scales, None, 128, "mxfp4")
    assert np.array_equal(D, Q.mxfp4_dequantize(E, oc).astype(np.float32))


@pytest.mark.parametrize("kind", KINDS)
def test_nvfp4_pack_matches_the_oracle(M, kind):
    W = _weights(kind, 24, 128, 2).astype(np.float32)
    if kind == "wide_range":                    # one tensor scale cannot span 60 decades: keep 4
        W = _weights("normal", 24, 128, 2).astype(np.float32) * np.logspace(-2, 2, 24)[:, None].astype(np.float32)
    codes, scales, ts = M.moe_quantize_fp4_host(W, "nvfp4", threads=2)
    st, sb, oc = Q.nvfp4_quantize(W)
    assert ts == st
    sb_lib = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).float().double().numpy()
    assert np.array_equal(sb_lib, sb)
    assert np.array_equal(_nibbles(codes), oc)
    D = M.moe_dequantize_fp4_host(codes, scales, ts, 128, "nvfp4")
    assert np.array_equal(D, Q.nvfp4_dequantize(st, sb, oc).astype(np.float32))


def test_e4m3_scale_bytes_decode_like_the_library_float8(M):
    # every positive finite E4M3 byte as a block scale, element code 2 (= 1.0), tensor scale 1
    scale_bytes = np.arange(1, 127, dtype=np.uint8)[:, None]
    codes = np.full((126, 8), 0x22, np.uint8)                  # two elements of 1.0 per byte
    D = M.moe_dequantize_fp4_host(codes, scale_bytes, 1.0, 16, "nvfp4")
    lib = torch.from_numpy(scale_bytes[:, 0].copy()).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(D[:, 0], lib) and (D == D[:, :1]).all()


def test_pack_does_not_depend_on_the_thread_count(M):
    W = _weights("outliers", 37, 256, 3).astype(np.float32)
    for fmt in ("mxfp4", "nvfp4"):
        ref = M.moe_quantize_fp4_host(W, fmt, threads=1)
        for th in (0, 2, 5, 64):
            got = M.moe_quantize_fp4_host(W, fmt, threads=th)
            assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1]) and got[2] == ref[2]


def test_fp4_host_validation(M):
    L = M.lib()
    assert L.moe_fp4_block_size(0) == 32 and L.moe_fp4_block_size(1) == 16 and L.moe_fp4_block_size(2) == -1
    buf = (ctypes.c_uint8 * 4096)()
    f = (ctypes.c_float * 4096)()
    P = ctypes.cast(buf, ctypes.c_void_p)
    F = ctypes.cast(f, ctypes.c_void_p)
    q = L.moe_quantize_fp4_host        # (W, rows, K, fmt, codes, scales, tensor_scale, threads)
    assert q(F, 2, 64, 2, P, P, F, 0) == 1                 # unknown format
    assert q(F, 2, 48, 0, P, P, None, 0) == 2              # K not a multiple of 32
    assert q(F, 2, 48, 1, P, P, F, 0) == 0                 # 48 = 3 NVFP4 blocks
    assert q(F, 2, 64, 1, P, P, None, 0) == 1              # NVFP4 without a tensor scale
    assert q(None, 2, 64, 0, P, P, None, 0) == 1
    assert q(F, -1, 64, 0, P, P, None, 0) == 1
    assert q(F, 2, 64, 0, P, P, None, -1) == 1
    assert q(None, 0, 64, 0, None, None, None, 0) == 0     # nothing to pack
    d = L.moe_dequantize_fp4_host      # (codes, scales, tensor_scale, rows, K, fmt, W, threads)
    assert d(P, P, None, 2, 64, 1, F, 0) == 1
    assert d(P, P, None, 2, 40, 0, F, 0) == 2
    assert d(None, P, None, 2, 64, 0, F, 0) == 1
    assert d(None, None, None, 0, 64, 0, None, 0) == 0


def test_pack_matches_the_oracle_on_random_blocks(M):
    """Randomised: rows of mixed magnitudes, signs, exact zeros and values on E2M1
    midpoints, for both formats."""
    from hypothesis import given, settings, strategies as st
    from hypothesis.extra import numpy as hnp

    vals = st.one_of(st.floats(-1e6, 1e6, width=32), st.sampled_from([0.0, -0.0, 0.25, 0.75, 2.5, 5.0, -3.5]))

    @settings(max_examples=60, deadline=None, derandomize=True)
    @given(hnp.arrays(np.float32, st.tuples(st.integers(1, 6), st.sampled_from([32, 64, 96])), elements=vals))
    def check(W):
        for fmt in ("mxfp4", "nvfp4"):
            codes, scales, ts = M.moe_quantize_fp4_host(W, fmt, threads=2)
            if fmt == "mxfp4":
                E, oc = Q.mxfp4_quantize(W)
                assert np.array_equal(scales.astype(np.int32) - 127, E)
            else:
                st_, sb, oc = Q.nvfp4_quantize(W)
                assert ts == st_
                assert np.array_equal(torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).double().numpy(), sb)
            assert np.array_equal(_nibbles(codes), oc)

    check()
