"""CPU oracle for 4-bit expert weights: the FP4 (E2M1) element format, the MXFP4 and
NVFP4 block-scaled encodings, and the expert FFN on dequantized weights.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline / reference arm may import this module.  It imports nothing
from the library.  Plain Python and numpy in float64, meant to be read by eye.

Sources (cited by title and section):
  [Handbook-Digest] "Hugging Face 发布 3 万词免费 MoE 训练手册" (agihunt.info), "已确认",
                    bullet "量化与推理": Kimi K3 quantizes its routed experts to MXFP4;
                    NVIDIA trains Nemotron 3 with NVFP4 and keeps key layers in BF16.
The pages name the formats only.  Readings taken (listed again in the design notes):
  R24 MXFP4 is the Open Compute Project microscaling format: blocks of 32 elements in
      FP4 E2M1 sharing one power-of-two scale (E8M0).  The scale exponent is
      floor(log2(amax)) - 2 (2 = the largest E2M1 exponent), each element is rounded to
      nearest-even in E2M1 after division by the scale, and magnitudes beyond 6
      saturate to 6.  An all-zero block takes the smallest scale, 2^-127.
  R25 NVFP4: blocks of 16 elements in E2M1, one FP8 E4M3 scale per block and one fp32
      scale per tensor: s_t = amax(tensor) / (6 * 448), s_b = E4M3(amax(block) / 6 / s_t)
      rounded to nearest-even (saturating at 448), elements E2M1(x / (s_b s_t)).  A
      block whose scale rounds to 0 is all zeros; an all-zero tensor takes s_t = 1.
  R26 the experts run on the dequantized weights (value = element x scales); the router,
      the shared expert and the activations stay as they are ("key layers in BF16").
Parity status: every function here is pinned by tests/test_oracle_fp4.py.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# FP4 E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; no infinity or NaN.
# ---------------------------------------------------------------------------
E2M1_MAX = 6.0


def e2m1_decode(code: int) -> float:
    """Value of a 4-bit code s|e e|m: subnormal (e = 0) m/2, normal 2^(e-1) (1 + m/2)."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m * 0.5)
    return -mag if s else mag


def e2m1_encode(v: float) -> int:
    """Nearest E2M1 code, ties to the even mantissa bit, magnitudes above 6 saturating."""
    s = 1 if (v < 0 or (v == 0 and math.copysign(1.0, v) < 0)) else 0
    a = min(abs(float(v)), E2M1_MAX)
    best, best_err = 0, math.inf
    for c in range(8):                          # the eight magnitudes, ascending
        err = abs(e2m1_decode(c) - a)
        if err < best_err or (err == best_err and (c & 1) == 0):
            best, best_err = c, err
    return (s << 3) | best


def e2m1_round(v):
    """Elementwise E2M1 rounding of an array (values, float64)."""
    v = np.asarray(v, np.float64)
    out = np.empty_like(v)
    for i, x in np.ndenumerate(v):
        out[i] = e2m1_decode(e2m1_encode(float(x)))
    return out


# ---------------------------------------------------------------------------
# FP8 E4M3 (the NVFP4 block scale): sign, 4 exponent bits (bias 7), 3 mantissa bits;
# largest finite 448 (exponent 15 with mantissa 7 is NaN); smallest subnormal 2^-9.
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_round(v: float) -> float:
    """Nearest E4M3 value, ties to the even mantissa, magnitudes above 448 saturating."""
    x = float(v)
    a = abs(x)
    if a == 0.0:
        return x
    if a >= E4M3_MAX:
        return math.copysign(E4M3_MAX, x)
    e = max(math.frexp(a)[1] - 1, -6)           # binade floor(log2 a); subnormals share 2^-6's spacing
    step = 2.0 ** (e - 3)                       # 3 mantissa bits
    q = a / step
    r = math.floor(q)
    frac = q - r
    if frac > 0.5 or (frac == 0.5 and r % 2 == 1):
        r += 1
    return math.copysign(min(r * step, E4M3_MAX), x)


# ---------------------------------------------------------------------------
# MXFP4 (R24)
# ---------------------------------------------------------------------------
MX_BLOCK = 32


def mxfp4_block(v) -> tuple:
    """One block: (scale exponent E, element codes); value_i = 2^E * e2m1(code_i)."""
    v = np.asarray(v, np.float64)
    amax = float(np.abs(v).max()) if v.size else 0.0
    if amax == 0.0:
        E = -127
    else:
        E = max(-127, min(127, (math.frexp(amax)[1] - 1) - 2))     # floor(log2 amax) - 2
    X = 2.0 ** E
    return E, [e2m1_encode(float(x) / X) for x in v]


def mxfp4_quantize(W, block: int = MX_BLOCK) -> tuple:
    """W [rows, K] (K a multiple of block): scale exponents [rows, K/block], codes [rows, K]."""
    W = np.asarray(W, np.float64)
    rows, K = W.shape
    if K % block:
        raise ValueError("K must be a multiple of the block size")
    E = np.empty((rows, K // block), np.int32)
    codes = np.empty((rows, K), np.uint8)
    for r in range(rows):
        for b in range(K // block):
            e, c = mxfp4_block(W[r, b * block:(b + 1) * block])
            E[r, b] = e
            codes[r, b * block:(b + 1) * block] = c
    return E, codes


def mxfp4_dequantize(E, codes, block: int = MX_BLOCK) -> np.ndarray:
    codes = np.asarray(codes)
    out = np.empty(codes.shape, np.float64)
    for (r, k), c in np.ndenumerate(codes):
        out[r, k] = math.ldexp(e2m1_decode(int(c)), int(E[r, k // block]))
    return out


# ---------------------------------------------------------------------------
# NVFP4 (R25)
# ---------------------------------------------------------------------------
NV_BLOCK = 16


def nvfp4_quantize(W, block: int = NV_BLOCK) -> tuple:
    """W [rows, K]: tensor scale s_t, block scales s_b [rows, K/block] (E4M3 values),
    element codes [rows, K]."""
    W = np.asarray(W, np.float64)
    rows, K = W.shape
    if K % block:
        raise ValueError("K must be a multiple of the block size")
    amax = float(np.abs(W).max()) if W.size else 0.0
    s_t = float(np.float32(amax / (E2M1_MAX * E4M3_MAX))) if amax > 0 else 1.0   # an fp32 scale (R25)
    s_b = np.empty((rows, K // block), np.float64)
    codes = np.empty((rows, K), np.uint8)
    for r in range(rows):
        for b in range(K // block):
            blk = W[r, b * block:(b + 1) * block]
            sb = e4m3_round(float(np.abs(blk).max()) / E2M1_MAX / s_t)
            s_b[r, b] = sb
            if sb == 0.0:
                codes[r, b * block:(b + 1) * block] = 0
            else:
                codes[r, b * block:(b + 1) * block] = [e2m1_encode(float(x) / (sb * s_t)) for x in blk]
    return s_t, s_b, codes


def nvfp4_dequantize(s_t: float, s_b, codes, block: int = NV_BLOCK) -> np.ndarray:
    codes = np.asarray(codes)
    out = np.empty(codes.shape, np.float64)
    for (r, k), c in np.ndenumerate(codes):
        out[r, k] = e2m1_decode(int(c)) * float(s_b[r, k // block]) * s_t
    return out


# ---------------------------------------------------------------------------
# The packed layout (what a 4-bit expert GEMM reads): codes [rows, K/2] bytes with element
# 2j in the low nibble of byte j; scale bytes [rows, K/block]: E8M0 (MXFP4, the byte E + 127)
# or FP8 E4M3 (NVFP4); and, for NVFP4, one fp32 tensor scale.
# ---------------------------------------------------------------------------
def e4m3_decode(byte: int) -> float:
    """Value of an FP8 E4M3 byte s|eeee|mmm: normal (e > 0) 2^(e-7) (1 + m/8), subnormal
    (e = 0) m 2^-9; exponent 15 with mantissa 7 is NaN (never written by the quantizer)."""
    s, e, m = (byte >> 7) & 1, (byte >> 3) & 15, byte & 7
    if e == 15 and m == 7:
        return math.nan
    mag = m * 2.0 ** -9 if e == 0 else 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return -mag if s else mag


def pack_codes(codes) -> np.ndarray:
    """Element codes [rows, K] -> bytes [rows, K/2], element 2j in the low nibble of byte j."""
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def decode_packed(codes, scales, fmt: str, tensor_scale: float = 1.0) -> np.ndarray:
    """Dequantized weights [rows, K] (float64) of the packed layout: code value x block
    scale (x tensor scale for NVFP4).  Table-driven: the 16 code values from e2m1_decode and
    the 256 scale values from their byte layouts."""
    codes = np.asarray(codes, np.uint8)
    scales = np.asarray(scales, np.uint8)
    rows, half = codes.shape
    K = 2 * half
    block = MX_BLOCK if fmt == "mxfp4" else NV_BLOCK
    if scales.shape != (rows, K // block):
        raise ValueError("scales must be [rows, K / block]")
    vals = np.array([e2m1_decode(c) for c in range(16)], np.float64)
    if fmt == "mxfp4":
        svals = np.array([2.0 ** (b - 127) for b in range(256)], np.float64)
    elif fmt == "nvfp4":
        svals = np.array([e4m3_decode(b) for b in range(256)], np.float64)
    else:
        raise ValueError(fmt)
    el = np.empty((rows, K), np.uint8)
    el[:, 0::2] = codes & 15
    el[:, 1::2] = codes >> 4
    W = vals[el] * np.repeat(svals[scales], block, axis=1)
    return W * (float(tensor_scale) if fmt == "nvfp4" else 1.0)


def fake_quantize(W, fmt: str) -> np.ndarray:
    """W -> its dequantized 4-bit form ("mxfp4" or "nvfp4"), the weights the experts run on (R26)."""
    if fmt == "mxfp4":
        return mxfp4_dequantize(*mxfp4_quantize(W))
    if fmt == "nvfp4":
        return nvfp4_dequantize(*nvfp4_quantize(W))
    raise ValueError(fmt)
