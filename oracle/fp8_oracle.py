"""Plain CPU oracle of the 8-bit (e4m3) GEMM path: per-tensor quantisation and the product.

TEST INFRASTRUCTURE ONLY.  Only the tests may import this module.  It shares no code with the CUDA
path and nothing in the product calls it.

The pages name FP8 matrix products for the d24 speedrun ("supa beginna nanochat", the 8×H100
speedrun) and for "alpha-nanochat-d24" (The run) but give no format details; the reading taken
here is the OCP 8-bit float E4M3 ("e4m3fn") with one scale per tensor:
  * E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no infinities, NaN = S.1111.111,
    largest finite 448 = 1.75·2^8, smallest normal 2^-6, subnormals m·2^-9 (m = 1..7);
  * a value is rounded to the nearest representable one, ties to the even mantissa, and values
    beyond ±448 saturate to ±448 ("satfinite");
  * per tensor: amax = max|x|, scale = 448/amax (1 when amax = 0), q = e4m3(x·scale) with the
    product formed in float32, dq = amax/448 (float32) so that x ≈ q·dq;
  * the product C = alpha·dq_a·dq_b·(A·Bᵀ) over the decoded codes, exactly (float64).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
MIN_NORMAL_EXP = -6
MANT_BITS = 3
BIAS = 7


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Values (float64) of uint8 codes; NaN for S.1111.111."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** (1 - BIAS - MANT_BITS),
                   (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - BIAS))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def e4m3_round(y: np.ndarray) -> np.ndarray:
    """Nearest E4M3 value (float64) of each finite y, ties to even, saturated to ±448."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), E4M3_MAX)
    # spacing of the grid around a: 2^(e−3) for normal a (e = ⌊log2 a⌋ ≥ −6), 2^−9 below 2^−6
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, MIN_NORMAL_EXP)
    step = np.exp2(e - MANT_BITS)
    r = np.round(a / step) * step  # np.round: ties to even on the integer multiple
    r = np.minimum(r, E4M3_MAX)
    return np.sign(y) * r


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """uint8 codes of e4m3_round(y)."""
    r = e4m3_round(y)
    a = np.abs(r)
    sign = (np.signbit(r)).astype(np.int64) << 7
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    normal = a >= 2.0 ** MIN_NORMAL_EXP
    ebits = np.where(normal, e + BIAS, 0)
    m = np.where(normal, np.round((a / np.exp2(e) - 1.0) * 8.0), np.round(a / 2.0 ** -9)).astype(np.int64)
    code = sign | (ebits << 3) | m
    return np.where(a == 0, sign, code).astype(np.uint8)


def quantize_per_tensor(x: np.ndarray):
    """(codes uint8, dq float32) of one tensor, the scale and the scaled values formed in float32."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    scale = np.float32(448.0) / amax if amax > 0 else np.float32(1.0)
    y = (x32 * np.float32(scale)).astype(np.float32)
    dq = amax / np.float32(448.0) if amax > 0 else np.float32(1.0)
    return e4m3_encode(y), np.float32(dq)


def gemm_e4m3(qa: np.ndarray, qb: np.ndarray, dq_a: float, dq_b: float, alpha: float = 1.0) -> np.ndarray:
    """alpha·dq_a·dq_b·(A·Bᵀ) with A [M,K], B [N,K] given as e4m3 codes, in float64."""
    return float(alpha) * float(dq_a) * float(dq_b) * (e4m3_decode(qa) @ e4m3_decode(qb).T)
