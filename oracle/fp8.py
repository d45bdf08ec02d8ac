"""FP8 E4M3 codec and per-output-channel weight quantiser (CPU oracle; test infrastructure only).

Follows the APXInf article ("开源 APXInf 把 VLA 推理压到 26 毫秒", section "CUDA Graph、FP8 和
Rust"): FP8 weights halve the bytes the expert streams.  The weight-only form used here
(e4m3 weights with one fp32 scale per output channel, bf16 activations, fp32
accumulation) is the workload definition of the FP8 variant.

The codec is written from the E4M3 format definition (OCP 8-bit floating point, "E4M3FN"):
1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no infinities; the only NaN
codes are S.1111.111; the largest finite magnitude is 1.75 * 2^8 = 448; subnormals are
m * 2^-9 for m = 1..7.  Encoding rounds to nearest, ties to even, and saturates to +-448.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Code (uint8) -> value (float64).  NaN codes decode to NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    sub = m * 2.0 ** -9
    nrm = (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64))
    val = np.where(e == 0, sub, nrm)
    val = np.where((e == 15) & ((c & 7) == 7), np.nan, val)
    return sign * val


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Value -> code (uint8): round to nearest even, saturate to +-448, NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    neg = np.signbit(x)
    code = np.zeros(x.shape, dtype=np.int64)

    pos = (a > 0) & np.isfinite(a) & (a < E4M3_MAX)
    # a = f * 2^ex with f in [0.5, 1): the unbiased exponent of a is ex - 1 (exact).
    _, ex = np.frexp(np.where(pos, a, 1.0))
    e = ex.astype(np.int64) - 1

    normal = pos & (e >= -6)
    frac = np.ldexp(np.where(normal, a, 1.0), -np.where(normal, e, 0))      # in [1, 2), exact
    mq = np.rint((frac - 1.0) * 8.0).astype(np.int64)                       # ties to even
    carry = mq == 8
    e_n = np.where(carry, e + 1, e)
    mq = np.where(carry, 0, mq)
    code_n = ((e_n + 7) << 3) | mq
    code_n = np.where(code_n >= 0x7F, 0x7E, code_n)                         # never reach NaN
    code = np.where(normal, code_n, code)

    subn = pos & (e < -6)
    msub = np.rint(np.ldexp(np.where(subn, a, 0.0), 9)).astype(np.int64)     # 0..8; 8 is 2^-6
    code = np.where(subn, msub, code)

    code = np.where(np.isfinite(a) & (a >= E4M3_MAX), 0x7E, code)
    code = np.where(np.isinf(a), 0x7E, code)
    code = np.where(neg, code | 0x80, code)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def quantize_rowwise_e4m3(w: np.ndarray):
    """Per-output-channel quantisation of a weight ``[out, in]`` given in fp32.

    scale[o] = max_i |w[o, i]| / 448 (fp32 division); a zero row takes scale 1.
    code[o, i] = e4m3(w[o, i] / scale[o]) with the quotient rounded to fp32 first.
    Returns ``(codes uint8 [out, in], scales float32 [out])``.
    """
    w32 = np.asarray(w, dtype=np.float32)
    amax = np.max(np.abs(w32), axis=1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    q = (w32 / scale[:, None]).astype(np.float32)
    return e4m3_encode(q), scale


def dequantize_rowwise_e4m3(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """W' = e4m3 value * scale, in float64."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[:, None]
