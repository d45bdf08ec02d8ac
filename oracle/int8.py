"""Row-wise symmetric INT8 weight quantiser (CPU oracle; test infrastructure only).

The APXInf article ("开源 APXInf 把 VLA 推理压到 26 毫秒", section "CUDA Graph、FP8 和 Rust") uses
INT8 quantisation on GPUs without FP8 tensor cores (Jetson Orin) in place of FP8.  It gives no
scheme; the reading used here is the plainest weight-only one, symmetric per output channel,
the same shape as the FP8 variant:

    scale[o]   = max_i |w[o, i]| / 127           (fp32 division; a zero row takes scale 1)
    code[o, i] = round_half_even(w[o, i] / scale[o])   (quotient rounded to fp32 first),
                 clamped to [-127, 127]           (code -128 is never produced)
    W'[o, i]   = code[o, i] * scale[o]
"""

from __future__ import annotations

import numpy as np

INT8_MAX = 127.0


def quantize_rowwise_int8(w: np.ndarray):
    """Per-output-channel quantisation of ``w [out, in]`` (given in fp32).

    Returns ``(codes int8 [out, in], scales float32 [out])``."""
    w32 = np.asarray(w, dtype=np.float32)
    amax = np.max(np.abs(w32), axis=1)
    scale = (amax / np.float32(INT8_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    q = (w32 / scale[:, None]).astype(np.float32)
    codes = np.clip(np.rint(q), -INT8_MAX, INT8_MAX).astype(np.int8)   # rint: half to even
    return codes, scale


def dequantize_rowwise_int8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """W' = code * scale, in float64."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[:, None]
