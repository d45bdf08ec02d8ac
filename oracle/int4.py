"""Group-wise symmetric INT4 weight quantiser, W4A16 (CPU oracle; test infrastructure only).

"AI Infra如何优化VLA" (section 后续工作) names FP8 and INT4 as the next quantisation steps and
warns that the action head's denoising is sensitive to accumulated quantisation error; it gives
no scheme.  The reading used here is the usual weight-only W4A16 form: one fp32 scale per
output row and group of G = 128 consecutive inputs,

    scale[o, g]  = max_{i in g} |w[o, i]| / 7     (fp32 division; a zero group takes scale 1)
    code[o, i]   = round_half_even(w[o, i] / scale[o, g]) clamped to [-7, 7]  (quotient in fp32)
    W'[o, i]     = bf16(code * scale)             (fp32 product rounded to nearest-even bf16)

W' is the bf16 weight the tensor cores multiply with bf16 activations: the scale varies along
the reduction, so it is applied when the codes are widened on chip, not after the dot product.
"""

from __future__ import annotations

import numpy as np

INT4_MAX = 7.0
GROUP = 128


def _bf16_round(x32: np.ndarray) -> np.ndarray:
    """fp32 -> nearest-even bf16, returned as float64 (finite inputs)."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def quantize_groupwise_int4(w: np.ndarray, group: int = GROUP):
    """``w [out, in]`` (fp32) -> ``(codes int8 [out, in] in [-7, 7], scales float32 [out, ceil(in/group)])``."""
    w32 = np.asarray(w, dtype=np.float32)
    out, n = w32.shape
    ng = -(-n // group)
    pad = np.zeros((out, ng * group), np.float32)
    pad[:, :n] = w32
    g = pad.reshape(out, ng, group)
    amax = np.max(np.abs(g), axis=2)
    scale = (amax / np.float32(INT4_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    q = (g / scale[:, :, None]).astype(np.float32)
    codes = np.clip(np.rint(q), -INT4_MAX, INT4_MAX).astype(np.int8).reshape(out, ng * group)[:, :n]
    return np.ascontiguousarray(codes), scale


def dequantize_groupwise_int4(codes: np.ndarray, scales: np.ndarray, group: int = GROUP) -> np.ndarray:
    """W' = bf16(code * scale) in float64."""
    c = np.asarray(codes, dtype=np.float32)
    s = np.repeat(np.asarray(scales, dtype=np.float32), group, axis=1)[:, : c.shape[1]]
    return _bf16_round((c * s).astype(np.float32))
