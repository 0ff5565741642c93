"""Per-tensor FP8 codec of the oracle (test infrastructure only).

Pages: "Efficient MoE training for biological foundation models" (news.bpdata.com,
section 2, "FP8 and MXFP8"; sitech.ge, "Reducing memory and quantisation cost"): besides
MXFP8's one scale per 32 values, FP8 training keeps ONE scale per tensor, with E4M3 for
the forward operands and E5M2 (more range, less precision) for the gradients.

Readings where the pages are silent:
  * formats: OCP FP8 E4M3 "fn" (bias 7, max 448, no infinities) and E5M2 (bias 15, max
    57344, IEEE-like infinities and NaNs, which are never produced here);
  * current scaling: for a tensor X, amax = max |X| and s = fmt_max / amax (s = 1 for an
    all-zero tensor); codes = the fp32 product X * s rounded to the format, nearest with
    ties to even, saturating at +-fmt_max; the value of a code c is decode(c) / s. The
    scale and the product are computed in fp32 (the precision the kernels decide codes
    in), so both sides encode identical inputs;
  * a "tensor" is one GEMM operand: a weight matrix of one expert (GroupedLinear keeps a
    weight per expert), or a whole activation / gradient over all routed rows.
"""
from __future__ import annotations

import numpy as np

from .mxfp8 import E4M3_VALUES, e4m3_encode

E4M3_MAX = 448.0
E5M2_MAX = 57344.0


def e5m2_decode_code(c: int) -> float:
    """Value of one E5M2 code (inf / NaN for exponent field 31)."""
    sign = -1.0 if c & 0x80 else 1.0
    exp = (c >> 2) & 0x1F
    man = c & 3
    if exp == 31:
        return sign * np.inf if man == 0 else np.nan
    if exp == 0:
        return sign * (man / 4.0) * 2.0 ** (1 - 15)
    return sign * (1.0 + man / 4.0) * 2.0 ** (exp - 15)


E5M2_VALUES = np.array([e5m2_decode_code(c) for c in range(256)], dtype=np.float64)
_POS5 = E5M2_VALUES[:124].copy()      # the finite non-negative values, ascending; index == code


def e5m2_encode(v) -> np.ndarray:
    """Round float64 values to E5M2 codes: nearest, ties to even, saturating at 57344."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v)
    a = np.minimum(np.abs(v), E5M2_MAX)
    i = np.clip(np.searchsorted(_POS5, a, side="right") - 1, 0, 123)
    lo = _POS5[i]
    hi = _POS5[np.minimum(i + 1, 123)]
    up = (i < 123) & (((hi - a) < (a - lo)) | (((hi - a) == (a - lo)) & ((i & 1) == 1)))
    code = np.where(up, i + 1, i).astype(np.uint8)
    return (code | (sign.astype(np.uint8) << 7)).astype(np.uint8)


FORMATS = {"e4m3": (E4M3_MAX, e4m3_encode, E4M3_VALUES), "e5m2": (E5M2_MAX, e5m2_encode, E5M2_VALUES)}


def tensor_scale(x, fmt: str) -> np.float32:
    """s = fmt_max / amax in fp32 (1 for an all-zero tensor)."""
    amax = np.float32(np.max(np.abs(np.asarray(x, dtype=np.float32)))) if np.size(x) else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(np.float32(FORMATS[fmt][0]) / amax)


def quantize_tensor(x, fmt: str, scale=None):
    """Codes of x (any shape) with one scale for the whole tensor. Returns (codes, s)."""
    s = tensor_scale(x, fmt) if scale is None else np.float32(scale)
    prod = np.asarray(x, dtype=np.float32) * s                  # fp32 product, rounded once
    return FORMATS[fmt][1](prod.astype(np.float64)), s


def dequantize_tensor(codes, s, fmt: str) -> np.ndarray:
    return FORMATS[fmt][2][np.asarray(codes, dtype=np.uint8)] / np.float64(s)


def qdq(x, fmt: str) -> np.ndarray:
    """x quantised and dequantised with its own current scale (fp64 values)."""
    c, s = quantize_tensor(x, fmt)
    return dequantize_tensor(c, s, fmt)
