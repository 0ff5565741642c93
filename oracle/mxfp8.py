"""MXFP8 codec of the oracle (test infrastructure only).

Pages: "Efficient MoE training for biological foundation models" (news.bpdata.com,
section 2 "model size and activation memory"; sitech.ge, section "Reducing memory and
quantisation cost"): MXFP8 stores 8-bit values with one scale factor per block of 32
consecutive values, and Blackwell tensor cores consume it directly.

Readings where the pages are silent (the OCP Microscaling v1.0 formats):
  * element format E4M3 "fn": sign, 4 exponent bits (bias 7), 3 mantissa bits,
    subnormals down to 2**-9, largest finite 448, code 0x7F/0xFF is NaN, no infinities;
  * encoding rounds to nearest, ties to even significand, and saturates: any magnitude
    above 448 encodes as 448 (sign kept; -0.0 and negative values that round to zero
    encode as 0x80);
  * scale format E8M0: code c means 2**(c - 127);
  * scale choice for a block with amax = max |v|: X = 2**(floor(log2(amax)) - 8), the
    exponent clamped to [-127, 127]; a block of zeros gets code 0 and all-zero codes
    (8 = exponent of 448, the largest E4M3 binade);
  * blocks run along one axis from index 0; that axis must be a multiple of 32.
Inputs are finite.
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0
BLOCK = 32
EMAX_E4M3 = 8


def e4m3_decode_code(c: int) -> float:
    """Value of one E4M3 code (NaN for 0x7F/0xFF)."""
    sign = -1.0 if c & 0x80 else 1.0
    mag = c & 0x7F
    if mag == 0x7F:
        return math.nan
    exp = mag >> 3
    man = mag & 7
    if exp == 0:
        return sign * (man / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


#: value of every code 0..255 (NaN at 0x7F and 0xFF)
E4M3_VALUES = np.array([e4m3_decode_code(c) for c in range(256)], dtype=np.float64)
#: the 127 finite non-negative values, ascending; index == code
_POS = E4M3_VALUES[:127].copy()


def e4m3_encode(v) -> np.ndarray:
    """Round float64 values to E4M3 codes: nearest, ties to even, saturating at 448."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v)
    a = np.minimum(np.abs(v), E4M3_MAX)
    i = np.searchsorted(_POS, a, side="right") - 1          # largest code with value <= a
    i = np.clip(i, 0, 126)
    lo = _POS[i]
    hi = _POS[np.minimum(i + 1, 126)]
    d_lo = a - lo
    d_hi = hi - a
    up = (i < 126) & ((d_hi < d_lo) | ((d_hi == d_lo) & ((i & 1) == 1)))
    code = np.where(up, i + 1, i).astype(np.uint8)
    return (code | (sign.astype(np.uint8) << 7)).astype(np.uint8)


def e8m0_value(code) -> np.ndarray:
    return np.ldexp(1.0, np.asarray(code, dtype=np.int64) - 127)


def e8m0_for_amax(amax) -> np.ndarray:
    """Scale code for each block maximum: floor(log2(amax)) - 8 + 127, clamped to [0, 254]."""
    amax = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(amax)                 # amax = m * 2**ex, 0.5 <= m < 1
    e = (ex.astype(np.int64) - 1) - EMAX_E4M3
    code = np.clip(e + 127, 0, 254)
    return np.where(amax == 0.0, 0, code).astype(np.uint8)


def quantize_blocks_last_axis(v) -> tuple[np.ndarray, np.ndarray]:
    """Quantise ``v[..., n]`` in blocks of 32 consecutive values along the last axis.

    Returns (codes uint8 [..., n], scales uint8 [..., n/32]).
    """
    v = np.asarray(v, dtype=np.float64)
    n = v.shape[-1]
    if n % BLOCK:
        raise ValueError("blocked axis must be a multiple of 32")
    blk = v.reshape(v.shape[:-1] + (n // BLOCK, BLOCK))
    amax = np.max(np.abs(blk), axis=-1)
    scales = e8m0_for_amax(amax)
    x = e8m0_value(scales)[..., None]
    codes = e4m3_encode(blk / x)
    return codes.reshape(v.shape), scales


def dequantize_blocks_last_axis(codes, scales) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    n = codes.shape[-1]
    vals = E4M3_VALUES[codes].reshape(codes.shape[:-1] + (n // BLOCK, BLOCK))
    return (vals * e8m0_value(scales)[..., None]).reshape(codes.shape)


def quantize(v, axis: int, transpose_out: bool = False) -> tuple[np.ndarray, np.ndarray]:
    """Quantise a batch of matrices ``v[..., rows, cols]``.

    axis 0: blocks of 32 along cols (each row on its own) -> codes [..., rows, cols],
            scales [..., rows, cols/32].
    axis 1: blocks of 32 along rows (each column on its own). With ``transpose_out`` the
            result is the transposed matrix quantised along its rows: codes
            [..., cols, rows], scales [..., cols, rows/32]; without it codes keep the
            input layout [..., rows, cols] and scales are [..., rows/32, cols].
    """
    v = np.asarray(v, dtype=np.float64)
    if axis == 0:
        if transpose_out:
            raise ValueError("transpose_out applies to axis 1 only")
        return quantize_blocks_last_axis(v)
    if axis != 1:
        raise ValueError("axis must be 0 or 1")
    vt = np.swapaxes(v, -1, -2)
    codes_t, scales_t = quantize_blocks_last_axis(vt)
    if transpose_out:
        return codes_t, scales_t
    return np.swapaxes(codes_t, -1, -2), np.swapaxes(scales_t, -1, -2)


def dequantize(codes, scales, axis: int, transpose_out: bool = False) -> np.ndarray:
    """Inverse of :func:`quantize` (returns the matrix in the layout the codes are in)."""
    if axis == 0 or transpose_out:
        return dequantize_blocks_last_axis(codes, scales)
    return np.swapaxes(dequantize_blocks_last_axis(np.swapaxes(codes, -1, -2),
                                                   np.swapaxes(scales, -1, -2)), -1, -2)


def quantize_grouped_rows(v, split_sizes) -> tuple[np.ndarray, list]:
    """Quantise expert-contiguous rows ``v[R, C]`` along the rows, per column, in blocks
    of 32 rows that restart at every expert's first row; an expert's last block covers
    its remaining rows, as if padded with zeros.

    Returns codes [R, C] and, per expert, its scales [ceil(n_e/32), C].
    """
    v = np.asarray(v, dtype=np.float64)
    codes = np.zeros(v.shape, dtype=np.uint8)
    scales = []
    start = 0
    for n in np.asarray(split_sizes, dtype=np.int64):
        nb = (n + BLOCK - 1) // BLOCK
        padded = np.zeros((nb * BLOCK, v.shape[1]))
        padded[:n] = v[start:start + n]
        c, s = quantize(padded, axis=1)
        codes[start:start + n] = c[:n]
        scales.append(s)
        start += n
    return codes, scales


def dequantize_grouped_rows(codes, scales, split_sizes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.zeros(codes.shape)
    start = 0
    for n, s in zip(np.asarray(split_sizes, dtype=np.int64), scales):
        nb = (n + BLOCK - 1) // BLOCK
        padded = np.zeros((nb * BLOCK, codes.shape[1]), dtype=np.uint8)
        padded[:n] = codes[start:start + n]
        out[start:start + n] = dequantize(padded, s, axis=1)[:n]
        start += n
    return out
