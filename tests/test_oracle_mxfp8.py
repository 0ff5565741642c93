"""Pins of the oracle's MXFP8 codec to a library routine, closed forms and hand values."""
import math

import ml_dtypes
import numpy as np
import pytest

from oracle import mxfp8
from tests.golden import load


def test_decode_table_matches_ml_dtypes():
    # every one of the 256 codes decodes like ml_dtypes' float8_e4m3fn
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ours = mxfp8.E4M3_VALUES
    both_nan = np.isnan(lib) & np.isnan(ours)
    assert np.all(both_nan | (lib == ours))
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(3)
    finite = mxfp8.E4M3_VALUES[np.isfinite(mxfp8.E4M3_VALUES)]
    pos = np.unique(np.abs(finite))
    mids = (pos[1:] + pos[:-1]) / 2.0                       # exact ties
    vals = np.concatenate([
        rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000), rng.normal(0, 0.01, 20000),
        mids, -mids, pos, -pos, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    vals = vals.astype(np.float32).astype(np.float64)       # what a cast from fp32 sees
    lib = vals.astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ours = mxfp8.e4m3_encode(vals)
    assert np.array_equal(lib, ours)


def test_ties_to_even_and_saturation():
    # 1.0625 sits halfway between 1.0 (0x38) and 1.125 (0x39): even code 0x38
    # 1.1875 sits halfway between 1.125 (0x39) and 1.25 (0x3A): even code 0x3A
    # 0.5 * 2**-9 sits halfway between 0 and the smallest subnormal: even code 0x00
    assert list(mxfp8.e4m3_encode([1.0625, 1.1875, 2.0 ** -10, -1.0625])) == [0x38, 0x3A, 0x00, 0xB8]
    # saturating: everything above 448 encodes as 448
    assert list(mxfp8.e4m3_encode([448.0, 449.0, 464.0, 500.0, 1e9, -1e9])) == [0x7E] * 5 + [0xFE]


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(mxfp8.e4m3_encode(mxfp8.E4M3_VALUES[codes]), codes)


def test_scale_rule_closed_forms():
    # amax 448 -> floor(log2) 8 -> X = 1 -> code 127; amax 1 -> X = 2**-8 -> code 119
    assert list(mxfp8.e8m0_for_amax([448.0, 1.0, 0.0, 3.0, 511.99, 2.0 ** -130, 2.0 ** 130])) == \
        [127, 119, 0, 120, 127, 0, 249]
    lib = np.arange(255, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert np.array_equal(lib, mxfp8.e8m0_value(np.arange(255)))


def test_golden_block():
    g = load("mxfp8_block.txt")
    v = np.zeros(32)
    v[:len(g["values"])] = g["values"]
    v[5] = -0.0
    codes, scales = mxfp8.quantize_blocks_last_axis(v[None, :])
    assert scales[0, 0] == g["scale"]
    assert list(codes[0, :6]) == g["codes"]
    assert np.all(codes[0, 6:] == 0)


@pytest.mark.parametrize("e", [-127, -100, -7, 0, 5, 100, 119])
def test_quantize_dequantize_exact_on_representable_blocks(e):
    # blocks built from E4M3 values times 2**e, with one element in the top binade
    # [256, 448], quantise to exactly those codes and dequantise to the same values
    rng = np.random.default_rng(e + 1000)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    top = np.array([c for c in range(0x78, 0x7F)], dtype=np.uint8)   # 256 .. 448
    codes = rng.choice(finite, size=(64, 32))
    codes[:, 7] = rng.choice(top, size=64)
    vals = mxfp8.E4M3_VALUES[codes] * 2.0 ** e
    q, s = mxfp8.quantize_blocks_last_axis(vals)
    assert np.all(s == e + 127)
    assert np.array_equal(mxfp8.dequantize_blocks_last_axis(q, s), vals)
    assert np.array_equal(q & 0x7F, codes & 0x7F)


def test_scaled_block_lands_in_top_binade():
    # invariant of the scale rule: the block maximum maps into [256, 512) before
    # saturation, so its code is one of 256..448 (0x78..0x7E)
    rng = np.random.default_rng(7)
    v = rng.normal(0, 1, (500, 64)) * np.exp(rng.uniform(-30, 30, (500, 1)))
    q, s = mxfp8.quantize_blocks_last_axis(v)
    mx = np.max(q.reshape(500, 2, 32) & 0x7F, axis=-1)
    assert np.all((mx >= 0x78) & (mx <= 0x7E))
    # error bound: |deq - v| <= half an ulp of the top binade (2**-4 relative to 2**8 X)
    d = mxfp8.dequantize_blocks_last_axis(q, s)
    x = mxfp8.e8m0_value(s).repeat(32, axis=1)
    sat = np.abs(v) > 448 * x
    err = np.abs(d - v)
    assert np.all(err[~sat] <= 16.0 * x[~sat])   # half the spacing 32 of [256, 512)
    assert np.all(np.abs(d[sat]) == 448 * x[sat])


def test_axis_and_transpose_layouts():
    rng = np.random.default_rng(11)
    w = rng.normal(0, 0.02, (3, 64, 96))
    c0, s0 = mxfp8.quantize(w, axis=0)
    assert c0.shape == (3, 64, 96) and s0.shape == (3, 64, 3)
    c1, s1 = mxfp8.quantize(w, axis=1)
    assert c1.shape == (3, 64, 96) and s1.shape == (3, 2, 96)
    ct, st = mxfp8.quantize(w, axis=1, transpose_out=True)
    assert ct.shape == (3, 96, 64) and st.shape == (3, 96, 2)
    assert np.array_equal(np.swapaxes(ct, 1, 2), c1)
    # blocks along rows: column j of rows 0..31 shares one scale
    j = 5
    col = w[1, :32, j]
    ref_scale = mxfp8.e8m0_for_amax(np.max(np.abs(col)))
    assert s1[1, 0, j] == ref_scale
    np.testing.assert_array_equal(mxfp8.dequantize(c1, s1, axis=1),
                                  np.swapaxes(mxfp8.dequantize(ct, st, axis=1, transpose_out=True), 1, 2))
    with pytest.raises(ValueError):
        mxfp8.quantize(rng.normal(size=(4, 33)), axis=0)
    assert math.isnan(mxfp8.e4m3_decode_code(0x7F))


def test_grouped_rows_quantiser_pins():
    rng = np.random.default_rng(21)
    split = [64, 0, 45, 7, 96]
    v = rng.normal(size=(sum(split), 40)) * np.exp(rng.uniform(-5, 5, (1, 40)))
    codes, scales = mxfp8.quantize_grouped_rows(v, split)
    # a group of whole blocks is the plain column quantiser on that group
    c0, s0 = mxfp8.quantize(v[:64], axis=1)
    assert np.array_equal(codes[:64], c0) and np.array_equal(scales[0], s0)
    assert scales[1].shape == (0, 40)
    # a partial block: the rows of the group padded with zeros (hand-built)
    g = v[64:109]
    pad = np.zeros((64, 40))
    pad[:45] = g
    c2, s2 = mxfp8.quantize(pad, axis=1)
    assert np.array_equal(codes[64:109], c2[:45]) and np.array_equal(scales[2], s2)
    # blocks never mix experts: quantising each group alone gives the same codes
    c3, s3 = mxfp8.quantize_grouped_rows(v[109:116], [7])
    assert np.array_equal(codes[109:116], c3) and np.array_equal(scales[3], s3[0])
    # dequantised values are within the MXFP8 rounding bound of the input
    d = mxfp8.dequantize_grouped_rows(codes, scales, split)
    assert np.max(np.abs(d - v) / np.maximum(np.abs(v), 1e-300)) <= 0.126 or np.allclose(d, v, rtol=0.126)
