"""Pins of the oracle's per-tensor FP8 codec and FP8 layer: library casts (ml_dtypes),
closed forms, and exactness on operands that are representable with their own scale."""
import ml_dtypes
import numpy as np
import pytest

from oracle import fp8, moe


def test_e5m2_decode_table_matches_ml_dtypes():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e5m2).astype(np.float64)
    ours = fp8.E5M2_VALUES
    same = (np.isnan(lib) & np.isnan(ours)) | (lib == ours)
    assert np.all(same)
    assert ours[0x7B] == 57344.0 and ours[0x01] == 2.0 ** -16 and np.isinf(ours[0x7C])


def test_e5m2_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(4)
    pos = np.unique(np.abs(fp8.E5M2_VALUES[np.isfinite(fp8.E5M2_VALUES)]))
    mids = (pos[1:] + pos[:-1]) / 2.0
    vals = np.concatenate([rng.uniform(-57344, 57344, 20000), rng.normal(0, 1, 20000), rng.normal(0, 1e-4, 20000),
                           mids, -mids, pos, -pos]).astype(np.float32).astype(np.float64)
    lib = vals.astype(np.float32).astype(ml_dtypes.float8_e5m2).view(np.uint8)
    assert np.array_equal(fp8.e5m2_encode(vals), lib)
    assert list(fp8.e5m2_encode([57344.0, 60000.0, 1e9, -1e9])) == [0x7B, 0x7B, 0x7B, 0xFB]


def test_tensor_scale_closed_forms():
    assert fp8.tensor_scale(np.array([448.0, -3.0]), "e4m3") == 1.0
    assert fp8.tensor_scale(np.array([-57344.0]), "e5m2") == 1.0
    assert fp8.tensor_scale(np.zeros(5), "e4m3") == 1.0
    assert fp8.tensor_scale(np.array([56.0]), "e4m3") == 8.0
    assert fp8.tensor_scale(np.array([3.0]), "e4m3") == np.float32(np.float32(448.0) / np.float32(3.0))


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_representable_tensor_round_trips(fmt):
    # codes times 1/s with the largest code at amax: quantising gives the codes back
    rng = np.random.default_rng(6)
    vmax, _, table = fp8.FORMATS[fmt]
    finite = np.nonzero(np.isfinite(table) & (np.abs(table) <= vmax))[0]
    codes = rng.choice(finite, size=(40, 24)).astype(np.uint8)
    codes[3, 5] = 0x7E if fmt == "e4m3" else 0x7B                 # amax = vmax / s
    s = np.float32(0.125)
    x = table[codes] / np.float64(s)
    c, s2 = fp8.quantize_tensor(x, fmt)
    assert s2 == s and np.array_equal(fp8.dequantize_tensor(c, s2, fmt), x)


def test_fp8_layer_exact_on_representable_operands():
    """Forward and backward with every operand representable under its own per-tensor
    scale (and a, dh given as such) equal the unquantised fp64 layer."""
    rng = np.random.default_rng(8)
    split, E, H, F = [20, 0, 12], 3, 32, 32
    R = sum(split)

    def rep(shape, fmt, s=0.25):
        vmax, _, table = fp8.FORMATS[fmt]
        finite = np.nonzero(np.isfinite(table) & (np.abs(table) <= vmax) & (np.abs(table) < vmax / 4))[0]
        c = rng.choice(finite, size=shape).astype(np.uint8)
        c.reshape(-1)[0] = 0x7E if fmt == "e4m3" else 0x7B
        return table[c] / s

    xp = rep((R, H), "e4m3", 32.0)
    # each expert's weights on their own scale (a scale shared by the stacked experts
    # would round the smaller experts' weights)
    w1 = np.stack([rep((H, 2 * F), "e4m3", 4096.0 / 8 ** e) for e in range(E)])
    w2 = np.stack([rep((F, H), "e4m3", 4096.0 / 8 ** e) for e in range(E)])
    assert not np.array_equal(fp8.qdq(w1, "e4m3"), w1)
    pp = rng.uniform(0.2, 1, R)
    yp, ac, asc, h = moe.grouped_mlp_fwd_fp8(xp, split, w1, w2, pp)
    a_given = rep((R, F), "e4m3", 8.0)
    ac2, as2 = fp8.quantize_tensor(a_given, "e4m3")
    yp2, _, _, h2 = moe.grouped_mlp_fwd_fp8(xp, split, w1, w2, pp, ac2, as2)
    ref_h, ref_y = np.zeros((R, 2 * F)), np.zeros((R, H))
    s0 = 0
    for e, n in enumerate(split):
        ref_h[s0:s0 + n] = xp[s0:s0 + n] @ w1[e]
        ref_y[s0:s0 + n] = a_given[s0:s0 + n] @ w2[e]
        s0 += n
    assert np.max(np.abs(h2 - ref_h)) <= 1e-12 * np.max(np.abs(ref_h))
    assert np.max(np.abs(yp2 - ref_y)) <= 1e-12 * np.max(np.abs(ref_y))
    dy = rep((R, H), "e5m2", 64.0)
    dh = rep((R, 2 * F), "e5m2", 64.0)
    dxp, dw1, dw2, _, _ = moe.grouped_mlp_bwd_fp8(dy, xp, split, w1, w2, pp, h2, ac2, as2, dh=dh)
    s0 = 0
    for e, n in enumerate(split):
        r = slice(s0, s0 + n)
        if n == 0:
            continue
        for got, ref in ((dxp[r], dh[r] @ w1[e].T), (dw1[e], xp[r].T @ dh[r]), (dw2[e], a_given[r].T @ dy[r])):
            assert np.max(np.abs(got - ref)) <= 1e-12 * max(np.max(np.abs(ref)), 1e-300)
        s0 += n
    assert np.all(dw1[1] == 0) and np.all(dw2[1] == 0)
