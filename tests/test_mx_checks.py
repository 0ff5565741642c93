"""The boundary-flip checker of the GPU MXFP8 tests accepts rounding-boundary flips and
rejects the mistakes it is there to catch (planted on the CPU)."""
import numpy as np

from oracle import mxfp8 as oq
from tests.mx_checks import E4M3, boundary_flips


def _exact_with_boundary_cases(rng, n=64, C=128):
    v = rng.normal(size=(n, C)) * np.exp2(rng.integers(-4, 4, size=(n, 1)))
    # put some elements exactly on rounding midpoints (in units of their block's scale)
    blk = v.reshape(n, C // 32, 32)
    X = oq.e8m0_value(oq.e8m0_for_amax(np.max(np.abs(blk), axis=-1)))
    pos = np.unique(np.abs(E4M3[np.isfinite(E4M3)]))
    mids = (pos[1:] + pos[:-1]) / 2
    for r in range(0, n, 3):
        b = r % (C // 32)
        m = rng.choice(mids[mids < 200])
        blk[r, b, 5] = m * X[r, b]
    # and one block whose maximum is a power of two (the scale boundary)
    blk[1, 0, :] = rng.uniform(-0.5, 0.5, 32)
    blk[1, 0, 7] = 1.0 - 2.0 ** -30
    return blk.reshape(n, C)


def test_fp32_rounding_of_exact_values_passes():
    rng = np.random.default_rng(0)
    exact = _exact_with_boundary_cases(rng)
    # what a kernel sees: the same values after fp32 arithmetic (a relative nudge of a few
    # fp32 ulps either way), quantised by the same rule
    nudged = exact * (1.0 + rng.choice([-3, -1, 1, 3], size=exact.shape) * 2.0 ** -24)
    nudged[1, 7] = 1.0                        # the block max rounds up to the power of two
    c, s = oq.quantize(nudged, axis=0)
    ok, rep = boundary_flips(c, s, exact)
    assert ok, rep
    assert rep["code_flips"] > 0 and rep["scale_flips"] == 1


def test_planted_mistakes_are_rejected():
    rng = np.random.default_rng(1)
    exact = rng.normal(size=(32, 128)) * 3.0
    c, s = oq.quantize(exact, axis=0)
    assert boundary_flips(c, s, exact)[0]
    # a scale one step off in a block whose maximum is far from a power of two
    s2 = s.copy()
    s2[4, 1] += 1
    assert not boundary_flips(c, s2, exact)[0]
    # the last 32 columns quantised with the previous block's scale (a wrong tail block)
    c3, s3 = c.copy(), s.copy()
    X = oq.e8m0_value(s[:, 2])[:, None]
    c3[:, 96:] = oq.e4m3_encode(exact[:, 96:] / X)
    s3[:, 3] = s[:, 2]
    assert not boundary_flips(c3, s3, exact)[0]
    # one code one step off where the exact value is nowhere near a midpoint
    c4 = c.copy()
    i = np.argmax(np.abs(exact[0, :32]) > 1.0)
    c4[0, i] = c4[0, i] + 1 if (c4[0, i] & 0x7F) < 0x7E else c4[0, i] - 1
    assert not boundary_flips(c4, s, exact)[0]
