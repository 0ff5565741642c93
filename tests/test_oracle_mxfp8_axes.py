"""Pins of the quantisation axes of the oracle's MXFP8 layer (forward and backward).

MXFP8 keeps one scale per 32 consecutive values ("Efficient MoE training for biological
foundation models", news.bpdata.com section 2, "FP8 and MXFP8"); a GEMM consumes its
operands blocked along its own contraction axis. Which axis that is for each operand of
each GEMM is a choice the pages leave open, so it is pinned here by a fact of the codec
rather than by a tolerance: quantising and dequantising a value that is already an E4M3
code times the block's power-of-two scale gives it back exactly.

Each test builds the operands of one GEMM so that they are exactly representable when
blocked along the axis the oracle is meant to use, and NOT representable along the other
axis. The oracle's MXFP8 result must then equal the unquantised fp64 result (torch fp64
autograd, or the exact oracle that torch autograd pins) to 1e-12; blocking along the wrong
axis, or letting a 32-row block run across an expert boundary, changes the result by a
full E4M3 step. The mutation tests at the end plant exactly those mistakes in the oracle
and check that the pins catch them.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import moe, mxfp8

# decode table from the library type, independent of the oracle's own table
E4M3 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
TOP_BINADE = np.arange(0x78, 0x7F)        # codes of 256 .. 448


def mx_blocks(rng, nblk: int, valid=32, lo=-5, hi=5) -> np.ndarray:
    """``nblk`` blocks of 32 values, each an E4M3 value times 2**s_b (random s_b per
    block) with one element of the top binade among the first ``valid`` positions, so the
    scale rule picks exactly 2**s_b and every element is representable."""
    codes = rng.integers(0, 0x7F, size=(nblk, 32))
    top = rng.integers(0, valid, size=nblk)
    codes[np.arange(nblk), top] = rng.choice(TOP_BINADE, size=nblk)
    sign = np.where(rng.random((nblk, 32)) < 0.5, -1.0, 1.0)
    s = rng.integers(lo, hi + 1, size=nblk)
    return E4M3[codes] * sign * np.ldexp(1.0, s)[:, None]


def along_cols(rng, r: int, c: int, lo=-5, hi=5) -> np.ndarray:
    """[r, c] matrix representable in 32-column blocks of each row."""
    return mx_blocks(rng, r * c // 32, lo=lo, hi=hi).reshape(r, c)


def along_rows(rng, r: int, c: int, lo=-5, hi=5) -> np.ndarray:
    """[r, c] matrix representable in 32-row blocks of each column."""
    return along_cols(rng, c, r, lo, hi).T.copy()


def along_expert_rows(rng, split, c: int) -> np.ndarray:
    """[sum(split), c] representable in 32-row blocks of each column that restart at each
    expert's first row (an expert's last block holds its remaining rows)."""
    out = np.zeros((int(np.sum(split)), c))
    start = 0
    for n in split:
        for b0 in range(0, n, 32):
            m = min(32, n - b0)
            out[start + b0:start + b0 + m] = mx_blocks(rng, c, valid=m)[:, :m].T
        start += n
    return out


# bound at import, so that the planted mistakes below do not reach these checks
_QUANTIZE, _DEQUANTIZE = mxfp8.quantize, mxfp8.dequantize


def _qdq_cols(v):
    return _DEQUANTIZE(*_QUANTIZE(v, axis=0), axis=0)


def _exactly_representable_along_cols(v) -> bool:
    return bool(np.array_equal(_qdq_cols(v), v))


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ------------------------------------------------------------------ the constructions
def test_constructions_are_representable_on_one_axis_only():
    rng = np.random.default_rng(0)
    v = along_cols(rng, 64, 96)
    assert _exactly_representable_along_cols(v)
    assert not _exactly_representable_along_cols(v.T.copy())
    split = [37, 0, 70]
    g = along_expert_rows(rng, split, 64)
    assert np.array_equal(mxfp8.dequantize_grouped_rows(*mxfp8.quantize_grouped_rows(g, split), split), g)
    # blocks of 32 global rows (ignoring the expert boundary at row 37) are lossy, and so
    # are blocks along the columns
    whole = [sum(split)]
    assert not np.array_equal(mxfp8.dequantize_grouped_rows(*mxfp8.quantize_grouped_rows(g, whole), whole), g)
    assert not _exactly_representable_along_cols(g)


# ---------------------------------------------------------- the four backward GEMMs
SPLIT_DENSE = [32, 0, 64]        # R = 96: every axis a multiple of 32 (used by the dgrads)
SPLIT_RAGGED = [37, 0, 70]       # ragged experts and an empty one (used by the wgrads)
H, F = 64, 64


def _torch_bilinear_grads(left, w, right, split):
    """Gradients of sum_e sum((left_e @ w[e]) * right_e) with respect to left and w,
    by torch fp64 autograd: d/dleft = right_e @ w[e]^T, d/dw[e] = left_e^T @ right_e."""
    lt = torch.tensor(left, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    rt = torch.tensor(right)
    total = 0
    s = 0
    for e, n in enumerate(split):
        total = total + ((lt[s:s + n] @ wt[e]) * rt[s:s + n]).sum()
        s += n
    total.backward()
    return lt.grad.numpy(), wt.grad.numpy()


def _fc2_dgrad_err(rng_seed=1):
    """fc2 dgrad: dy blocked along H times w2 blocked along H. dh and dprob depend on
    the data gradient of fc2 only; the exact oracle (pinned by torch autograd) gives them
    from the same h."""
    rng = np.random.default_rng(rng_seed)
    split, E = SPLIT_DENSE, len(SPLIT_DENSE)
    R = sum(split)
    xp = rng.normal(size=(R, H))
    w1 = rng.normal(0, 0.2, size=(E, H, 2 * F))
    pp = rng.uniform(0.1, 1.0, size=R)
    dy = along_cols(rng, R, H)
    w2 = np.stack([along_cols(rng, F, H) for _ in range(E)])       # [E, F, H] along H
    assert not _exactly_representable_along_cols(dy.T.copy())
    _, h, _ = moe.grouped_mlp_fwd(xp, split, w1, w2, pp, a_round="f64")
    exact = moe.grouped_mlp_bwd(dy, xp, split, w1, w2, pp, a_round="f64")
    got = moe.grouped_mlp_bwd_mxfp8(dy, xp, split, w1, w2, pp, h)
    return max(_rel(got[4], exact[4]), _rel(got[3], exact[3]))


def _fc1_dgrad_err(rng_seed=2):
    """fc1 dgrad: dh blocked along 2F times w1 blocked along 2F."""
    rng = np.random.default_rng(rng_seed)
    split, E = SPLIT_DENSE, len(SPLIT_DENSE)
    R = sum(split)
    dh = along_cols(rng, R, 2 * F)
    w1 = np.stack([along_cols(rng, H, 2 * F) for _ in range(E)])   # [E, H, 2F] along 2F
    xp = rng.normal(size=(R, H))
    got = moe.grouped_mlp_bwd_mxfp8(rng.normal(size=(R, H)), xp, split, w1, rng.normal(size=(E, F, H)),
                                    rng.uniform(0.1, 1, R), rng.normal(size=(R, 2 * F)), dh=dh,
                                    a=rng.normal(size=(R, F)))
    ref_dxp, _ = _torch_bilinear_grads(xp, w1, dh, split)
    return _rel(got[0], ref_dxp)


def _fc2_wgrad_err(rng_seed=3):
    """fc2 wgrad: a and dy blocked along each expert's rows."""
    rng = np.random.default_rng(rng_seed)
    split, E = SPLIT_RAGGED, len(SPLIT_RAGGED)
    R = sum(split)
    a = along_expert_rows(rng, split, F)
    dy = along_expert_rows(rng, split, H)
    w2 = rng.normal(size=(E, F, H))
    got = moe.grouped_mlp_bwd_mxfp8(dy, rng.normal(size=(R, H)), split, rng.normal(size=(E, H, 2 * F)), w2,
                                    rng.uniform(0.1, 1, R), rng.normal(size=(R, 2 * F)),
                                    dh=rng.normal(size=(R, 2 * F)), a=a)
    _, ref_dw2 = _torch_bilinear_grads(a, w2, dy, split)
    assert np.all(got[2][1] == 0.0)          # the empty expert's gradient
    return _rel(got[2], ref_dw2)


def _fc1_wgrad_err(rng_seed=4):
    """fc1 wgrad: xp and dh blocked along each expert's rows."""
    rng = np.random.default_rng(rng_seed)
    split, E = SPLIT_RAGGED, len(SPLIT_RAGGED)
    R = sum(split)
    xp = along_expert_rows(rng, split, H)
    dh = along_expert_rows(rng, split, 2 * F)
    w1 = rng.normal(size=(E, H, 2 * F))
    got = moe.grouped_mlp_bwd_mxfp8(rng.normal(size=(R, H)), xp, split, w1, rng.normal(size=(E, F, H)),
                                    rng.uniform(0.1, 1, R), rng.normal(size=(R, 2 * F)), dh=dh,
                                    a=rng.normal(size=(R, F)))
    _, ref_dw1 = _torch_bilinear_grads(xp, w1, dh, split)
    assert np.all(got[1][1] == 0.0)
    return _rel(got[1], ref_dw1)


CHECKS = {"fc2_dgrad": _fc2_dgrad_err, "fc1_dgrad": _fc1_dgrad_err, "fc2_wgrad": _fc2_wgrad_err,
          "fc1_wgrad": _fc1_wgrad_err}


@pytest.mark.parametrize("gemm", sorted(CHECKS))
def test_backward_gemm_axis_is_exact_on_representable_operands(gemm):
    assert CHECKS[gemm]() <= 1e-12


# --------------------------------------------------------------------------- forward
def test_forward_axes_exact_on_representable_operands():
    """fc1: xp blocked along H times w1 blocked along H (k-major codes [E, 2F, H]); fc2:
    the given `a` codes times w2 blocked along F. The grouped and the per-row forms."""
    rng = np.random.default_rng(5)
    split, E = [40, 0, 24], 3
    R = sum(split)
    x = along_cols(rng, R, H, -8, -6)
    w1 = np.stack([along_rows(rng, H, 2 * F, -10, -7) for _ in range(E)])   # [E, H, 2F] along H
    w2 = np.stack([along_rows(rng, F, H) for _ in range(E)])                 # [E, F, H] along F
    assert not _exactly_representable_along_cols(w1[0])
    pp = rng.uniform(0.1, 1, R)
    xc, xs = mxfp8.quantize(x, axis=0)
    w1c, w1s = moe.quantize_weights_kmajor(w1, "rows")
    w2c, w2s = moe.quantize_weights_kmajor(w2, "rows")
    a_codes = rng.integers(0, 0x7F, size=(R, F)).astype(np.uint8) | \
        (rng.integers(0, 2, size=(R, F)).astype(np.uint8) << 7)
    a_scales = rng.integers(120, 130, size=(R, F // 32)).astype(np.uint8)
    aq = E4M3[a_codes] * np.repeat(np.ldexp(1.0, a_scales.astype(np.int64) - 127), 32, axis=1)
    yp, _, _, h = moe.grouped_mlp_fwd_mxfp8(xc, xs, split, w1c, w1s, w2c, w2s, pp, a_codes, a_scales)
    ref_h = np.zeros((R, 2 * F))
    ref_y = np.zeros((R, H))
    s = 0
    for e, n in enumerate(split):
        ref_h[s:s + n] = (torch.tensor(x[s:s + n]) @ torch.tensor(w1[e])).numpy()
        ref_y[s:s + n] = (torch.tensor(aq[s:s + n]) @ torch.tensor(w2[e])).numpy()
        s += n
    assert _rel(h, ref_h) <= 1e-12 and _rel(yp, ref_y) <= 1e-12
    experts = np.repeat(np.arange(E), split)
    ypr, _, _ = moe.fwd_rows_mxfp8(x, pp, experts, w1, w2, a_codes=a_codes, a_scales=a_scales)
    assert _rel(ypr, ref_y) <= 1e-12


# -------------------------------------------------------------- planted mistakes
def _swap_plain_axes(monkeypatch):
    q, dq = mxfp8.quantize, mxfp8.dequantize
    monkeypatch.setattr(mxfp8, "quantize", lambda v, axis, transpose_out=False: q(v, 1 - axis, transpose_out))
    monkeypatch.setattr(mxfp8, "dequantize", lambda c, s, axis, transpose_out=False: dq(c, s, 1 - axis,
                                                                                         transpose_out))


def _global_row_blocks(monkeypatch):
    q, dq = mxfp8.quantize_grouped_rows, mxfp8.dequantize_grouped_rows
    monkeypatch.setattr(mxfp8, "quantize_grouped_rows", lambda v, split: q(v, [int(np.sum(split))]))
    monkeypatch.setattr(mxfp8, "dequantize_grouped_rows", lambda c, s, split: dq(c, s, [int(np.sum(split))]))


def _row_blocks_along_cols(monkeypatch):
    monkeypatch.setattr(mxfp8, "quantize_grouped_rows", lambda v, split: mxfp8.quantize(v, axis=0))
    monkeypatch.setattr(mxfp8, "dequantize_grouped_rows", lambda c, s, split: mxfp8.dequantize(c, s, axis=0))


@pytest.mark.parametrize("plant,gemms", [
    (_swap_plain_axes, ["fc2_dgrad", "fc1_dgrad"]),
    (_global_row_blocks, ["fc2_wgrad", "fc1_wgrad"]),
    (_row_blocks_along_cols, ["fc2_wgrad", "fc1_wgrad"]),
])
def test_planted_axis_mistakes_are_caught(monkeypatch, plant, gemms):
    plant(monkeypatch)
    for g in gemms:
        assert CHECKS[g]() > 1e-4, g
