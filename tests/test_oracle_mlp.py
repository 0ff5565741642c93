"""Pins of the oracle's grouped expert MLP (forward and backward)."""
import math

import numpy as np
import pytest
import torch

from oracle import moe, mxfp8


def _layer(T, H, F, E, k, seed=0, empty=()):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, H))
    lg = rng.normal(size=(T, E))
    for e in empty:
        lg[:, e] -= 100.0
    w1 = rng.normal(0, 0.3, size=(E, H, 2 * F))
    w2 = rng.normal(0, 0.3, size=(E, F, H))
    idx, prob = moe.route(lg, k)
    return x, idx, prob, w1, w2


def _grouped_layer(x, idx, prob, w1, w2, a_round):
    T, k = idx.shape
    E = w1.shape[0]
    row_map, split, _ = moe.permute_index(idx, E)
    xp = moe.permute_rows(x, row_map, k)
    pp = moe.permute_probs(prob, row_map)
    yp, _, _ = moe.grouped_mlp_fwd(xp, split, w1, w2, pp, a_round)
    return moe.unpermute(yp, row_map, T, k)


@pytest.mark.parametrize("a_round", ["f64", "bf16"])
@pytest.mark.parametrize("T,H,F,E,k,empty", [(16, 8, 6, 4, 2, (1,)), (40, 12, 8, 6, 3, (0, 5)),
                                             (9, 4, 3, 1, 1, ())])
def test_per_token_definition_equals_grouped_loop(T, H, F, E, k, empty, a_round):
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=T, empty=empty)
    ref = moe.moe_forward_per_token(x, idx, prob, w1, w2, a_round)
    got = _grouped_layer(x, idx, prob, w1, w2, a_round)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def _pure_python_layer(x, idx, prob, w1, w2):
    """Brute force with scalar loops only (no numpy linear algebra)."""
    T, H = x.shape
    F = w2.shape[1]
    out = [[0.0] * H for _ in range(T)]
    for t in range(T):
        for j in range(idx.shape[1]):
            e = int(idx[t, j])
            h = [sum(float(x[t, i]) * float(w1[e, i, c]) for i in range(H)) for c in range(2 * F)]
            a = [h[f] / (1.0 + math.exp(-h[f])) * h[F + f] * float(prob[t, j]) for f in range(F)]
            for o in range(H):
                out[t][o] += sum(a[f] * float(w2[e, f, o]) for f in range(F))
    return np.array(out)


def test_brute_force_tiny_with_empty_expert():
    x, idx, prob, w1, w2 = _layer(8, 5, 4, 4, 2, seed=3, empty=(2,))
    assert not np.any(idx == 2)
    ref = _pure_python_layer(x, idx, prob, w1, w2)
    got = _grouped_layer(x, idx, prob, w1, w2, "f64")
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_single_expert_reduces_to_dense_swiglu_mlp():
    # E=1, k=1: p = 1 and the layer is the textbook SwiGLU MLP, checked with torch fp64
    x, idx, prob, w1, w2 = _layer(32, 16, 12, 1, 1, seed=9)
    assert np.all(prob == 1.0)
    xt, w1t, w2t = (torch.from_numpy(a) for a in (x, w1[0], w2[0]))
    ref = (torch.nn.functional.silu(xt @ w1t[:, :12]) * (xt @ w1t[:, 12:])) @ w2t
    got = _grouped_layer(x, idx, prob, w1, w2, "f64")
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_round_to_bf16_matches_torch_cast():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.normal(size=5000), rng.normal(size=5000) * 1e-30,
                        rng.normal(size=5000) * 1e20, [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(moe.round_to_bf16(v32.astype(np.float64)), ref)


def _torch_layer_grads(x, idx, prob, w1, w2, dy):
    """Autograd of the per-expert loop written with torch fp64 ops."""
    T, k = idx.shape
    E, F = w2.shape[0], w2.shape[1]
    row_map, split, _ = moe.permute_index(idx, E)
    xp = torch.tensor(moe.permute_rows(x, row_map, k), requires_grad=True)
    pp = torch.tensor(moe.permute_probs(prob, row_map), requires_grad=True)
    w1t = torch.tensor(w1, requires_grad=True)
    w2t = torch.tensor(w2, requires_grad=True)
    outs = []
    s = 0
    for e, n in enumerate(split):
        h = xp[s:s + n] @ w1t[e]
        a = torch.nn.functional.silu(h[:, :F]) * h[:, F:] * pp[s:s + n, None]
        outs.append(a @ w2t[e])
        s += n
    yp = torch.cat(outs)
    dyp = torch.tensor(moe.permute_rows(dy, row_map, k))
    (yp * dyp).sum().backward()
    return xp.grad.numpy(), w1t.grad.numpy(), w2t.grad.numpy(), pp.grad.numpy(), split, dyp.numpy(), \
        xp.detach().numpy(), pp.detach().numpy(), row_map


@pytest.mark.parametrize("T,H,F,E,k", [(12, 6, 4, 3, 2), (30, 8, 8, 5, 3)])
def test_backward_matches_torch_autograd(T, H, F, E, k):
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=T + 1, empty=(E - 1,))
    dy = np.random.default_rng(4).normal(size=(T, H))
    gx, gw1, gw2, gp, split, dyp, xp, pp, row_map = _torch_layer_grads(x, idx, prob, w1, w2, dy)
    dxp, dw1, dw2, dpp, _ = moe.grouped_mlp_bwd(dyp, xp, split, w1, w2, pp, a_round="f64")
    for got, ref in ((dxp, gx), (dw1, gw1), (dw2, gw2), (dpp, gp)):
        np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
    assert np.all(dw1[E - 1] == 0) and np.all(dw2[E - 1] == 0)    # empty expert: zero grads
    dx, dprob = moe.moe_backward_tokens(dxp, dpp, row_map, T, k)
    assert dx.shape == (T, H) and dprob.shape == (T, k)


def test_backward_matches_finite_differences():
    T, H, F, E, k = 6, 4, 3, 2, 2
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=21)
    row_map, split, _ = moe.permute_index(idx, E)
    xp = moe.permute_rows(x, row_map, k)
    pp = moe.permute_probs(prob, row_map)
    dy = np.random.default_rng(8).normal(size=xp.shape)

    def loss(xp_, w1_, w2_, pp_):
        yp, _, _ = moe.grouped_mlp_fwd(xp_, split, w1_, w2_, pp_, a_round="f64")
        return float(np.sum(yp * dy))

    dxp, dw1, dw2, dpp, _ = moe.grouped_mlp_bwd(dy, xp, split, w1, w2, pp, a_round="f64")
    eps = 1e-6
    for arr, grad, at in ((xp, dxp, (3, 2)), (w1, dw1, (1, 2, 5)), (w2, dw2, (0, 1, 3)), (pp, dpp, (4,))):
        args = [xp, w1, w2, pp]
        pos = [a is arr for a in args].index(True)
        plus = [a.copy() for a in args]
        minus = [a.copy() for a in args]
        plus[pos][at] += eps
        minus[pos][at] -= eps
        fd = (loss(*plus) - loss(*minus)) / (2 * eps)
        assert abs(fd - grad[at]) <= 1e-7 * max(1.0, abs(fd))


def test_mxfp8_grouped_equals_per_token_on_quantised_operands():
    T, H, F, E, k = 24, 64, 64, 3, 2
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=31)
    xc, xs = mxfp8.quantize(x, axis=0)
    w1c, w1s = moe.quantize_weights_kmajor(w1, "rows")           # [E, 2F, H]
    w2c, w2s = moe.quantize_weights_kmajor(w2, "rows")           # [E, H, F]
    row_map, split, _ = moe.permute_index(idx, E)
    xpc = moe.permute_rows(xc, row_map, k)
    xps = moe.permute_rows(xs, row_map, k)
    pp = moe.permute_probs(prob, row_map)
    yp, ac, asc, _ = moe.grouped_mlp_fwd_mxfp8(xpc, xps, split, w1c, w1s, w2c, w2s, pp)
    got = moe.unpermute(yp, row_map, T, k)
    # definition (per token) on the dequantised operands with `a` rounded to MXFP8
    xq = mxfp8.dequantize(xc, xs, axis=0)
    w1q = np.swapaxes(mxfp8.dequantize_blocks_last_axis(w1c, w1s), 1, 2)
    w2q = np.swapaxes(mxfp8.dequantize_blocks_last_axis(w2c, w2s), 1, 2)
    ref = moe.moe_forward_per_token(xq, idx, prob, w1q, w2q, a_round="mxfp8")
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))
    # feeding the layer's own quantised `a` back in reproduces the same output
    yp2, _, _, _ = moe.grouped_mlp_fwd_mxfp8(xpc, xps, split, w1c, w1s, w2c, w2s, pp, ac, asc)
    assert np.array_equal(yp, yp2)


def test_sampled_forward_equals_per_token_definition():
    x, idx, prob, w1, w2 = _layer(30, 8, 6, 4, 2, seed=41)
    toks = np.array([0, 3, 7, 29])
    ref = moe.moe_forward_per_token(x, idx, prob, w1, w2, "bf16", tokens=toks)
    got = moe.moe_forward_sampled(x, idx, prob, w1, w2, toks, "bf16")
    assert np.max(np.abs(got - ref)) <= 1e-13 * np.max(np.abs(ref))


def test_mxfp8_backward_close_to_exact_backward():
    # the MXFP8 backward is the exact backward up to MXFP8 quantisation error (catches
    # transposed operands, wrong terms or mixed-up axes, which give O(1) differences)
    T, H, F, E, k = 40, 64, 64, 3, 2
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=51)
    row_map, split, _ = moe.permute_index(idx, E)
    xp = moe.permute_rows(x, row_map, k)
    pp = moe.permute_probs(prob, row_map)
    _, h, _ = moe.grouped_mlp_fwd(xp, split, w1, w2, pp, a_round="f64")
    dy = np.random.default_rng(3).normal(size=xp.shape)
    ref = moe.grouped_mlp_bwd(dy, xp, split, w1, w2, pp, a_round="f64")
    got = moe.grouped_mlp_bwd_mxfp8(dy, xp, split, w1, w2, pp, h)
    for g, r in zip(got[:4], ref[:4]):
        rel = np.max(np.abs(g - r)) / np.max(np.abs(r))
        assert rel < 0.08, rel
    # dh before quantisation is the exact SwiGLU backward of the quantised da
    assert got[4].shape == (xp.shape[0], 2 * F)
    assert np.allclose(got[5], moe.silu(h[:, :F]) * h[:, F:] * pp[:, None])


def test_sampled_backward_equals_full_backward():
    rng = np.random.default_rng(0)
    T, H, F, E, k = 30, 16, 8, 3, 2
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=61)
    rm, split, _ = moe.permute_index(idx, E)
    xp = moe.permute_rows(x, rm, k)
    pp = moe.permute_probs(prob, rm)
    dy = rng.normal(size=xp.shape)
    ref = moe.grouped_mlp_bwd(dy, xp, split, w1, w2, pp, a_round="bf16")
    rows, c1, c2 = np.array([0, 5, 17, 59]), [0, 3, 7], [1, 2]
    dxp, dpp, dw1, dw2 = moe.bwd_sampled_bf16(dy, xp, split, w1, w2, pp, rows, [0, 2], c1, c2)
    assert np.allclose(dxp, ref[0][rows], rtol=0, atol=1e-12) and np.allclose(dpp, ref[3][rows], atol=1e-12)
    assert np.allclose(dw1[2], ref[1][2][:, c1], atol=1e-12) and np.allclose(dw2[0], ref[2][0][:, c2], atol=1e-12)


def test_sampled_mxfp8_backward_equals_full_mxfp8_backward():
    rng = np.random.default_rng(1)
    T, H, F, E, k = 40, 64, 64, 3, 2
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=71)
    rm, split, _ = moe.permute_index(idx, E)
    xp = moe.permute_rows(x, rm, k)
    pp = moe.permute_probs(prob, rm)
    _, h, _ = moe.grouped_mlp_fwd(xp, split, w1, w2, pp, a_round="f64")
    dy = rng.normal(size=xp.shape)
    full = moe.grouped_mlp_bwd_mxfp8(dy, xp, split, w1, w2, pp, h)
    dh, a = full[4], full[5]
    rows = np.array([1, 7, 33, 79])
    cols = ([3, 9], [0, 63], [5, 6], [2, 100])
    s = moe.bwd_sampled_mxfp8(dy, xp, split, w1, w2, pp, h, dh, a, rows, [0, 1, 2], cols)
    assert np.allclose(s["dxp"], full[0][rows], atol=1e-12) and np.allclose(s["dp"], full[3][rows], atol=1e-12)
    assert np.allclose(s["dh"], full[4][rows], atol=1e-12)
    for e in range(3):
        assert np.allclose(s["dw2"][e], full[2][e][np.ix_(cols[0], cols[1])], atol=1e-12)
        assert np.allclose(s["dw1"][e], full[1][e][np.ix_(cols[2], cols[3])], atol=1e-12)


def test_mxfp8_forward_rows_equal_grouped_forward():
    T, H, F, E, k = 24, 64, 64, 3, 2
    x, idx, prob, w1, w2 = _layer(T, H, F, E, k, seed=81)
    rm, split, _ = moe.permute_index(idx, E)
    xc, xs = mxfp8.quantize(x, axis=0)
    w1c, w1s = moe.quantize_weights_kmajor(w1, "rows")
    w2c, w2s = moe.quantize_weights_kmajor(w2, "rows")
    yp, ac, asc, _ = moe.grouped_mlp_fwd_mxfp8(moe.permute_rows(xc, rm, k), moe.permute_rows(xs, rm, k), split,
                                               w1c, w1s, w2c, w2s, moe.permute_probs(prob, rm))
    # rows of token t, slot j live at rm[t*k + j]
    toks = np.repeat(np.arange(T), k)
    rows = rm
    ypr, c, s = moe.fwd_rows_mxfp8(x[toks], prob.reshape(-1), idx.reshape(-1), w1, w2)
    assert np.allclose(ypr, yp[rows], atol=1e-12) and np.array_equal(c, ac[rows]) and np.array_equal(s, asc[rows])


# ------------------------------------------------------------ capacity-padded dispatch
def test_capacity_keep_is_first_C_slots_per_expert():
    rng = np.random.default_rng(12)
    T, E, k = 50, 5, 2
    idx, _ = moe.route(rng.normal(size=(T, E)) + np.array([2.0, 1.0, 0, 0, -3.0]), k)
    for C in (0, 1, 7, 20, 100):
        keep = moe.capacity_keep(idx, E, C)
        flat, kf = idx.reshape(-1), keep.reshape(-1)
        for e in range(E):
            slots = np.nonzero(flat == e)[0]               # ascending slot order
            assert np.array_equal(np.nonzero(kf & (flat == e))[0], slots[:C])
        assert kf.sum() == sum(min(int((flat == e).sum()), C) for e in range(E))


def test_capacity_forward_special_cases():
    x, idx, prob, w1, w2 = _layer(24, 8, 6, 4, 2, seed=13)
    ref = moe.moe_forward_per_token(x, idx, prob, w1, w2, "f64")
    # a capacity that holds every slot is the dropless layer
    big = moe.moe_forward_capacity(x, idx, prob, w1, w2, C=24 * 2, a_round="f64")
    np.testing.assert_allclose(big, ref, rtol=1e-13, atol=1e-13)
    # no capacity: nothing is computed
    assert np.all(moe.moe_forward_capacity(x, idx, prob, w1, w2, C=0, a_round="f64") == 0)
    # a dropped slot is the same as a zero routing probability (p scales a inside ScaledSwiGLU)
    keep = moe.capacity_keep(idx, 4, 5)
    assert not keep.all()
    got = moe.moe_forward_capacity(x, idx, prob, w1, w2, C=5, a_round="f64")
    np.testing.assert_allclose(got, moe.moe_forward_per_token(x, idx, np.where(keep, prob, 0.0), w1, w2, "f64"),
                               rtol=1e-13, atol=1e-13)
