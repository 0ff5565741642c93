"""Routing, permutation, grouped expert MLP (forward and backward) — fp64 oracle.

Test infrastructure only (see the package docstring). Pages and sections followed:

* routing and combine — "Efficient MoE training for biological foundation models"
  (sitech.ge, introduction and section "Grouped experts instead of a Python loop"):
  each token is sent to a few experts and their outputs are weighted by the routing
  weights, which the fused GroupedMLP kernel applies itself;
* grouping — same section, and news.bpdata.com section 1): tokens are grouped per
  expert and the grouped GEMM takes per-expert token counts (``split_sizes``); the
  result equals running every expert in a loop. "NeMo AutoModel" (seventnews.com,
  section on Transformers v5 expert back-ends): ``grouped_mm`` runs on tokens sorted by
  expert;
* fused chain — news.bpdata.com section 3): GroupedLinear -> ScaledSwiGLU ->
  GroupedLinear; sitech.ge section "Reducing memory and quantisation cost": the
  backward pass has a fused counterpart.

Readings where the pages are silent:
  * router input is fp32 logits [T, E]; softmax over all E experts; the k experts with
    the largest logits are selected (ties -> lower expert index), slot j holds the
    j-th largest; with ``renorm`` the k selected probabilities are divided by their sum;
  * permutation is a stable counting sort of the T*k slots (flat slot s = t*k + j) by
    expert: ``row_map[s]`` is the slot's row in the expert-contiguous order, rows of one
    expert keep ascending slot order; ``split_sizes[e]`` counts them, ``offsets`` is
    their exclusive prefix sum (length E+1);
  * w1[e] is [H, 2F] with gate columns [0, F) and up columns [F, 2F); w2[e] is [F, H];
  * ScaledSwiGLU: a = SiLU(gate) * up * p with SiLU(z) = z / (1 + exp(-z)) and p the
    slot's routing probability; the probability is applied there only, so the combine
    that follows sums the k expert outputs with weight 1;
  * the BF16 path stores ``a`` in bf16 (round to nearest even) before fc2; the oracle
    reproduces that rounding when ``a_round="bf16"``; everything else stays fp64.
"""
from __future__ import annotations

import numpy as np

from . import fp8, mxfp8


# ----------------------------------------------------------------------------- helpers
def round_to_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even (fp64 result)."""
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)                             # |v| in [2**(ex-1), 2**ex)
    q = np.ldexp(1.0, np.maximum(ex.astype(np.int64) - 8, -133))   # bf16 spacing
    return np.where(v == 0.0, v, np.rint(v / q) * q)


def silu(z):
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def silu_grad(z):
    """d/dz SiLU(z) = s(z) * (1 + z * (1 - s(z))) with s the logistic sigmoid."""
    z = np.asarray(z, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def f64(t) -> np.ndarray:
    """Any CPU tensor or array as float64 numpy."""
    if hasattr(t, "detach"):
        import torch
        return t.detach().to(torch.float64).cpu().numpy()
    return np.asarray(t, dtype=np.float64)


# ----------------------------------------------------------------------------- routing
def route(logits, k: int, renorm: bool = True):
    """Top-k router softmax. Returns idx int32 [T, k] and prob float64 [T, k]."""
    lg = f64(logits)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    m = lg.max(axis=1, keepdims=True)
    ex = np.exp(lg - m)
    soft = ex / ex.sum(axis=1, keepdims=True)
    # stable sort of the negated logits: largest first, equal logits keep index order
    order = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    prob = np.take_along_axis(soft, order, axis=1)
    if renorm:
        prob = prob / prob.sum(axis=1, keepdims=True)
    return order.astype(np.int32), prob


def route_bwd(logits, idx, dprob, renorm: bool = True) -> np.ndarray:
    """Gradient of the router's probabilities with respect to its logits.

    The forward's steps, in order (``route``): s = softmax(l) over all E experts; the
    selected probabilities q_j = s[idx_j]; with ``renorm`` p_j = q_j / Z, Z = sum_j q_j
    (else p_j = q_j). Given dL/dp_j (``dprob`` [T, k]) and the forward's ``idx``, the
    chain rule runs those steps backwards:
        renorm:  dq_j = (dprob_j - sum_m dprob_m p_m) / Z      else  dq_j = dprob_j
        gather:  ds_b = sum_j [idx_j == b] dq_j
        softmax: dl_b = s_b * (ds_b - sum_c ds_c s_c)
    Returns dlogits float64 [T, E]. The routing weights are what trains the router: each
    token's expert outputs are weighted by them (sitech.ge, introduction).
    """
    lg = f64(logits)
    idx = np.asarray(idx, dtype=np.int64)
    dp = f64(dprob)
    T, E = lg.shape
    m = lg.max(axis=1, keepdims=True)
    ex = np.exp(lg - m)
    soft = ex / ex.sum(axis=1, keepdims=True)
    q = np.take_along_axis(soft, idx, axis=1)
    if renorm:
        Z = q.sum(axis=1, keepdims=True)
        p = q / Z
        dq = (dp - np.sum(dp * p, axis=1, keepdims=True)) / Z
    else:
        dq = dp
    ds = np.zeros((T, E))
    for j in range(idx.shape[1]):
        ds[np.arange(T), idx[:, j]] += dq[:, j]
    return soft * (ds - np.sum(ds * soft, axis=1, keepdims=True))


# ------------------------------------------------------------------------- permutation
def permute_index(idx, E: int):
    """Stable counting sort of the flat slots by expert.

    Returns row_map int32 [T*k], split_sizes int32 [E], offsets int32 [E+1].
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert index out of range")
    split_sizes = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(split_sizes)])
    order = np.argsort(flat, kind="stable")          # slots in expert-contiguous order
    row_map = np.empty(flat.size, dtype=np.int64)
    row_map[order] = np.arange(flat.size)
    return row_map.astype(np.int32), split_sizes.astype(np.int32), offsets.astype(np.int32)


def permute_rows(x, row_map, k: int) -> np.ndarray:
    """xp[row_map[t*k + j]] = x[t] (works on any dtype; rows are copied unchanged)."""
    x = np.asarray(x)
    row_map = np.asarray(row_map, dtype=np.int64)
    R = row_map.size
    xp = np.empty((R,) + x.shape[1:], dtype=x.dtype)
    xp[row_map] = np.repeat(x, k, axis=0)
    return xp


def permute_probs(prob, row_map) -> np.ndarray:
    pp = np.empty(np.asarray(row_map).size, dtype=np.float64)
    pp[np.asarray(row_map, dtype=np.int64)] = f64(prob).reshape(-1)
    return pp


def unpermute(yp, row_map, T: int, k: int, prob=None) -> np.ndarray:
    """out[t] = sum_j w_tj * yp[row_map[t*k + j]], w = 1 unless ``prob`` is given."""
    yp = f64(yp)
    rm = np.asarray(row_map, dtype=np.int64).reshape(T, k)
    out = np.zeros((T,) + yp.shape[1:], dtype=np.float64)
    for j in range(k):
        w = 1.0 if prob is None else f64(prob)[:, j][:, None]
        out += w * yp[rm[:, j]]
    return out


# ------------------------------------------------------------- capacity-padded dispatch
def capacity_keep(idx, E: int, C: int) -> np.ndarray:
    """Capacity-padded dispatch: every expert takes at most C of the slots routed to it,
    the first ones in flat slot order s = t*k + j; later slots are dropped (the padded
    ``batched_mm`` expert back-end of Transformers v5 named on the "NeMo AutoModel" page,
    section on Transformers v5 features, runs one batched GEMM over [E, C] rows).
    Returns keep, bool [T, k]."""
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    keep = np.zeros(flat.size, dtype=bool)
    taken = np.zeros(E, dtype=np.int64)
    for s, e in enumerate(flat):
        if taken[e] < C:
            keep[s] = True
            taken[e] += 1
    return keep.reshape(np.asarray(idx).shape)


def moe_forward_capacity(x, idx, prob, w1, w2, C: int, a_round="bf16") -> np.ndarray:
    """The layer with expert capacity C: out[t] = sum over the token's KEPT slots j of
    (SiLU(x_t W1g_e) * (x_t W1u_e) * p_tj) W2_e; a dropped slot contributes nothing."""
    x = f64(x)
    idx = np.asarray(idx, dtype=np.int64)
    prob = f64(prob)
    w1 = f64(w1)
    w2 = f64(w2)
    F = w2.shape[1]
    keep = capacity_keep(idx, w1.shape[0], C)
    out = np.zeros((x.shape[0], x.shape[1]))
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            if not keep[t, j]:
                continue
            e = idx[t, j]
            h = x[t] @ w1[e]
            out[t] += _round_a(silu(h[:F]) * h[F:] * prob[t, j], a_round) @ w2[e]
    return out


# -------------------------------------------------------------------- expert MLP (fwd)
def _round_a(a, a_round):
    if a_round is None or a_round == "f64":
        return a
    if a_round == "bf16":
        return round_to_bf16(a)
    if a_round == "mxfp8":
        codes, scales = mxfp8.quantize_blocks_last_axis(a)
        return mxfp8.dequantize_blocks_last_axis(codes, scales)
    raise ValueError(a_round)


def moe_forward_per_token(x, idx, prob, w1, w2, a_round="bf16", tokens=None) -> np.ndarray:
    """Definition of the layer, one token at a time, no permutation.

    out[t] = sum_j ( SiLU(x_t W1g_e) * (x_t W1u_e) * p_tj ) W2_e, with e = idx[t, j].
    ``tokens`` restricts the computation to those token indices (rows of the result
    follow that order).
    """
    x = f64(x)
    idx = np.asarray(idx, dtype=np.int64)
    prob = f64(prob)
    w1 = f64(w1) if not isinstance(w1, list) else w1
    w2 = f64(w2) if not isinstance(w2, list) else w2
    F = w2[0].shape[0]
    toks = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens, dtype=np.int64)
    out = np.zeros((toks.size, x.shape[1]), dtype=np.float64)
    for n, t in enumerate(toks):
        for j in range(idx.shape[1]):
            e = idx[t, j]
            h = x[t] @ w1[e]
            a = silu(h[:F]) * h[F:] * prob[t, j]
            out[n] += _round_a(a, a_round) @ w2[e]
    return out


def grouped_mlp_fwd(xp, split_sizes, w1, w2, probs_perm, a_round="bf16"):
    """The per-expert loop over expert-contiguous rows (grouped GEMM semantics).

    Returns (yp [R,H], h [R,2F], a [R,F]) in float64; ``a`` carries the path rounding.
    """
    xp = f64(xp)
    w1 = f64(w1)
    w2 = f64(w2)
    pp = f64(probs_perm)
    R, H = xp.shape
    F = w2.shape[1]
    yp = np.zeros((R, w2.shape[2]), dtype=np.float64)
    hh = np.zeros((R, 2 * F), dtype=np.float64)
    aa = np.zeros((R, F), dtype=np.float64)
    start = 0
    for e, n in enumerate(np.asarray(split_sizes, dtype=np.int64)):
        rows = slice(start, start + n)
        h = xp[rows] @ w1[e]
        a = _round_a(silu(h[:, :F]) * h[:, F:] * pp[rows, None], a_round)
        yp[rows] = a @ w2[e]
        hh[rows] = h
        aa[rows] = a
        start += n
    if start != R:
        raise ValueError("split_sizes must sum to the number of rows")
    return yp, hh, aa


def grouped_mlp_bwd(dy_perm, xp, split_sizes, w1, w2, probs_perm, a_round="bf16"):
    """Analytic gradient of :func:`grouped_mlp_fwd` with respect to xp, w1, w2, probs_perm.

    Per expert e (rows of the group, a = SiLU(g) * u * p):
        da = dy W2_e^T;  dg = da * p * u * SiLU'(g);  du = da * p * SiLU(g);
        dp = sum_f da * SiLU(g) * u;  dW2_e = a^T dy;  dxp = [dg|du] W1_e^T;
        dW1_e = xp^T [dg|du].
    Returns (dxp [R,H], dw1 [E,H,2F], dw2 [E,F,H], dprobs_perm [R], dh [R,2F]).
    """
    dy = f64(dy_perm)
    xp = f64(xp)
    w1 = f64(w1)
    w2 = f64(w2)
    pp = f64(probs_perm)
    R, H = xp.shape
    E, F = w2.shape[0], w2.shape[1]
    dxp = np.zeros_like(xp)
    dw1 = np.zeros_like(w1)
    dw2 = np.zeros_like(w2)
    dpp = np.zeros(R, dtype=np.float64)
    dhh = np.zeros((R, 2 * F), dtype=np.float64)
    start = 0
    for e, n in enumerate(np.asarray(split_sizes, dtype=np.int64)):
        rows = slice(start, start + n)
        h = xp[rows] @ w1[e]
        g, u = h[:, :F], h[:, F:]
        p = pp[rows, None]
        a = _round_a(silu(g) * u * p, a_round)
        da = dy[rows] @ w2[e].T
        dg = da * p * u * silu_grad(g)
        du = da * p * silu(g)
        dpp[rows] = np.sum(da * silu(g) * u, axis=1)
        dh = np.concatenate([dg, du], axis=1)
        dw2[e] = a.T @ dy[rows]
        dxp[rows] = dh @ w1[e].T
        dw1[e] = xp[rows].T @ dh
        dhh[rows] = dh
        start += n
    return dxp, dw1, dw2, dpp, dhh


def moe_backward_tokens(dx_perm, dprobs_perm, row_map, T: int, k: int):
    """dx[t] = sum_j dxp[row_map[t*k+j]];  dprob[t, j] = dprobs_perm[row_map[t*k+j]]."""
    dx = unpermute(dx_perm, row_map, T, k)
    dprob = f64(dprobs_perm)[np.asarray(row_map, dtype=np.int64)].reshape(T, k)
    return dx, dprob


# ------------------------------------------------------------------ MXFP8 expert MLP
def quantize_weights_kmajor(w, along: str):
    """MXFP8 codes of stacked expert weights, transposed so the contraction axis is last.

    ``w1`` [E, H, 2F] quantised along H gives codes [E, 2F, H] (``along="rows"``);
    the same call serves w2 [E, F, H] along F, giving [E, H, F].
    """
    if along != "rows":
        raise ValueError(along)
    return mxfp8.quantize(f64(w), axis=1, transpose_out=True)


def grouped_mlp_fwd_mxfp8(xp_codes, xp_scales, split_sizes, w1_codes, w1_scales, w2_codes,
                          w2_scales, probs_perm, a_codes=None, a_scales=None):
    """MXFP8 forward on quantised operands, computed in float64.

    xp codes [R,H] / scales [R,H/32] (blocks along H); w1 codes [E,2F,H] / scales
    [E,2F,H/32]; w2 codes [E,H,F] / scales [E,H,F/32]. The fc1 epilogue output
    a = SiLU(g)*u*p is quantised along F with the same rule, unless ``a_codes`` /
    ``a_scales`` (an externally produced quantised ``a``) are given, in which case fc2
    runs on those. Returns (yp [R,H], a_codes, a_scales, h [R,2F]).
    """
    xq = mxfp8.dequantize_blocks_last_axis(xp_codes, xp_scales)
    w1q = mxfp8.dequantize_blocks_last_axis(w1_codes, w1_scales)     # [E, 2F, H]
    w2q = mxfp8.dequantize_blocks_last_axis(w2_codes, w2_scales)     # [E, H, F]
    pp = f64(probs_perm)
    R = xq.shape[0]
    E, H, F = w2q.shape
    h_all = np.zeros((R, 2 * F))
    a_all = np.zeros((R, F))
    start = 0
    for e, n in enumerate(np.asarray(split_sizes, dtype=np.int64)):
        rows = slice(start, start + n)
        h = xq[rows] @ w1q[e].T
        h_all[rows] = h
        a_all[rows] = silu(h[:, :F]) * h[:, F:] * pp[rows, None]
        start += n
    if a_codes is None:
        a_codes, a_scales = mxfp8.quantize_blocks_last_axis(a_all)
    aq = mxfp8.dequantize_blocks_last_axis(a_codes, a_scales)
    yp = np.zeros((R, H))
    start = 0
    for e, n in enumerate(np.asarray(split_sizes, dtype=np.int64)):
        rows = slice(start, start + n)
        yp[rows] = aq[rows] @ w2q[e].T
        start += n
    return yp, a_codes, a_scales, h_all


def moe_forward_sampled(x, idx, prob, w1, w2, tokens, a_round="bf16") -> np.ndarray:
    """The per-token definition restricted to ``tokens``, computed expert by expert.

    Same sum as :func:`moe_forward_per_token` (the k terms of a token are added in slot
    order j = 0..k-1), but each expert's weights are converted to float64 once, so the
    full-size layers fit in host memory. ``w1``/``w2`` may be bf16 CPU tensors.
    """
    toks = np.asarray(tokens, dtype=np.int64)
    idx = np.asarray(idx, dtype=np.int64)[toks]
    prob = f64(prob)[toks]
    xs = f64(x[toks]) if hasattr(x, "detach") else f64(x)[toks]
    E = w1.shape[0]
    F = w2.shape[1]
    terms = np.zeros((idx.shape[1], toks.size, xs.shape[1]), dtype=np.float64)
    for e in range(E):
        sel = np.nonzero(idx == e)
        if sel[0].size == 0:
            continue
        w1e = f64(w1[e])
        w2e = f64(w2[e])
        n, j = sel
        h = xs[n] @ w1e
        a = _round_a(silu(h[:, :F]) * h[:, F:] * prob[n, j][:, None], a_round)
        terms[j, n] = a @ w2e
    out = np.zeros((toks.size, xs.shape[1]), dtype=np.float64)
    for j in range(idx.shape[1]):
        out += terms[j]
    return out


def grouped_mlp_bwd_mxfp8(dy_perm, xp, split_sizes, w1, w2, probs_perm, h, dh=None, a=None, dh_wgrad=None):
    """Backward of the MXFP8 layer: every GEMM on operands quantised along its own
    contraction axis, computed in float64.

    fc2 dgrad: dy along H times w2 along H (transposed);  fc2 wgrad: a and dy along rows
    (32-row blocks restarting at each expert);  fc1 dgrad: dh along 2F times w1 along 2F;
    fc1 wgrad: xp and dh along rows. h = [g | u] is the forward's saved pre-activation.
    dh and the recomputed a are quantised from their exact values (the fused backward
    quantises them in the kernel that computes them; they are never stored at a lower
    precision first). ``a`` is the forward's fc1 output (a fused forward quantises it
    along rows for this GEMM in its own epilogue); by default it is recomputed from h.
    ``dh`` / ``a`` replace those values (e.g. by the dequantised codes a GPU produced,
    which quantise to themselves along their own axis); ``dh_wgrad`` replaces dh for the
    fc1 weight gradient only (default: ``dh``).
    Returns (dxp, dw1, dw2, dprobs_perm, dh_exact, a_exact).
    """
    dy = f64(dy_perm)
    xp = f64(xp)
    w1 = f64(w1)
    w2 = f64(w2)
    pp = f64(probs_perm)
    h = f64(h)
    split = np.asarray(split_sizes, dtype=np.int64)
    E, F, H = w2.shape
    w2q = mxfp8.dequantize(*mxfp8.quantize(w2, axis=0), axis=0)        # [E, F, H] along H
    w1q = mxfp8.dequantize(*mxfp8.quantize(w1, axis=0), axis=0)        # [E, H, 2F] along 2F
    dyq = mxfp8.dequantize(*mxfp8.quantize(dy, axis=0), axis=0)        # along H
    da = np.zeros((dy.shape[0], F))
    start = 0
    for e, n in enumerate(split):
        da[start:start + n] = dyq[start:start + n] @ w2q[e].T
        start += n
    g, u = h[:, :F], h[:, F:]
    p = pp[:, None]
    dh_exact = np.concatenate([da * p * u * silu_grad(g), da * p * silu(g)], axis=1)
    dprob = np.sum(da * silu(g) * u, axis=1)
    a_exact = silu(g) * u * p
    dh_use = dh_exact if dh is None else f64(dh)
    a_use = a_exact if a is None else f64(a)
    dh_w = dh_use if dh_wgrad is None else f64(dh_wgrad)
    deq_rows = lambda v: mxfp8.dequantize_grouped_rows(*mxfp8.quantize_grouped_rows(v, split), split)
    aq, dyc, xc, dhc = deq_rows(a_use), deq_rows(dy), deq_rows(xp), deq_rows(dh_w)
    dhq = mxfp8.dequantize(*mxfp8.quantize(dh_use, axis=0), axis=0)    # along 2F
    dxp = np.zeros_like(xp)
    dw1 = np.zeros_like(w1)
    dw2 = np.zeros_like(w2)
    start = 0
    for e, n in enumerate(split):
        rows = slice(start, start + n)
        dw2[e] = aq[rows].T @ dyc[rows]
        dxp[rows] = dhq[rows] @ w1q[e].T
        dw1[e] = xc[rows].T @ dhc[rows]
        start += n
    return dxp, dw1, dw2, dprob, dh_exact, a_exact


def expert_rows(split_sizes, e) -> slice:
    off = int(np.sum(np.asarray(split_sizes, dtype=np.int64)[:e]))
    return slice(off, off + int(np.asarray(split_sizes)[e]))


def bwd_sampled_bf16(dy_perm, xp, split_sizes, w1, w2, probs_perm, rows, experts, cols1, cols2):
    """Sampled entries of the BF16 backward (the analytic gradient of
    :func:`grouped_mlp_fwd` with `a` rounded to bf16), computed in float64:

    dxp and dprobs_perm for the permuted ``rows``; for every expert in ``experts``,
    dw2[e][:, cols2] and dw1[e][:, cols1] over all of that expert's rows.
    """
    split = np.asarray(split_sizes, dtype=np.int64)
    offs = np.concatenate([[0], np.cumsum(split)])
    F = w2.shape[1]

    def swiglu_bwd(rsel, e):
        x_r = f64(xp[rsel])
        w1e = f64(w1[e])
        w2e = f64(w2[e])
        h = x_r @ w1e
        g, u = h[:, :F], h[:, F:]
        p = f64(probs_perm[rsel])[:, None] if not isinstance(rsel, slice) else f64(probs_perm)[rsel][:, None]
        da = f64(dy_perm[rsel]) @ w2e.T
        dh = np.concatenate([da * p * u * silu_grad(g), da * p * silu(g)], axis=1)
        a = round_to_bf16(silu(g) * u * p)
        dp = np.sum(da * silu(g) * u, axis=1)
        return x_r, w1e, dh, a, dp

    rows = np.asarray(rows, dtype=np.int64)
    dxp = np.zeros((rows.size, xp.shape[1]))
    dpp = np.zeros(rows.size)
    for e in range(len(split)):
        sel = np.nonzero((rows >= offs[e]) & (rows < offs[e + 1]))[0]
        if sel.size == 0:
            continue
        _, w1e, dh, _, dp = swiglu_bwd(rows[sel], e)
        dxp[sel] = dh @ w1e.T
        dpp[sel] = dp
    dw1, dw2 = {}, {}
    for e in experts:
        rs = slice(int(offs[e]), int(offs[e + 1]))
        if rs.stop == rs.start:
            dw1[e] = np.zeros((xp.shape[1], len(cols1)))
            dw2[e] = np.zeros((F, len(cols2)))
            continue
        x_r, _, dh, a, _ = swiglu_bwd(rs, e)
        dw2[e] = a.T @ f64(dy_perm[rs])[:, cols2]
        dw1[e] = x_r.T @ dh[:, cols1]
    return dxp, dpp, dw1, dw2


def fwd_rows_mxfp8(x_rows, prob_rows, expert_of_rows, w1, w2, a_codes=None, a_scales=None, details=False):
    """MXFP8 forward of individual routed rows (x_rows[i] is the token's bf16 row routed
    to expert expert_of_rows[i] with probability prob_rows[i]), float64 on quantised
    operands. The oracle quantises x along H and each needed expert's weights along their
    contraction axis itself. fc2 runs on the oracle's own `a` codes unless ``a_codes`` /
    ``a_scales`` (rows x F, F/32) are given. Returns (yp, a_codes, a_scales); with
    ``details`` also a dict with fc1's exact output ``h`` [rows, 2F] and ``sum_abs``, the
    sum over H of |x_q * w1_q| per element of h (the magnitude an fp32 accumulation of
    that dot product is rounded against)."""
    xr = f64(x_rows)
    prob_rows = f64(prob_rows)
    experts = np.asarray(expert_of_rows, dtype=np.int64)
    F = w2.shape[1]
    xq = mxfp8.dequantize(*mxfp8.quantize(xr, axis=0), axis=0)
    yp = np.zeros((xr.shape[0], w2.shape[2]))
    own_c = np.zeros((xr.shape[0], F), dtype=np.uint8)
    own_s = np.zeros((xr.shape[0], F // 32), dtype=np.uint8)
    h_all = np.zeros((xr.shape[0], 2 * F)) if details else None
    sabs = np.zeros((xr.shape[0], 2 * F)) if details else None
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        w1q = mxfp8.dequantize(*mxfp8.quantize(f64(w1[e]), axis=1), axis=1)     # along H
        w2q = mxfp8.dequantize(*mxfp8.quantize(f64(w2[e]), axis=1), axis=1)     # along F
        hh = xq[sel] @ w1q
        if details:
            h_all[sel] = hh
            sabs[sel] = np.abs(xq[sel]) @ np.abs(w1q)
        a = silu(hh[:, :F]) * hh[:, F:] * prob_rows[sel, None]
        c, s = mxfp8.quantize(a, axis=0)
        own_c[sel], own_s[sel] = c, s
        if a_codes is None:
            aq = mxfp8.dequantize(c, s, axis=0)
        else:
            aq = mxfp8.dequantize(np.asarray(a_codes)[sel], np.asarray(a_scales)[sel], axis=0)
        yp[sel] = aq @ w2q
    if details:
        return yp, own_c, own_s, {"h": h_all, "sum_abs": sabs}
    return yp, own_c, own_s


def bwd_sampled_mxfp8(dy_perm, xp, split_sizes, w1, w2, probs_perm, h, dh, a, rows, experts, cols, dh_wgrad=None):
    """Sampled entries of :func:`grouped_mlp_bwd_mxfp8`, float64 on quantised operands.

    For the permuted ``rows``: dh_exact (from dy along H and w2 along H), dprobs, and dxp
    (from ``dh`` along 2F and w1 along 2F). For every expert in ``experts`` and the column
    samples ``cols = (f_cols, h_cols, hh_cols, j_cols)``: dw2[e][f_cols][:, h_cols] (``a``
    and dy along the expert's rows) and dw1[e][hh_cols][:, j_cols] (xp and ``dh_wgrad``,
    default ``dh``, along rows). ``h`` is the forward's [g | u]; ``dh`` and ``a`` are the
    values the GEMMs consume (e.g. dequantised GPU codes), indexed as ``dh[rows]`` and
    ``a[rows_slice, cols]`` / ``dh_wgrad[rows_slice, cols]`` only.
    """
    split = np.asarray(split_sizes, dtype=np.int64)
    offs = np.concatenate([[0], np.cumsum(split)])
    F = w2.shape[1]
    rows = np.asarray(rows, dtype=np.int64)
    out = {"dh": np.zeros((rows.size, 2 * F)), "dp": np.zeros(rows.size), "dxp": np.zeros((rows.size, xp.shape[1]))}
    for e in range(len(split)):
        sel = np.nonzero((rows >= offs[e]) & (rows < offs[e + 1]))[0]
        if sel.size == 0:
            continue
        r = rows[sel]
        w2q = mxfp8.dequantize(*mxfp8.quantize(f64(w2[e]), axis=0), axis=0)      # [F, H] along H
        w1q = mxfp8.dequantize(*mxfp8.quantize(f64(w1[e]), axis=0), axis=0)      # [H, 2F] along 2F
        dyq = mxfp8.dequantize(*mxfp8.quantize(f64(dy_perm[r]), axis=0), axis=0)
        da = dyq @ w2q.T
        hh = f64(h[r])
        g, u = hh[:, :F], hh[:, F:]
        p = f64(probs_perm[r])[:, None]
        out["dh"][sel] = np.concatenate([da * p * u * silu_grad(g), da * p * silu(g)], axis=1)
        out["dp"][sel] = np.sum(da * silu(g) * u, axis=1)
        dhq = mxfp8.dequantize(*mxfp8.quantize(f64(dh[r]), axis=0), axis=0)
        out["dxp"][sel] = dhq @ w1q.T
    f_cols, h_cols, hh_cols, j_cols = cols
    out["dw2"], out["dw1"] = {}, {}
    for e in experts:
        rs = slice(int(offs[e]), int(offs[e + 1]))
        n = rs.stop - rs.start
        deq_rows = lambda v: mxfp8.dequantize_grouped_rows(*mxfp8.quantize_grouped_rows(v, [n]), [n])
        if n == 0:
            out["dw2"][e] = np.zeros((len(f_cols), len(h_cols)))
            out["dw1"][e] = np.zeros((len(hh_cols), len(j_cols)))
            continue
        out["dw2"][e] = deq_rows(f64(a[rs, f_cols])).T @ deq_rows(f64(dy_perm[rs][:, h_cols]))
        dhw = dh if dh_wgrad is None else dh_wgrad
        out["dw1"][e] = deq_rows(f64(xp[rs][:, hh_cols])).T @ deq_rows(f64(dhw[rs, j_cols]))
    return out


# ------------------------------------------------------------ per-tensor FP8 expert MLP
def grouped_mlp_fwd_fp8(xp, split_sizes, w1, w2, probs_perm, a_codes=None, a_scale=None):
    """The layer with per-tensor FP8 (current scaling, E4M3), float64 on quantised
    operands: xp one scale over all rows, each expert's w1[e] / w2[e] its own scale; the
    fc1 output a = SiLU(g) * u * p is stored in bf16 (its amax is only known once all of it
    exists) and quantised with one scale over [R, F], unless ``a_codes`` / ``a_scale`` (a
    GPU's) are given. Returns (yp, a_codes, a_scale, h)."""
    xq = fp8.qdq(f64(xp), "e4m3")
    w1 = f64(w1)
    w2 = f64(w2)
    pp = f64(probs_perm)
    E, F, H = w2.shape[0], w2.shape[1], w2.shape[2]
    w1q = np.stack([fp8.qdq(w1[e], "e4m3") for e in range(E)])
    w2q = np.stack([fp8.qdq(w2[e], "e4m3") for e in range(E)])
    R = xq.shape[0]
    h_all = np.zeros((R, 2 * F))
    a_all = np.zeros((R, F))
    start = 0
    for e, n in enumerate(np.asarray(split_sizes, dtype=np.int64)):
        rows = slice(start, start + n)
        h = xq[rows] @ w1q[e]
        h_all[rows] = h
        a_all[rows] = silu(h[:, :F]) * h[:, F:] * pp[rows, None]
        start += n
    if a_codes is None:
        a_codes, a_scale = fp8.quantize_tensor(round_to_bf16(a_all), "e4m3")
    aq = fp8.dequantize_tensor(a_codes, a_scale, "e4m3")
    yp = np.zeros((R, H))
    start = 0
    for e, n in enumerate(np.asarray(split_sizes, dtype=np.int64)):
        rows = slice(start, start + n)
        yp[rows] = aq[rows] @ w2q[e]
        start += n
    return yp, a_codes, a_scale, h_all


def grouped_mlp_bwd_fp8(dy_perm, xp, split_sizes, w1, w2, probs_perm, h, a_codes, a_scale, dh=None):
    """Backward of :func:`grouped_mlp_fwd_fp8`: gradients in E5M2 with one scale per
    tensor (dy over [R, H], dh over [R, 2F]), forward operands in E4M3 as in the forward
    (per-tensor scales have no axis, so the forward's codes of xp, a and the weights serve
    the backward's GEMMs too). dh is stored in bf16 before its quantisation unless ``dh``
    (e.g. a GPU's values) is given. Returns (dxp, dw1, dw2, dprobs_perm, dh_exact)."""
    dyq = fp8.qdq(f64(dy_perm), "e5m2")
    xq = fp8.qdq(f64(xp), "e4m3")
    aq = fp8.dequantize_tensor(a_codes, a_scale, "e4m3")
    w1 = f64(w1)
    w2 = f64(w2)
    pp = f64(probs_perm)
    h = f64(h)
    E, F = w2.shape[0], w2.shape[1]
    w1q = np.stack([fp8.qdq(w1[e], "e4m3") for e in range(E)])
    w2q = np.stack([fp8.qdq(w2[e], "e4m3") for e in range(E)])
    split = np.asarray(split_sizes, dtype=np.int64)
    da = np.zeros((dyq.shape[0], F))
    start = 0
    for e, n in enumerate(split):
        da[start:start + n] = dyq[start:start + n] @ w2q[e].T
        start += n
    g, u = h[:, :F], h[:, F:]
    p = pp[:, None]
    dh_exact = np.concatenate([da * p * u * silu_grad(g), da * p * silu(g)], axis=1)
    dprob = np.sum(da * silu(g) * u, axis=1)
    dhq = fp8.qdq(round_to_bf16(dh_exact) if dh is None else f64(dh), "e5m2")
    dxp = np.zeros_like(xq)
    dw1 = np.zeros_like(w1)
    dw2 = np.zeros_like(w2)
    start = 0
    for e, n in enumerate(split):
        rows = slice(start, start + n)
        dw2[e] = aq[rows].T @ dyq[rows]
        dxp[rows] = dhq[rows] @ w1q[e].T
        dw1[e] = xq[rows].T @ dhq[rows]
        start += n
    return dxp, dw1, dw2, dprob, dh_exact
