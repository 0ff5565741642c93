"""GPU parity of the MXFP8 backward: the grouped (row-wise, per-expert) quantiser bit for
bit, and each backward GEMM against the fp64 oracle on the same quantised operands.

The fc2-dgrad epilogue quantises dh = [dg | du] (along 2F and along the expert's rows),
and the forward's fc1 epilogue a along the expert's rows, from fp32: their codes and
scales may differ from the oracle's quantisation of the exact values only by
rounding-boundary flips within the fp32 error bound (tests/mx_checks.py). The other GEMMs are checked on the GPU's own
codes: dxp, dw1, dw2 (bf16) within 2e-3 * max|ref| plus their own bf16 storage rounding
(half an ulp, at most 2^-8 |ref|); dprobs (fp32) within 2e-3 * max|ref|.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
from oracle import mxfp8 as oq
import workloads
from tests.mx_checks import (assert_boundary_flips, boundary_flips_grouped_rows, dswiglu_fp32_error_bounds,
                             swiglu_fp32_error_bound)
from tests.gather import permuted
from tests.mx_layout import grouped_atoms_to_scales, grouped_scales_to_atoms, tile_atoms_to_plain

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def within(got, ref, name):
    g = got.float().cpu().numpy() if hasattr(got, "cpu") else np.asarray(got)
    bound = TOL * np.max(np.abs(ref)) + 2.0 ** -8 * np.abs(ref)
    bad = np.abs(g - ref) > bound
    assert not bad.any(), f"{name}: {bad.sum()} elements off, worst {np.max(np.abs(g - ref) - bound):.3e}"


@pytest.mark.parametrize("split", [[64, 0, 45, 7, 96, 300], [128, 128], [1, 2, 3, 250]])
@pytest.mark.parametrize("C", [128, 384])
def test_grouped_quantiser_bit_exact(split, C):
    rng = np.random.default_rng(sum(split) + C)
    R = sum(split)
    v = (rng.standard_normal((R, C), dtype=np.float32) * np.exp(rng.uniform(-8, 8, (1, C)))).astype(np.float32)
    x = torch.from_numpy(v).to(torch.bfloat16)
    codes, atoms = mb.mxfp8_quantize_grouped(x.to(DEV), torch.tensor(split, dtype=torch.int32, device=DEV))
    rc, rs = oq.quantize_grouped_rows(om.f64(x), split)
    assert np.array_equal(codes.cpu().numpy(), rc)
    ref_atoms = grouped_scales_to_atoms(rs, split, C)
    assert np.array_equal(atoms.cpu().numpy()[: ref_atoms.size], ref_atoms)
    assert mb.moe_device_status() == 0


BWD_CASES = [
    (256, 128, 256, 4, 2, ()),
    (600, 256, 384, 5, 2, (3,)),
    (300, 384, 256, 8, 2, (1, 6)),
    (300, 256, 256, 1, 1, ()),              # one expert
    (257, 256, 256, 5, 1, (0, 1, 2, 4)),    # every row on one expert
    (300, 256, 256, 4, 2, (0, 2)),          # every token on the same two experts
]


def fused_operands(layer, E, R, H, F, split):
    """The MXFP8 operands quantised inside the GEMM epilogues: dh along 2F (codes, plain
    scales) and dh along rows (codes, per-expert scales) from the fc2-dgrad epilogue (the
    backward workspace), a along rows from the fc1 epilogue (the forward's saved buffer)."""
    ws, saved = layer._bwd["ws"], layer.saved

    def part(buf, off, ncols, atoms_off=None):
        codes = buf[off: off + R * ncols].view(R, ncols).cpu().numpy()
        a0 = off + (R * ncols + 255) // 256 * 256 if atoms_off is None else atoms_off
        return codes, buf[a0:].cpu().numpy()

    dhr, dhr_at = part(ws, mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "mxfp8", 8), 2 * F)
    dhr_s, _, _ = tile_atoms_to_plain(dhr_at, split, 2 * F // 32)
    dhc, dhc_at = part(ws, mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "mxfp8", 9), 2 * F)
    ac, ac_at = part(saved, mb.grouped_mlp_saved_offset(E, R, H, F, "mxfp8", 3), F,
                     mb.grouped_mlp_saved_offset(E, R, H, F, "mxfp8", 4))
    return (dhr, dhr_s), (dhc, grouped_atoms_to_scales(dhc_at, split, 2 * F)), \
        (ac, grouped_atoms_to_scales(ac_at, split, F))


def forward_a(layer, d, split, F, H):
    """The forward's exact a (fp64 on the same MXFP8 operands) and its fp32 error bound,
    for the codes the fc1 epilogue quantised along rows."""
    xc, xs = layer.perm["xp"].cpu().numpy(), layer.perm["xp_scale"].cpu().numpy()
    w1c, w1s = om.quantize_weights_kmajor(d["w1"], "rows")
    w2c, w2s = om.quantize_weights_kmajor(d["w2"], "rows")
    pp = om.f64(layer.perm["probs_perm"].cpu())[:, None]
    _, _, _, h = om.grouped_mlp_fwd_mxfp8(xc, xs, split, w1c, w1s, w2c, w2s, pp[:, 0])
    xq = np.abs(oq.dequantize_blocks_last_axis(xc, xs))
    w1q = np.abs(oq.dequantize_blocks_last_axis(w1c, w1s))
    sabs = np.zeros((xq.shape[0], 2 * F))
    s0 = 0
    for e, n in enumerate(split):
        sabs[s0:s0 + n] = xq[s0:s0 + n] @ w1q[e].T
        s0 += n
    a = om.silu(h[:, :F]) * h[:, F:] * pp
    return a, swiglu_fp32_error_bound(h[:, :F], h[:, F:], pp, sabs[:, :F], sabs[:, F:], H)


def fused_bounds(dy, w2, split, h, pp, F, H):
    """fp32 error bounds of dg, du and a (see tests/mx_checks.py): |da| magnitudes from
    the oracle's own MXFP8 operands of fc2 dgrad (dy and w2 along H)."""
    dyq = np.abs(oq.dequantize(*oq.quantize(om.f64(dy), axis=0), axis=0))
    w2q = np.abs(oq.dequantize(*oq.quantize(om.f64(w2), axis=0), axis=0))
    sabs = np.zeros((dyq.shape[0], F))
    s0 = 0
    for e, n in enumerate(split):
        sabs[s0:s0 + n] = dyq[s0:s0 + n] @ w2q[e].T
        s0 += n
    hh = om.f64(h)
    p = om.f64(pp)[:, None]
    e_dg, e_du, e_a = dswiglu_fp32_error_bounds(hh[:, :F], hh[:, F:], p, sabs, H)
    return np.concatenate([e_dg, e_du], axis=1), e_a


def check_fused_backward(layer, d, E, R, H, F):
    """dh and a codes (boundary flips only, against the oracle's exact values), then the
    remaining GEMMs on the GPU's own codes (2e-3 + bf16 storage), dprobs (2e-3)."""
    split = layer.perm["split_sizes"].cpu().numpy()
    b = layer._bwd
    h = layer.saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F).cpu()
    row_map = layer.perm["row_map"]
    dy, xp = permuted(d["grad_out"], row_map, layer.k), permuted(d["x"], row_map, layer.k)
    pp = layer.perm["probs_perm"].cpu()
    (dhr, dhr_s), (dhc, dhc_s), (ac, ac_s) = fused_operands(layer, E, R, H, F, split)
    exact = om.grouped_mlp_bwd_mxfp8(dy, xp, split, d["w1"], d["w2"], pp, h)
    dh_exact = exact[4]
    err_dh, _ = fused_bounds(dy, d["w2"], split, h, pp, F, H)
    a_exact, err_a = forward_a(layer, d, split, F, H)
    assert_boundary_flips(dhr, dhr_s, dh_exact, "dh along 2F", err=err_dh)
    for name, (c, sc), ex, er in (("dh along rows", (dhc, dhc_s), dh_exact, err_dh),
                                  ("a along rows", (ac, ac_s), a_exact, err_a)):
        ok, rep = boundary_flips_grouped_rows(c, sc, ex, split, err=er)
        assert ok, f"{name}: {rep}"
    # the GEMMs that consume them, on the GPU's own codes
    dh_rows = oq.dequantize_blocks_last_axis(dhr, dhr_s)
    dh_cols = oq.dequantize_grouped_rows(dhc, dhc_s, split)
    a_cols = oq.dequantize_grouped_rows(ac, ac_s, split)
    ref = om.grouped_mlp_bwd_mxfp8(dy, xp, split, d["w1"], d["w2"], pp, h, dh=dh_rows, a=a_cols, dh_wgrad=dh_cols)
    rdxp, rdw1, rdw2, rdp = ref[:4]
    within(b["dxp"], rdxp, "dxp")
    within(b["dw1"], rdw1, "dw1")
    within(b["dw2"], rdw2, "dw2")
    gp = b["dprobs_perm"].cpu().numpy()
    assert np.max(np.abs(gp - rdp)) <= TOL * np.max(np.abs(rdp))
    return split


@pytest.mark.parametrize("T,H,F,E,k,empty", BWD_CASES)
def test_mxfp8_backward_parity(T, H, F, E, k, empty):
    bias = np.zeros(E)
    bias[list(empty)] = -1e4
    d = workloads.small_layer(T, H, F, E, k, seed=T + 11, with_grad=True, logits_bias=bias)
    layer = mb.MoEExpertLayer(T, H, F, E, k, precision="mxfp8", training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    dx, dw1, dw2, dprob = layer.backward(d["grad_out"].to(DEV))
    assert mb.moe_device_status() == 0
    split = check_fused_backward(layer, d, E, T * k, H, F)
    for e in empty:
        assert split[e] == 0
        assert torch.count_nonzero(dw1[e]) == 0 and torch.count_nonzero(dw2[e]) == 0


def test_mxfp8_backward_close_to_bf16_definition():
    """Reported, loosely gated: MXFP8 gradients against the unquantised definition."""
    T, H, F, E, k = 256, 256, 256, 4, 2
    d = workloads.small_layer(T, H, F, E, k, seed=3, with_grad=True)
    layer = mb.MoEExpertLayer(T, H, F, E, k, precision="mxfp8", training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    dx, dw1, dw2, dprob = layer.backward(d["grad_out"].to(DEV))
    ridx, rprob = om.route(d["logits"], k)
    row_map, split, _ = om.permute_index(ridx, E)
    xp = om.permute_rows(om.f64(d["x"]), row_map, k)
    pp = om.permute_probs(rprob, row_map)
    dyp = om.permute_rows(om.f64(d["grad_out"]), row_map, k)
    rdxp, rdw1, rdw2, rdpp, _ = om.grouped_mlp_bwd(dyp, xp, split, d["w1"], d["w2"], pp, a_round="f64")
    rdx, rdprob = om.moe_backward_tokens(rdxp, rdpp, row_map, T, k)
    for name, g, r in (("dx", dx, rdx), ("dw1", dw1, rdw1), ("dw2", dw2, rdw2), ("dprob", dprob, rdprob)):
        err = np.max(np.abs(g.float().cpu().numpy() - r)) / np.max(np.abs(r))
        print(f"MXFP8 backward {name}: rel err vs unquantised definition {err:.3e}")
        assert err <= 0.25   # MXFP8 rounding of the method itself (dw2 contracts over ~128 rows here)


def test_mxfp8_layer_bitwise_deterministic():
    """Two forward+backward passes over the same inputs give the same bits, fused codes
    included. A race between a producer and a consumer inside a kernel (for instance the
    staging of the saved h for the fc2-dgrad epilogue) shows up here as run-to-run
    differences in a few strips long before it breaks a tolerance; the size gives each
    CTA pair tens of tiles."""
    T, H, F, E, k = 16384, 2048, 4096, 8, 2
    g = torch.Generator(device=DEV)
    g.manual_seed(7)
    x = torch.randn(T, H, device=DEV, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, device=DEV, generator=g)
    w1 = (torch.randn(E, H, 2 * F, device=DEV, generator=g) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn(E, F, H, device=DEV, generator=g) * 0.02).to(torch.bfloat16)
    gy = torch.randn(T, H, device=DEV, generator=g).to(torch.bfloat16)
    layer = mb.MoEExpertLayer(T, H, F, E, k, precision="mxfp8", training=True)
    layer.set_weights(w1, w2)
    R = T * k
    parts = [mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "mxfp8", i) for i in (8, 9)]
    runs = []
    for _ in range(2):
        out = layer.forward(x, logits).clone()
        dx, dw1, dw2, dprob = (t.clone() for t in layer.backward(gy))
        ws = layer._bwd["ws"]
        codes = [ws[o: o + R * 2 * F].clone() for o in parts]
        runs.append([out, dx, dw1, dw2, dprob, layer.saved.clone()] + codes)
        assert mb.moe_device_status() == 0
    names = ["out", "dx", "dw1", "dw2", "dprob", "saved", "dh codes (2F)", "dh codes (rows)"]
    for name, a, b in zip(names, *runs):
        assert torch.equal(a.view(torch.uint8) if a.dtype != torch.uint8 else a,
                           b.view(torch.uint8) if b.dtype != torch.uint8 else b), f"{name} differs between runs"


@pytest.mark.parametrize("batch,rows,cols", [(3, 256, 384), (2, 384, 256), (1, 128, 128)])
def test_quantize_weights_both_forms_bit_exact(batch, rows, cols):
    """mxfp8_quantize_weights' two forms are the bytes of the two one-orientation
    quantisers (whose codes and scales the oracle pins bit for bit)."""
    g = torch.Generator(device=DEV)
    g.manual_seed(rows + cols)
    w = (torch.randn(batch, rows, cols, device=DEV, generator=g) *
         torch.exp(torch.randn(batch, 1, cols, device=DEV, generator=g) * 3)).to(torch.bfloat16)
    ct, at, cr, ar = mb.mxfp8_quantize_weights(w)
    ct_ref, at_ref = mb.mxfp8_quantize(w, axis=1, transpose_out=True, mma_scales=True)
    cr_ref, ar_ref = mb.mxfp8_quantize(w.reshape(batch * rows, cols), axis=0, mma_scales=True)
    assert mb.moe_device_status() == 0
    assert torch.equal(ct, ct_ref) and torch.equal(at, at_ref)
    assert torch.equal(cr.reshape(batch * rows, cols), cr_ref) and torch.equal(ar, ar_ref)
    # and the oracle's quantisation along each axis, on one matrix
    rc, rs = oq.quantize(om.f64(w[0].cpu()), axis=1)
    assert np.array_equal(ct[0].cpu().numpy(), rc.T)


def test_mxfp8_backward_with_prequantised_operands_is_identical():
    """The layer's backward (grouped_mlp_bwd_mxfp8_operands on the weights quantised both
    ways at once, xp and dy permuted and quantised in one pass) gives the same bits as
    grouped_mlp_bwd quantising the bf16 masters and bf16 permuted tensors itself."""
    T, H, F, E, k = 600, 256, 384, 5, 2
    d = workloads.small_layer(T, H, F, E, k, seed=41, with_grad=True)
    layer = mb.MoEExpertLayer(T, H, F, E, k, precision="mxfp8", training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    dx, dw1, dw2, dprob = (t.clone() for t in layer.backward(d["grad_out"].to(DEV)))
    b = layer._bwd
    row_map = layer.perm["row_map"]
    dy_perm = mb.moe_permute_rows(d["grad_out"].to(DEV), row_map, k)
    xp = mb.moe_permute_rows(d["x"].to(DEV), row_map, k)
    ref = mb.grouped_mlp_bwd(dy_perm, layer.perm["split_sizes"], xp, layer.w1_master, layer.w2_master,
                             layer.perm["probs_perm"], layer.saved, "mxfp8")
    assert mb.moe_device_status() == 0
    for got, want in zip((b["dxp"], dw1, dw2, b["dprobs_perm"]), ref):
        assert torch.equal(got, want)


@pytest.mark.parametrize("T,H,E,k,empty", [(300, 256, 5, 2, (3,)), (257, 384, 4, 1, (0, 2)), (96, 128, 8, 4, ())])
def test_permute_rows_mxfp8_both_forms_bit_exact(T, H, E, k, empty):
    """moe_permute_rows_mxfp8: the permuted rows quantised along H (tile atoms) and along
    each expert's rows (grouped atoms), bit for bit against the oracle's quantisers of the
    gathered bf16 rows; empty experts and ragged expert ends included."""
    bias = np.zeros(E)
    bias[list(empty)] = -1e4
    d = workloads.small_layer(T, H, 256, E, k, seed=T + H, with_grad=True, logits_bias=bias)
    ridx, _ = om.route(d["logits"], k)
    row_map, split, _ = om.permute_index(ridx, E)
    rm = torch.from_numpy(row_map.astype(np.int32)).to(DEV)
    sp = torch.from_numpy(split.astype(np.int32)).to(DEV)
    out = mb.moe_permute_rows_mxfp8(d["grad_out"].to(DEV), rm, k, sp)
    assert mb.moe_device_status() == 0
    dyp = om.f64(permuted(d["grad_out"], row_map, k))
    # rows form: blocks of 32 along H; atoms per 128-row expert tile
    rc, rs = oq.quantize(dyp, axis=0)
    assert np.array_equal(out["rows"].cpu().numpy(), rc)
    got_s, _, _ = tile_atoms_to_plain(out["rows_atoms"].cpu().numpy(), split, H // 32)
    assert np.array_equal(got_s, rs)
    # cols form: blocks of 32 rows restarting at every expert
    cc, cs = oq.quantize_grouped_rows(dyp, split)
    assert np.array_equal(out["cols"].cpu().numpy(), cc)
    ref_atoms = grouped_scales_to_atoms(cs, split, H)
    assert np.array_equal(out["cols_atoms"].cpu().numpy()[: ref_atoms.size], ref_atoms)
