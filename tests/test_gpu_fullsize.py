"""Full-size parity of the benchmark workloads (same shapes and launch configuration as
bench.py), checked on outputs the oracle can compute one by one: sampled tokens/rows and
sampled weight-gradient entries (each depends only on its own column over one expert).

Tolerances: BF16 outputs max|err| / max|ref| <= 1e-2 over the sampled set; MXFP8 outputs
within 2e-3 * max|ref| plus their own bf16 storage rounding (2^-8 |ref|) against the
oracle on the same quantised operands.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
import workloads
from oracle import mxfp8 as oq
from tests.gather import permuted
from tests.mx_checks import assert_boundary_flips, dswiglu_fp32_error_bounds, swiglu_fp32_error_bound
from tests.mx_layout import grouped_atoms_to_scales, tile_atoms_to_plain

pytestmark = pytest.mark.gpu
DEV = "cuda"


def rel(got, ref):
    g = got.float().cpu().numpy() if hasattr(got, "cpu") else np.asarray(got)
    return float(np.max(np.abs(g - ref)) / np.max(np.abs(ref)))


def within_mx(got, ref, name, tol=2e-3):
    g = got.float().cpu().numpy() if hasattr(got, "cpu") else np.asarray(got)
    bound = tol * np.max(np.abs(ref)) + 2.0 ** -8 * np.abs(ref)
    assert np.all(np.abs(g - ref) <= bound), f"{name}: worst excess {np.max(np.abs(g - ref) - bound):.3e}"


def sample_rows(split, n, seed):
    """n seeded permuted rows plus the first and last row of the smallest non-empty and
    of the largest expert."""
    rng = np.random.default_rng(seed)
    R = int(np.sum(split))
    offs = np.concatenate([[0], np.cumsum(split)])
    nz = [e for e in range(len(split)) if split[e] > 0]
    small = min(nz, key=lambda e: split[e])
    large = max(nz, key=lambda e: split[e])
    extra = [offs[small], offs[small + 1] - 1, offs[large], offs[large + 1] - 1]
    return np.unique(np.concatenate([rng.choice(R, size=n, replace=False), extra])).astype(np.int64), small, large


def test_qwen3_full_size_fwd_bwd_bf16():
    cfg = workloads.CONFIGS["qwen3_30b_a3b_bf16_fwdbwd"]
    d = workloads.make_layer_inputs(cfg)
    layer = mb.MoEExpertLayer(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    out = layer.forward(d["x"].to(DEV), d["logits"].to(DEV)).cpu()
    dx, dw1, dw2, dprob = layer.backward(d["grad_out"].to(DEV))
    assert mb.moe_device_status() == 0
    split = layer.perm["split_sizes"].cpu().numpy()
    assert split.sum() == cfg.R and np.all(split[-4:] == 0)          # the forced-empty experts
    ridx, rprob = om.route(d["logits"], cfg.k)
    assert np.array_equal(layer.idx.cpu().numpy(), ridx)
    toks = workloads.sample_tokens(cfg.T, 256, seed=3)
    ref = om.moe_forward_sampled(d["x"], ridx, rprob, d["w1"], d["w2"], toks, a_round="bf16")
    assert rel(out[toks], ref) <= 1e-2
    # backward on the GPU's own permuted inputs (bit-exact by the permutation tests)
    b = layer._bwd
    rows, small, large = sample_rows(split, 512, seed=4)
    experts = [small, large, cfg.E - 1, 17, 60]
    c1 = np.sort(np.random.default_rng(5).choice(2 * cfg.F, 16, replace=False))
    c2 = np.sort(np.random.default_rng(6).choice(cfg.H, 16, replace=False))
    xp, dyp, pp = layer.perm["xp"].cpu(), b["dy_perm"].cpu(), layer.perm["probs_perm"].cpu()
    rdxp, rdpp, rdw1, rdw2 = om.bwd_sampled_bf16(dyp, xp, split, d["w1"], d["w2"], pp, rows, experts, c1, c2)
    assert rel(b["dxp"].cpu()[rows], rdxp) <= 1e-2
    assert rel(b["dprobs_perm"].cpu()[rows], rdpp) <= 1e-2
    for e in experts:
        g1, g2 = dw1[e][:, c1].cpu(), dw2[e][:, c2].cpu()
        if split[e] == 0:
            assert torch.count_nonzero(g1) == 0 and torch.count_nonzero(g2) == 0
        else:
            assert rel(g1, rdw1[e]) <= 1e-2 and rel(g2, rdw2[e]) <= 1e-2


def test_mixtral_mxfp8_full_size_fwd():
    cfg = workloads.CONFIGS["mixtral_mxfp8_fwd"]
    d = workloads.make_layer_inputs(cfg)
    layer = mb.MoEExpertLayer(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, "mxfp8", training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    assert mb.moe_device_status() == 0
    R, F = cfg.R, cfg.F
    split = layer.perm["split_sizes"].cpu().numpy()
    ridx, rprob = om.route(d["logits"], cfg.k)
    row_map = layer.perm["row_map"].cpu().numpy()
    assert np.array_equal(row_map, om.permute_index(ridx, cfg.E)[0])
    # sampled routed rows of the smallest and the largest expert
    rows_all, small, large = sample_rows(split, 4096, seed=7)
    offs = np.concatenate([[0], np.cumsum(split)])
    keep = ((rows_all >= offs[small]) & (rows_all < offs[small + 1])) | \
           ((rows_all >= offs[large]) & (rows_all < offs[large + 1]))
    rows = rows_all[keep]
    slot_of_row = np.empty(R, dtype=np.int64)
    slot_of_row[row_map] = np.arange(R)
    slots = slot_of_row[rows]
    toks, js = slots // cfg.k, slots % cfg.k
    off_a = (R * 2 * F * 2 + 255) // 256 * 256
    a_codes = layer.saved[off_a: off_a + R * F].view(R, F).cpu().numpy()
    off_s = off_a + (R * F + 255) // 256 * 256
    a_scales, _, _ = tile_atoms_to_plain(layer.saved[off_s:].cpu().numpy(), split, F // 32)
    pr = rprob[toks, js]
    yp_ref, own_c, own_s, det = om.fwd_rows_mxfp8(d["x"][toks], pr, ridx[toks, js], d["w1"], d["w2"],
                                                  a_codes=a_codes[rows], a_scales=a_scales[rows], details=True)
    # the fused epilogue's codes differ from the oracle's only by rounding-boundary flips
    h, sabs = det["h"], det["sum_abs"]
    p = pr.astype(np.float64)[:, None]
    a_exact = om.silu(h[:, :F]) * h[:, F:] * p
    err = swiglu_fp32_error_bound(h[:, :F], h[:, F:], p, sabs[:, :F], sabs[:, F:], cfg.H)
    rep = assert_boundary_flips(a_codes[rows], a_scales[rows], a_exact, "a", err=err)
    assert rep["code_flips"] <= 0.01 * own_c.size
    within_mx(layer.yp.cpu()[rows], yp_ref, "yp")


def test_genomic_mxfp8_full_size_fwd_bwd():
    cfg = workloads.CONFIGS["genomic_mixtral_mxfp8_fwdbwd"]
    d = workloads.make_layer_inputs(cfg)
    layer = mb.MoEExpertLayer(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, "mxfp8", training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    dx, dw1, dw2, dprob = layer.backward(d["grad_out"].to(DEV))
    assert mb.moe_device_status() == 0
    R, H, F, E = cfg.R, cfg.H, cfg.F, cfg.E
    split = layer.perm["split_sizes"].cpu().numpy()
    assert split[0] > 0.4 * R                                            # expert 0 carries the skew
    b = layer._bwd
    h = layer.saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F).cpu()
    ws = b["ws"]

    def part(i, ncols):
        off = mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "mxfp8", i)
        codes = ws[off: off + R * ncols].view(R, ncols)                      # stays on the device
        atoms = ws[off + (R * ncols + 255) // 256 * 256:].cpu().numpy()
        return codes, atoms

    dhr, dhr_at = part(8, 2 * F)
    dhr_s, _, _ = tile_atoms_to_plain(dhr_at, split, 2 * F // 32)
    dhc, dhc_at = part(9, 2 * F)
    dhc_s = grouped_atoms_to_scales(dhc_at, split, 2 * F)
    off3 = mb.grouped_mlp_saved_offset(E, R, H, F, "mxfp8", 3)
    ac = layer.saved[off3: off3 + R * F].view(R, F)                            # stays on the device
    ac_s = grouped_atoms_to_scales(layer.saved[mb.grouped_mlp_saved_offset(E, R, H, F, "mxfp8", 4):].cpu().numpy(),
                                   split, F)
    offs = np.concatenate([[0], np.cumsum(split)])

    class RowsDeq:
        """dh along 2F, dequantised on demand for the rows asked for."""
        def __getitem__(self, rows):
            return oq.dequantize_blocks_last_axis(dhr[torch.as_tensor(rows, device=DEV)].cpu().numpy(),
                                                  dhr_s[rows])

    class ColsDeq:
        """codes along each expert's rows, dequantised on demand for one expert's rows and
        the columns asked for."""
        def __init__(self, codes, scales):
            self.codes, self.scales = codes, scales

        def __getitem__(self, key):
            rs, cols = key
            e = int(np.searchsorted(offs, rs.start, side="right") - 1)
            c = self.codes[rs][:, torch.as_tensor(cols, device=DEV)].cpu().numpy()
            return oq.dequantize_grouped_rows(c, [self.scales[e][:, cols]], [rs.stop - rs.start])

    rows_all, small, large = sample_rows(split, 2048, seed=8)
    keep = ((rows_all >= offs[small]) & (rows_all < offs[small + 1])) | \
           ((rows_all >= offs[large]) & (rows_all < offs[large + 1]))
    rows = rows_all[keep]
    rng = np.random.default_rng(9)
    cols = (np.sort(rng.choice(F, 16, replace=False)), np.sort(rng.choice(H, 16, replace=False)),
            np.sort(rng.choice(H, 16, replace=False)), np.sort(rng.choice(2 * F, 16, replace=False)))
    row_map = layer.perm["row_map"]
    dy_cpu = permuted(d["grad_out"], row_map, cfg.k)   # the bf16 rows the fused quantiser read
    ref = om.bwd_sampled_mxfp8(dy_cpu, permuted(d["x"], row_map, cfg.k), split, d["w1"], d["w2"],
                               layer.perm["probs_perm"].cpu(), h, RowsDeq(), ColsDeq(ac, ac_s), rows,
                               [small, large], cols, dh_wgrad=ColsDeq(dhc, dhc_s))
    # dh along 2F at the sampled rows: only rounding-boundary flips against the exact dh;
    # the fp32 error bound takes |da| magnitudes from the oracle's fc2-dgrad operands
    sabs = np.zeros((rows.size, F))
    dyq = np.abs(oq.dequantize(*oq.quantize(om.f64(dy_cpu[torch.as_tensor(rows)]), axis=0),
                               axis=0))
    for e in (small, large):
        sel = (rows >= offs[e]) & (rows < offs[e + 1])
        w2q = np.abs(oq.dequantize(*oq.quantize(om.f64(d["w2"][e]), axis=0), axis=0))
        sabs[sel] = dyq[sel] @ w2q.T
    hh = om.f64(h[torch.as_tensor(rows)])
    pp = om.f64(layer.perm["probs_perm"].cpu()[torch.as_tensor(rows)])[:, None]
    e_dg, e_du, _ = dswiglu_fp32_error_bounds(hh[:, :F], hh[:, F:], pp, sabs, H)
    assert_boundary_flips(dhr[torch.as_tensor(rows, device=DEV)].cpu().numpy(), dhr_s[rows], ref["dh"], "dh",
                          err=np.concatenate([e_dg, e_du], axis=1))
    within_mx(b["dxp"].cpu()[rows], ref["dxp"], "dxp")
    gp = b["dprobs_perm"].cpu().numpy()[rows]
    assert np.max(np.abs(gp - ref["dp"])) <= 2e-3 * np.max(np.abs(ref["dp"]))
    for e in (small, large):
        within_mx(dw2[e].cpu()[np.ix_(cols[0], cols[1])], ref["dw2"][e], f"dw2[{e}]")
        within_mx(dw1[e].cpu()[np.ix_(cols[2], cols[3])], ref["dw1"][e], f"dw1[{e}]")
