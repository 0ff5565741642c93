"""GPU parity of the MXFP8 grouped expert MLP against the fp64 oracle.

fc2's output is compared with the oracle run on the same quantised operands (xp and
weight codes, which are bit-exact by the quantiser tests, and the `a` codes the fc1
epilogue emitted): max|err| / max|ref| <= 2e-3. fc1's quantised `a` is compared with the
oracle's own quantisation of its fp64 `a`: codes and scales may differ only where fp32
and fp64 land on opposite sides of a rounding boundary (one E4M3 step, with the exact
value within the fp32 error bound of the midpoint; see tests/mx_checks.py).
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
from oracle import mxfp8 as oq
import workloads
from tests.mx_checks import assert_boundary_flips, swiglu_fp32_error_bound
from tests.mx_layout import plain_to_atoms, tile_atoms_to_plain

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_MXFP8 = 2e-3


def rel_err(got, ref):
    got = got.float().cpu().numpy() if hasattr(got, "cpu") else got
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _align(n):
    return (n + 255) // 256 * 256


def _bias(E, empty):
    b = np.zeros(E)
    b[list(empty)] = -1e4
    return b


def run_mx_layer(T, H, F, E, k, empty=(), seed=0):
    d = workloads.small_layer(T, H, F, E, k, seed=seed, with_grad=False, logits_bias=_bias(E, empty))
    ridx, rprob = om.route(d["logits"], k)
    idx = torch.from_numpy(ridx).to(DEV)
    prob = torch.from_numpy(rprob.astype(np.float32)).to(DEV)
    o = mb.moe_permute(d["x"].to(DEV), idx, prob, E, precision="mxfp8")
    # weights: MMA-layout scales for the GEMM, plain ones for the oracle (same codes)
    w1c, w1a = mb.mxfp8_quantize(d["w1"].to(DEV), axis=1, transpose_out=True, mma_scales=True)
    w2c, w2a = mb.mxfp8_quantize(d["w2"].to(DEV), axis=1, transpose_out=True, mma_scales=True)
    _, w1s = mb.mxfp8_quantize(d["w1"].to(DEV), axis=1, transpose_out=True)
    _, w2s = mb.mxfp8_quantize(d["w2"].to(DEV), axis=1, transpose_out=True)
    assert np.array_equal(w1a.cpu().numpy(), plain_to_atoms(w1s.cpu().numpy().reshape(-1, H // 32)))
    yp, saved = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1c, w2c, o["probs_perm"], "mxfp8",
                                   xp_scale=o["xp_scale"], w1_scale=w1a, w2_scale=w2a, training=True, F=F)
    yp32, _ = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1c, w2c, o["probs_perm"], "mxfp8",
                                 xp_scale=o["xp_scale"], w1_scale=w1a, w2_scale=w2a, F=F, out_f32=True)
    R = T * k
    h = saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F)
    off = _align(R * 2 * F * 2)
    a_codes = saved[off: off + R * F].view(R, F)
    off2 = off + _align(R * F)
    a_scales, padded, groups = tile_atoms_to_plain(saved[off2:].cpu().numpy(), o["split_sizes"].cpu().numpy(),
                                                   F // 32)
    # rows of the last, partial tile of each expert carry zero scales
    assert int(padded.astype(np.int64).sum()) == int(a_scales.astype(np.int64).sum())
    a_scales = torch.from_numpy(a_scales)
    assert mb.moe_device_status() == 0
    return dict(d=d, ridx=ridx, rprob=rprob, o=o, w1c=w1c, w1s=w1s, w2c=w2c, w2s=w2s, yp=yp, yp32=yp32, h=h,
                a_codes=a_codes, a_scales=a_scales)


MX_CASES = [
    (256, 128, 256, 4, 2, ()),
    (300, 256, 256, 4, 2, ()),
    (600, 512, 384, 5, 2, (3,)),
    (1000, 384, 640, 16, 2, (2, 5, 11)),
    (300, 256, 256, 1, 1, ()),              # one expert
    (257, 256, 256, 5, 1, (0, 1, 2, 4)),    # every row on one expert
    (300, 256, 256, 4, 2, (0, 2)),          # every token on the same two experts
]


@pytest.mark.parametrize("T,H,F,E,k,empty", MX_CASES)
def test_grouped_mlp_fwd_mxfp8_parity(T, H, F, E, k, empty):
    r = run_mx_layer(T, H, F, E, k, empty, seed=T + F)
    o = r["o"]
    split = o["split_sizes"].cpu().numpy()
    cpu = lambda t: t.cpu().numpy()
    # fc2 on the GPU-emitted `a` codes: the 2e-3 gate applies to the GEMM's arithmetic,
    # i.e. the fp32 accumulator (MOE_OUT_F32) against the fp64 oracle on the same operands
    ryp, rac, ras, rh = om.grouped_mlp_fwd_mxfp8(
        cpu(o["xp"]), cpu(o["xp_scale"]), split, cpu(r["w1c"]), cpu(r["w1s"]), cpu(r["w2c"]), cpu(r["w2s"]),
        cpu(o["probs_perm"]), a_codes=cpu(r["a_codes"]), a_scales=cpu(r["a_scales"]))
    assert rel_err(r["yp32"], ryp) <= TOL_MXFP8
    # the bf16 output is that accumulator rounded once (nearest even) ...
    assert torch.equal(r["yp"], r["yp32"].to(torch.bfloat16))
    # ... so it meets the same bound plus its own storage rounding (half a bf16 ulp, <= 2^-8 |y|)
    yb = r["yp"].float().cpu().numpy()
    assert np.all(np.abs(yb - ryp) <= TOL_MXFP8 * np.max(np.abs(ryp)) + 2.0 ** -8 * np.abs(ryp))
    # fc1: saved pre-activations (bf16) against the oracle's fp64 h
    assert rel_err(r["h"], rh) <= 1e-2
    # fc1 epilogue quantisation of a = SiLU(g) * u * p against the oracle's own codes
    _, rac_own, ras_own, _ = om.grouped_mlp_fwd_mxfp8(
        cpu(o["xp"]), cpu(o["xp_scale"]), split, cpu(r["w1c"]), cpu(r["w1s"]), cpu(r["w2c"]), cpu(r["w2s"]),
        cpu(o["probs_perm"]))
    gc, gs = cpu(r["a_codes"]), cpu(r["a_scales"])
    pp = cpu(o["probs_perm"]).astype(np.float64)[:, None]
    a_exact = om.silu(rh[:, :F]) * rh[:, F:] * pp
    # codes and scales may differ from the oracle's only by rounding-boundary flips of the
    # fp32 arithmetic, bounded per element from the magnitudes of fc1's products
    xq = np.abs(oq.dequantize_blocks_last_axis(cpu(o["xp"]), cpu(o["xp_scale"])))
    w1q = np.abs(oq.dequantize_blocks_last_axis(cpu(r["w1c"]), cpu(r["w1s"])))       # [E, 2F, H]
    sabs = np.zeros((xq.shape[0], 2 * F))
    s0 = 0
    for e, n in enumerate(split):
        sabs[s0:s0 + n] = xq[s0:s0 + n] @ w1q[e].T
        s0 += n
    err = swiglu_fp32_error_bound(rh[:, :F], rh[:, F:], pp, sabs[:, :F], sabs[:, F:], H)
    rep = assert_boundary_flips(gc, gs, a_exact, "a", err=err)
    assert rep["code_flips"] <= 0.01 * gc.size


def test_mxfp8_layer_end_to_end_against_fully_oracle_chain():
    """Reported, loosely gated: the whole MXFP8 layer (own quantisation of x, weights and
    a) against the oracle's fully quantised chain on the per-token definition."""
    T, H, F, E, k = 256, 256, 256, 4, 2
    d = workloads.small_layer(T, H, F, E, k, seed=9, with_grad=False)
    layer = mb.MoEExpertLayer(T, H, F, E, k, precision="mxfp8")
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    out = layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    ridx, rprob = om.route(d["logits"], k)
    xc, xs = oq.quantize(om.f64(d["x"]), axis=0)
    w1c, w1s = om.quantize_weights_kmajor(d["w1"], "rows")
    w2c, w2s = om.quantize_weights_kmajor(d["w2"], "rows")
    xq = oq.dequantize(xc, xs, axis=0)
    w1q = np.swapaxes(oq.dequantize_blocks_last_axis(w1c, w1s), 1, 2)
    w2q = np.swapaxes(oq.dequantize_blocks_last_axis(w2c, w2s), 1, 2)
    ref = om.moe_forward_per_token(xq, ridx, rprob, w1q, w2q, a_round="mxfp8")
    err = rel_err(out, ref)
    print(f"MXFP8 end-to-end rel err vs fully quantised oracle chain: {err:.3e}")
    assert err <= 2e-2
    # and against the unquantised BF16 definition (quantisation error of the method itself)
    ref_bf16 = om.moe_forward_per_token(d["x"], ridx, rprob, d["w1"], d["w2"], a_round="f64")
    assert rel_err(out, ref_bf16) <= 0.15
