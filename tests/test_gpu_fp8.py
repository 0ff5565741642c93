"""GPU parity of the per-tensor FP8 path (current scaling: E4M3 forward operands, E5M2
gradients) against the fp64 oracle (oracle.fp8, oracle.moe.*_fp8).

* fp8_quantize: codes and scales bit-exact (both sides take the scale and the product in
  fp32), for both formats, batched and transposed, with an all-zero tensor;
* forward: the saved h (bf16) within 1e-2 of the oracle's; a's scale within one bf16
  rounding of amax, and every dequantised code of a within half an E4M3 step of the
  exact a (plus that bf16 rounding); fc2's fp32 accumulator against the oracle on the
  GPU's own a codes and scale within 2e-3 * max|ref|;
* backward: dh (bf16) within 1e-2; dh's E5M2 codes and scale bit-exact with the oracle's
  quantisation of the GPU's dh; dxp, dw1, dw2 within 2e-3 * max|ref| plus their bf16
  storage rounding, dprobs within 2e-3, against the oracle on the GPU's dh.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import fp8 as of
from oracle import moe as om
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("shape,transpose", [((3, 64, 96), False), ((2, 128, 64), True), ((256, 512), False)])
def test_fp8_quantize_bit_exact(fmt, shape, transpose):
    rng = np.random.default_rng(sum(shape))
    v = (rng.standard_normal(shape) * np.exp(rng.uniform(-6, 6, shape[:-2] + (1, 1) if len(shape) == 3 else (1, 1))))
    x = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
    if len(shape) == 3:
        x[1] = 0                                        # an all-zero tensor: scale 1, codes 0
    codes, scales = mb.fp8_quantize(x.to(DEV), fmt, transpose_out=transpose)
    assert mb.moe_device_status() == 0
    xs = om.f64(x).reshape((-1,) + shape[-2:])
    for b in range(xs.shape[0]):
        rc, rs = of.quantize_tensor(xs[b], fmt)
        assert scales.cpu().numpy()[b] == rs
        got = codes.cpu().numpy().reshape((-1,) + codes.shape[-2:])[b]
        assert np.array_equal(got, rc.T if transpose else rc)


def _fp8_layer(T, H, F, E, k, seed, empty=()):
    bias = np.zeros(E)
    bias[list(empty)] = -1e4
    d = workloads.small_layer(T, H, F, E, k, seed=seed, with_grad=True, logits_bias=bias)
    layer = mb.MoEExpertLayer(T, H, F, E, k, "fp8", training=True, device=DEV)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    assert mb.moe_device_status() == 0
    return d, layer


CASES = [(256, 128, 256, 4, 2, ()), (600, 256, 384, 5, 2, (3,)), (300, 256, 256, 1, 1, ()),
         (300, 384, 256, 8, 2, (1, 6))]


@pytest.mark.parametrize("T,H,F,E,k,empty", CASES)
def test_fp8_forward_parity(T, H, F, E, k, empty):
    d, layer = _fp8_layer(T, H, F, E, k, seed=T + 3, empty=empty)
    R = T * k
    split = layer.perm["split_sizes"].cpu().numpy()
    xp = layer.perm["xp"].cpu()
    pp = layer.perm["probs_perm"].cpu()
    saved = layer.saved
    h = saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F).float().cpu().numpy()
    off_a = (R * 2 * F * 2 + 255) // 256 * 256
    a_codes = saved[off_a: off_a + R * F].view(R, F).cpu().numpy()
    a_scale = saved[off_a + (R * F + 255) // 256 * 256:][:4].view(torch.float32).cpu().numpy()[0]
    # fc1 against the oracle on the same E4M3 operands
    ryp, rac, ras, rh = om.grouped_mlp_fwd_fp8(xp, split, d["w1"], d["w2"], pp)
    assert np.max(np.abs(h - rh)) <= 1e-2 * np.max(np.abs(rh))
    a_exact = om.silu(rh[:, :F]) * rh[:, F:] * om.f64(pp)[:, None]
    assert abs(a_scale / ras - 1.0) <= 2.0 ** -7
    deq = of.dequantize_tensor(a_codes, a_scale, "e4m3")
    bound = (2.0 ** -4 + 2.0 ** -7) * np.abs(a_exact) + 2.0 ** -9 / a_scale
    assert np.all(np.abs(deq - a_exact) <= bound)
    # fc2 on the GPU's own a codes: the fp32 accumulator (MOE_OUT_F32)
    yp32, _ = mb.grouped_mlp_fwd(layer.xq, layer.perm["split_sizes"], layer.w1, layer.w2, layer.perm["probs_perm"],
                                 "fp8", xp_scale=layer.xq_scale, w1_scale=layer.w1_scale, w2_scale=layer.w2_scale,
                                 F=F, out_f32=True)
    ref, _, _, _ = om.grouped_mlp_fwd_fp8(xp, split, d["w1"], d["w2"], pp, a_codes=a_codes, a_scale=a_scale)
    assert mb.moe_device_status() == 0
    assert np.max(np.abs(yp32.cpu().numpy() - ref)) <= TOL * np.max(np.abs(ref))
    for e in empty:
        assert split[e] == 0


def _within(got, ref, name):
    g = got.float().cpu().numpy() if hasattr(got, "cpu") else np.asarray(got)
    bound = TOL * np.max(np.abs(ref)) + 2.0 ** -8 * np.abs(ref)
    bad = np.abs(g - ref) > bound
    assert not bad.any(), f"{name}: {bad.sum()} off, worst excess {np.max(np.abs(g - ref) - bound):.3e}"


@pytest.mark.parametrize("T,H,F,E,k,empty", CASES)
def test_fp8_backward_parity(T, H, F, E, k, empty):
    d, layer = _fp8_layer(T, H, F, E, k, seed=T + 4, empty=empty)
    dx, dw1, dw2, dprob = layer.backward(d["grad_out"].to(DEV))
    assert mb.moe_device_status() == 0
    R = T * k
    split = layer.perm["split_sizes"].cpu().numpy()
    b = layer._bwd
    ws = b["ws"]
    saved = layer.saved
    h = saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F).cpu()
    off_a = (R * 2 * F * 2 + 255) // 256 * 256
    a_codes = saved[off_a: off_a + R * F].view(R, F).cpu().numpy()
    a_scale = saved[off_a + (R * F + 255) // 256 * 256:][:4].view(torch.float32).cpu().numpy()[0]
    off_dh = mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "fp8", 0)
    dh = ws[off_dh: off_dh + R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F).cpu()
    off_q = mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "fp8", 8)
    dhq = ws[off_q: off_q + R * 2 * F].view(R, 2 * F).cpu().numpy()
    dhs = ws[off_q + (R * 2 * F + 255) // 256 * 256:][:4].view(torch.float32).cpu().numpy()[0]
    dy, xp, pp = b["dy_perm"].cpu(), layer.perm["xp"].cpu(), layer.perm["probs_perm"].cpu()
    exact = om.grouped_mlp_bwd_fp8(dy, xp, split, d["w1"], d["w2"], pp, h, a_codes, a_scale)
    assert np.max(np.abs(dh.float().numpy() - exact[4])) <= 1e-2 * np.max(np.abs(exact[4]))
    # dh's E5M2 codes: the oracle's quantisation of the GPU's bf16 dh, bit for bit
    rc, rs = of.quantize_tensor(om.f64(dh), "e5m2")
    assert dhs == rs and np.array_equal(dhq, rc)
    ref = om.grouped_mlp_bwd_fp8(dy, xp, split, d["w1"], d["w2"], pp, h, a_codes, a_scale, dh=dh)
    _within(b["dxp"], ref[0], "dxp")
    _within(dw1, ref[1], "dw1")
    _within(dw2, ref[2], "dw2")
    gp = b["dprobs_perm"].cpu().numpy()
    assert np.max(np.abs(gp - ref[3])) <= TOL * np.max(np.abs(ref[3]))
    for e in empty:
        assert torch.count_nonzero(dw1[e]) == 0 and torch.count_nonzero(dw2[e]) == 0


def test_fp8_layer_close_to_bf16_definition():
    """Reported, loosely gated: the FP8 layer output against the unquantised definition."""
    T, H, F, E, k = 256, 256, 256, 4, 2
    d, layer = _fp8_layer(T, H, F, E, k, seed=5)
    ridx, rprob = om.route(d["logits"], k)
    ref = om.moe_forward_per_token(d["x"], ridx, rprob, d["w1"], d["w2"], a_round="f64")
    err = np.max(np.abs(layer.out.float().cpu().numpy() - ref)) / np.max(np.abs(ref))
    print(f"FP8 layer rel err vs the unquantised definition: {err:.3e}")
    assert err <= 0.15
