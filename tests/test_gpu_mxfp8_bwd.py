"""GPU parity of the MXFP8 backward: the grouped (row-wise, per-expert) quantiser bit for
bit, and each backward GEMM against the fp64 oracle on the same quantised operands.

Outputs are bf16 (dh, the recomputed a, dxp, dw1, dw2): each element must lie within
2e-3 * max|ref| of the oracle plus its own bf16 storage rounding (half an ulp, at most
2^-8 |ref|); dprobs (fp32) within 2e-3 * max|ref|.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
from oracle import mxfp8 as oq
import workloads
from tests.mx_layout import grouped_scales_to_atoms

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
]


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
    R = T * k
    split = layer.perm["split_sizes"].cpu().numpy()
    for e in empty:
        assert split[e] == 0
        assert torch.count_nonzero(dw1[e]) == 0 and torch.count_nonzero(dw2[e]) == 0
    b = layer._bwd
    ws = b["ws"]
    off_dh = mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "mxfp8", 0)
    off_a = mb.grouped_mlp_bwd_workspace_offset(E, R, H, F, "mxfp8", 1)
    dh = ws[off_dh: off_dh + R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F)
    a = ws[off_a: off_a + R * F * 2].view(torch.bfloat16).view(R, F)
    h = layer.saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F)
    cpu = lambda t: t.cpu()
    ref = om.grouped_mlp_bwd_mxfp8(cpu(b["dy_perm"]), cpu(layer.xp_bf16), split, d["w1"], d["w2"],
                                   cpu(layer.perm["probs_perm"]), cpu(h), dh=cpu(dh), a=cpu(a))
    rdxp, rdw1, rdw2, rdp, rdh, ra = ref
    within(dh, rdh, "dh")
    within(a, ra, "a")
    within(b["dxp"], rdxp, "dxp")
    within(dw1, rdw1, "dw1")
    within(dw2, rdw2, "dw2")
    gp = b["dprobs_perm"].cpu().numpy()
    assert np.max(np.abs(gp - rdp)) <= TOL * np.max(np.abs(rdp))


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
