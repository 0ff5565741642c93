"""GPU parity of the combine fused into fc2's epilogue (grouped_mlp_fwd_combine): the
layer output without the permuted yp ever being written.

BF16: max|err| / max|ref| <= 1e-2 against the oracle's per-token definition (the same
bound as the unfused layer). MXFP8: the fc2 accumulators of a token's k rows are summed in
fp32 and rounded once, so out is checked against the oracle's sum of the fc2 rows computed
on the same quantised operands (the GPU's own `a` codes): within 2e-3 * max|ref| plus one
bf16 rounding of the element. For k = 2 the fp32 sum does not depend on the order of the
two adds: two runs are bit-identical.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
import workloads
from tests.mx_layout import tile_atoms_to_plain

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [(300, 256, 256, 4, 2), (257, 128, 256, 5, 1), (200, 192, 256, 8, 8), (513, 320, 384, 16, 2)]


def _rel(got, ref):
    return float(np.max(np.abs(got.float().cpu().numpy() - ref)) / np.max(np.abs(ref)))


@pytest.mark.parametrize("T,H,F,E,k", CASES)
def test_fused_combine_bf16(T, H, F, E, k):
    d = workloads.small_layer(T, H, F, E, k, seed=T + 5, with_grad=False)
    layer = mb.MoEExpertLayer(T, H, F, E, k, device=DEV, fused_combine=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    out = layer.forward(d["x"].to(DEV), d["logits"].to(DEV)).clone()
    assert mb.moe_device_status() == 0
    ridx, rprob = om.route(d["logits"], k)
    ref = om.moe_forward_per_token(d["x"], ridx, rprob, d["w1"], d["w2"], a_round="bf16")
    assert _rel(out, ref) <= 1e-2
    out2 = layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    if k <= 2:
        assert torch.equal(out, out2)


@pytest.mark.parametrize("T,H,F,E,k", [(300, 256, 256, 4, 2), (200, 256, 384, 8, 8)])
def test_fused_combine_mxfp8(T, H, F, E, k):
    d = workloads.small_layer(T, H, F, E, k, seed=T + 6, with_grad=False)
    layer = mb.MoEExpertLayer(T, H, F, E, k, "mxfp8", training=True, device=DEV, fused_combine=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    out = layer.forward(d["x"].to(DEV), d["logits"].to(DEV)).clone()
    assert mb.moe_device_status() == 0
    R = T * k
    ridx, rprob = om.route(d["logits"], k)
    split = layer.perm["split_sizes"].cpu().numpy()
    row_map = layer.perm["row_map"].cpu().numpy()
    off_a = (R * 2 * F * 2 + 255) // 256 * 256
    a_codes = layer.saved[off_a: off_a + R * F].view(R, F).cpu().numpy()
    a_scales, _, _ = tile_atoms_to_plain(layer.saved[off_a + (R * F + 255) // 256 * 256:].cpu().numpy(), split, F // 32)
    slots = np.arange(R)
    toks, js = slots // k, slots % k
    rows = row_map[slots]
    yp, _, _ = om.fwd_rows_mxfp8(d["x"][toks], rprob[toks, js], ridx[toks, js], d["w1"], d["w2"],
                                 a_codes=a_codes[rows], a_scales=a_scales[rows])
    ref = yp.reshape(T, k, H).sum(axis=1)
    g = out.float().cpu().numpy()
    assert np.all(np.abs(g - ref) <= 2e-3 * np.max(np.abs(ref)) + 2.0 ** -8 * np.abs(ref))
    out2 = layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    if k <= 2:
        assert torch.equal(out, out2)
