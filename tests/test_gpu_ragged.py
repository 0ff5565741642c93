"""GPU parity of the backward at expert sizes around the weight-gradient GEMMs' MMA steps
(16 rows for BF16, 32 for MXFP8) and stages (64 / 128 rows), plus an empty expert.

Each token is routed to a chosen expert (top-1, one-hot logits), so split_sizes are
exact. Every expert's weight gradients are checked on their own scale: BF16
max|err| / max|ref| <= 1e-2 per expert; MXFP8 within 2e-3 * max|ref| of the expert plus
the bf16 storage rounding of the element, against the oracle on the same operands.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"

SPLIT_BF16 = [1, 15, 16, 17, 0, 63, 64, 65, 128, 200]
SPLIT_MX = [1, 31, 32, 33, 0, 127, 128, 129, 300]


def routed_inputs(split, H, F, seed):
    E, T = len(split), int(sum(split))
    d = workloads.small_layer(T, H, F, E, 1, seed=seed, with_grad=True)
    rng = np.random.default_rng(seed)
    owner = np.repeat(np.arange(E), split)
    rng.shuffle(owner)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[np.arange(T), owner] += 50.0
    d["logits"] = torch.from_numpy(lg)
    return d, E, T


def run_layer(d, T, H, F, E, precision):
    layer = mb.MoEExpertLayer(T, H, F, E, 1, precision=precision, training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    grads = layer.backward(d["grad_out"].to(DEV))
    assert mb.moe_device_status() == 0
    return layer, grads


def per_expert_rel(got, ref, e):
    g = got[e].float().cpu().numpy()
    r = ref[e]
    return float(np.max(np.abs(g - r)) / np.max(np.abs(r)))


def test_bf16_backward_ragged_expert_sizes():
    H, F = 128, 128
    d, E, T = routed_inputs(SPLIT_BF16, H, F, seed=21)
    layer, (dx, dw1, dw2, dprob) = run_layer(d, T, H, F, E, "bf16")
    split = layer.perm["split_sizes"].cpu().numpy()
    assert list(split) == SPLIT_BF16
    b = layer._bwd
    rdxp, rdw1, rdw2, rdpp, _ = om.grouped_mlp_bwd(b["dy_perm"].cpu(), layer.perm["xp"].cpu(), split, d["w1"],
                                                    d["w2"], layer.perm["probs_perm"].cpu(), a_round="bf16")
    for e, n in enumerate(SPLIT_BF16):
        if n == 0:
            assert torch.count_nonzero(dw1[e]) == 0 and torch.count_nonzero(dw2[e]) == 0
            continue
        assert per_expert_rel(dw1, rdw1, e) <= 1e-2, (e, n)
        assert per_expert_rel(dw2, rdw2, e) <= 1e-2, (e, n)
    got = b["dxp"].float().cpu().numpy()
    assert np.max(np.abs(got - rdxp)) <= 1e-2 * np.max(np.abs(rdxp))


# experts that span more than the weight-gradient ring's three 128-row stages and end
# ragged, and sizes around one and two stages; H = F = 384 puts a ragged 128-column tail
# in the second CTA of each pair's last output tile
SPLIT_BF16_DEEP = [4 * 128 + 5, 3 * 128 + 17, 255, 256, 257, 0, 1]


def test_bf16_backward_ragged_deep_experts():
    H, F = 384, 384
    d, E, T = routed_inputs(SPLIT_BF16_DEEP, H, F, seed=23)
    layer, (dx, dw1, dw2, dprob) = run_layer(d, T, H, F, E, "bf16")
    split = layer.perm["split_sizes"].cpu().numpy()
    assert list(split) == SPLIT_BF16_DEEP
    b = layer._bwd
    rdxp, rdw1, rdw2, rdpp, _ = om.grouped_mlp_bwd(b["dy_perm"].cpu(), layer.perm["xp"].cpu(), split, d["w1"],
                                                    d["w2"], layer.perm["probs_perm"].cpu(), a_round="bf16")
    for e, n in enumerate(SPLIT_BF16_DEEP):
        if n == 0:
            assert torch.count_nonzero(dw1[e]) == 0 and torch.count_nonzero(dw2[e]) == 0
            continue
        assert per_expert_rel(dw1, rdw1, e) <= 1e-2, (e, n)
        assert per_expert_rel(dw2, rdw2, e) <= 1e-2, (e, n)


def within_expert(got, ref, e, name, tol=2e-3):
    g = got[e].float().cpu().numpy()
    r = ref[e]
    bound = tol * np.max(np.abs(r)) + 2.0 ** -8 * np.abs(r)
    assert np.all(np.abs(g - r) <= bound), f"{name}[{e}]: worst excess {np.max(np.abs(g - r) - bound):.3e}"


def test_mxfp8_backward_ragged_expert_sizes():
    from tests.test_gpu_mxfp8_bwd import fused_operands
    from oracle import mxfp8 as oq
    H, F = 256, 128
    d, E, T = routed_inputs(SPLIT_MX, H, F, seed=22)
    layer, (dx, dw1, dw2, dprob) = run_layer(d, T, H, F, E, "mxfp8")
    split = layer.perm["split_sizes"].cpu().numpy()
    assert list(split) == SPLIT_MX
    R = T
    b = layer._bwd
    h = layer.saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F).cpu()
    (dhr, dhr_s), (dhc, dhc_s), (ac, ac_s) = fused_operands(layer, E, R, H, F, split)
    from tests.gather import permuted
    row_map = layer.perm["row_map"]
    ref = om.grouped_mlp_bwd_mxfp8(permuted(d["grad_out"], row_map, layer.k), permuted(d["x"], row_map, layer.k),
                                   split, d["w1"], d["w2"],
                                   layer.perm["probs_perm"].cpu(), h,
                                   dh=oq.dequantize_blocks_last_axis(dhr, dhr_s),
                                   a=oq.dequantize_grouped_rows(ac, ac_s, split),
                                   dh_wgrad=oq.dequantize_grouped_rows(dhc, dhc_s, split))
    _, rdw1, rdw2, _, _, _ = ref
    for e, n in enumerate(SPLIT_MX):
        if n == 0:
            assert torch.count_nonzero(dw1[e]) == 0 and torch.count_nonzero(dw2[e]) == 0
            continue
        within_expert(dw1, rdw1, e, "dw1")
        within_expert(dw2, rdw2, e, "dw2")
