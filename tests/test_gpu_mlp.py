"""GPU parity of the grouped expert MLP (tcgen05 grouped GEMMs) against the fp64 oracle.

Tolerance for BF16 outputs: max|err| / max|ref| <= 1e-2 (bf16 operands and outputs,
fp32 accumulation, against the oracle in fp64 with the same bf16 rounding of `a`).
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 1e-2


def rel_err(got, ref):
    got = got.float().cpu().numpy() if hasattr(got, "cpu") else got
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _route_and_permute(d, E, k):
    ridx, rprob = om.route(d["logits"], k)
    idx = torch.from_numpy(ridx).to(DEV)
    prob = torch.from_numpy(rprob.astype(np.float32)).to(DEV)
    o = mb.moe_permute(d["x"].to(DEV), idx, prob, E)
    return ridx, rprob, o


# (T, H, F, E, k, empty experts): several M tiles per expert with ragged tails, several
# N tiles, H not a multiple of 256 (fc2 column tail), an expert with no rows
FWD_CASES = [
    (256, 128, 256, 4, 2, ()),
    (600, 256, 384, 5, 2, (3,)),
    (300, 512, 256, 3, 1, ()),
    (100, 192, 128, 8, 4, (0, 7)),
    (1000, 320, 512, 16, 2, (2, 5, 11)),
    # degenerate routings: one expert (E=1, k=1, p=1); every row on one expert (k=1);
    # every token on the same two experts (k=2), each of them holding all T rows
    (300, 256, 256, 1, 1, ()),
    (257, 128, 256, 5, 1, (0, 1, 2, 4)),
    (300, 128, 256, 4, 2, (0, 2)),
]


def _bias(E, empty):
    b = np.zeros(E)
    b[list(empty)] = -1e4
    return b


@pytest.mark.parametrize("T,H,F,E,k,empty", FWD_CASES)
def test_grouped_mlp_fwd_bf16_parity(T, H, F, E, k, empty):
    d = workloads.small_layer(T, H, F, E, k, seed=T + H, with_grad=False, logits_bias=_bias(E, empty))
    ridx, rprob, o = _route_and_permute(d, E, k)
    split = o["split_sizes"].cpu().numpy()
    for e in empty:
        assert split[e] == 0
    w1, w2 = d["w1"].to(DEV), d["w2"].to(DEV)
    yp, saved = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, o["probs_perm"], training=True)
    ryp, rh, ra = om.grouped_mlp_fwd(o["xp"].cpu(), split, d["w1"], d["w2"], o["probs_perm"].cpu(), a_round="bf16")
    assert rel_err(yp, ryp) <= TOL_BF16
    R = T * k
    h = saved[: R * 2 * F * 2].view(torch.bfloat16).view(R, 2 * F)
    off = (R * 2 * F * 2 + 255) // 256 * 256
    a = saved[off: off + R * F * 2].view(torch.bfloat16).view(R, F)
    assert rel_err(h, rh) <= TOL_BF16
    assert rel_err(a, ra) <= TOL_BF16
    # inference mode (no saved buffer) gives the same output bit for bit
    yp2, _ = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, o["probs_perm"])
    assert torch.equal(yp, yp2)
    assert mb.moe_device_status() == 0


def test_tiny_config_layer_forward_against_definition():
    cfg = workloads.CONFIGS["tiny_bf16_fwd"]
    d = workloads.make_layer_inputs(cfg)
    layer = mb.MoEExpertLayer(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    out = layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    ridx, rprob = om.route(d["logits"], cfg.k)
    assert np.array_equal(layer.idx.cpu().numpy(), ridx)
    ref = om.moe_forward_per_token(d["x"], ridx, rprob, d["w1"], d["w2"], a_round="bf16")
    assert rel_err(out, ref) <= TOL_BF16
    assert mb.moe_device_status() == 0


def test_probabilities_move_between_mlp_and_combine():
    # invariant: MLP(p) + sum-combine == MLP(1) + p-weighted combine (up to rounding)
    T, H, F, E, k = 200, 128, 256, 4, 2
    d = workloads.small_layer(T, H, F, E, k, seed=5, with_grad=False)
    ridx, rprob, o = _route_and_permute(d, E, k)
    w1, w2 = d["w1"].to(DEV), d["w2"].to(DEV)
    yp_p, _ = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, o["probs_perm"])
    out_p = mb.moe_unpermute(yp_p, o["row_map"], T, k)
    yp_1, _ = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, None)
    out_1 = mb.moe_unpermute(yp_1, o["row_map"], T, k, prob=torch.from_numpy(rprob.astype(np.float32)).to(DEV))
    ref = om.moe_forward_per_token(d["x"], ridx, rprob, d["w1"], d["w2"], a_round="f64")
    assert rel_err(out_p, ref) <= TOL_BF16
    assert rel_err(out_1, ref) <= TOL_BF16


BWD_CASES = [
    (256, 128, 256, 4, 2, ()),
    (600, 256, 384, 5, 2, (3,)),
    (300, 192, 256, 8, 4, (1, 6)),
    (300, 256, 256, 1, 1, ()),
    (257, 128, 256, 5, 1, (0, 1, 2, 4)),
    (300, 128, 256, 4, 2, (0, 2)),
]


@pytest.mark.parametrize("T,H,F,E,k,empty", BWD_CASES)
def test_grouped_mlp_bwd_bf16_parity(T, H, F, E, k, empty):
    d = workloads.small_layer(T, H, F, E, k, seed=T + 3, with_grad=True, logits_bias=_bias(E, empty))
    ridx, rprob, o = _route_and_permute(d, E, k)
    split = o["split_sizes"].cpu().numpy()
    w1, w2 = d["w1"].to(DEV), d["w2"].to(DEV)
    _, saved = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, o["probs_perm"], training=True)
    dy_perm = mb.moe_permute_rows(d["grad_out"].to(DEV), o["row_map"], k)
    dxp, dw1, dw2, dpp = mb.grouped_mlp_bwd(dy_perm, o["split_sizes"], o["xp"], w1, w2, o["probs_perm"], saved)
    rdxp, rdw1, rdw2, rdpp, _ = om.grouped_mlp_bwd(dy_perm.cpu(), o["xp"].cpu(), split, d["w1"], d["w2"],
                                                    o["probs_perm"].cpu(), a_round="bf16")
    assert rel_err(dxp, rdxp) <= TOL_BF16
    assert rel_err(dw1, rdw1) <= TOL_BF16
    assert rel_err(dw2, rdw2) <= TOL_BF16
    assert rel_err(dpp, rdpp) <= TOL_BF16
    for e in empty:
        assert torch.count_nonzero(dw1[e]) == 0 and torch.count_nonzero(dw2[e]) == 0
    assert mb.moe_device_status() == 0


def test_layer_backward_token_outputs():
    T, H, F, E, k = 300, 128, 256, 6, 2
    d = workloads.small_layer(T, H, F, E, k, seed=77, with_grad=True)
    layer = mb.MoEExpertLayer(T, H, F, E, k, training=True)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    layer.forward(d["x"].to(DEV), d["logits"].to(DEV))
    dx, dw1, dw2, dprob = layer.backward(d["grad_out"].to(DEV))
    ridx, rprob = om.route(d["logits"], k)
    row_map, split, _ = om.permute_index(ridx, E)
    xp = om.permute_rows(om.f64(d["x"]), row_map, k)
    pp = om.permute_probs(rprob, row_map)
    dyp = om.permute_rows(om.f64(d["grad_out"]), row_map, k)
    rdxp, rdw1, rdw2, rdpp, _ = om.grouped_mlp_bwd(dyp, xp, split, d["w1"], d["w2"], pp, a_round="bf16")
    rdx, rdprob = om.moe_backward_tokens(rdxp, rdpp, row_map, T, k)
    assert rel_err(dx, rdx) <= TOL_BF16
    assert rel_err(dprob, rdprob) <= TOL_BF16
    assert rel_err(dw1, rdw1) <= TOL_BF16 and rel_err(dw2, rdw2) <= TOL_BF16


def test_mixtral_full_size_sampled_parity():
    """The Mixtral-shaped BF16 layer at full size, launched exactly as the benchmark does;
    512 sampled tokens (plus the first rows of the smallest and largest experts) are
    compared against the oracle's per-token definition."""
    cfg = workloads.CONFIGS["mixtral_bf16_fwd"]
    d = workloads.make_layer_inputs(cfg)
    layer = mb.MoEExpertLayer(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    out = layer.forward(d["x"].to(DEV), d["logits"].to(DEV)).cpu()
    assert mb.moe_device_status() == 0
    ridx, rprob = om.route(d["logits"], cfg.k)
    assert np.array_equal(layer.idx.cpu().numpy(), ridx)
    row_map, split, offsets = om.permute_index(ridx, cfg.E)
    assert np.array_equal(layer.perm["row_map"].cpu().numpy(), row_map)
    assert np.array_equal(layer.perm["split_sizes"].cpu().numpy(), split)
    toks = set(workloads.sample_tokens(cfg.T, 512).tolist())
    flat = ridx.reshape(-1)
    for e in (int(np.argmin(split)), int(np.argmax(split))):
        toks.add(int(np.nonzero(flat == e)[0][0]) // cfg.k)
    toks = np.array(sorted(toks))
    ref = om.moe_forward_sampled(d["x"], ridx, rprob, d["w1"], d["w2"], toks, a_round="bf16")
    assert rel_err(out[toks], ref) <= TOL_BF16
