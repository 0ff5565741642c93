"""GPU parity of the capacity-padded dispatch (moe_permute_capacity) that feeds the same
grouped GEMMs with exactly C rows per expert, against the oracle's capacity definition.

Indices (row_map with -1 for dropped slots, kept counts, split sizes, offsets) are
bit-exact; the layer output within 1e-2 * max|ref| of oracle.moe.moe_forward_capacity
(BF16) or against the MXFP8 oracle on the same quantised operands (2e-3 + bf16 storage);
with a capacity that holds every slot, the output is bit-identical to the dropless path
(every output row depends only on its own input row). The BF16 weight gradients through
the padded rows equal the oracle's backward over the kept rows alone.
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


def _expected_rows(ridx, E, C):
    """The padded row of every slot (e*C + its rank among the expert's slots) or -1."""
    row_map, split, offs = om.permute_index(ridx, E)
    flat = ridx.reshape(-1).astype(np.int64)
    rank = row_map.astype(np.int64) - offs[flat]
    keep = om.capacity_keep(ridx, E, C).reshape(-1)
    assert np.array_equal(keep, rank < C)            # the stable order is the slot order
    return np.where(keep, flat * C + rank, -1).astype(np.int32), np.minimum(split, C)


def _route(d, k):
    ridx, rprob = om.route(d["logits"], k)
    return ridx, rprob, torch.from_numpy(ridx).to(DEV), torch.from_numpy(rprob.astype(np.float32)).to(DEV)


@pytest.mark.parametrize("T,H,F,E,k,factor", [(300, 256, 256, 4, 2, 1.0), (500, 128, 256, 8, 2, 0.6),
                                              (256, 192, 128, 16, 4, 1.25), (200, 128, 256, 4, 1, 3.0)])
def test_capacity_forward_bf16(T, H, F, E, k, factor):
    bias = np.array([1.5] + [0.0] * (E - 1))          # a favoured expert overflows its capacity
    d = workloads.small_layer(T, H, F, E, k, seed=T + E, with_grad=False, logits_bias=bias)
    C = int(np.ceil(factor * T * k / E))
    ridx, rprob, idx, prob = _route(d, k)
    o = mb.moe_permute_capacity(d["x"].to(DEV), idx, prob, E, C)
    rows, kept = _expected_rows(ridx, E, C)
    assert np.array_equal(o["row_map"].cpu().numpy(), rows)
    assert np.array_equal(o["kept"].cpu().numpy(), kept)
    assert np.all(o["split_sizes"].cpu().numpy() == C)
    assert np.array_equal(o["offsets"].cpu().numpy(), np.arange(E + 1) * C)
    yp, _ = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], d["w1"].to(DEV), d["w2"].to(DEV), o["probs_perm"])
    out = mb.moe_unpermute(yp, o["row_map"], T, k)
    assert mb.moe_device_status() == 0
    ref = om.moe_forward_capacity(d["x"], ridx, rprob, d["w1"], d["w2"], C, a_round="bf16")
    err = np.max(np.abs(out.float().cpu().numpy() - ref)) / np.max(np.abs(ref))
    assert err <= 1e-2
    if factor >= 1.0 and kept.sum() == T * k:
        # nothing dropped: bit-identical with the dropless layer
        dl = mb.moe_permute(d["x"].to(DEV), idx, prob, E)
        yd, _ = mb.grouped_mlp_fwd(dl["xp"], dl["split_sizes"], d["w1"].to(DEV), d["w2"].to(DEV), dl["probs_perm"])
        assert torch.equal(out, mb.moe_unpermute(yd, dl["row_map"], T, k))


def test_capacity_large_enough_is_the_dropless_layer():
    T, H, F, E, k = 300, 256, 256, 4, 2
    d = workloads.small_layer(T, H, F, E, k, seed=3, with_grad=False)
    ridx, rprob, idx, prob = _route(d, k)
    C = T * k                                            # holds every slot
    o = mb.moe_permute_capacity(d["x"].to(DEV), idx, prob, E, C)
    w1, w2 = d["w1"].to(DEV), d["w2"].to(DEV)
    yp, _ = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, o["probs_perm"])
    dl = mb.moe_permute(d["x"].to(DEV), idx, prob, E)
    yd, _ = mb.grouped_mlp_fwd(dl["xp"], dl["split_sizes"], w1, w2, dl["probs_perm"])
    assert torch.equal(mb.moe_unpermute(yp, o["row_map"], T, k), mb.moe_unpermute(yd, dl["row_map"], T, k))
    assert mb.moe_device_status() == 0


def test_capacity_backward_bf16():
    T, H, F, E, k = 400, 128, 256, 4, 2
    bias = np.array([2.0, 0.0, 0.0, -1.0])
    d = workloads.small_layer(T, H, F, E, k, seed=19, with_grad=True, logits_bias=bias)
    C = int(np.ceil(0.8 * T * k / E))
    ridx, rprob, idx, prob = _route(d, k)
    o = mb.moe_permute_capacity(d["x"].to(DEV), idx, prob, E, C)
    w1, w2 = d["w1"].to(DEV), d["w2"].to(DEV)
    _, saved = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, o["probs_perm"], training=True)
    dy = torch.zeros((E * C, H), dtype=torch.bfloat16, device=DEV)     # padded rows: zero gradient
    mb.moe_permute_rows(d["grad_out"].to(DEV), o["row_map"], k, out=dy)
    dxp, dw1, dw2, _ = mb.grouped_mlp_bwd(dy, o["split_sizes"], o["xp"], w1, w2, o["probs_perm"], saved)
    assert mb.moe_device_status() == 0
    # the oracle over the kept rows only: the first min(n_e, C) rows of each expert in
    # the dropless order
    row_map, split, offs = om.permute_index(ridx, E)
    xp = om.permute_rows(om.f64(d["x"]), row_map, k)
    pp = om.permute_probs(rprob, row_map)
    dyp = om.permute_rows(om.f64(d["grad_out"]), row_map, k)
    kept = np.minimum(split, C)
    sel = np.concatenate([np.arange(offs[e], offs[e] + kept[e]) for e in range(E)])
    _, rdw1, rdw2, _, _ = om.grouped_mlp_bwd(dyp[sel], xp[sel], kept, d["w1"], d["w2"], pp[sel], a_round="bf16")
    for g, r in ((dw1, rdw1), (dw2, rdw2)):
        assert np.max(np.abs(g.float().cpu().numpy() - r)) <= 1e-2 * np.max(np.abs(r))


def test_capacity_forward_mxfp8():
    T, H, F, E, k = 300, 256, 256, 4, 2
    d = workloads.small_layer(T, H, F, E, k, seed=29, with_grad=False, logits_bias=np.array([1.5, 0, 0, 0]))
    C = int(np.ceil(0.9 * T * k / E))
    ridx, rprob, idx, prob = _route(d, k)
    o = mb.moe_permute_capacity(d["x"].to(DEV), idx, prob, E, C, precision="mxfp8")
    rows, kept = _expected_rows(ridx, E, C)
    assert np.array_equal(o["row_map"].cpu().numpy(), rows)
    w1c, w1a = mb.mxfp8_quantize(d["w1"].to(DEV), axis=1, transpose_out=True, mma_scales=True)
    w2c, w2a = mb.mxfp8_quantize(d["w2"].to(DEV), axis=1, transpose_out=True, mma_scales=True)
    RC = E * C
    yp, saved = mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1c, w2c, o["probs_perm"], "mxfp8",
                                   xp_scale=o["xp_scale"], w1_scale=w1a, w2_scale=w2a, training=True, F=F)
    out = mb.moe_unpermute(yp, o["row_map"], T, k)
    assert mb.moe_device_status() == 0
    off_a = (RC * 2 * F * 2 + 255) // 256 * 256
    a_codes = saved[off_a: off_a + RC * F].view(RC, F).cpu().numpy()
    a_scales, _, _ = tile_atoms_to_plain(saved[off_a + (RC * F + 255) // 256 * 256:].cpu().numpy(), [C] * E, F // 32)
    slots = np.nonzero(rows >= 0)[0]
    toks, js = slots // k, slots % k
    r = rows[slots]
    yk, _, _ = om.fwd_rows_mxfp8(d["x"][toks], rprob[toks, js], ridx[toks, js], d["w1"], d["w2"],
                                 a_codes=a_codes[r], a_scales=a_scales[r])
    ref = np.zeros((T, H))
    mag = np.zeros((T, H))
    np.add.at(ref, toks, yk)
    np.add.at(mag, toks, np.abs(yk))
    g = out.float().cpu().numpy()
    # the GEMM bound, plus the bf16 rounding of every kept row and of their sum
    assert np.all(np.abs(g - ref) <= 2e-3 * np.max(np.abs(ref)) + 2.0 ** -8 * (mag + np.abs(ref)))
