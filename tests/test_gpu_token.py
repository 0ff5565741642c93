"""GPU parity of routing, permutation, combine and the MXFP8 quantiser against the oracle.

Integer/index/code outputs are compared bit-exactly; probabilities within 1e-6 absolute
(fp32 softmax against the fp64 oracle); the combine within one bf16 rounding.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
from oracle import mxfp8 as oq
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _status_ok():
    assert mb.moe_device_status() == 0


ROUTE_CASES = [(256, 4, 2), (1000, 8, 2), (777, 128, 8), (64, 1, 1), (33, 5, 5), (1, 40, 3), (513, 1024, 32),
               (300, 33, 7)]


@pytest.mark.parametrize("T,E,k", ROUTE_CASES)
@pytest.mark.parametrize("renorm", [True, False])
def test_route_parity(T, E, k, renorm):
    rng = np.random.default_rng(T * 7 + E)
    lg = rng.standard_normal((T, E), dtype=np.float32)
    lg[: T // 4] = np.round(lg[: T // 4])            # exact ties on a quarter of the tokens
    idx, prob = mb.moe_route(torch.from_numpy(lg).to(DEV), k, renorm)
    ridx, rprob = om.route(lg, k, renorm)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.max(np.abs(prob.cpu().numpy() - rprob)) <= 1e-6
    _status_ok()


PERMUTE_CASES = [(256, 128, 4, 2), (1000, 64, 8, 2), (777, 256, 128, 8), (5, 64, 3, 1), (2049, 8, 16, 4),
                 (1, 32, 1, 1), (4096, 136, 32, 8)]


@pytest.mark.parametrize("T,H,E,k", PERMUTE_CASES)
def test_permute_parity_bf16(T, H, E, k):
    d = workloads.small_layer(T, H, 128, E, k, seed=T, with_grad=False,
                              logits_bias=np.where(np.arange(E) % 3 == 1, -30.0, 0.0) if E > k + 2 else None)
    x, lg = d["x"], d["logits"]
    ridx, rprob = om.route(lg, k)
    idx = torch.from_numpy(ridx).to(DEV)
    prob = torch.from_numpy(rprob.astype(np.float32)).to(DEV)
    o = mb.moe_permute(x.to(DEV), idx, prob, E)
    row_map, split, offsets = om.permute_index(ridx, E)
    assert np.array_equal(o["row_map"].cpu().numpy(), row_map)
    assert np.array_equal(o["split_sizes"].cpu().numpy(), split)
    assert np.array_equal(o["offsets"].cpu().numpy(), offsets)
    ref_xp = om.permute_rows(x.view(torch.int16).numpy(), row_map, k)
    assert np.array_equal(o["xp"].cpu().view(torch.int16).numpy(), ref_xp)
    assert np.array_equal(o["probs_perm"].cpu().numpy(), om.permute_probs(rprob.astype(np.float32), row_map))
    _status_ok()


@pytest.mark.parametrize("T,H,E,k", [(300, 256, 8, 2), (64, 128, 4, 2), (100, 4096, 16, 8)])
def test_permute_parity_mxfp8(T, H, E, k):
    d = workloads.small_layer(T, H, 128, E, k, seed=T + 1, with_grad=False)
    x = d["x"]
    x[0, :32] = 0                                   # an all-zero block
    x[1, 32:64] = torch.tensor(4.0e37)              # a huge block
    ridx, rprob = om.route(d["logits"], k)
    o = mb.moe_permute(x.to(DEV), torch.from_numpy(ridx).to(DEV), torch.from_numpy(rprob.astype(np.float32)).to(DEV),
                       E, precision="mxfp8")
    row_map, _, _ = om.permute_index(ridx, E)
    codes, scales = oq.quantize(om.f64(x), axis=0)
    assert np.array_equal(o["xp"].cpu().numpy(), om.permute_rows(codes, row_map, k))
    assert np.array_equal(o["xp_scale"].cpu().numpy(), om.permute_rows(scales, row_map, k))
    _status_ok()


@pytest.mark.parametrize("T,H,k,weighted", [(300, 256, 2, False), (300, 256, 2, True), (77, 64, 8, False),
                                            (1, 8, 1, True), (1025, 136, 3, True)])
def test_unpermute_parity(T, H, k, weighted):
    rng = np.random.default_rng(T + k)
    R = T * k
    yp = torch.from_numpy(rng.standard_normal((R, H), dtype=np.float32)).to(torch.bfloat16)
    row_map = rng.permutation(R).astype(np.int32)
    prob = rng.random((T, k), dtype=np.float32) if weighted else None
    out = mb.moe_unpermute(yp.to(DEV), torch.from_numpy(row_map).to(DEV), T, k,
                           prob=None if prob is None else torch.from_numpy(prob).to(DEV))
    ref = om.unpermute(yp, row_map, T, k, prob)
    got = out.float().cpu().numpy()
    # one bf16 rounding of the result plus fp32 accumulation
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * k)
    _status_ok()


@pytest.mark.parametrize("k", [1, 2, 8])
def test_unpermute_of_permute_is_exact(k):
    T, H, E = 500, 192, 16
    d = workloads.small_layer(T, H, 128, E, k, seed=k, with_grad=False)
    ridx, _ = om.route(d["logits"], k)
    o = mb.moe_permute(d["x"].to(DEV), torch.from_numpy(ridx).to(DEV), None, E)
    w = torch.full((T, k), 1.0 / k, device=DEV)
    back = mb.moe_unpermute(o["xp"], o["row_map"], T, k, prob=w)
    assert torch.equal(back.cpu(), d["x"])


@pytest.mark.parametrize("B,rows,cols", [(1, 64, 256), (3, 128, 96), (2, 32, 4096)])
def test_quantize_axis0_bit_exact(B, rows, cols):
    rng = np.random.default_rng(rows + cols)
    v = rng.standard_normal((B, rows, cols), dtype=np.float32) * np.exp(
        rng.uniform(-20, 20, (B, rows, 1))).astype(np.float32)
    v[0, 0, :32] = 0.0
    v[0, 1, :] *= 1e-38                           # subnormal bf16 inputs
    x = torch.from_numpy(v).to(torch.bfloat16)
    codes, scales = mb.mxfp8_quantize(x.to(DEV), axis=0)
    rc, rs = oq.quantize(om.f64(x), axis=0)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)
    _status_ok()


@pytest.mark.parametrize("B,rows,cols,transpose", [(2, 64, 256, True), (3, 96, 320, True), (2, 64, 256, False),
                                                   (1, 128, 100, False), (4, 4096, 512, True)])
def test_quantize_axis1_bit_exact(B, rows, cols, transpose):
    rng = np.random.default_rng(rows * 3 + cols)
    v = (rng.standard_normal((B, rows, cols), dtype=np.float32) * 0.02).astype(np.float32)
    x = torch.from_numpy(v).to(torch.bfloat16)
    codes, scales = mb.mxfp8_quantize(x.to(DEV), axis=1, transpose_out=transpose)
    rc, rs = oq.quantize(om.f64(x), axis=1, transpose_out=transpose)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)
    _status_ok()


@pytest.mark.parametrize("B,rows,cols", [(2, 128, 256), (3, 256, 384), (8, 512, 128)])
def test_quantize_mma_scale_layout_bit_exact(B, rows, cols):
    from tests.mx_layout import plain_to_atoms
    rng = np.random.default_rng(rows + 7 * cols)
    x = torch.from_numpy((rng.standard_normal((B, rows, cols), dtype=np.float32) * 0.02)).to(torch.bfloat16)
    codes, atoms = mb.mxfp8_quantize(x.to(DEV), axis=1, transpose_out=True, mma_scales=True)
    rc, rs = oq.quantize(om.f64(x), axis=1, transpose_out=True)          # [B, cols, rows], [B, cols, rows/32]
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(atoms.cpu().numpy(), plain_to_atoms(rs.reshape(B * cols, rows // 32)))


def test_quantize_golden_block_and_edges():
    # the hand-worked block of tests/golden/mxfp8_block.txt (values exact in bf16 except 0.1)
    from tests.golden import load
    g = load("mxfp8_block.txt")
    v = torch.zeros(1, 32)
    v[0, :6] = torch.tensor(g["values"])
    v[0, 5] = -0.0
    x = v.to(torch.bfloat16)
    codes, scales = mb.mxfp8_quantize(x.to(DEV), axis=0)
    rc, rs = oq.quantize(om.f64(x), axis=0)
    assert np.array_equal(codes.cpu().numpy(), rc) and np.array_equal(scales.cpu().numpy(), rs)
    assert scales.item() == g["scale"]
    assert list(codes.cpu().numpy()[0, :6]) == [0x70, 0xFA, rc[0, 2], 0x7C, 0x38, 0x80]


def test_bad_expert_index_sets_device_error():
    T, H, E, k = 64, 64, 4, 2
    x = torch.zeros((T, H), dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros((T, k), dtype=torch.int32, device=DEV)
    idx[3, 1] = 7                                  # out of range
    o = mb.moe_permute(x, idx, None, E)
    assert mb.moe_device_status() == 4             # MOE_ERR_DEVICE_CHECK, and cleared
    assert o["row_map"].cpu()[7].item() == -1
    assert mb.moe_device_status() == 0
