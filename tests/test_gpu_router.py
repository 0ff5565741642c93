"""GPU parity of the router backward (moe_route_bwd) and of the fused route + permutation
(moe_route_permute) against the fp64 oracle.

moe_route_bwd: dlogits within 1e-5 * max|ref| + 1e-6 of oracle.moe.route_bwd. The bound
comes from the inputs: the kernel takes the forward's fp32 probabilities (within 1e-6 of
the exact ones, the routing parity bound) and dlogits is linear in them with coefficients
|dprob_j - D| of order max|dprob|; fp32 rounding of the few products and sums adds a few
ulps.

moe_route_permute: every output bit-exact with the oracle's route / permutation (and so
with the two separate calls), on shapes that take the fused launch and shapes that fall
back to the separate kernels, with the workspace reused across calls.
"""
import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"

ROUTE_BWD_CASES = [(256, 4, 2), (1000, 8, 2), (777, 128, 8), (64, 1, 1), (33, 5, 5), (1, 40, 3), (513, 1024, 32),
                   (300, 33, 7), (4096, 256, 16)]


def _within(got, ref, name):
    err = np.max(np.abs(got - ref))
    bound = 1e-5 * np.max(np.abs(ref)) + 1e-6
    assert err <= bound, f"{name}: max err {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("T,E,k", ROUTE_BWD_CASES)
@pytest.mark.parametrize("renorm", [True, False])
def test_route_bwd_parity(T, E, k, renorm):
    rng = np.random.default_rng(T * 3 + E + k)
    lg = rng.standard_normal((T, E), dtype=np.float32)
    lg[: T // 4] = np.round(lg[: T // 4])            # exact ties on a quarter of the tokens
    dprob = rng.standard_normal((T, k), dtype=np.float32)
    lg_d = torch.from_numpy(lg).to(DEV)
    idx, prob = mb.moe_route(lg_d, k, renorm)
    ridx, _ = om.route(lg, k, renorm)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    dl = mb.moe_route_bwd(lg_d if not renorm else None, idx, prob, torch.from_numpy(dprob).to(DEV), renorm,
                          dlogits=torch.full((T, E), float("nan"), device=DEV))
    assert mb.moe_device_status() == 0
    ref = om.route_bwd(lg, ridx, dprob, renorm)
    got = dl.cpu().numpy()
    assert np.all(np.isfinite(got))                  # every entry written
    _within(got, ref, "dlogits")
    if renorm:
        sel = np.zeros((T, E), dtype=bool)
        sel[np.arange(T)[:, None], ridx] = True
        assert np.all(got[~sel] == 0.0)
    # shift invariance of the softmax: every row sums to zero
    assert np.max(np.abs(got.sum(axis=1))) <= 1e-5 * max(1.0, np.max(np.abs(ref))) * np.sqrt(E)


@pytest.mark.parametrize("renorm", [True, False])
def test_route_bwd_repeated_experts(renorm):
    """The call accepts any idx in range, repeated experts included (their slots add)."""
    rng = np.random.default_rng(5)
    T, E, k = 200, 6, 4
    lg = rng.standard_normal((T, E))
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[:, 1] = idx[:, 0]                            # at least one repeat per token
    s = np.exp(lg - lg.max(axis=1, keepdims=True))
    s /= s.sum(axis=1, keepdims=True)
    q = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    p = q / q.sum(axis=1, keepdims=True) if renorm else q
    dprob = rng.standard_normal((T, k))
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)
    dl = mb.moe_route_bwd(f32(lg), torch.from_numpy(idx).to(DEV), f32(p), f32(dprob), renorm)
    assert mb.moe_device_status() == 0
    _within(dl.cpu().numpy(), om.route_bwd(lg.astype(np.float32), idx, dprob.astype(np.float32), renorm),
            "dlogits")


def test_route_bwd_bad_index_sets_device_error():
    T, E, k = 8, 4, 2
    idx = torch.zeros((T, k), dtype=torch.int32, device=DEV)
    idx[3, 1] = 7                                    # out of range: flagged, slot skipped
    ones = torch.ones((T, k), dtype=torch.float32, device=DEV)
    mb.moe_route_bwd(None, idx, ones * 0.5, ones, True, dlogits=torch.empty((T, E), device=DEV))
    assert mb.moe_device_status() == 4             # MOE_ERR_DEVICE_CHECK
    assert mb.moe_device_status() == 0               # the word was cleared


FUSED_CASES = [
    (256, 128, 4, 2, "bf16"),       # fused (8 lanes per token)
    (8192, 64, 8, 2, "bf16"),       # fused, several blocks (8 lanes per token)
    (3001, 64, 5, 4, "mxfp8"),      # fused, 8 lanes per token, k = 4, ragged last block
    (4096, 64, 16, 4, "bf16"),      # fused, 16 lanes per token
    (2000, 64, 13, 2, "mxfp8"),     # fused, 16 lanes per token, E not a power of two
    (600, 64, 32, 4, "bf16"),       # fused, a warp per token
    (16384, 64, 128, 8, "bf16"),    # fused, Qwen3's routing shape
    (3000, 96, 256, 16, "mxfp8"),   # fused, largest E of the fused launch, ragged last block
    (1, 32, 1, 1, "bf16"),          # fused, one token
    (777, 64, 1024, 32, "bf16"),    # E > 256: separate kernels
    (500, 64, 12, 3, "mxfp8"),      # k does not divide 1024: separate kernels
]


@pytest.mark.parametrize("T,H,E,k,prec", FUSED_CASES)
def test_route_permute_matches_oracle(T, H, E, k, prec):
    ws = torch.empty(mb.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    for seed in (T, T + 1):                          # two calls reuse the workspace and its counter
        d = workloads.small_layer(T, H, 128, E, k, seed=seed, with_grad=False)
        lg = d["logits"].numpy()
        lg[: T // 5] = np.round(lg[: T // 5])
        o = mb.moe_route_permute(torch.from_numpy(lg).to(DEV), d["x"].to(DEV), k, True, prec, workspace=ws)
        assert mb.moe_device_status() == 0
        ridx, rprob = om.route(lg, k)
        assert np.array_equal(o["idx"].cpu().numpy(), ridx)
        # the fused launch routes 32 / W tokens per warp for E <= 16: the same bits as the
        # warp-per-token routing kernel
        uidx, uprob = mb.moe_route(torch.from_numpy(lg).to(DEV), k, True)
        assert torch.equal(uidx, o["idx"]) and torch.equal(uprob, o["prob"])
        assert np.max(np.abs(o["prob"].cpu().numpy() - rprob)) <= 1e-6
        row_map, split, offsets = om.permute_index(ridx, E)
        assert np.array_equal(o["row_map"].cpu().numpy(), row_map)
        assert np.array_equal(o["split_sizes"].cpu().numpy(), split)
        assert np.array_equal(o["offsets"].cpu().numpy(), offsets)
        assert np.array_equal(o["probs_perm"].cpu().numpy(), o["prob"].cpu().numpy().reshape(-1)[np.argsort(row_map)])
        # the data rows against the separate permutation call on the same routing
        sep = mb.moe_permute(d["x"].to(DEV), o["idx"], o["prob"], E, prec)
        assert torch.equal(sep["xp"], o["xp"])
        if prec == "mxfp8":
            assert torch.equal(sep["xp_scale"], o["xp_scale"])


@pytest.mark.parametrize("T,E,k", [(2048, 8, 2), (999, 13, 3), (64, 2, 2)])
def test_route_permute_no_renorm_narrow(T, E, k):
    """Fused routing with 8 / 16 lanes per token and renorm off: idx bit-exact and prob
    within 1e-6 of the oracle, and the same bits as the warp-per-token routing kernel."""
    rng = np.random.default_rng(T + E)
    lg = rng.standard_normal((T, E), dtype=np.float32)
    lg[: T // 4] = np.round(lg[: T // 4])            # exact ties between experts
    x = torch.from_numpy(rng.standard_normal((T, 64), dtype=np.float32)).to(torch.bfloat16)
    ws = torch.empty(mb.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    o = mb.moe_route_permute(torch.from_numpy(lg).to(DEV), x.to(DEV), k, False, "bf16", workspace=ws)
    assert mb.moe_device_status() == 0
    ridx, rprob = om.route(lg, k, renorm=False)
    assert np.array_equal(o["idx"].cpu().numpy(), ridx)
    assert np.max(np.abs(o["prob"].cpu().numpy() - rprob)) <= 1e-6
    uidx, uprob = mb.moe_route(torch.from_numpy(lg).to(DEV), k, False)
    assert torch.equal(uidx, o["idx"]) and torch.equal(uprob, o["prob"])
