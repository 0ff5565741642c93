"""The bounded waits of the grouped GEMMs: a launch whose data never arrives reports
MOE_ERR_TIMEOUT and returns, and the next call on the same context is correct.

The stall is made on the host side (moe_test_stall_gemm: the chosen launch's producers
issue no copies, so nothing is ever in flight and the first wait for data runs out after
a short budget). No fault, trap or endless loop is involved.
"""
import time

import numpy as np
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
from oracle import moe as om
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
MOE_OK, MOE_ERR_TIMEOUT = 0, 5
BUDGET_NS = 2_000_000     # 2 ms


def _layer(prec):
    T, H, F, E, k = 512, 256, 256, 4, 2
    d = workloads.small_layer(T, H, F, E, k, seed=17, with_grad=True)
    layer = mb.MoEExpertLayer(T, H, F, E, k, prec, training=True, device=DEV)
    layer.set_weights(d["w1"].to(DEV), d["w2"].to(DEV))
    return layer, d


def _rel(got, ref):
    return float(np.max(np.abs(got.float().cpu().numpy() - ref)) / np.max(np.abs(ref)))


@pytest.mark.parametrize("prec", ["bf16", "mxfp8"])
@pytest.mark.parametrize("which", [0, 1, 2, 3, 4, 5])
def test_stalled_gemm_times_out_then_next_call_is_correct(prec, which):
    """which: 0/1 = fc1/fc2 of the forward; 2..5 = fc2 dgrad, fc2 wgrad, fc1 dgrad, fc1
    wgrad of the backward (every grouped GEMM kernel of both precisions)."""
    layer, d = _layer(prec)
    x, lg, g = d["x"].to(DEV), d["logits"].to(DEV), d["grad_out"].to(DEV)
    layer.forward(x, lg)
    layer.backward(g)
    assert mb.moe_device_status() == MOE_OK
    mb.moe_test_stall_gemm(which, BUDGET_NS)
    t0 = time.perf_counter()
    layer.forward(x, lg)
    layer.backward(g)
    status = mb.moe_device_status()           # synchronises
    elapsed = time.perf_counter() - t0
    assert status == MOE_ERR_TIMEOUT
    # the stalled launch used the short budget, not the 4 s default (a few waits in turn)
    assert elapsed < 1.0, elapsed
    # the context is usable and the next pass is correct
    out = layer.forward(x, lg).clone()
    dx, dw1, dw2, _ = layer.backward(g)
    assert mb.moe_device_status() == MOE_OK
    ridx, rprob = om.route(d["logits"], 2)
    if prec == "bf16":
        ref = om.moe_forward_per_token(d["x"], ridx, rprob, d["w1"], d["w2"], a_round="bf16")
        assert _rel(out, ref) <= 1e-2
        row_map, split, _ = om.permute_index(ridx, 4)
        xp = om.permute_rows(om.f64(d["x"]), row_map, 2)
        pp = om.permute_probs(rprob, row_map)
        dyp = om.permute_rows(om.f64(d["grad_out"]), row_map, 2)
        rdxp, rdw1, rdw2, _, _ = om.grouped_mlp_bwd(dyp, xp, split, d["w1"], d["w2"], pp, a_round="bf16")
        rdx, _ = om.moe_backward_tokens(rdxp, np.zeros(xp.shape[0]), row_map, 512, 2)
        assert _rel(dx, rdx) <= 1e-2 and _rel(dw1, rdw1) <= 1e-2 and _rel(dw2, rdw2) <= 1e-2
    else:
        # the MXFP8 layer against the unquantised definition, at its quantisation error
        ref = om.moe_forward_per_token(d["x"], ridx, rprob, d["w1"], d["w2"], a_round="f64")
        assert _rel(out, ref) <= 0.15


def test_stall_hook_rejects_bad_budgets():
    with pytest.raises(mb.MoEError):
        mb.moe_test_stall_gemm(0, 10)
    with pytest.raises(mb.MoEError):
        mb.moe_test_stall_gemm(-1, 1_000_000)
