"""HostPipeline: overlapped host<->device transfers give exactly the layer's results."""
import pytest
import torch

import mixture_experts_grouped_top_b200 as mb
import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("training", [False, True])
def test_host_pipeline_matches_direct_calls(training):
    T, H, F, E, k = 300, 256, 256, 6, 2
    layer = mb.MoEExpertLayer(T, H, F, E, k, training=training)
    batches = [workloads.small_layer(T, H, F, E, k, seed=s, with_grad=True) for s in range(4)]
    layer.set_weights(batches[0]["w1"].cuda(), batches[0]["w2"].cuda())
    ref_out, ref_dx = [], []
    for d in batches:
        ref_out.append(layer.forward(d["x"].cuda(), d["logits"].cuda()).cpu().clone())
        if training:
            ref_dx.append(layer.backward(d["grad_out"].cuda())[0].cpu().clone())
    pipe = mb.HostPipeline(layer)
    outs = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in batches]
    dxs = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in batches]
    ins = [(d["x"].pin_memory(), d["logits"].pin_memory(), d["grad_out"].pin_memory()) for d in batches]
    for (x_h, lg_h, g_h), o_h, dx_h in zip(ins, outs, dxs):
        pipe.step(x_h, lg_h, o_h, g_h if training else None, dx_h if training else None)
    pipe.flush()
    torch.cuda.synchronize()
    for i in range(len(batches)):
        assert torch.equal(outs[i], ref_out[i])
        if training:
            assert torch.equal(dxs[i], ref_dx[i])
    assert mb.moe_device_status() == 0
