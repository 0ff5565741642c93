"""One MoE expert-MLP layer on preallocated device buffers, sequencing the C-ABI calls.

forward:  moe_route_permute (route + permutation) -> grouped_mlp_fwd -> moe_unpermute
backward: moe_permute_rows(grad_out) -> grouped_mlp_bwd -> moe_unpermute(dxp) -> moe_gather_slots
          -> moe_route_bwd (dlogits)
MXFP8 training: the weights are quantised in both orientations at once (mxfp8_quantize_weights),
the forward also quantises the permuted x along the expert rows and the backward permutes and
quantises grad_out both ways (moe_permute_rows_mxfp8), so grouped_mlp_bwd gets every operand
already quantised (grouped_mlp_bwd_mxfp8_operands) and no bf16 permuted copy is written.

All arithmetic runs in libmoe_grouped.so; this module only owns buffers and call order.
"""
from __future__ import annotations

import torch

from . import (BF16, FP8, MXFP8, _PREC, fp8_quantize, grouped_mlp_bwd, grouped_mlp_bwd_workspace_size, grouped_mlp_fwd,
               grouped_mlp_fwd_combine, grouped_mlp_fwd_combine_workspace_size, grouped_mlp_saved_size, grouped_mlp_workspace_size, moe_gather_slots, moe_permute_rows,
               moe_permute_rows_mxfp8, moe_permute_workspace_size, moe_route_bwd, moe_route_permute, moe_unpermute,
               mxfp8_quantize, mxfp8_quantize_weights)


def lib_ws_bytes(T: int, k: int) -> int:
    from . import lib
    return max(int(lib().moe_permute_rows_mxfp8_workspace_size(T, k)), 1)


class MoEExpertLayer:
    def __init__(self, T: int, H: int, F: int, E: int, k: int, precision="bf16", training: bool = False,
                 renorm: bool = True, device="cuda", fused_combine: bool = False):
        self.T, self.H, self.F, self.E, self.k = T, H, F, E, k
        self.R = T * k
        self.prec = _PREC[precision]
        self.precision = {BF16: "bf16", MXFP8: "mxfp8", FP8: "fp8"}[self.prec]
        # the permutation moves bf16 rows except for MXFP8, whose permute quantises them
        self.perm_precision = "mxfp8" if self.prec == MXFP8 else "bf16"
        self.training = training
        self.renorm = renorm
        # fused_combine: fc2's epilogue adds its rows into the token outputs (no yp)
        self.fused_combine = fused_combine
        dev = torch.device(device)
        self.device = dev
        R = self.R
        u8, i32, f32, bf = torch.uint8, torch.int32, torch.float32, torch.bfloat16
        self.idx = torch.empty((T, k), dtype=i32, device=dev)
        self.prob = torch.empty((T, k), dtype=f32, device=dev)
        self.perm = {
            "xp": torch.empty((R, H), dtype=u8 if self.prec == MXFP8 else bf, device=dev),
            "row_map": torch.empty(R, dtype=i32, device=dev),
            "probs_perm": torch.empty(R, dtype=f32, device=dev),
            "split_sizes": torch.empty(E, dtype=i32, device=dev),
            "offsets": torch.empty(E + 1, dtype=i32, device=dev),
        }
        if self.prec == MXFP8:
            self.perm["xp_scale"] = torch.empty((R, H // 32), dtype=u8, device=dev)
        if self.prec == FP8:
            # per-tensor E4M3 codes of the permuted rows and their scale
            self.xq = torch.empty((R, H), dtype=u8, device=dev)
            self.xq_scale = torch.empty(1, dtype=f32, device=dev)
        self.perm_ws = torch.empty(max(moe_permute_workspace_size(T, k, E), 1), dtype=u8, device=dev)
        self.yp = None if fused_combine else torch.empty((R, H), dtype=bf, device=dev)
        self.out = torch.empty((T, H), dtype=bf, device=dev)
        ws_bytes = (grouped_mlp_fwd_combine_workspace_size(E, R, H, F, self.precision, training, T) if fused_combine
                    else grouped_mlp_workspace_size(E, R, H, F, self.precision, training))
        self.mlp_ws = torch.empty(ws_bytes, dtype=u8, device=dev)
        self.saved = (torch.empty(grouped_mlp_saved_size(E, R, H, F, self.precision), dtype=u8, device=dev)
                      if training else None)
        self.w1 = self.w2 = None
        self.w1_scale = self.w2_scale = None
        self.w_rows = None
        self.xp_cols = None
        self._perm_q_ws = (torch.empty(int(lib_ws_bytes(T, k)), dtype=u8, device=dev)
                           if training and self.prec == MXFP8 else None)
        self._bwd = None

    # --------------------------------------------------------------- weights
    def set_weights(self, w1: torch.Tensor, w2: torch.Tensor, stream=None):
        """w1 [E, H, 2F] and w2 [E, F, H] bf16 masters on the device. The MXFP8 layer
        quantises them here (once per optimizer step) into K-major E4M3 codes."""
        self.w1_master, self.w2_master = w1, w2
        if self.prec == BF16:
            self.w1, self.w2 = w1, w2
        elif self.prec == FP8:
            # one E4M3 scale per expert, codes K-major for the forward GEMMs
            self.w1, self.w1_scale = fp8_quantize(w1, "e4m3", transpose_out=True, stream=stream)
            self.w2, self.w2_scale = fp8_quantize(w2, "e4m3", transpose_out=True, stream=stream)
        elif self.training:
            # both MXFP8 forms in one pass: K-major along H / F for the forward, along the
            # other axis for the backward's data-gradient GEMMs
            self.w1, self.w1_scale, w1r, w1ra = mxfp8_quantize_weights(w1, stream=stream)
            self.w2, self.w2_scale, w2r, w2ra = mxfp8_quantize_weights(w2, stream=stream)
            self.w_rows = {"w1_rows": w1r, "w1_rows_atoms": w1ra, "w2_rows": w2r, "w2_rows_atoms": w2ra}
        else:
            self.w1, self.w1_scale = mxfp8_quantize(w1, axis=1, transpose_out=True, mma_scales=True, stream=stream)
            self.w2, self.w2_scale = mxfp8_quantize(w2, axis=1, transpose_out=True, mma_scales=True, stream=stream)

    # --------------------------------------------------------------- forward
    def forward(self, x: torch.Tensor, logits: torch.Tensor, stream=None) -> torch.Tensor:
        self.perm["idx"], self.perm["prob"] = self.idx, self.prob
        moe_route_permute(logits, x, self.k, self.renorm, self.perm_precision, out=self.perm,
                          workspace=self.perm_ws, stream=stream)
        self.logits = logits
        xp, xp_scale = self.perm["xp"], self.perm.get("xp_scale")
        if self.prec == FP8:
            fp8_quantize(self.perm["xp"], "e4m3", codes=self.xq, scales=self.xq_scale, stream=stream)
            xp, xp_scale = self.xq, self.xq_scale
        if self.fused_combine:
            grouped_mlp_fwd_combine(xp, self.perm["split_sizes"], self.w1, self.w2,
                                    self.perm["probs_perm"], self.perm["row_map"], self.T, self.k, self.precision,
                                    xp_scale=xp_scale, w1_scale=self.w1_scale,
                                    w2_scale=self.w2_scale, out=self.out, saved=self.saved, workspace=self.mlp_ws,
                                    F=self.F, stream=stream)
        else:
            grouped_mlp_fwd(xp, self.perm["split_sizes"], self.w1, self.w2, self.perm["probs_perm"],
                            self.precision, xp_scale=xp_scale, w1_scale=self.w1_scale,
                            w2_scale=self.w2_scale, yp=self.yp, saved=self.saved, workspace=self.mlp_ws, F=self.F,
                            stream=stream)
            moe_unpermute(self.yp, self.perm["row_map"], self.T, self.k, out=self.out, stream=stream)
        if self.training and self.prec == MXFP8:
            self.permute_for_backward(x, stream=stream)
        return self.out

    def bwd_operands(self):
        """MXFP8 backward operands this layer already holds quantised (None otherwise)."""
        if self.prec != MXFP8 or self.w_rows is None:
            return None
        ops = dict(self.w_rows)
        if self.xp_cols is not None:
            ops.update(xp_cols=self.xp_cols["cols"], xp_cols_atoms=self.xp_cols["cols_atoms"])
        if self._bwd is not None and self._bwd.get("dyq") is not None:
            q = self._bwd["dyq"]
            ops.update(dy_rows=q["rows"], dy_rows_atoms=q["rows_atoms"], dy_cols=q["cols"],
                       dy_cols_atoms=q["cols_atoms"])
        return ops

    def permute_for_backward(self, x: torch.Tensor, stream=None):
        """The MXFP8 fc1 weight gradient reads xp quantised along each expert's rows:
        permute and quantise x that way (no bf16 copy of the permuted rows)."""
        if self.xp_cols is None:
            self.xp_cols = {}
            self._perm_q_ws = None
        self.xp_cols = moe_permute_rows_mxfp8(x, self.perm["row_map"], self.k, self.perm["split_sizes"], rows=False,
                                              cols=True, out=self.xp_cols, workspace=self._perm_q_ws, stream=stream)

    def permute_grad(self, grad_out: torch.Tensor, stream=None):
        """The MXFP8 backward's dy in both forms (along H and along each expert's rows)."""
        b = self._bwd
        b["dyq"] = moe_permute_rows_mxfp8(grad_out, self.perm["row_map"], self.k, self.perm["split_sizes"],
                                          out=b.get("dyq"), workspace=self._perm_q_ws, stream=stream)

    # -------------------------------------------------------------- backward
    def _alloc_bwd(self):
        T, H, F, E, R = self.T, self.H, self.F, self.E, self.R
        dev, bf = self.device, torch.bfloat16
        self._bwd = {
            "dy_perm": torch.empty((R, H), dtype=bf, device=dev) if self.prec != MXFP8 else None,
            "dxp": torch.empty((R, H), dtype=bf, device=dev),
            "dw1": torch.empty((E, H, 2 * F), dtype=bf, device=dev),
            "dw2": torch.empty((E, F, H), dtype=bf, device=dev),
            "dprobs_perm": torch.empty(R, dtype=torch.float32, device=dev),
            "dx": torch.empty((T, H), dtype=bf, device=dev),
            "dprob": torch.empty((T, self.k), dtype=torch.float32, device=dev),
            "dlogits": torch.empty((T, E), dtype=torch.float32, device=dev),
            "ws": torch.empty(grouped_mlp_bwd_workspace_size(E, R, H, F, self.precision), dtype=torch.uint8,
                              device=dev),
        }

    def backward(self, grad_out: torch.Tensor, stream=None, router: bool = True):
        """Gradients of the last forward: returns (dx [T,H], dw1, dw2, dprob [T,k]); with
        ``router`` the router's dlogits [T,E] are in ``self.dlogits`` too."""
        if not self.training:
            raise RuntimeError("layer was built without training=True")
        if self._bwd is None:
            self._alloc_bwd()
        b = self._bwd
        if self.prec == MXFP8:
            self.permute_grad(grad_out, stream=stream)
            grouped_mlp_bwd(None, self.perm["split_sizes"], None, self.w1_master, self.w2_master,
                            self.perm["probs_perm"], self.saved, self.precision, dxp=b["dxp"], dw1=b["dw1"],
                            dw2=b["dw2"], dprobs_perm=b["dprobs_perm"], workspace=b["ws"], stream=stream,
                            operands=self.bwd_operands(), shape=(self.R, self.H, self.F))
        else:
            moe_permute_rows(grad_out, self.perm["row_map"], self.k, out=b["dy_perm"], stream=stream)
            grouped_mlp_bwd(b["dy_perm"], self.perm["split_sizes"], self.perm["xp"], self.w1_master,
                            self.w2_master, self.perm["probs_perm"], self.saved, self.precision, dxp=b["dxp"],
                            dw1=b["dw1"], dw2=b["dw2"], dprobs_perm=b["dprobs_perm"], workspace=b["ws"],
                            stream=stream)
        moe_unpermute(b["dxp"], self.perm["row_map"], self.T, self.k, out=b["dx"], stream=stream)
        moe_gather_slots(b["dprobs_perm"], self.perm["row_map"], out=b["dprob"].view(-1), stream=stream)
        if router:
            moe_route_bwd(None if self.renorm else self.logits, self.idx, self.prob, b["dprob"], self.renorm,
                          dlogits=b["dlogits"], stream=stream)
        self.dlogits = b["dlogits"] if router else None
        return b["dx"], b["dw1"], b["dw2"], b["dprob"]

    def allreduce_weight_grads(self, group=None, average: bool = False):
        """Sum (or average) dw1 and dw2 of the last backward over the data-parallel group."""
        return allreduce_grads([self._bwd["dw1"], self._bwd["dw2"]], group=group, average=average)


def allreduce_grads(tensors, group=None, average: bool = False):
    """The data-parallel backward's one exchange: sum (or average) gradients over the
    replicas of `group` in place with torch.distributed (NCCL over NVLink on GPUs, gloo on
    CPU), one all-reduce per tensor, enqueued on the current stream."""
    import torch.distributed as dist
    n = dist.get_world_size(group)
    for t in tensors:
        dist.all_reduce(t, group=group)
        if average and n > 1:
            t.div_(n)
    return tensors


def moe_layer_forward(x, logits, w1, w2, k: int, precision="bf16", stream=None):
    """One-shot forward of a layer (allocates its buffers; use MoEExpertLayer to reuse them)."""
    T, H = x.shape
    E, _, F2 = w1.shape
    layer = MoEExpertLayer(T, H, F2 // 2, E, k, precision, device=x.device)
    layer.set_weights(w1, w2, stream=stream)
    return layer.forward(x, logits, stream=stream), layer


class HostPipeline:
    """Run a layer on host (pinned) buffers with the transfers overlapped.

    Each call to :meth:`step` uploads one batch (x, logits, and grad_out for a training
    layer) on an upload stream, runs the layer on the compute stream, and downloads its
    result (the output; with backward also dx) on a download stream. Device input and
    output buffers are double-buffered, so step i's upload and step i-1's download run
    while step i-1 / i compute. :meth:`flush` waits for everything issued.
    """

    def __init__(self, layer: MoEExpertLayer):
        self.layer = layer
        dev = layer.device
        T, H, E = layer.T, layer.H, layer.E
        bf = torch.bfloat16
        self.compute = torch.cuda.current_stream(dev)
        self.up = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.x = [torch.empty((T, H), dtype=bf, device=dev) for _ in range(2)]
        self.lg = [torch.empty((T, E), dtype=torch.float32, device=dev) for _ in range(2)]
        self.g = [torch.empty((T, H), dtype=bf, device=dev) for _ in range(2)] if layer.training else None
        self.out = [torch.empty((T, H), dtype=bf, device=dev) for _ in range(2)]
        self.dx = [torch.empty((T, H), dtype=bf, device=dev) for _ in range(2)] if layer.training else None
        self.uploaded = [torch.cuda.Event() for _ in range(2)]
        self.inputs_free = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.downloaded = [torch.cuda.Event() for _ in range(2)]
        self.i = 0

    def step(self, x_h, logits_h, out_h, grad_h=None, dx_h=None):
        b = self.i & 1
        # upload into buffer b once the step that last used it has consumed its inputs
        self.up.wait_event(self.inputs_free[b])
        with torch.cuda.stream(self.up):
            self.x[b].copy_(x_h, non_blocking=True)
            self.lg[b].copy_(logits_h, non_blocking=True)
            if self.g is not None:
                self.g[b].copy_(grad_h, non_blocking=True)
            self.uploaded[b].record(self.up)
        # compute once the inputs are there and the previous download of buffer b is done
        self.compute.wait_event(self.uploaded[b])
        self.compute.wait_event(self.downloaded[b])
        with torch.cuda.stream(self.compute):
            out = self.layer.forward(self.x[b], self.lg[b], stream=self.compute)
            self.out[b].copy_(out, non_blocking=True)
            if self.g is not None:
                dx = self.layer.backward(self.g[b], stream=self.compute)[0]
                self.dx[b].copy_(dx, non_blocking=True)
            self.inputs_free[b].record(self.compute)
            self.computed[b].record(self.compute)
        # download the result
        self.down.wait_event(self.computed[b])
        with torch.cuda.stream(self.down):
            out_h.copy_(self.out[b], non_blocking=True)
            if self.dx is not None:
                dx_h.copy_(self.dx[b], non_blocking=True)
            self.downloaded[b].record(self.down)
        self.i += 1

    def flush(self):
        self.compute.wait_stream(self.up)
        self.compute.wait_stream(self.down)
