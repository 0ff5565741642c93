"""B200 (sm_100a) MoE expert-MLP hot path: Python binding of the C ABI in include/moe_grouped.h.

Every function here only marshals arguments (torch CUDA tensors -> device pointers and
the current CUDA stream) and calls the function of the same name in libmoe_grouped.so;
all computation runs in the library's CUDA kernels. Output and scratch buffers are
allocated here with torch when the caller does not pass them (the library itself never
allocates). There is no CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

BF16 = 0
MXFP8 = 1
FP8 = 2
OUT_F32 = 0x100
_PREC = {"bf16": BF16, "mxfp8": MXFP8, "fp8": FP8, BF16: BF16, MXFP8: MXFP8, FP8: FP8}
_FP8_FMT = {"e4m3": 0, "e5m2": 1}

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
          4: "MOE_ERR_DEVICE_CHECK", 5: "MOE_ERR_TIMEOUT"}


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


def lib():
    return _lib.load()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(name: str, rc: int):
    if rc != 0:
        raise MoEError(name, rc)


def _need(t, dtype, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ------------------------------------------------------------------ status helpers
def moe_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return lib().moe_device_status(_stream(stream))


def moe_launch_count() -> int:
    return int(lib().moe_launch_count())


def moe_test_stall_gemm(skip: int, timeout_ns: int) -> None:
    """Test hook: after `skip` grouped GEMM launches, the next one issues no loads and its
    waits run out after timeout_ns (it then reports MOE_ERR_TIMEOUT through
    moe_device_status)."""
    _check("moe_test_stall_gemm", lib().moe_test_stall_gemm(int(skip), int(timeout_ns)))


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


# ------------------------------------------------------------------------ routing
def moe_route(logits, k: int, renorm: bool = True, idx=None, prob=None, stream=None):
    _need(logits, torch.float32, "logits")
    T, E = logits.shape
    idx = torch.empty((T, k), dtype=torch.int32, device=logits.device) if idx is None else idx
    prob = torch.empty((T, k), dtype=torch.float32, device=logits.device) if prob is None else prob
    _check("moe_route", lib().moe_route(_p(logits), T, E, k, int(bool(renorm)), _p(idx), _p(prob), _stream(stream)))
    return idx, prob


def moe_route_bwd(logits, idx, prob, dprob, renorm: bool = True, dlogits=None, stream=None):
    """dL/dlogits [T, E] fp32 from dL/dprob [T, k] and the forward's idx / prob (logits
    may be None with renorm)."""
    _need(idx, torch.int32, "idx")
    _need(prob, torch.float32, "prob")
    _need(dprob, torch.float32, "dprob")
    T, k = idx.shape
    if logits is not None:
        _need(logits, torch.float32, "logits")
        E = logits.shape[1]
    elif dlogits is not None:
        E = dlogits.shape[1]
    else:
        raise ValueError("pass logits or dlogits (to give E)")
    dlogits = torch.empty((T, E), dtype=torch.float32, device=idx.device) if dlogits is None else dlogits
    _check("moe_route_bwd", lib().moe_route_bwd(_p(logits), _p(idx), _p(prob), _p(dprob), T, E, k,
                                                int(bool(renorm)), _p(dlogits), _stream(stream)))
    return dlogits


def moe_route_permute(logits, x, k: int, renorm: bool = True, precision="bf16", out=None, workspace=None,
                      stream=None):
    """moe_route + moe_permute with the routing and index build fused. Returns the
    moe_permute dict plus idx and prob."""
    _need(logits, torch.float32, "logits")
    _need(x, torch.bfloat16, "x")
    prec = _PREC[precision]
    T, E = logits.shape
    H = x.shape[1]
    R = T * k
    dev = x.device
    o = dict(out or {})
    o.setdefault("idx", torch.empty((T, k), dtype=torch.int32, device=dev))
    o.setdefault("prob", torch.empty((T, k), dtype=torch.float32, device=dev))
    if "xp" not in o:
        o["xp"] = torch.empty((R, H), dtype=torch.bfloat16 if prec == BF16 else torch.uint8, device=dev)
    if prec == MXFP8 and "xp_scale" not in o:
        o["xp_scale"] = torch.empty((R, H // 32), dtype=torch.uint8, device=dev)
    o.setdefault("row_map", torch.empty(R, dtype=torch.int32, device=dev))
    o.setdefault("probs_perm", torch.empty(R, dtype=torch.float32, device=dev))
    o.setdefault("split_sizes", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = torch.empty(moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=dev)
    rc = lib().moe_route_permute(_p(logits), _p(x), T, H, E, k, int(bool(renorm)), prec, _p(o["idx"]), _p(o["prob"]),
                                 _p(o["xp"]), _p(o.get("xp_scale")), _p(o["row_map"]), _p(o["probs_perm"]),
                                 _p(o["split_sizes"]), _p(o["offsets"]), _p(workspace), workspace.numel(),
                                 _stream(stream))
    _check("moe_route_permute", rc)
    o.setdefault("xp_scale", None)
    return o


def moe_permute_workspace_size(T: int, k: int, E: int) -> int:
    return int(lib().moe_permute_workspace_size(T, k, E))


def moe_permute(x, idx, prob, E: int, precision="bf16", out=None, workspace=None, stream=None):
    """Permute tokens into expert-contiguous rows. Returns a dict with xp, xp_scale
    (MXFP8 only), row_map, probs_perm (None when prob is None), split_sizes, offsets."""
    _need(x, torch.bfloat16, "x")
    _need(idx, torch.int32, "idx")
    prec = _PREC[precision]
    T, H = x.shape
    k = idx.shape[1]
    R = T * k
    dev = x.device
    o = dict(out or {})
    if "xp" not in o:
        o["xp"] = torch.empty((R, H), dtype=torch.bfloat16 if prec == BF16 else torch.uint8, device=dev)
    if prec == MXFP8 and "xp_scale" not in o:
        o["xp_scale"] = torch.empty((R, H // 32), dtype=torch.uint8, device=dev)
    o.setdefault("row_map", torch.empty(R, dtype=torch.int32, device=dev))
    if prob is not None:
        o.setdefault("probs_perm", torch.empty(R, dtype=torch.float32, device=dev))
    o.setdefault("split_sizes", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    ws_bytes = moe_permute_workspace_size(T, k, E)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    rc = lib().moe_permute(_p(x), _p(idx), _p(prob), T, H, E, k, prec, _p(o["xp"]), _p(o.get("xp_scale")),
                           _p(o["row_map"]), _p(o.get("probs_perm")), _p(o["split_sizes"]), _p(o["offsets"]),
                           _p(workspace), workspace.numel(), _stream(stream))
    _check("moe_permute", rc)
    o.setdefault("xp_scale", None)
    o.setdefault("probs_perm", None)
    return o


def moe_permute_noalloc(x, idx, prob, E: int, precision="bf16", out=None, stream=None):
    """moe_permute with the library's static scratch table instead of a workspace (for
    callers that must not allocate device memory); outputs as moe_permute."""
    _need(x, torch.bfloat16, "x")
    _need(idx, torch.int32, "idx")
    prec = _PREC[precision]
    T, H = x.shape
    k = idx.shape[1]
    o = dict(out)   # every output buffer is passed by the caller
    rc = lib().moe_permute_noalloc(_p(x), _p(idx), _p(prob), T, H, E, k, prec, _p(o["xp"]), _p(o.get("xp_scale")),
                                   _p(o["row_map"]), _p(o.get("probs_perm")), _p(o["split_sizes"]),
                                   _p(o["offsets"]), _stream(stream))
    _check("moe_permute_noalloc", rc)
    return o


def moe_permute_capacity_workspace_size(T: int, k: int, E: int) -> int:
    return int(lib().moe_permute_capacity_workspace_size(T, k, E))


def moe_permute_capacity(x, idx, prob, E: int, C: int, precision="bf16", out=None, workspace=None, stream=None):
    """Capacity-padded dispatch into [E*C] rows (slots past an expert's capacity dropped).
    Returns a dict with xp, xp_scale (MXFP8), row_map, probs_perm, split_sizes, offsets, kept."""
    _need(x, torch.bfloat16, "x")
    _need(idx, torch.int32, "idx")
    prec = _PREC[precision]
    T, H = x.shape
    k = idx.shape[1]
    dev = x.device
    o = dict(out or {})
    RC = E * C
    if "xp" not in o:
        o["xp"] = torch.empty((RC, H), dtype=torch.bfloat16 if prec == BF16 else torch.uint8, device=dev)
    if prec == MXFP8 and "xp_scale" not in o:
        o["xp_scale"] = torch.empty((RC, H // 32), dtype=torch.uint8, device=dev)
    o.setdefault("row_map", torch.empty(T * k, dtype=torch.int32, device=dev))
    if prob is not None:
        o.setdefault("probs_perm", torch.empty(RC, dtype=torch.float32, device=dev))
    o.setdefault("split_sizes", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    o.setdefault("kept", torch.empty(E, dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = torch.empty(max(moe_permute_capacity_workspace_size(T, k, E), 1), dtype=torch.uint8, device=dev)
    rc = lib().moe_permute_capacity(_p(x), _p(idx), _p(prob), T, H, E, k, C, prec, _p(o["xp"]),
                                    _p(o.get("xp_scale")), _p(o["row_map"]), _p(o.get("probs_perm")),
                                    _p(o["split_sizes"]), _p(o["offsets"]), _p(o["kept"]), _p(workspace),
                                    workspace.numel(), _stream(stream))
    _check("moe_permute_capacity", rc)
    o.setdefault("xp_scale", None)
    o.setdefault("probs_perm", None)
    return o


def moe_permute_rows(src, row_map, k: int, out=None, stream=None):
    _need(src, torch.bfloat16, "src")
    T, H = src.shape
    out = torch.empty((T * k, H), dtype=torch.bfloat16, device=src.device) if out is None else out
    _check("moe_permute_rows", lib().moe_permute_rows(_p(src), _p(row_map), T, H, k, _p(out), _stream(stream)))
    return out


def moe_unpermute(yp, row_map, T: int, k: int, prob=None, out=None, stream=None):
    _need(yp, torch.bfloat16, "yp")
    H = yp.shape[1]
    out = torch.empty((T, H), dtype=torch.bfloat16, device=yp.device) if out is None else out
    _check("moe_unpermute",
           lib().moe_unpermute(_p(yp), _p(row_map), _p(prob), T, H, k, _p(out), _stream(stream)))
    return out


def moe_gather_slots(src, row_map, out=None, stream=None):
    R = row_map.numel()
    out = torch.empty(R, dtype=torch.float32, device=src.device) if out is None else out
    _check("moe_gather_slots", lib().moe_gather_slots(_p(src), _p(row_map), R, _p(out), _stream(stream)))
    return out


# ------------------------------------------------------------------------- MXFP8
SCALES_PLAIN = 0
SCALES_MMA = 1


def mma_scale_bytes(groups: int, K: int) -> int:
    return groups * (K // 128) * 512


def mxfp8_quantize(x, axis: int = 0, transpose_out: bool = False, codes=None, scales=None, mma_scales=False,
                   stream=None):
    """Quantise bf16 [batch, rows, cols] (or [rows, cols]). Returns (codes, scales) uint8.
    With ``mma_scales`` (axis 1, transpose_out) the scales come in the MMA atom layout
    (a flat uint8 tensor) that grouped_mlp_fwd expects for weights."""
    _need(x, torch.bfloat16, "x")
    squeeze = x.dim() == 2
    x3 = x.unsqueeze(0) if squeeze else x
    B, rows, cols = x3.shape
    dev = x.device
    if axis == 0:
        cshape, sshape = (B, rows, cols), (B, rows, cols // 32)
    elif transpose_out:
        cshape, sshape = (B, cols, rows), (B, cols, rows // 32)
    else:
        cshape, sshape = (B, rows, cols), (B, rows // 32, cols)
    if mma_scales:
        sshape = (B * cols * rows // 32,)
    codes = torch.empty(cshape, dtype=torch.uint8, device=dev) if codes is None else codes
    scales = torch.empty(sshape, dtype=torch.uint8, device=dev) if scales is None else scales
    rc = lib().mxfp8_quantize(_p(x3), B, rows, cols, axis, int(bool(transpose_out)),
                              SCALES_MMA if mma_scales else SCALES_PLAIN, _p(codes), _p(scales), _stream(stream))
    _check("mxfp8_quantize", rc)
    if squeeze:
        return codes.reshape(cshape[1:]), (scales if mma_scales else scales.reshape(sshape[1:]))
    return codes, scales


def moe_permute_rows_mxfp8(src, row_map, k, split_sizes, rows=True, cols=True, out=None, workspace=None,
                           stream=None):
    """moe_permute_rows fused with the MXFP8 quantisation of the permuted rows in the rows
    form (along H, tile atoms) and / or the cols form (along each expert's rows, grouped
    atoms). Returns a dict with "rows", "rows_atoms", "cols", "cols_atoms" (None where not
    asked for); ``out`` may hold preallocated tensors under those names."""
    _need(src, torch.bfloat16, "src")
    T, H = src.shape
    R = T * k
    E = split_sizes.numel()
    dev = src.device
    out = {} if out is None else out
    nat = int(lib().mxfp8_grouped_atoms_bytes(E, R, H))
    for name, want, shape in (("rows", rows, (R, H)), ("cols", cols, (R, H))):
        if want:
            if out.get(name) is None:
                out[name] = torch.empty(shape, dtype=torch.uint8, device=dev)
            if out.get(name + "_atoms") is None:
                out[name + "_atoms"] = torch.empty(max(nat, 1), dtype=torch.uint8, device=dev)
        else:
            out[name] = out[name + "_atoms"] = None
    if workspace is None:
        workspace = torch.empty(int(lib().moe_permute_rows_mxfp8_workspace_size(T, k)), dtype=torch.uint8,
                                device=dev)
    rc = lib().moe_permute_rows_mxfp8(_p(src), _p(row_map), T, H, k, _p(split_sizes), E, _p(out["rows"]),
                                      _p(out["rows_atoms"]), _p(out["cols"]), _p(out["cols_atoms"]), _p(workspace),
                                      workspace.numel(), _stream(stream))
    _check("moe_permute_rows_mxfp8", rc)
    return out


def mxfp8_quantize_weights(w, codes_t=None, atoms_t=None, codes_r=None, atoms_r=None, stream=None):
    """Both MXFP8 forms of bf16 weights [batch, rows, cols] in one pass: (codes_t
    [batch, cols, rows], atoms_t) blocked along rows (the forward's K-major operand, as
    mxfp8_quantize(axis=1, transpose_out=True, mma_scales=True)) and (codes_r
    [batch, rows, cols], atoms_r) blocked along cols (the backward's data-gradient
    operand). Returns (codes_t, atoms_t, codes_r, atoms_r)."""
    _need(w, torch.bfloat16, "w")
    B, rows, cols = w.shape
    dev = w.device
    n = B * rows * cols
    codes_t = torch.empty((B, cols, rows), dtype=torch.uint8, device=dev) if codes_t is None else codes_t
    codes_r = torch.empty((B, rows, cols), dtype=torch.uint8, device=dev) if codes_r is None else codes_r
    atoms_t = torch.empty(n // 32, dtype=torch.uint8, device=dev) if atoms_t is None else atoms_t
    atoms_r = torch.empty(n // 32, dtype=torch.uint8, device=dev) if atoms_r is None else atoms_r
    rc = lib().mxfp8_quantize_weights(_p(w), B, rows, cols, _p(codes_t), _p(atoms_t), _p(codes_r), _p(atoms_r),
                                      _stream(stream))
    _check("mxfp8_quantize_weights", rc)
    return codes_t, atoms_t, codes_r, atoms_r


def fp8_quantize(x, fmt="e4m3", transpose_out=False, codes=None, scales=None, stream=None):
    """Per-tensor FP8 (current scaling) of bf16 [batch, rows, cols] (or [rows, cols]): one
    fp32 scale per batch matrix. Returns (codes uint8, scales fp32 [batch])."""
    _need(x, torch.bfloat16, "x")
    squeeze = x.dim() == 2
    x3 = x.unsqueeze(0) if squeeze else x
    B, rows, cols = x3.shape
    cshape = (B, cols, rows) if transpose_out else (B, rows, cols)
    codes = torch.empty(cshape, dtype=torch.uint8, device=x.device) if codes is None else codes
    scales = torch.empty(B, dtype=torch.float32, device=x.device) if scales is None else scales
    ws = torch.empty(max(int(lib().fp8_quantize_workspace_size(B)), 1), dtype=torch.uint8, device=x.device)
    rc = lib().fp8_quantize(_p(x3), B, rows, cols, _FP8_FMT[fmt], int(bool(transpose_out)), _p(codes), _p(scales),
                            _p(ws), ws.numel(), _stream(stream))
    _check("fp8_quantize", rc)
    return (codes.reshape(cshape[1:]) if squeeze else codes), scales


def mxfp8_quantize_grouped(x, split_sizes, codes=None, atoms=None, stream=None):
    """Quantise expert-contiguous rows x [R, C] along the rows (32-row blocks restarting
    at every expert). Returns (codes [R, C] uint8, scale atoms (flat uint8))."""
    _need(x, torch.bfloat16, "x")
    R, C = x.shape
    E = split_sizes.numel()
    codes = torch.empty((R, C), dtype=torch.uint8, device=x.device) if codes is None else codes
    if atoms is None:
        atoms = torch.zeros(int(lib().mxfp8_grouped_atoms_bytes(E, R, C)), dtype=torch.uint8, device=x.device)
    _check("mxfp8_quantize_grouped", lib().mxfp8_quantize_grouped(_p(x), R, C, _p(split_sizes), E, _p(codes),
                                                                   _p(atoms), _stream(stream)))
    return codes, atoms


# ------------------------------------------------------------- grouped expert MLP
def grouped_mlp_workspace_size(E, R, H, F, precision="bf16", training=False) -> int:
    return int(lib().grouped_mlp_workspace_size(E, R, H, F, _PREC[precision], int(bool(training))))


def grouped_mlp_saved_size(E, R, H, F, precision="bf16") -> int:
    return int(lib().grouped_mlp_saved_size(E, R, H, F, _PREC[precision]))


def grouped_mlp_saved_offset(E, R, H, F, precision, part) -> int:
    return int(lib().grouped_mlp_saved_offset(E, R, H, F, _PREC[precision], part))


def grouped_mlp_fwd(xp, split_sizes, w1, w2, probs_perm=None, precision="bf16", xp_scale=None, w1_scale=None,
                    w2_scale=None, yp=None, saved=None, training=False, workspace=None, F=None, out_f32=False,
                    stream=None):
    """fc1 (gate|up) -> ScaledSwiGLU -> fc2 over expert-contiguous rows.

    BF16: w1 [E, H, 2F], w2 [E, F, H] bf16. MXFP8: xp/w1/w2 are E4M3 codes with scales
    (w1 [E, 2F, H], w2 [E, H, F]). Returns (yp, saved); ``saved`` is None unless
    ``training`` (or a saved buffer is passed).
    """
    prec = _PREC[precision]
    R, H = xp.shape
    E = split_sizes.numel()
    if F is None:
        F = w2.shape[1] if prec == BF16 else w2.shape[2]
    dev = xp.device
    if yp is None:
        yp = torch.empty((R, H), dtype=torch.float32 if out_f32 else torch.bfloat16, device=dev)
    if training and saved is None:
        saved = torch.empty(grouped_mlp_saved_size(E, R, H, F, precision), dtype=torch.uint8, device=dev)
    ws_bytes = grouped_mlp_workspace_size(E, R, H, F, precision, saved is not None)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    rc = lib().grouped_mlp_fwd(_p(xp), _p(xp_scale), _p(split_sizes), E, R, H, F, _p(w1), _p(w1_scale), _p(w2),
                               _p(w2_scale), _p(probs_perm), prec | (OUT_F32 if out_f32 else 0), _p(yp), _p(saved),
                               _p(workspace),
                               workspace.numel(), _stream(stream))
    _check("grouped_mlp_fwd", rc)
    return yp, saved


def grouped_mlp_fwd_combine_workspace_size(E, R, H, F, precision="bf16", training=False, T=0) -> int:
    return int(lib().grouped_mlp_fwd_combine_workspace_size(E, R, H, F, _PREC[precision], int(bool(training)), T))


def grouped_mlp_fwd_combine(xp, split_sizes, w1, w2, probs_perm, row_map, T, k, precision="bf16", xp_scale=None,
                            w1_scale=None, w2_scale=None, out=None, saved=None, workspace=None, F=None, stream=None):
    """grouped_mlp_fwd + moe_unpermute with the combine fused into fc2's epilogue: returns
    out [T, H] bf16 (and writes `saved` when given)."""
    prec = _PREC[precision]
    R, H = xp.shape
    E = split_sizes.numel()
    if F is None:
        F = w2.shape[1] if prec == BF16 else w2.shape[2]
    dev = xp.device
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    ws_bytes = grouped_mlp_fwd_combine_workspace_size(E, R, H, F, precision, saved is not None, T)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    rc = lib().grouped_mlp_fwd_combine(_p(xp), _p(xp_scale), _p(split_sizes), E, R, H, F, _p(w1), _p(w1_scale),
                                       _p(w2), _p(w2_scale), _p(probs_perm), prec, _p(row_map), T, k, _p(out),
                                       _p(saved), _p(workspace), workspace.numel(), _stream(stream))
    _check("grouped_mlp_fwd_combine", rc)
    return out


def grouped_mlp_bwd_workspace_size(E, R, H, F, precision="bf16") -> int:
    return int(lib().grouped_mlp_bwd_workspace_size(E, R, H, F, _PREC[precision]))


def grouped_mlp_bwd_workspace_offset(E, R, H, F, precision, part) -> int:
    return int(lib().grouped_mlp_bwd_workspace_offset(E, R, H, F, _PREC[precision], part))


def grouped_mlp_bwd(dy_perm, split_sizes, xp, w1, w2, probs_perm, saved, precision="bf16", dxp=None, dw1=None,
                    dw2=None, dprobs_perm=None, workspace=None, stream=None, operands=None, shape=None):
    """Backward of grouped_mlp_fwd. Returns (dxp, dw1, dw2, dprobs_perm). xp, w1 and w2
    are bf16 on both paths (the MXFP8 path quantises what it needs). MXFP8 only:
    ``operands`` maps names of moe_mxfp8_bwd_operands ("w1_rows", "w1_rows_atoms", ...,
    "dy_rows", "dy_cols", "xp_cols" and their atoms) to tensors already quantised; their
    bf16 sources may then be None, and ``shape`` = (R, H, F) names the sizes."""
    prec = _PREC[precision]
    if shape is not None:
        R, H, F = shape
    else:
        R, H = dy_perm.shape
        F = w2.shape[1]
    E = split_sizes.numel()
    dev = split_sizes.device
    dxp = torch.empty((R, H), dtype=torch.bfloat16, device=dev) if dxp is None else dxp
    dw1 = torch.empty((E, H, 2 * F), dtype=torch.bfloat16, device=dev) if dw1 is None else dw1
    dw2 = torch.empty((E, F, H), dtype=torch.bfloat16, device=dev) if dw2 is None else dw2
    if dprobs_perm is None and probs_perm is not None:
        dprobs_perm = torch.empty(R, dtype=torch.float32, device=dev)
    ws_bytes = grouped_mlp_bwd_workspace_size(E, R, H, F, precision)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if operands:
        if prec != MXFP8:
            raise ValueError("pre-quantised operands are for the MXFP8 backward")
        q = _lib.MxBwdOperands(**{k: (v.data_ptr() if v is not None else None) for k, v in operands.items()})
        rc = lib().grouped_mlp_bwd_mxfp8_operands(ctypes.byref(q), _p(dy_perm), _p(split_sizes), E, R, H, F, _p(xp),
                                                  _p(w1), _p(w2), _p(probs_perm), _p(saved), _p(dxp), _p(dw1),
                                                  _p(dw2), _p(dprobs_perm), _p(workspace), workspace.numel(),
                                                  _stream(stream))
        _check("grouped_mlp_bwd_mxfp8_operands", rc)
    else:
        rc = lib().grouped_mlp_bwd(_p(dy_perm), _p(split_sizes), E, R, H, F, _p(xp), _p(w1), _p(w2),
                                   _p(probs_perm), prec, _p(saved), _p(dxp), _p(dw1), _p(dw2), _p(dprobs_perm),
                                   _p(workspace), workspace.numel(), _stream(stream))
        _check("grouped_mlp_bwd", rc)
    return dxp, dw1, dw2, dprobs_perm


from .layer import HostPipeline, MoEExpertLayer, allreduce_grads, moe_layer_forward  # noqa: E402,F401
