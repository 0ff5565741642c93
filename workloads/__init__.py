"""Seeded synthetic MoE-layer workloads shared by the tests, the bench and the oracle.

This module only draws random numbers and defines shapes. It contains none of the
layer's arithmetic (no routing, no permutation, no GEMM, no quantisation), so the
CUDA path and the CPU oracle can both take their inputs from here without sharing
any computation.

Recipe (all configurations):
  * generator: numpy ``default_rng(seed)`` (PCG64), ``standard_normal(dtype=float32)``;
  * draw order: x, router logits, w1, w2, grad_out — each drawn in row-major order in
    chunks of ``_CHUNK`` elements (one continuous stream);
  * x ~ N(0,1); logits ~ N(0,1) (+ a per-expert bias where the workload is skewed);
    w1, w2 ~ N(0, 0.02); grad_out ~ N(0,1);
  * bf16 tensors are the fp32 draws rounded to nearest-even by torch's CPU cast.

The layer shapes follow the pages' workloads (Mixtral-8x7B and Qwen3-30B-A3B expert
MLPs; the genomic long-sequence Mixtral case). No model weights or datasets are used.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

_CHUNK = 1 << 24


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int          # tokens
    H: int          # hidden size (fc1 K, fc2 N)
    F: int          # expert FFN size (fc1 N = 2F for gate|up, fc2 K)
    E: int          # experts
    k: int          # top-k
    precision: str  # "bf16" or "mxfp8"
    passes: str     # "fwd" or "fwd+bwd"
    skew: str = "none"  # "none", "zipf_log_rank", "expert0_plus2"
    seed: int = 0

    @property
    def R(self) -> int:
        return self.T * self.k

    def gemm_flops(self, backward: bool | None = None) -> float:
        """Algorithmic GEMM flops of the layer: fc1 (2F wide) + fc2, times 3 with backward."""
        bwd = (self.passes == "fwd+bwd") if backward is None else backward
        fwd = 6.0 * self.H * self.F * self.R
        return 3.0 * fwd if bwd else fwd


CONFIGS = {
    "tiny_bf16_fwd": LayerConfig("tiny_bf16_fwd", 256, 128, 256, 4, 2, "bf16", "fwd"),
    "mixtral_bf16_fwd": LayerConfig("mixtral_bf16_fwd", 8192, 4096, 14336, 8, 2, "bf16", "fwd"),
    "mixtral_mxfp8_fwd": LayerConfig("mixtral_mxfp8_fwd", 8192, 4096, 14336, 8, 2, "mxfp8", "fwd"),
    "qwen3_30b_a3b_bf16_fwdbwd": LayerConfig(
        "qwen3_30b_a3b_bf16_fwdbwd", 16384, 2048, 768, 128, 8, "bf16", "fwd+bwd", "zipf_log_rank"),
    "genomic_mixtral_mxfp8_fwdbwd": LayerConfig(
        "genomic_mixtral_mxfp8_fwdbwd", 32768, 4096, 14336, 8, 2, "mxfp8", "fwd+bwd", "expert0_plus2"),
}


def expert_bias(E: int, skew: str) -> np.ndarray:
    """Per-expert additive logit bias that shapes the routing load.

    * ``zipf_log_rank``: bias_e = 0.5 * ln(rank_e ** -1.1) with rank_e = e + 1, and the
      last four experts pushed to -1e4 so that some experts receive no tokens.
    * ``expert0_plus2``: expert 0 gets +2.0.
    """
    b = np.zeros(E, dtype=np.float32)
    if skew == "zipf_log_rank":
        r = np.arange(1, E + 1, dtype=np.float64)
        b = (0.5 * np.log(r ** -1.1)).astype(np.float32)
        if E > 4:
            b[-4:] = np.float32(-1.0e4)
    elif skew == "expert0_plus2":
        b[0] = np.float32(2.0)
    elif skew != "none":
        raise ValueError(f"unknown skew {skew!r}")
    return b


class _Stream:
    """One continuous float32 N(0,1) stream drawn in fixed-size chunks."""

    def __init__(self, seed: int):
        self.rng = np.random.default_rng(seed)

    def normal(self, shape, scale: float = 1.0) -> np.ndarray:
        n = int(np.prod(shape))
        out = np.empty(n, dtype=np.float32)
        for s in range(0, n, _CHUNK):
            m = min(_CHUNK, n - s)
            out[s:s + m] = self.rng.standard_normal(m, dtype=np.float32)
        if scale != 1.0:
            out *= np.float32(scale)
        return out.reshape(shape)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a).to(torch.bfloat16)


def make_layer_inputs(cfg: LayerConfig, *, with_grad: bool | None = None, T: int | None = None,
                      seed: int | None = None) -> dict:
    """Draw the CPU inputs of one MoE expert-MLP layer.

    Returns a dict of CPU tensors: x [T,H] bf16, logits [T,E] fp32, w1 [E,H,2F] bf16
    (gate columns [0,F), up columns [F,2F)), w2 [E,F,H] bf16 and, with ``with_grad``,
    grad_out [T,H] bf16. ``T`` overrides the token count (the draw order is unchanged).
    """
    T = cfg.T if T is None else T
    seed = cfg.seed if seed is None else seed
    with_grad = (cfg.passes == "fwd+bwd") if with_grad is None else with_grad
    st = _Stream(seed)
    x = _bf16(st.normal((T, cfg.H)))
    logits = st.normal((T, cfg.E)) + expert_bias(cfg.E, cfg.skew)[None, :]
    w1 = _bf16(st.normal((cfg.E, cfg.H, 2 * cfg.F), 0.02))
    w2 = _bf16(st.normal((cfg.E, cfg.F, cfg.H), 0.02))
    out = {"x": x, "logits": torch.from_numpy(np.ascontiguousarray(logits, dtype=np.float32)),
           "w1": w1, "w2": w2}
    if with_grad:
        out["grad_out"] = _bf16(st.normal((T, cfg.H)))
    return out


def small_layer(T: int, H: int, F: int, E: int, k: int, *, seed: int = 0, skew: str = "none",
                with_grad: bool = True, logits_bias: np.ndarray | None = None) -> dict:
    """Inputs of an arbitrary small layer with the same distributions (parity cases)."""
    cfg = LayerConfig("custom", T, H, F, E, k, "bf16", "fwd+bwd" if with_grad else "fwd", skew, seed)
    d = make_layer_inputs(cfg, with_grad=with_grad)
    if logits_bias is not None:
        d["logits"] = d["logits"] + torch.from_numpy(np.asarray(logits_bias, dtype=np.float32))[None, :]
    return d


def sample_tokens(T: int, n: int, seed: int = 1) -> np.ndarray:
    """Sorted, distinct, seeded token indices used for sampled checks at large sizes."""
    rng = np.random.default_rng(seed)
    n = min(n, T)
    return np.sort(rng.choice(T, size=n, replace=False)).astype(np.int64)


def bytes_of(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


__all__ = ["LayerConfig", "CONFIGS", "expert_bias", "make_layer_inputs", "small_layer",
           "sample_tokens", "bytes_of"]
