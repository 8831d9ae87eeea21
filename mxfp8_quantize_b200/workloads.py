"""Seeded synthetic workloads for the grouped MoE expert MLP.

This module only draws inputs. It holds none of the layer's arithmetic (no
quantisation, no routing bookkeeping, no matmuls), so the CPU oracle and the
CUDA path can both be fed from it without sharing any of the method.

The pages (NVIDIA's BioNeMo / Transformer Engine MoE tutorial, as summarised by
the sitech.ge, andresseo.expert, hyper.ai, ai4snews and ai.kitmori.com pages)
describe Mixtral-8x7B training on genomic sequences but publish no shapes beyond
the model name and no data, so every tensor here is synthetic:

* x, dy      ~ N(0, 1), drawn in fp32 and rounded to bf16 (round-to-nearest-even)
* w_gate_up  [E, 2f, d] and w_down [E, d, f] ~ N(0, sigma): sigma = 1/sqrt(fan_in)
  for the small shapes, 0.02 for the Mixtral-layer shapes; rounded to bf16
* router     logits ~ N(0, 1) [T, E] plus an optional per-expert bias, softmax in
  fp64, top-k (ties -> lower expert index), probabilities renormalised over the
  k picks, stored fp32.  The router itself is upstream of the expert MLP; only
  its outputs (topk_idx, topk_prob) enter the layer.

Draw order from ``numpy.random.default_rng(seed)``: x, w_gate_up, w_down,
logits, bias, dy.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int          # tokens
    d: int          # hidden size
    f: int          # expert ffn size (gate and up are f wide each)
    E: int          # experts
    k: int          # experts per token
    precision: str  # "bf16", "mxfp8" or "fp8" (per-tensor)
    backward: bool  # whether the workload includes the backward pass
    w_std: Optional[float]  # None -> 1/sqrt(fan_in)
    routing: str    # "uniform" | "zipf" | "dirichlet"
    seed: int
    empty_expert: Optional[int] = None  # expert forced to receive no tokens

    @property
    def Tk(self) -> int:
        return self.T * self.k

    def flops_fwd(self) -> float:
        """Algorithmic forward FLOPs: 2*Tk*d*2f (gate_up) + 2*Tk*f*d (down)."""
        return 6.0 * self.Tk * self.d * self.f

    def flops_fwd_bwd(self) -> float:
        """Forward + dgrad + wgrad of both grouped linears: 18*Tk*d*f."""
        return 18.0 * self.Tk * self.d * self.f


CONFIGS = {
    # Tiny forward, BF16 (+ MXFP8 quantisation of x and the weights).
    "tiny_bf16": MoEConfig("tiny_bf16", 256, 256, 512, 4, 2, "bf16", False, None, "uniform", 0),
    # Small forward+backward, MXFP8, Zipf(1.2)-skewed routing, expert 7 empty.
    "small_mxfp8": MoEConfig("small_mxfp8", 4096, 1024, 2048, 8, 2, "mxfp8", True, None, "zipf", 1,
                             empty_expert=7),
    # Mixtral-8x7B layer shape (batch 2 x seq 4096), BF16 forward+backward.
    "mixtral_bf16": MoEConfig("mixtral_bf16", 8192, 4096, 14336, 8, 2, "bf16", True, 0.02, "uniform", 2),
    # Same layer, MXFP8 forward+backward, weights quantised every step.
    "mixtral_mxfp8": MoEConfig("mixtral_mxfp8", 8192, 4096, 14336, 8, 2, "mxfp8", True, 0.02, "uniform", 3),
    # Same layer with per-tensor FP8 operands (one scale per expert operand, current scaling).
    "mixtral_fp8": MoEConfig("mixtral_fp8", 8192, 4096, 14336, 8, 2, "fp8", True, 0.02, "uniform", 3),
    # Long-sequence genomics-style layer: one sequence of 32768 tokens, Dirichlet-skewed routing.
    "longseq_mxfp8": MoEConfig("longseq_mxfp8", 32768, 4096, 14336, 8, 2, "mxfp8", True, 0.02, "dirichlet", 4),
}


def _bf16_from_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _route(logits: np.ndarray, k: int):
    """softmax (fp64) -> top-k (stable: ties go to the lower expert index) -> renormalise."""
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    order = np.argsort(-p, axis=1, kind="stable")[:, :k]
    topk_p = np.take_along_axis(p, order, axis=1)
    topk_p = topk_p / topk_p.sum(axis=1, keepdims=True)
    return order.astype(np.int32), topk_p.astype(np.float32)


def make_routing(cfg: MoEConfig, rng: np.random.Generator):
    logits = rng.standard_normal((cfg.T, cfg.E))  # fp64 draws
    if cfg.routing == "zipf":
        bias = rng.zipf(1.2, cfg.E).astype(np.float64)
        logits = logits + bias[None, :]
    elif cfg.routing == "dirichlet":
        bias = rng.dirichlet([0.5] * cfg.E) * 4.0
        logits = logits + bias[None, :]
    elif cfg.routing != "uniform":
        raise ValueError(cfg.routing)
    if cfg.empty_expert is not None:
        logits[:, cfg.empty_expert] = -np.inf
    return _route(logits, cfg.k)


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> torch.Tensor:
    """N(0, std) drawn in fp32, scaled, rounded to bf16; filled in slabs to bound host memory."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    n = flat.numel()
    slab = 1 << 26
    for s in range(0, n, slab):
        m = min(slab, n - s)
        a = rng.standard_normal(m, dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        flat[s:s + m] = _bf16_from_f32(a)
    return out


def make_inputs(cfg: MoEConfig, with_dy: Optional[bool] = None):
    """All layer inputs on the host, as torch tensors (bf16 / int32 / fp32).

    Returns dict with x [T,d], w_gate_up [E,2f,d], w_down [E,d,f], topk_idx [T,k] int32,
    topk_prob [T,k] fp32 and, for backward workloads, dy [T,d].
    """
    rng = np.random.default_rng(cfg.seed)
    std1 = cfg.w_std if cfg.w_std is not None else 1.0 / np.sqrt(cfg.d)
    std2 = cfg.w_std if cfg.w_std is not None else 1.0 / np.sqrt(cfg.f)
    x = _normal_bf16(rng, (cfg.T, cfg.d), 1.0)
    w1 = _normal_bf16(rng, (cfg.E, 2 * cfg.f, cfg.d), float(std1))
    w2 = _normal_bf16(rng, (cfg.E, cfg.d, cfg.f), float(std2))
    idx, prob = make_routing(cfg, rng)
    out = dict(x=x, w_gate_up=w1, w_down=w2,
               topk_idx=torch.from_numpy(idx), topk_prob=torch.from_numpy(prob))
    if with_dy is None:
        with_dy = cfg.backward
    if with_dy:
        out["dy"] = _normal_bf16(rng, (cfg.T, cfg.d), 1.0)
    return out


def scaled_config(cfg: MoEConfig, **changes) -> MoEConfig:
    return dataclasses.replace(cfg, **changes)


def random_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """Generic seeded bf16 tensor (quantiser tests)."""
    return _normal_bf16(np.random.default_rng(seed), shape, std)


def random_topk(T: int, E: int, k: int, seed: int, skew: str = "uniform"):
    """Generic seeded routing (routing tests): returns (topk_idx int32 [T,k], topk_prob fp32 [T,k])."""
    cfg = MoEConfig("adhoc", T, 0, 0, E, k, "bf16", False, None, skew, seed)
    rng = np.random.default_rng(seed)
    return tuple(torch.from_numpy(a) for a in make_routing(cfg, rng))
