"""Seeded synthetic inputs for MoE dispatch/combine -- shared by tests, bench
and the oracle checks.

This module holds no part of the method's arithmetic: it draws token rows,
router logits and routing choices (the router is upstream of dispatch), the
stand-in experts' scales and an output gradient, all on the CPU with a seeded
``torch.Generator``.  It imports nothing else from the package, so the oracle
side can use it without touching the CUDA path.

Workload shapes (tokens T, hidden H, experts E, logical ranks R, top_k K,
alignment) follow the model families the AutoEP base PR presets (Mixtral,
Qwen3-MoE, DeepSeek-V3; DeepSpeed AutoEP PR, "Supported presets"), the
count-exchange measurement of the DeepSpeed PR "Derive AutoEP rank splits from
the per-expert count exchange" (Measurements: 256 experts, 1024 tokens per
rank, top_k 8, balanced / skewed token distributions) and the benchmark table
of the DeepSpeed fused-restore folding PR (page_*).  No dataset is used.

Recipe (fixed draw order per config: x, logits, bias, zipf permutation,
scales, grad_out):
  x          ~ N(0, 1) in fp32, rounded to bf16 (RNE by torch).
  logits     ~ N(0, 1) fp32 [T, E]; "mild skew" adds a per-expert bias
               b_e ~ N(0, bias_std); "severe skew" adds beta*log(z_e) with
               z_e proportional to rank_e^-s over a seeded random ranking of
               the experts, beta found by bisection so that the fraction of
               all assignments on the 8 most favoured experts is hot_fraction.
  topk_idx   = the K largest logits per token (stable sort, so a tie goes to
               the lower expert id); softmax and sigmoid are monotone, so
               ranking by logits equals ranking by router scores.
  weights    softmax router: the selected softmax probabilities (fp32, not
               renormalised); sigmoid router: sigma / sum of selected sigma.
  scales     s_e ~ U(0.5, 1.5) fp32 (stand-in expert y = x * s_e).
  grad_out   ~ N(0, 1) fp32 rounded to bf16 (the combine's output gradient).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    T: int
    H: int
    E: int
    R: int
    K: int
    align: int
    seed: int
    router: str = "softmax"          # "softmax" | "sigmoid"
    bias_std: float = 0.0            # mild skew: per-expert logit bias std
    zipf_s: float = 0.0              # severe skew: Zipf exponent (0 = off)
    hot_experts: int = 8
    hot_fraction: float = 0.5
    backward: bool = False           # the config includes the backward pass
    description: str = ""


CONFIGS = {
    "tiny": Config("tiny", T=64, H=128, E=8, R=2, K=2, align=8, seed=1000,
                   description="T=64 H=128 E=8 R=2 top-2 softmax, align 8"),
    "mixtral": Config("mixtral", T=4096, H=4096, E=8, R=1, K=2, align=16, seed=1001,
                      description="Mixtral-shaped: T=4096 H=4096 E=8 R=1 top-2 softmax, align 16"),
    "dsv3": Config("dsv3", T=8192, H=7168, E=256, R=8, K=8, align=128, seed=1002, router="sigmoid",
                   description="DeepSeek-V3-shaped: T=8192 (8x1024) H=7168 E=256 (8x32) top-8 "
                               "sigmoid-normalised, balanced, align 128"),
    "dsv3_skew": Config("dsv3_skew", T=8192, H=7168, E=256, R=8, K=8, align=128, seed=1003,
                        router="sigmoid", zipf_s=1.2,
                        description="DeepSeek-V3-shaped, severe skew: Zipf(1.2) logit bias, "
                                    "~50% of assignments on 8 experts"),
    "qwen3": Config("qwen3", T=16384, H=2048, E=128, R=8, K=8, align=16, seed=1004, bias_std=0.5,
                    backward=True,
                    description="Qwen3-MoE-shaped fwd+bwd: T=16384 H=2048 E=128 (8x16) top-8 "
                                "softmax, mild skew N(0,0.5) bias, align 16"),
    # The benchmark shapes of the DeepSpeed PR "AutoEP: support
    # combine_impl=fused_weighted_sum with AutoEP+AutoTP folding" (Benchmark:
    # hidden 6144; top-4 of 128 and top-8 of 256 experts, the MiniMax-M3 and
    # GLM-5.2 values; 8,192 and 32,768 tokens; random routing with distinct
    # experts per token, FP32 weights).  No expert ranks, no group alignment.
    "page_k4": Config("page_k4", T=8192, H=6144, E=128, R=1, K=4, align=1, seed=1005,
                      router="sigmoid", backward=True,
                      description="fused-restore benchmark shape (MiniMax-M3 values) fwd+bwd: "
                                  "T=8192 H=6144 E=128 top-4 sigmoid-normalised"),
    "page_k8": Config("page_k8", T=8192, H=6144, E=256, R=1, K=8, align=1, seed=1006,
                      router="sigmoid", backward=True,
                      description="fused-restore benchmark shape (GLM-5.2 values) fwd+bwd: "
                                  "T=8192 H=6144 E=256 top-8 sigmoid-normalised"),
    "page_k4_32k": Config("page_k4_32k", T=32768, H=6144, E=128, R=1, K=4, align=1, seed=1007,
                          router="sigmoid", backward=True,
                          description="fused-restore benchmark shape (MiniMax-M3 values) fwd+bwd: "
                                      "T=32768 H=6144 E=128 top-4 sigmoid-normalised"),
    "page_k8_32k": Config("page_k8_32k", T=32768, H=6144, E=256, R=1, K=8, align=1, seed=1008,
                          router="sigmoid", backward=True,
                          description="fused-restore benchmark shape (GLM-5.2 values) fwd+bwd: "
                                      "T=32768 H=6144 E=256 top-8 sigmoid-normalised"),
}


def _topk_from_logits(logits: torch.Tensor, K: int) -> torch.Tensor:
    order = torch.sort(logits, dim=-1, descending=True, stable=True).indices
    return order[:, :K].contiguous()


def _weights(logits: torch.Tensor, idx: torch.Tensor, router: str) -> torch.Tensor:
    if router == "softmax":
        probs = torch.softmax(logits, dim=-1)
        return torch.gather(probs, 1, idx).contiguous()
    if router == "sigmoid":
        sel = torch.gather(torch.sigmoid(logits), 1, idx)
        return (sel / sel.sum(dim=-1, keepdim=True)).contiguous()
    raise ValueError(f"unknown router {router!r}")


def _hot_share(logits: torch.Tensor, K: int, hot: torch.Tensor) -> float:
    idx = _topk_from_logits(logits, K)
    return float(hot[idx].float().mean())


def _zipf_bias(g: torch.Generator, base: torch.Tensor, cfg: Config) -> tuple[torch.Tensor, dict]:
    E = cfg.E
    ranking = torch.randperm(E, generator=g) + 1                 # rank_e in 1..E
    z = ranking.double().pow(-cfg.zipf_s)
    logz = torch.log(z / z.sum()).float()
    hot = ranking <= cfg.hot_experts
    lo, hi = 0.0, 1.0
    while _hot_share(base + hi * logz, cfg.K, hot) < cfg.hot_fraction and hi < 1e3:
        hi *= 2.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if _hot_share(base + mid * logz, cfg.K, hot) < cfg.hot_fraction:
            lo = mid
        else:
            hi = mid
    beta = 0.5 * (lo + hi)
    info = dict(beta=beta, hot_share=_hot_share(base + beta * logz, cfg.K, hot))
    return beta * logz, info


def make_inputs(cfg: Config | str, *, T: int | None = None, H: int | None = None,
                seed: int | None = None, with_grad: bool | None = None) -> dict:
    """Draw one seeded problem.  ``T``/``H``/``seed`` override the config (for
    edge-case tests); returns CPU tensors:

      x [T,H] bf16, topk_idx [T,K] int64, weights [T,K] fp32, scales [E] fp32,
      grad_out [T,H] bf16 (when with_grad, default: cfg.backward), and 'info'.
    """
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    if T is not None or H is not None or seed is not None:
        cfg = dataclasses.replace(cfg, T=cfg.T if T is None else T, H=cfg.H if H is None else H,
                                  seed=cfg.seed if seed is None else seed)
    if with_grad is None:
        with_grad = cfg.backward
    g = torch.Generator().manual_seed(cfg.seed)
    x = torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16)
    logits = torch.randn(cfg.T, cfg.E, generator=g)
    info: dict = {}
    if cfg.bias_std > 0:
        logits = logits + torch.randn(cfg.E, generator=g) * cfg.bias_std
    if cfg.zipf_s > 0:
        bias, zinfo = _zipf_bias(g, logits, cfg)
        logits = logits + bias
        info.update(zinfo)
    scales = (torch.rand(cfg.E, generator=g) + 0.5).float()
    grad_out = torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16) if with_grad else None
    topk_idx = _topk_from_logits(logits, cfg.K).to(torch.int64)
    weights = _weights(logits, topk_idx, cfg.router).float()
    return dict(cfg=cfg, x=x, topk_idx=topk_idx, weights=weights, scales=scales, grad_out=grad_out,
                info=info)


def custom_inputs(T: int, H: int, E: int, K: int, seed: int, *, router: str = "softmax",
                  topk_idx: torch.Tensor | None = None, with_grad: bool = True) -> dict:
    """Same recipe at an arbitrary shape; ``topk_idx`` may be imposed (edge
    cases such as all tokens on one expert, or repeated experts per token)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g)
    scales = (torch.rand(E, generator=g) + 0.5).float()
    grad_out = torch.randn(T, H, generator=g).to(torch.bfloat16) if with_grad else None
    if topk_idx is None:
        topk_idx = _topk_from_logits(logits, K).to(torch.int64)
        weights = _weights(logits, topk_idx, router).float()
    else:
        topk_idx = topk_idx.to(torch.int64).contiguous()
        weights = torch.rand(T, K, generator=g).float()
    return dict(cfg=None, x=x, topk_idx=topk_idx, weights=weights, scales=scales,
                grad_out=grad_out, info={})


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CPU tensor -> uint16 numpy bit patterns (no copy of values)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(
        torch.bfloat16)


def capacity_rows(T: int, K: int, E: int, align: int) -> int:
    """A worst-case row capacity for the expert-grouped buffer: every expert
    may need up to align-1 pad rows on top of the T*K assignment rows."""
    return T * K + E * (align - 1)


__all__ = ["Config", "CONFIGS", "make_inputs", "custom_inputs", "bf16_bits", "bits_to_bf16",
           "capacity_rows"]
