"""Seeded synthetic workloads for the NVFP4 MoE expert layer.

Shared by the tests, the bench and the CPU oracle's callers.  This module
draws random numbers and routes tokens; it holds none of the NVFP4 arithmetic
(no quantization, no GEMM, no SwiGLU, no combine).

The pages measure on Qwen3-4B and Qwen3-30B-A3B during GRPO on DAPO math
(www.aib.vote "miniTE report", paragraph 2); neither the checkpoints nor the
dataset are available, so these tensors stand in for them with the models'
shapes only:

  toy          E=4, T=256, top-2 (two distinct experts per token drawn
               uniformly), K=256, N=512; one grouped GEMM
  dense4b      Qwen3-4B MLP as W4A4 linears: T=8192, H=2560, I=9728, E=1, k=1;
               0.1% of the H channels (3 channels) scaled x30 as outliers
  moe30b       Qwen3-30B-A3B expert layer: T=16384, H=2048, I=768, E=128, k=8,
               router logits N(0,1), softmax top-8, renormalised weights
  moe30b_skew  the same layer with T=65536 and a per-expert logit bias
               beta * ln p, p_r ~ r^-1.2 (Zipf s=1.2) over a seeded expert order
  strict       the moe30b layer on 4096 tokens (batch-invariance check)

Activations are BF16 N(0,1), weights BF16 N(0,0.02).  All draws come from a
CPU torch.Generator, so every machine produces the same bytes.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int            # tokens
    H: int            # hidden size (K of gate_up, N of down)
    I: int            # expert intermediate size (gate_up N = 2I, down K = I)
    E: int            # experts
    k: int            # experts per token
    seed: int
    routing: str = "softmax"     # softmax | uniform | identity
    zipf_s: float = 0.0
    zipf_beta: float = 0.0
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0

    @property
    def rows(self) -> int:
        return self.T * self.k


CONFIGS = {
    "toy": LayerConfig("toy", T=256, H=256, I=256, E=4, k=2, seed=1, routing="uniform"),
    "dense4b": LayerConfig("dense4b", T=8192, H=2560, I=9728, E=1, k=1, seed=2,
                           routing="identity", outlier_frac=0.001, outlier_scale=30.0),
    "moe30b": LayerConfig("moe30b", T=16384, H=2048, I=768, E=128, k=8, seed=3),
    "moe30b_skew": LayerConfig("moe30b_skew", T=65536, H=2048, I=768, E=128, k=8, seed=4,
                               zipf_s=1.2, zipf_beta=1.28),
    "strict": LayerConfig("strict", T=4096, H=2048, I=768, E=128, k=8, seed=5),
}


def scaled(cfg: LayerConfig, **kw) -> LayerConfig:
    """A copy of cfg with some fields replaced (small parity cases)."""
    return replace(cfg, **kw)


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1000 + stream)
    return g


def activations(cfg: LayerConfig) -> torch.Tensor:
    """x [T][H] BF16 ~ N(0,1), with outlier channels scaled if configured."""
    x = torch.randn(cfg.T, cfg.H, generator=_gen(cfg.seed, 1), dtype=torch.float32)
    if cfg.outlier_frac > 0:
        n_out = max(1, round(cfg.outlier_frac * cfg.H))
        ch = torch.randperm(cfg.H, generator=_gen(cfg.seed, 2))[:n_out]
        x[:, ch] *= cfg.outlier_scale
    return x.to(torch.bfloat16)


def weights(cfg: LayerConfig, which: str) -> torch.Tensor:
    """gate_up [E][2I][H] or down [E][H][I], BF16 ~ N(0, 0.02).

    gate_up rows 0..I-1 are the gate projection and I..2I-1 the up projection.
    Drawn one expert at a time to bound host memory.
    """
    if which == "gate_up":
        shape, stream = (2 * cfg.I, cfg.H), 10
    elif which == "down":
        shape, stream = (cfg.H, cfg.I), 20
    else:
        raise ValueError(which)
    g = _gen(cfg.seed, stream)
    out = torch.empty((cfg.E,) + shape, dtype=torch.bfloat16)
    for e in range(cfg.E):
        out[e] = (torch.randn(shape, generator=g, dtype=torch.float32) * 0.02).to(torch.bfloat16)
    return out


def routing(cfg: LayerConfig):
    """(topk_idx int32 [T][k], topk_w float32 [T][k]).

    softmax: logits ~ N(0,1) (plus beta * ln p_zipf[perm[e]] when skewed),
    p = softmax(logits) in fp64, the k largest (ties to the lower expert
    index, slots in descending probability), weights renormalised over the k.
    uniform: k distinct experts drawn uniformly, weights 1/k.
    identity: E == k == 1.
    """
    T, E, k = cfg.T, cfg.E, cfg.k
    if cfg.routing == "identity":
        if E != 1 or k != 1:
            raise ValueError("identity routing needs E == k == 1")
        return torch.zeros(T, 1, dtype=torch.int32), torch.ones(T, 1, dtype=torch.float32)
    if cfg.routing == "uniform":
        keys = torch.rand(T, E, generator=_gen(cfg.seed, 3), dtype=torch.float64)
        idx = torch.argsort(keys, dim=1, stable=True)[:, :k]
        return idx.to(torch.int32).contiguous(), torch.full((T, k), 1.0 / k, dtype=torch.float32)
    logits = torch.randn(T, E, generator=_gen(cfg.seed, 3), dtype=torch.float32).to(torch.float64)
    if cfg.zipf_s > 0:
        ranks = torch.arange(1, E + 1, dtype=torch.float64)
        p = ranks.pow(-cfg.zipf_s)
        p = p / p.sum()
        order = torch.randperm(E, generator=_gen(cfg.seed, 4))
        bias = torch.empty(E, dtype=torch.float64)
        bias[order] = cfg.zipf_beta * torch.log(p)
        logits = logits + bias
    prob = torch.softmax(logits, dim=1)
    vals, idx = torch.sort(prob, dim=1, descending=True, stable=True)
    vals, idx = vals[:, :k], idx[:, :k]
    w = vals / vals.sum(dim=1, keepdim=True)
    return idx.to(torch.int32).contiguous(), w.to(torch.float32).contiguous()


def layer_inputs(cfg: LayerConfig, with_weights: bool = True):
    """Everything one layer call needs, on the CPU."""
    out = {"x": activations(cfg)}
    out["topk_idx"], out["topk_w"] = routing(cfg)
    if with_weights:
        out["w_gate_up"] = weights(cfg, "gate_up")
        out["w_down"] = weights(cfg, "down")
    return out


def expert_histogram(topk_idx: torch.Tensor, E: int) -> torch.Tensor:
    return torch.bincount(topk_idx.reshape(-1).to(torch.int64), minlength=E)
