"""Seeded synthetic inputs for the MoE routing path.

This module only draws random numbers and lays them out; it holds none of the
routing arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle
(tests) take their inputs from here, so the two never generate inputs for each
other.

Recipe (one reading for every workload):
  * one ``torch.Generator`` on the CPU, ``manual_seed(seed)``;
  * normal draws are ``randn * std + mean`` in fp32, uniform draws
    ``rand * (hi - lo) + lo`` in fp32, taken in the order the workload lists
    its tensors;
  * bf16 tensors are the RNE cast (``Tensor.to(torch.bfloat16)``) of the fp32
    draw.

The five workloads mirror the problem statements the routing pages describe:
a tiny softmax route, a DeepSeek-V3-style grouped sigmoid route with a
correction bias, a Mixtral-style route + dispatch + combine, a Qwen3-MoE-like
aux-loss batch, and a decode-size fused RMSNorm + router + top-k batch.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

SOFTMAX = 0
SIGMOID = 1
F32 = 0
BF16 = 1

_TORCH_DTYPE = {F32: torch.float32, BF16: torch.bfloat16}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(g: torch.Generator, shape, mean: float, std: float, dtype: int) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32) * std + mean
    return x.to(_TORCH_DTYPE[dtype])


def uniform(g: torch.Generator, shape, lo: float, hi: float, dtype: int) -> torch.Tensor:
    x = torch.rand(shape, generator=g, dtype=torch.float32) * (hi - lo) + lo
    return x.to(_TORCH_DTYPE[dtype])


@dataclass(frozen=True)
class RouteSpec:
    """Parameters of one routing call (score, groups, top-k, weights, tiles)."""
    T: int
    E: int
    k: int
    score_fn: int = SOFTMAX
    softmax_before_topk: int = 1
    n_group: int = 0
    topk_group: int = 0
    group_score_topn: int = 2
    renormalize: int = 1
    scaling_factor: float = 1.0
    tile_tokens_dim: int = 8
    logits_dtype: int = F32
    bias_dtype: int = F32
    weights_dtype: int = F32
    local_expert_offset: int = 0  # expert-parallel shard (local_num_experts 0: all experts local)
    local_num_experts: int = 0
    has_bias: bool = False
    # distributions
    logit_mean: float = 0.0
    logit_std: float = 1.0
    bias_lo: float = -0.1
    bias_hi: float = 0.1
    seed: int = 0

    def with_(self, **kw) -> "RouteSpec":
        return replace(self, **kw)


# Workload 1: tiny softmax route (oracle finishes instantly).
TINY_SOFTMAX = RouteSpec(T=16, E=8, k=2, score_fn=SOFTMAX, softmax_before_topk=1,
                         renormalize=1, scaling_factor=1.0, tile_tokens_dim=4,
                         logits_dtype=F32, weights_dtype=F32, seed=0)

# Workload 2: DeepSeek-V3-style grouped sigmoid route with correction bias.
DSV3_GROUPED_SIGMOID = RouteSpec(T=16384, E=256, k=8, score_fn=SIGMOID, softmax_before_topk=1,
                                 n_group=8, topk_group=4, group_score_topn=2,
                                 renormalize=1, scaling_factor=2.5, tile_tokens_dim=128,
                                 logits_dtype=BF16, bias_dtype=F32, weights_dtype=BF16,
                                 has_bias=True, logit_std=2.0, bias_lo=-0.1, bias_hi=0.1,
                                 seed=1)

# Workload 3: Mixtral-style route (top-k on logits, softmax over the selected 2).
MIXTRAL_ROUTE = RouteSpec(T=65536, E=8, k=2, score_fn=SOFTMAX, softmax_before_topk=0,
                          renormalize=0, scaling_factor=1.0, tile_tokens_dim=128,
                          logits_dtype=BF16, weights_dtype=F32, seed=2)
MIXTRAL_HIDDEN = 4096


@dataclass(frozen=True)
class AuxSpec:
    T: int = 32768
    E: int = 128
    k: int = 8
    score_fn: int = SOFTMAX
    coeff: float = 1e-2
    grad_loss: float = 1.0
    seed: int = 3


QWEN3_AUX = AuxSpec()


@dataclass(frozen=True)
class DecodeSpec:
    T: int = 128
    H: int = 7168
    E: int = 256
    k: int = 8
    eps: float = 1e-6
    act: int = SIGMOID
    has_bias: bool = True
    seed: int = 4

    def with_(self, **kw) -> "DecodeSpec":
        return replace(self, **kw)


DECODE_FUSED = DecodeSpec()


def route_inputs(spec: RouteSpec) -> Dict[str, Optional[torch.Tensor]]:
    """logits [T,E] ~ N(mean, std) in the logits dtype, then bias [E] ~ U(lo, hi)."""
    g = generator(spec.seed)
    logits = normal(g, (spec.T, spec.E), spec.logit_mean, spec.logit_std, spec.logits_dtype)
    bias = uniform(g, (spec.E,), spec.bias_lo, spec.bias_hi, spec.bias_dtype) if spec.has_bias else None
    return {"logits": logits, "bias": bias}


def mixtral_inputs(T: int = MIXTRAL_ROUTE.T, H: int = MIXTRAL_HIDDEN, seed: int = MIXTRAL_ROUTE.seed,
                   E: int = MIXTRAL_ROUTE.E, k: int = MIXTRAL_ROUTE.k) -> Dict[str, torch.Tensor]:
    """logits [T,E] bf16 ~N(0,1); hidden [T,H] bf16 ~N(0,1); expert outputs [T*k,H] bf16 ~N(0,1)."""
    g = generator(seed)
    logits = normal(g, (T, E), 0.0, 1.0, BF16)
    hidden = normal(g, (T, H), 0.0, 1.0, BF16)
    expert_rows = normal(g, (T * k, H), 0.0, 1.0, BF16)
    return {"logits": logits, "hidden": hidden, "expert_rows": expert_rows}


def place_expert_rows(expert_rows: torch.Tensor, permuted_to_token: torch.Tensor,
                      total_padded: int, max_padded: int) -> torch.Tensor:
    """Lay the drawn expert-output rows into the padded permuted buffer.

    The r-th drawn row fills the r-th valid (non-padding) permuted row in
    increasing row order; padding rows and rows past the padded total are NaN so
    that a combine which reads them shows it.  Pure layout: no arithmetic.
    """
    H = expert_rows.shape[1]
    out = torch.full((max_padded, H), float("nan"), dtype=expert_rows.dtype)
    valid = torch.nonzero(permuted_to_token[:total_padded] >= 0).flatten()
    assert valid.numel() == expert_rows.shape[0]
    out[valid] = expert_rows
    return out


def aux_inputs(spec: AuxSpec = QWEN3_AUX) -> Dict[str, torch.Tensor]:
    g = generator(spec.seed)
    return {"logits": normal(g, (spec.T, spec.E), 0.0, 1.0, F32)}


def decode_inputs(spec: DecodeSpec = DECODE_FUSED) -> Dict[str, Optional[torch.Tensor]]:
    """hidden [T,H] ~N(0,1), gamma [H] ~N(1,0.1), W [H,E] ~N(0,0.02), bias [E] ~N(0,0.01); all bf16."""
    g = generator(spec.seed)
    hidden = normal(g, (spec.T, spec.H), 0.0, 1.0, BF16)
    gamma = normal(g, (spec.H,), 1.0, 0.1, BF16)
    W = normal(g, (spec.H, spec.E), 0.0, 0.02, BF16)
    bias = normal(g, (spec.E,), 0.0, 0.01, BF16) if spec.has_bias else None
    return {"hidden": hidden, "gamma": gamma, "W": W, "bias": bias}
