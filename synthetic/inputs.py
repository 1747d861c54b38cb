"""Workload shapes and seeded input tensors for the MoE FFN layer.

The five named workloads follow the shapes the reference pages discuss:
a tiny fp32 layer, a Mixtral-8x7B-shaped layer (8 experts, top-2; p1
"MoEアーキテクチャの概要" and p3 model table), a DeepSeekMoE-style
fine-grained layer with shared experts and a capacity limit (p5
"細粒度エキスパート分割", "共有エキスパート機構"; p3 "解決策2"), and
DeepSeek-V3-shaped prefill / decode layers (256 experts, 8 per token, one
shared expert; p1 DeepSeek-V3 config dict; p4 "DeepEP の性能" token counts
4096 and 128 with hidden size 7168 and FP8 dispatch).

Distributions: x ~ N(0, 1); router, W1 and W2 weights ~ N(0, 1/fan_in) with
fan_in = d_model for the router and W1 and d_ff for W2; every bias ~ N(0, 0.01)
(variance 0.01, i.e. standard deviation 0.1).  In the FP8 workloads the expert
weights are drawn in fp32 and then encoded offline as e4m3 codes with one
power-of-two fp32 scale per 128x128 block; the encoded weights are the layer's
inputs.  The decode workload adds a per-expert logit bias
b_e = 1.5 * ln(1 / rank_e) over a seeded random ranking of the experts.

Nothing here implements a step of the layer itself.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

DTYPE_F32 = 0   # activations and weights fp32
DTYPE_BF16 = 1  # activations and weights bf16, fp32 accumulation
DTYPE_FP8 = 2   # FP8 e4m3 dispatch and weights with block scales, bf16 combine


@dataclasses.dataclass(frozen=True)
class MoEShape:
    name: str
    T: int
    d_model: int
    n_routed: int
    top_k: int
    d_ff: int
    n_shared: int = 0
    d_ff_shared: int = 0
    capacity_factor: float = 0.0   # 0 means no capacity limit
    alpha: float = 0.01
    dtype: int = DTYPE_BF16
    zipf_logit_bias: bool = False
    # how the per-expert bias is used: 0 = added to the logits (softmax, top-K,
    # gates and P all see it); 1 = selection only (top-K on logits + bias,
    # softmax, gates and P on the unbiased logits)
    bias_mode: int = 0
    selection_bias: bool = False   # draw a N(0, 0.5^2) per-expert bias
    # capacity variants: which slots an expert keeps first (0 = token order,
    # 1 = slot-major: every token's first choice before any second choice),
    # and what a slot dropped by the capacity limit contributes (0 = nothing,
    # 1 = the token's own input times its gate: the token passes through)
    capacity_priority: int = 0
    overflow_mode: int = 0

    def replace(self, **kw) -> "MoEShape":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[int, MoEShape] = {
    1: MoEShape("tiny-fp32 T64 d128 E8 k2 ff256", 64, 128, 8, 2, 256,
                dtype=DTYPE_F32),
    2: MoEShape("mixtral-8x7b-shaped T4096 d4096 E8 k2 ff14336 bf16",
                4096, 4096, 8, 2, 14336, dtype=DTYPE_BF16),
    3: MoEShape("deepseekmoe-style T8192 d2048 E64 k8 ff1408 +2 shared cf1.25 bf16",
                8192, 2048, 64, 8, 1408, n_shared=2, d_ff_shared=1408,
                capacity_factor=1.25, dtype=DTYPE_BF16),
    4: MoEShape("deepseek-v3-prefill T4096 d7168 E256 k8 ff2048 +1 shared fp8",
                4096, 7168, 256, 8, 2048, n_shared=1, d_ff_shared=2048,
                dtype=DTYPE_FP8),
    5: MoEShape("deepseek-v3-decode-skewed T128 d7168 E256 k8 ff2048 +1 shared fp8",
                128, 7168, 256, 8, 2048, n_shared=1, d_ff_shared=2048,
                dtype=DTYPE_FP8, zipf_logit_bias=True),
}

_FP8_BLOCK = 128


def encode_fp8_blocks(w: torch.Tensor):
    """Offline weight encoding: (rows, cols) fp32 -> e4m3 codes (uint8) and
    fp32 scales of shape (rows/128, cols/128).

    Each 128x128 block gets the smallest power of two 2^k with
    amax / 2^k <= 448 (the largest finite e4m3 value); an all-zero block gets
    scale 1.  The codes are torch's round-to-nearest-even e4m3 conversion of
    w / scale, which never exceeds 448 in magnitude by construction.
    """
    rows, cols = w.shape
    assert rows % _FP8_BLOCK == 0 and cols % _FP8_BLOCK == 0
    wb = w.reshape(rows // _FP8_BLOCK, _FP8_BLOCK, cols // _FP8_BLOCK, _FP8_BLOCK)
    amax = wb.abs().amax(dim=(1, 3)).double()
    mant, expo = torch.frexp(amax)            # amax = mant * 2^expo, mant in [0.5, 1)
    k = expo.to(torch.int64) - 9 + (mant > 0.875).to(torch.int64)   # 448 = 0.875 * 2^9
    scale = torch.ldexp(torch.ones_like(amax), k)
    scale = torch.where(amax == 0, torch.ones_like(scale), scale).float()
    q = (wb / scale[:, None, :, None]).to(torch.float8_e4m3fn)
    codes = q.reshape(rows, cols).view(torch.uint8)
    return codes, scale


def _normal(gen, shape, std, device):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=gen)
    return t


def _weights(gen, n_mats, rows, cols, std, dtype, device):
    """Stack of n_mats (rows, cols) matrices, generated one matrix at a time so
    that the fp32 masters of the largest workloads never coexist in memory."""
    if dtype == DTYPE_FP8:
        codes = torch.empty((n_mats, rows, cols), dtype=torch.uint8, device=device)
        scales = torch.empty((n_mats, rows // _FP8_BLOCK, cols // _FP8_BLOCK),
                             dtype=torch.float32, device=device)
        for e in range(n_mats):
            c, s = encode_fp8_blocks(_normal(gen, (rows, cols), std, device))
            codes[e].copy_(c)
            scales[e].copy_(s)
        return codes, scales
    tdt = torch.float32 if dtype == DTYPE_F32 else torch.bfloat16
    out = torch.empty((n_mats, rows, cols), dtype=tdt, device=device)
    for e in range(n_mats):
        out[e].copy_(_normal(gen, (rows, cols), std, device).to(tdt))
    return out, None


def make_inputs(shape: MoEShape, seed: int = 0, device="cpu",
                route_only: bool = False) -> Dict[str, Optional[torch.Tensor]]:
    """All layer inputs for `shape`, drawn from one seeded generator on
    `device`.  The same seed on another device gives other (equally
    distributed) values; callers hand the oracle a host copy of exactly the
    tensors the GPU received.

    route_only=True skips the expert weights (router-only workloads).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    T, d, E, dff = shape.T, shape.d_model, shape.n_routed, shape.d_ff
    act = torch.float32 if shape.dtype == DTYPE_F32 else torch.bfloat16
    out: Dict[str, Optional[torch.Tensor]] = {}
    out["x"] = _normal(gen, (T, d), 1.0, device).to(act)
    out["W_r"] = _normal(gen, (E, d), 1.0 / math.sqrt(d), device)
    out["logit_bias"] = None
    if shape.zipf_logit_bias:
        rank = torch.randperm(E, generator=gen, device=device).to(torch.float64) + 1.0
        out["logit_bias"] = (1.5 * torch.log(1.0 / rank)).float()
    elif shape.selection_bias:
        out["logit_bias"] = _normal(gen, (E,), 0.5, device)
    if route_only:
        return out
    bias_std = 0.1  # N(0, 0.01): variance 0.01
    out["W1"], out["W1_scales"] = _weights(gen, E, dff, d, 1.0 / math.sqrt(d), shape.dtype, device)
    out["b1"] = _normal(gen, (E, dff), bias_std, device)
    out["W2"], out["W2_scales"] = _weights(gen, E, d, dff, 1.0 / math.sqrt(dff), shape.dtype, device)
    out["b2"] = _normal(gen, (E, d), bias_std, device)
    S, dfs = shape.n_shared, shape.d_ff_shared
    if S > 0:
        out["Ws1"], out["Ws1_scales"] = _weights(gen, S, dfs, d, 1.0 / math.sqrt(d), shape.dtype, device)
        out["bs1"] = _normal(gen, (S, dfs), bias_std, device)
        out["Ws2"], out["Ws2_scales"] = _weights(gen, S, d, dfs, 1.0 / math.sqrt(dfs), shape.dtype, device)
        out["bs2"] = _normal(gen, (S, d), bias_std, device)
    else:
        for k in ("Ws1", "Ws1_scales", "bs1", "Ws2", "Ws2_scales", "bs2"):
            out[k] = None
    return out
