"""Seeded synthetic inputs: weight matrices, activation batches and the layer
shapes of the benchmarked decode linears.

This module holds only random-number recipes and shapes -- none of the
quantization arithmetic -- so that the CUDA path and the CPU oracle can be fed
identical inputs without sharing any method code.

Shapes are those of Llama-3-8B and Llama-3-70B decoder linears ([out, in],
W row-major, y = x W^T); weight statistics follow the pages' examples
(N(0, 0.02^2) fp16 weights in the quantize_per_group example of "LLM 后训练量化
深度实战", section 二) and a heavy-tailed variant (0.02 * Student-t with 3
degrees of freedom, clipped at +-1) for the heavy-tail discussion of
arganzheng.life post-training-quantization-gptq-awq-and-rotation, section 四.1.
"""
from __future__ import annotations

import torch

# Llama-3-8B decoder linears: name -> (out, in)
LLAMA3_8B = {
    "q_proj": (4096, 4096),
    "k_proj": (1024, 4096),
    "v_proj": (1024, 4096),
    "o_proj": (4096, 4096),
    "gate_proj": (14336, 4096),
    "up_proj": (14336, 4096),
    "down_proj": (4096, 14336),
}
LLAMA3_8B_LAYERS = 32

# Llama-3-70B decoder linears: name -> (out, in)
LLAMA3_70B = {
    "q_proj": (8192, 8192),
    "k_proj": (1024, 8192),
    "v_proj": (1024, 8192),
    "o_proj": (8192, 8192),
    "gate_proj": (28672, 8192),
    "up_proj": (28672, 8192),
    "down_proj": (8192, 28672),
}
LLAMA3_70B_LAYERS = 80
LLAMA3_70B_MLP = ("gate_proj", "up_proj", "down_proj")


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_weight(out: int, inn: int, seed: int, std: float = 0.02,
                  device="cpu") -> torch.Tensor:
    """W = (N(0,1) * std).half(), [out, in]."""
    g = _gen(seed, device)
    w = torch.randn(out, inn, generator=g, device=device, dtype=torch.float32)
    return (w * std).to(torch.float16)


def student_t_weight(out: int, inn: int, seed: int, std: float = 0.02, df: int = 3,
                     clip: float = 1.0, device="cpu") -> torch.Tensor:
    """W = clamp(std * t_df, -clip, clip).half() with t_df = z / sqrt(chi2_df / df),
    chi2_df the sum of df squared standard normals."""
    g = _gen(seed, device)
    z = torch.randn(out, inn, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(out, inn, device=device, dtype=torch.float32)
    for _ in range(df):
        u = torch.randn(out, inn, generator=g, device=device, dtype=torch.float32)
        chi2.add_(u * u)
    t = z / torch.sqrt(chi2 / df)
    return torch.clamp(t * std, -clip, clip).to(torch.float16)


def uniform_weight(out: int, inn: int, seed: int, amp: float = 0.05,
                   device="cpu") -> torch.Tensor:
    """W ~ U(-amp, amp) fp16."""
    g = _gen(seed, device)
    w = torch.rand(out, inn, generator=g, device=device, dtype=torch.float32)
    return ((w * 2 - 1) * amp).to(torch.float16)


def activations(B: int, inn: int, seed: int, dtype=torch.bfloat16, n_outliers: int = 0,
                outlier_seed: int | None = None, outlier_scale: float = 20.0,
                device="cpu") -> torch.Tensor:
    """x = N(0,1) [B, in] in ``dtype``; optionally ``n_outliers`` fixed input
    channels (the first of a seeded permutation) scaled by ``outlier_scale``."""
    g = _gen(seed, device)
    x = torch.randn(B, inn, generator=g, device=device, dtype=torch.float32)
    if n_outliers:
        gp = _gen(outlier_seed if outlier_seed is not None else seed + 1, "cpu")
        ch = torch.randperm(inn, generator=gp)[:n_outliers].to(device)
        x[:, ch] *= outlier_scale
    return x.to(dtype)


def outlier_channels(inn: int, n_outliers: int, outlier_seed: int) -> torch.Tensor:
    gp = _gen(outlier_seed, "cpu")
    return torch.randperm(inn, generator=gp)[:n_outliers]


def llama3_8b_layer_seeds(layer: int) -> dict:
    """Distinct seeds for the seven linears of one layer (10..16 for layer 0)."""
    return {name: 10 + 7 * layer + i for i, name in enumerate(LLAMA3_8B)}


def llama3_70b_stack_seed(layer: int, idx: int) -> int:
    """Seed of linear ``idx`` (0..6 in LLAMA3_70B order) of layer ``layer``."""
    return 1000 * layer + idx


# Llama-3-70B KV cache geometry: 8 KV heads of head_dim 128 per layer
# ("LLM 后训练量化深度实战" (ybb.press) section 七, the KV bytes per token).
LLAMA3_70B_KV_HEADS = 8
LLAMA3_70B_HEAD_DIM = 128


def kv_cache(batch: int, heads: int, seq: int, head_dim: int, seed: int, dtype=torch.float16,
             n_sink: int = 4, sink_scale: float = 30.0, device="cpu") -> torch.Tensor:
    """A synthetic K or V cache [batch, heads, seq, head_dim]: N(0, 1) values
    times a per-head magnitude drawn log-uniformly from [0.1, 10], with the
    first ``n_sink`` tokens of every head scaled by ``sink_scale`` (the
    large-magnitude attention-sink tokens of ybb.press section 七)."""
    g = _gen(seed, device)
    x = torch.randn(batch, heads, seq, head_dim, generator=g, device=device, dtype=torch.float32)
    mag = torch.exp(torch.empty(1, heads, 1, 1, device=device).uniform_(-2.3026, 2.3026, generator=g))
    x = x * mag
    if n_sink:
        x[:, :, :n_sink, :] *= sink_scale
    return x.to(dtype)


# FP4 operands drawn directly as bytes, for the W4A4 product: every E2M1
# code equally likely (both signs, -0 included) and scale bytes uniform over
# a range -- E4M3 bytes 0x00..0x7E (zero, subnormal and normal scales up to
# 448) for NVFP4, E8M0 bytes 112..136 (2^-15 .. 2^9) for MXFP4 -- with the
# NVFP4 tensor scales of a weight (max |W| ~ 0.1) and of an activation
# (max |x| ~ 20) matrix.
FP4_BLOCK = {"mxfp4": 32, "nvfp4": 16}
FP4_SCALE_BYTES = {"mxfp4": (112, 136), "nvfp4": (0x00, 0x7E)}
FP4_W_TENSOR_SCALE = 0.1 / 2688.0
FP4_X_TENSOR_SCALE = 20.0 / 2688.0


def fp4_operand(rows: int, inn: int, fmt: str, seed: int):
    """(packed codes uint8 [rows, in/2], scale bytes uint8 [rows, in/block]) on the CPU."""
    g = _gen(seed, "cpu")
    packed = torch.randint(0, 256, (rows, inn // 2), generator=g, dtype=torch.uint8)
    lo, hi = FP4_SCALE_BYTES[fmt]
    scales = torch.randint(lo, hi + 1, (rows, inn // FP4_BLOCK[fmt]), generator=g,
                           dtype=torch.uint8)
    return packed, scales
