"""Seeded synthetic workloads (shapes and value distributions only).

This module draws the inputs -- keys, values and queries -- that both the CUDA
library and the CPU oracle receive. It contains none of the method's
arithmetic: no quantization, packing or attention.

The five workloads mirror the decode-attention configurations studied on the
KIVI README ("Example": Llama-2-7B; GQA update: Llama-3 family) and the
"Quantize What Counts" page (Qwen3-8B, per-layer bit budgets, "more for
keys"): model shapes stand in for those models, whose weights are not used.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    context: list            # cached tokens per sequence before the measured decode
    k_bits: list             # per layer
    v_bits: list
    group_k: int
    group_v: int
    residual: int
    kv_dtype: torch.dtype
    key_dist: str            # "fixed_outliers" | "random_outliers" | "lognormal"
    value_std: float
    seed: int
    num_layers: int = 1
    outlier_channels: tuple = ()
    outlier_scale: float = 1.0
    outliers_per_head: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


def tiny_mha() -> Workload:
    """Tiny KIVI-2bit decode: 1 x 8 heads (MHA) x 128, 1024 tokens, fp16, keys
    with outlier channels 3, 17, 64, 101 scaled by 10; K2 G32, V2 group 32, R32."""
    return Workload("tiny_mha_k2v2_g32_r32_ctx1024", 1, 8, 8, 128, [1024], [2], [2], 32, 32, 32, torch.float16,
                    "fixed_outliers", 1.0, seed=0, outlier_channels=(3, 17, 64, 101), outlier_scale=10.0)


def llama2_7b_mha() -> Workload:
    """Llama-2-7B-shaped layer: 8 x 32 heads (MHA) x 128, context 4096, bf16;
    8 outlier key channels per head x8, values N(0, 0.5); K2 G32, V2 group 32,
    R128; then 256 single-token append + decode steps."""
    return Workload("llama2_7b_mha_k2v2_g32_r128_b8_ctx4096", 8, 32, 32, 128, [4096] * 8, [2], [2], 32, 32, 128,
                    torch.bfloat16, "random_outliers", 0.5, seed=1, outliers_per_head=8, outlier_scale=8.0,
                    extra={"decode_steps": 256})


def llama3_8b_gqa() -> Workload:
    """Llama-3-8B-shaped GQA layer: 32 x (32 q / 8 kv heads) x 128, context 8192,
    bf16; keys N(0,1) times log-normal(0,1) channel magnitudes, values N(0,1);
    K2 G64, V4 group 64, R128."""
    return Workload("llama3_8b_gqa_k2v4_g64_r128_b32_ctx8192", 32, 32, 8, 128, [8192] * 32, [2], [4], 64, 64, 128,
                    torch.bfloat16, "lognormal", 1.0, seed=2)


def kv1_bq2_gqa() -> Workload:
    """The Llama-3-8B-shaped GQA layer with the KV1 card's BQ2_0 cache: keys
    and values 2-bit per token over one whole head vector (group 128), the
    Hadamard rotation, 4 sink tokens; G64 blocks, R128."""
    return Workload("kv1_bq2_gqa_k2v2_tok_gv128_rot_s4_r128_b32_ctx8192", 32, 32, 8, 128, [8192] * 32, [2], [2], 64,
                    128, 128, torch.bfloat16, "lognormal", 1.0, seed=2,
                    extra={"k_axis": [1], "hadamard": 1, "sinks": 4})


def long_context_gqa() -> Workload:
    """Long-context GQA decode: 1 x (32 q / 8 kv) x 128, context 131072, bf16
    distributed as the Llama-2 layer; K2 V2, G128, R128; plus a 4096-token
    prefill chunk appended in one call."""
    return Workload("long_gqa_k2v2_g128_r128_b1_ctx131072", 1, 32, 8, 128, [131072], [2], [2], 128, 128, 128,
                    torch.bfloat16, "random_outliers", 0.5, seed=3, outliers_per_head=8, outlier_scale=8.0,
                    extra={"prefill_chunk": 4096})


def qwen3_8b_layers(seed: int = 4) -> Workload:
    """Qwen3-8B-shaped 36-layer KV path: 64 ragged sequences with context
    uniform in [1024, 32768], (32 q / 8 kv) x 128, bf16; keys N(0,1) times
    log-normal channel magnitudes, values N(0, 0.5); K4 V2 with layers 0-3 at
    K8 V4; G64 for keys and values, R64."""
    g = torch.Generator().manual_seed(seed)
    ctx = torch.randint(1024, 32768 + 1, (64,), generator=g).tolist()
    kb = [8] * 4 + [4] * 32
    vb = [4] * 4 + [2] * 32
    return Workload("qwen3_8b_36L_k4v2_l0to3_k8v4_g64_r64_b64_ragged", 64, 32, 8, 128, ctx, kb, vb, 64, 64, 64,
                    torch.bfloat16, "lognormal", 0.5, seed=seed, num_layers=36)


ALL = {"tiny": tiny_mha, "llama2": llama2_7b_mha, "llama3": llama3_8b_gqa, "long": long_context_gqa,
       "qwen3": qwen3_8b_layers, "kv1": kv1_bq2_gqa}


def key_channel_scale(wl: Workload, layer: int, gen: torch.Generator) -> torch.Tensor:
    """Per-(KV head, channel) multiplier of the keys, float32 [Hkv, D]."""
    H, D = wl.num_kv_heads, wl.head_dim
    s = torch.ones(H, D)
    if wl.key_dist == "fixed_outliers":
        s[:, list(wl.outlier_channels)] = wl.outlier_scale
    elif wl.key_dist == "random_outliers":
        for h in range(H):
            idx = torch.randperm(D, generator=gen)[: wl.outliers_per_head]
            s[h, idx] = wl.outlier_scale
    elif wl.key_dist == "lognormal":
        s = torch.exp(torch.randn(H, D, generator=gen))
    else:
        raise ValueError(wl.key_dist)
    return s


def generate_tokens(wl: Workload, layer: int, lengths, device="cpu", seed_offset: int = 0):
    """Keys and values of `sum(lengths)` tokens, token-major [T, Hkv, D] in the
    workload dtype, drawn in order: channel scales, keys, values. Sequences are
    concatenated in order. Deterministic in (seed, layer, seed_offset, lengths)."""
    T = int(sum(lengths))
    H, D = wl.num_kv_heads, wl.head_dim
    cpu_gen = torch.Generator().manual_seed(wl.seed * 1000003 + layer * 7919 + seed_offset)
    scale = key_channel_scale(wl, layer, cpu_gen)
    if str(device).startswith("cuda"):
        gen = torch.Generator(device=device).manual_seed(wl.seed * 1000003 + layer * 7919 + seed_offset + 1)
    else:
        gen = cpu_gen
    k = torch.randn(T, H, D, generator=gen, device=device)
    k.mul_(scale.to(device))
    v = torch.randn(T, H, D, generator=gen, device=device)
    if wl.value_std != 1.0:
        v.mul_(wl.value_std)
    return k.to(wl.kv_dtype), v.to(wl.kv_dtype)


def generate_queries(wl: Workload, layer: int, batch: int, step: int = 0, device="cpu"):
    """Decode queries [batch, Hq, D] ~ N(0, 1) in the workload dtype."""
    gen = torch.Generator().manual_seed(wl.seed * 1000003 + layer * 7919 + 104729 * (step + 1))
    q = torch.randn(batch, wl.num_q_heads, wl.head_dim, generator=gen)
    return q.to(wl.kv_dtype).to(device)
