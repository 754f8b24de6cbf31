"""The KV1 card's BQ2_0 layout on the GPU against the oracle: keys quantized
per token (grouped like values) and, optionally, the Hadamard rotation of K
and V before quantization ("KV1-1.2B" card, Quantization Format: KV1.cpp
BQ2_0), with and without sinks.

Codes, scales, zero points and dequantized values (in the rotated basis, as
stored) must match the oracle bit for bit -- the rotation is the same fp32
butterfly on both sides; attention within the usual tolerance (max-abs 2e-3,
max-rel 1e-2 against max(|ref|, 0.2)). Layers with one key group per head
vector (group_v = head_dim, group_k >= 64) decode on the tensor-core kernel,
which multiplies the quantized tokens' part of the output by H itself; the
others on the CUDA-core split kernel, whose combine rotates that part back.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig
from kvq_testutil import Twin, assert_attention_close

pytestmark = pytest.mark.gpu

# (k bits, v bits, group_k, group_v, residual, dtype, hadamard, sinks)
CASES = [
    (2, 2, 64, 128, 128, torch.bfloat16, 1, 4),   # KV1-like: 2-bit, one group per head vector, rotation, 4 sinks (TC)
    (2, 4, 32, 64, 64, torch.float16, 0, 0),      # per-token keys, no rotation (split)
    (4, 2, 64, 32, 64, torch.bfloat16, 1, 0),     # rotation, 4 value groups (split)
    (8, 8, 128, 64, 128, torch.bfloat16, 1, 2),   # (split)
    (4, 4, 64, 128, 64, torch.float16, 1, 0),     # rotation, f16 (TC)
    (8, 2, 64, 128, 128, torch.bfloat16, 0, 2),   # per-token keys without rotation, 2 sinks (TC)
    (8, 4, 128, 128, 128, torch.bfloat16, 1, 0),  # two stages of 8-bit 128-token blocks do not fit: split
    (4, 2, 128, 128, 128, torch.float16, 1, 3),   # 128-token blocks (TC)
]
IDS = ["kv1_k2v2_gv128_rot_s4", "k2v4_g32_norot", "k4v2_gv32_rot", "k8v8_g128_rot_s2", "tc_k4v4_rot_f16",
       "tc_k8v2_norot_s2", "k8v4_g128_rot", "tc_k4v2_g128_rot_s3"]


def _cfg(case, batch=4, hq=8, hkv=2, layers=1):
    kb, vb, G, Gv, R, dtype, rot, S = case
    return CacheConfig(layers, batch, hq, hkv, 128, 4096, G, Gv, R, dtype, [kb] * layers, [vb] * layers,
                       sink_tokens=S, k_axis=[1] * layers, hadamard=rot)


def _tokens(T, H, dtype, gen):
    k = torch.randn(T, H, 128, generator=gen) * torch.exp(torch.randn(1, H, 128, generator=gen))
    v = torch.randn(T, H, 128, generator=gen)
    return k.to(dtype), v.to(dtype)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_bq2_codes_and_dequant_bit_exact(case):
    cfg = _cfg(case)
    G, R = cfg.group_k, cfg.residual
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(200 + G)
    plans = [[3 * G + 5, 1, R - 3, 2 * G + 1], [0, 7, 1, 0], [R + 2 * G + 1, G - 1, 1, 3], [2, 0, 0, 1]]
    for step in range(len(plans[0])):
        lens = [p[step] for p in plans]
        k, v = _tokens(sum(lens), cfg.num_kv_heads, cfg.kv_dtype, gen)
        tw.append(0, k, v, lens)
        tw.check_lengths(0, cfg.max_batch)
    torch.cuda.synchronize()
    for b in range(cfg.max_batch):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
    tw.flush_residual(0, cfg.max_batch)
    for b in range(cfg.max_batch):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)


@pytest.mark.parametrize("g", [1, 4, 8])
@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_bq2_decode_matches_oracle(case, g):
    G, R = case[2], case[4]
    hkv = 2
    lens = [0, 3, R // 2, 5 * G + R - 3, 17 * G + 11]
    cfg = _cfg(case, batch=len(lens), hq=hkv * g, hkv=hkv)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(300 + g + G)
    k, v = _tokens(sum(lens), hkv, cfg.kv_dtype, gen)
    tw.append(0, k, v, lens)
    q = torch.randn(cfg.max_batch, cfg.num_q_heads, 128, generator=gen).to(cfg.kv_dtype)
    scale = 128 ** -0.5
    out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    qn = q.float().numpy()
    for b in range(cfg.max_batch):
        assert_attention_close(out[b], tw.oracle_decode(0, b, qn[b], scale), f"seq {b} len {lens[b]}")
    assert np.all(out[0] == 0.0)


def test_bq2_next_to_kivi_layers_and_decode_steps():
    # a rotated cache with group_v 64: layer 0 per-channel keys, layer 1
    # per-token keys, both on the split kernel (append-then-decode steps)
    cfg = CacheConfig(2, 3, 8, 2, 128, 2048, 64, 64, 128, torch.bfloat16, [2, 2], [4, 2], k_axis=[0, 1], hadamard=1)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(7)
    lens = [500, 64, 129]
    scale = 128 ** -0.5
    for layer in (0, 1):
        k, v = _tokens(sum(lens), 2, cfg.kv_dtype, gen)
        tw.append(layer, k, v, lens)
    for step in range(70):
        for layer in (0, 1):
            k, v = _tokens(3, 2, cfg.kv_dtype, gen)
            q = torch.randn(3, 8, 128, generator=gen).to(cfg.kv_dtype)
            out = tw.gpu.decode_step(layer, k.cuda(), v.cuda(), q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
            for b in range(3):
                tw.ora[(layer, b)].append(k[b:b + 1].float().numpy(), v[b:b + 1].float().numpy())
            if step % 23 == 0:
                o = out.cpu().numpy()
                for b in range(3):
                    assert_attention_close(o[b], tw.oracle_decode(layer, b, q[b].float().numpy(), scale),
                                           f"layer {layer} step {step} seq {b}")
    for layer in (0, 1):
        tw.check_lengths(layer, 3)
        for b in range(3):
            tw.check_codes(layer, b)


def test_bq2_whole_vector_layers_take_the_fused_step():
    # the KV1 layout (2-bit per-token keys and values over whole head vectors,
    # rotation, 4 sinks) on the tensor-core kernel: fused decode steps between
    # flushes, append-then-decode steps at them; 8 and 4 query heads per KV head
    for hq in (16, 8):
        cfg = CacheConfig(2, 3, hq, 2, 128, 2048, 64, 128, 128, torch.bfloat16, [2, 2], [2, 4], sink_tokens=4,
                          k_axis=[1, 1], hadamard=1)
        tw = Twin(cfg)
        gen = torch.Generator().manual_seed(17 + hq)
        lens = [300, 2, 191]
        scale = 128 ** -0.5
        for layer in (0, 1):
            k, v = _tokens(sum(lens), 2, cfg.kv_dtype, gen)
            tw.append(layer, k, v, lens)
        for step in range(80):
            for layer in (0, 1):
                k, v = _tokens(3, 2, cfg.kv_dtype, gen)
                q = torch.randn(3, hq, 128, generator=gen).to(cfg.kv_dtype)
                out = tw.gpu.decode_step(layer, k.cuda(), v.cuda(), q.cuda(), out_dtype=torch.float32,
                                         softmax_scale=scale)
                for b in range(3):
                    tw.ora[(layer, b)].append(k[b:b + 1].float().numpy(), v[b:b + 1].float().numpy())
                if step % 13 == 0 or step == 79:
                    o = out.cpu().numpy()
                    for b in range(3):
                        assert_attention_close(o[b], tw.oracle_decode(layer, b, q[b].float().numpy(), scale),
                                               f"hq {hq} layer {layer} step {step} seq {b}")
        assert tw.gpu.device_errors() == 0
        for layer in (0, 1):
            tw.check_lengths(layer, 3)
            for b in range(3):
                tw.check_codes(layer, b)
