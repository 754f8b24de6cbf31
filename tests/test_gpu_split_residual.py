"""Separate residual windows for keys and values ("Quantize What Counts", KV
Cache Quantization: residual_length {"k", "v"}) against the oracle.

Each tensor keeps its own ring and flushes its own oldest G tokens when that
ring is full, so a block record may hold its key part before its value part
(or the reverse). Codes, scales, zero points, both rings and the dequantized
tokens must match the oracle bit for bit; attention within the tolerance.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KVCache, KvqError
from kvq_testutil import Twin, assert_attention_close

pytestmark = pytest.mark.gpu

# (k bits, v bits, G, group_v, R keys, R values, dtype, sinks, key axis, paged)
CASES = [
    (2, 2, 32, 32, 64, 128, torch.bfloat16, 0, 0, 0),
    (2, 4, 64, 64, 128, 64, torch.bfloat16, 0, 0, 0),
    (4, 2, 32, 64, 32, 96, torch.float16, 2, 0, 0),
    (2, 2, 64, 128, 192, 64, torch.bfloat16, 4, 1, 0),
    (4, 4, 32, 32, 96, 32, torch.bfloat16, 0, 0, 2),
]


def _ids(c):
    return f"k{c[0]}v{c[1]}_G{c[2]}_Rk{c[4]}_Rv{c[5]}_S{c[7]}_ax{c[8]}_pg{c[9]}"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_split_windows_codes_rings_dequant_and_decode(case):
    kb, vb, G, Gv, R, RV, dtype, S, ax, pg = case
    H, g, B = 2, 4, 3
    cap = 2048
    cfg = CacheConfig(1, B, H * g, H, 128, cap, G, Gv, R, dtype, [kb], [vb], sink_tokens=S, k_axis=[ax],
                      page_blocks=pg, pool_pages=B * (cap // G // pg + 1) if pg else 0, residual_v=RV)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(R + 3 * RV + G + kb)
    scale = 128 ** -0.5
    plans = [[3 * G + 5, 1, 1, max(R, RV) - 3, 7, 2 * G + 1],
             [0, 7, 0, 1, 0, 0],
             [max(R, RV) + 2 * G + 1, G - 1, 1, 1, 3, 0]]
    for step in range(len(plans[0])):
        lens = [p[step] for p in plans]
        T = sum(lens)
        k = (torch.randn(T, H, 128, generator=gen) * torch.exp(torch.randn(1, H, 128, generator=gen))).to(dtype)
        v = torch.randn(T, H, 128, generator=gen).to(dtype)
        tw.append(0, k, v, lens)
        tw.check_lengths(0, B)
        q = torch.randn(B, H * g, 128, generator=gen).to(dtype)
        out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale).cpu().numpy()
        for b in range(B):
            assert_attention_close(out[b], tw.oracle_decode(0, b, q[b].float().numpy(), scale), f"step {step} seq {b}")
    # the two windows really differ for the long sequences
    assert any(tw.gpu.lengths(0, b)[0] != tw.gpu.value_lengths(0, b)[0] for b in range(B))
    for b in range(B):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
    # decode steps (append + decode: this layer runs on the CUDA-core kernel)
    for step in range(G + 3):
        k = torch.randn(B, H, 128, generator=gen).to(dtype)
        v = torch.randn(B, H, 128, generator=gen).to(dtype)
        q = torch.randn(B, H * g, 128, generator=gen).to(dtype)
        out = tw.gpu.decode_step(0, k.cuda(), v.cuda(), q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
        for b in range(B):
            tw.ora[(0, b)].append(k[b:b + 1].float().numpy(), v[b:b + 1].float().numpy())
        if step % 7 == 0:
            o = out.cpu().numpy()
            for b in range(B):
                assert_attention_close(o[b], tw.oracle_decode(0, b, q[b].float().numpy(), scale), f"dstep {step} seq {b}")
    tw.check_lengths(0, B)
    for b in range(B):
        tw.check_codes(0, b)
    tw.flush_residual(0, B)
    tw.check_lengths(0, B)
    q = torch.randn(B, H * g, 128, generator=gen).to(dtype)
    out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale).cpu().numpy()
    for b in range(B):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
        assert_attention_close(out[b], tw.oracle_decode(0, b, q[b].float().numpy(), scale), f"flushed seq {b}")
    assert tw.gpu.device_errors() == 0


def test_split_windows_multi_query_decode():
    # verify-style decode of 2 query tokens per sequence: both tokens must be
    # in both rings; causal among them
    from oracle import kvq_oracle as O

    dtype, G, R, RV, H, g, B, T = torch.bfloat16, 32, 64, 96, 2, 2, 2, 2
    cfg = CacheConfig(1, B, H * g, H, 128, 1024, G, 32, R, dtype, [2], [4], residual_v=RV)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(77)
    lens = [5 * G + 9, 3 * G + 1]
    k = torch.randn(sum(lens), H, 128, generator=gen).to(dtype)
    v = torch.randn(sum(lens), H, 128, generator=gen).to(dtype)
    tw.append(0, k, v, lens)
    q = torch.randn(B, T, H * g, 128, generator=gen).to(dtype)
    out = tw.gpu.decode_attention_multi(0, q.cuda(), out_dtype=torch.float32, softmax_scale=0.1).cpu().numpy()
    for b in range(B):
        ref = O.decode_attention_multi(tw.ora[(0, b)], q[b].float().numpy(), 0.1)
        assert_attention_close(out[b], ref, f"seq {b}")


def test_split_windows_rejected_with_rotation_and_bad_length():
    base = dict(num_layers=1, max_batch=1, num_q_heads=4, num_kv_heads=2, head_dim=128, max_tokens=512,
                group_k=64, group_v=128, residual=128, kv_dtype=torch.bfloat16, k_bits=[2], v_bits=[2])
    with pytest.raises(KvqError, match="Hadamard"):
        KVCache(CacheConfig(**base, k_axis=[1], hadamard=1, residual_v=64), "cuda")
    with pytest.raises(KvqError, match="residual_v"):
        KVCache(CacheConfig(**base, residual_v=96), "cuda")
