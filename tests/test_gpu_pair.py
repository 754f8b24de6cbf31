"""The tensor-core kernel for 32-token key groups with 2-bit keys (the pair
layout: channels d and d + 64 share a 16-byte key row; "KIVI" README,
Example: group_size 32) against the oracle.

Every (value bits, value groups) instance, one and two query rows per KV
head, both cache dtypes, sinks, paged records, fused decode steps through
flushes and two query tokens per sequence. The cache contents must match
the oracle bit for bit in the pair layout, the outputs within the attention
tolerance, and each case must really run on that kernel.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KVCache
from kvq_testutil import Twin, assert_attention_close

pytestmark = pytest.mark.gpu

# (v bits, group_v, query rows per KV head, dtype, sinks, page blocks)
CASES = [
    (2, 32, 1, torch.bfloat16, 0, 0),
    (2, 32, 2, torch.float16, 0, 0),
    (2, 64, 1, torch.float16, 4, 0),
    (2, 128, 2, torch.bfloat16, 0, 3),
    (4, 32, 1, torch.bfloat16, 0, 0),
    (4, 64, 2, torch.bfloat16, 2, 0),
    (4, 128, 1, torch.float16, 0, 0),
    (8, 32, 2, torch.float16, 0, 0),
    (8, 64, 1, torch.bfloat16, 0, 2),
    (8, 128, 1, torch.bfloat16, 8, 0),
]


def _ids(c):
    return f"v{c[0]}_gv{c[1]}_rows{c[2]}_{str(c[3])[6:]}_S{c[4]}_pg{c[5]}"


def _cfg(vb, gv, rows, dtype, sinks, pg, *, B, H=2, R=128, cap=4096):
    return CacheConfig(1, B, H * rows, H, 128, cap, 32, gv, R, dtype, [2], [vb], sink_tokens=sinks, page_blocks=pg,
                       pool_pages=B * (cap // 32 // pg + 1) if pg else 0)


def _tokens(T, H, dtype, gen, outliers=True):
    k = torch.randn(T, H, 128, generator=gen)
    if outliers:  # a few key channels with large magnitudes, as KIVI's keys have
        k = k * torch.exp(torch.randn(1, H, 128, generator=gen))
    v = torch.randn(T, H, 128, generator=gen) * 0.5
    return k.to(dtype), v.to(dtype)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_pair_decode_matches_oracle(case):
    vb, gv, rows, dtype, S, pg = case
    lens = [0, 3, 64, 5 * 32 + 128 - 3, 40 * 32 + 11, 97 * 32 + 5]
    B, H = len(lens), 2
    cfg = _cfg(*case, B=B, H=H)
    tw = Twin(cfg)
    assert tw.gpu.decode_kernel(0) == "tensor_core_pair"
    gen = torch.Generator().manual_seed(vb * 1000 + gv + rows)
    k, v = _tokens(sum(lens), H, dtype, gen)
    tw.append(0, k, v, lens)
    tw.check_lengths(0, B)
    q = torch.randn(B, H * rows, 128, generator=gen).to(dtype)
    scale = 128 ** -0.5
    out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
    torch.cuda.synchronize()
    assert tw.gpu.device_errors() == 0
    out = out.cpu().numpy()
    for b in range(B):
        tw.check_codes(0, b)
        assert_attention_close(out[b], tw.oracle_decode(0, b, q[b].float().numpy(), scale), f"seq {b} len {lens[b]}")
    assert np.all(out[0] == 0.0)  # empty sequence


@pytest.mark.parametrize("case", [CASES[0], CASES[1], CASES[5]], ids=_ids)
def test_pair_decode_steps_through_flushes(case):
    """Fused decode steps on the pair kernel (the flush kernel writes the pair
    layout), bit for bit with kvq_append + kvq_decode_attention."""
    vb, gv, rows, dtype, S, pg = case
    R = 64
    init = [0, 5, R - 1, R, 3 * 32 + R - 2]
    B, H = len(init), 2
    cfg = _cfg(*case, B=B, H=H, R=R)
    tw = Twin(cfg)
    ref = KVCache(cfg, "cuda")
    gen = torch.Generator().manual_seed(321 + vb + rows)
    k0, v0 = _tokens(sum(init), H, dtype, gen)
    tw.append(0, k0, v0, init)
    ref.append(0, k0.cuda(), v0.cuda(), init)
    scale = 128 ** -0.5
    steps = R + 32 + 5
    for step in range(steps):
        k, v = _tokens(B, H, dtype, gen, outliers=False)
        q = torch.randn(B, H * rows, 128, generator=gen).to(dtype)
        out = tw.gpu.decode_step(0, k.cuda(), v.cuda(), q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
        for b in range(B):
            tw.ora[(0, b)].append(k[b:b + 1].float().numpy(), v[b:b + 1].float().numpy())
        ref.append(0, k.cuda(), v.cuda(), [1] * B)
        want = ref.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(out, want), f"step {step}: fused and two-call outputs differ"
        if step % 19 == 0 or step == steps - 1:
            o = out.cpu().numpy()
            for b in range(B):
                assert_attention_close(o[b], tw.oracle_decode(0, b, q[b].float().numpy(), scale), f"step {step} seq {b}")
    assert tw.gpu.device_errors() == 0
    tw.check_lengths(0, B)
    for b in range(B):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
    ref.close()


@pytest.mark.parametrize("T", [2, 3])
def test_pair_multi_query(T):
    """T query tokens per sequence on a multi-head layer: launches of two
    query rows per KV head (the last one of one row for odd T)."""
    from oracle import kvq_oracle as O

    dtype, H, B = torch.bfloat16, 4, 3
    cfg = CacheConfig(1, B, H, H, 128, 2048, 32, 32, 128, dtype, [2], [2])
    tw = Twin(cfg)
    assert tw.gpu.decode_kernel(0, rows_per_kv_head=2) == "tensor_core_pair"
    gen = torch.Generator().manual_seed(40 + T)
    lens = [9 * 32 + 7, 128 + 3, 30 * 32]
    k, v = _tokens(sum(lens), H, dtype, gen)
    tw.append(0, k, v, lens)
    q = torch.randn(B, T, H, 128, generator=gen).to(dtype)
    out = tw.gpu.decode_attention_multi(0, q.cuda(), out_dtype=torch.float32, softmax_scale=0.1).cpu().numpy()
    for b in range(B):
        ref = O.decode_attention_multi(tw.ora[(0, b)], q[b].float().numpy(), 0.1)
        assert_attention_close(out[b], ref, f"seq {b}")


def test_pair_not_taken_beyond_two_rows_or_with_per_token_keys():
    base = dict(num_layers=1, max_batch=1, num_kv_heads=2, head_dim=128, max_tokens=512, group_k=32, group_v=32,
                residual=64, kv_dtype=torch.bfloat16, v_bits=[2])
    c = KVCache(CacheConfig(num_q_heads=8, k_bits=[2], **base), "cuda")
    assert c.decode_kernel(0) == "cuda_core"  # four query rows per KV head
    c.close()
    c = KVCache(CacheConfig(num_q_heads=2, k_bits=[4], **base), "cuda")
    assert c.decode_kernel(0) == "cuda_core"  # 4-bit keys in 32-token groups
    c.close()
    c = KVCache(CacheConfig(num_q_heads=2, k_bits=[2], k_axis=[1], **base), "cuda")
    assert c.decode_kernel(0) == "cuda_core"  # per-token keys
    c.close()
