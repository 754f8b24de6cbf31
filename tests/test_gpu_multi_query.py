"""Several query tokens per sequence (kvq_decode_attention_multi) against the
oracle's causal decode.

The T query tokens' keys and values are appended first; query t attends to
the sequence's tokens up to its own position (oracle reading 8). Covered:
the tensor-core kernel with 4 and 1 query heads per KV head (query rows of
one launch up to 8: T = 2 per launch, or 8), groups split over several
launches (T = 3, 5), the CUDA-core split kernel, the KV1 layout (per-token
keys, rotation, sinks) and a paged cache; a sequence whose ring holds fewer
than T tokens is refused before anything runs.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig
from asymmetric_bit_kv_b200 import kvq as K
from kvq_testutil import Twin, assert_attention_close
from oracle import kvq_oracle as O

pytestmark = pytest.mark.gpu

# (k bits, v bits, G, group_v, R, Hq, Hkv, k_axis, hadamard, sinks, page_blocks, T values)
CASES = [
    (2, 4, 64, 64, 128, 8, 2, 0, 0, 0, 0, [1, 2, 3, 5]),     # tensor cores, 4 heads per KV head
    (2, 4, 64, 64, 128, 2, 2, 0, 0, 0, 0, [8, 6]),           # tensor cores, 8 query rows per KV head
    (2, 2, 32, 32, 64, 8, 2, 0, 0, 0, 0, [2, 3]),            # CUDA-core split kernel
    (2, 2, 64, 128, 128, 8, 2, 1, 1, 4, 0, [4]),             # KV1 layout
    (4, 2, 64, 64, 128, 8, 2, 0, 0, 0, 2, [3]),              # paged
]
IDS = ["tc_g4", "tc_g1_t8", "split_g32", "kv1", "paged"]


def _tokens(T, H, dtype, gen):
    k = torch.randn(T, H, 128, generator=gen) * torch.exp(torch.randn(1, H, 128, generator=gen))
    v = torch.randn(T, H, 128, generator=gen)
    return k.to(dtype), v.to(dtype)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_multi_query_matches_causal_oracle(case):
    kb, vb, G, Gv, R, Hq, Hkv, ka, rot, S, P, Ts = case
    cfg = CacheConfig(1, 4, Hq, Hkv, 128, 4096, G, Gv, R, torch.bfloat16, [kb], [vb], sink_tokens=S, k_axis=[ka],
                      hadamard=rot, page_blocks=P, pool_pages=64 if P else 0)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(70 + G + Hq)
    lens = [9 * G + 3, 12, R // 2 + 1, 3 * G + R - 9]
    k, v = _tokens(sum(lens), Hkv, cfg.kv_dtype, gen)
    tw.append(0, k, v, lens)
    scale = 128 ** -0.5
    for T in Ts:
        # each sequence's T query tokens enter the cache first (the ring must keep them)
        k, v = _tokens(4 * T, Hkv, cfg.kv_dtype, gen)
        tw.append(0, k, v, [T] * 4)
        q = torch.randn(4, T, Hq, 128, generator=gen).to(cfg.kv_dtype)
        out = tw.gpu.decode_attention_multi(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
        torch.cuda.synchronize()
        out = out.cpu().numpy()
        for b in range(4):
            assert tw.gpu.lengths(0, b)[1] >= T
            ref = O.decode_attention_multi(tw.ora[(0, b)], q[b].float().numpy(), scale)
            assert_attention_close(out[b], ref, f"T {T} seq {b}")
        if T == 1:
            one = tw.gpu.decode_attention(0, q[:, 0].cuda(), out_dtype=torch.float32, softmax_scale=scale)
            assert_attention_close(out[:, 0], one.cpu().numpy(), "T 1 against the single-token decode")
    assert tw.gpu.device_errors() == 0


def test_multi_query_needs_its_tokens_in_the_ring():
    cfg = CacheConfig(1, 2, 8, 2, 128, 1024, 64, 64, 64, torch.bfloat16, [2], [4])
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(3)
    lens = [64 + 3, 100]       # R = G = 64: sequence 0 keeps 3 ring tokens
    k, v = _tokens(sum(lens), 2, cfg.kv_dtype, gen)
    tw.append(0, k, v, lens)
    assert tw.gpu.lengths(0, 0)[1] == 3
    q = torch.randn(2, 4, 8, 128, generator=gen).to(cfg.kv_dtype).cuda()
    with pytest.raises(K.KvqError) as ei:
        tw.gpu.decode_attention_multi(0, q)
    assert ei.value.status == K.KVQ_ERR_UNSUPPORTED and "ring" in str(ei.value)
    out = tw.gpu.decode_attention_multi(0, q[:, :3].contiguous(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    for b in range(2):
        ref = O.decode_attention_multi(tw.ora[(0, b)], q[b, :3].float().cpu().numpy(), 128 ** -0.5)
        assert_attention_close(out[b].cpu().numpy(), ref, f"seq {b}")
