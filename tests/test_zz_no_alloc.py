"""kvq_decode_attention_noalloc through the C ABI.

This entry point is for callers that cannot allocate device memory when they
decode (for example an engine that gives all of its device memory to its own
pool at start-up): its split partials go to a fixed-size array that the library
itself holds on the device. Its output must agree with kvq_decode_attention on
the same cache, within the attention tolerance, on consecutive calls (the array
keeps the previous call's contents): between the two checked calls a call on
another cache, with another layout and values a hundred times larger, fills the
array with very different contents, so a partial left over from an earlier call
would show. A call that needs more scratch than the array holds must be refused
before anything runs.

The file name makes pytest collect it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KVCache
from asymmetric_bit_kv_b200 import kvq as K
from kvq_testutil import assert_attention_close

pytestmark = pytest.mark.gpu


def _call(cache: KVCache, fn: str, q: torch.Tensor, out: torch.Tensor, scale: float) -> int:
    lib = K.load_library()
    return getattr(lib, fn)(cache.handle, 0, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                            K.KVQ_F32, ctypes.c_float(scale), q.shape[0],
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# (k bits, v bits, group_k, group_v, residual, batch, query heads, KV heads, lengths):
# the tensor-core kernel (group_k 64) and the CUDA-core split kernel (group_k 32)
CASES = [
    (2, 4, 64, 64, 128, 4, 32, 8, [3000, 1, 700, 5000]),
    (2, 2, 32, 32, 64, 3, 8, 2, [2100, 64, 900]),
]


def _filled(case, gen, magnitude=1.0):
    kb, vb, G, Gv, R, B, Hq, Hkv, lens = case
    cfg = CacheConfig(1, B, Hq, Hkv, 128, 8192, G, Gv, R, torch.bfloat16, [kb], [vb])
    cache = KVCache(cfg, "cuda")
    k = (torch.randn(sum(lens), Hkv, 128, generator=gen) * torch.exp(torch.randn(1, Hkv, 128, generator=gen)))
    v = torch.randn(sum(lens), Hkv, 128, generator=gen) * magnitude
    cache.append(0, (k * magnitude).to(torch.bfloat16).cuda(), v.to(torch.bfloat16).cuda(), lens)
    return cache


@pytest.mark.parametrize("case", CASES, ids=["tensor_core_G64", "cuda_core_G32"])
def test_noalloc_matches_decode_attention_on_consecutive_calls(case):
    kb, vb, G, Gv, R, B, Hq, Hkv, lens = case
    gen = torch.Generator().manual_seed(11)
    cache = _filled(case, gen)
    other_case = CASES[1] if case is CASES[0] else CASES[0]
    other = _filled(other_case, gen, magnitude=100.0)
    scale = 128 ** -0.5
    for call in range(2):
        q = torch.randn(B, Hq, 128, generator=gen).to(torch.bfloat16).cuda()
        ref = torch.full((B, Hq, 128), float("nan"), device="cuda")
        got = torch.full((B, Hq, 128), float("nan"), device="cuda")
        assert _call(cache, "kvq_decode_attention", q, ref, scale) == K.KVQ_OK
        assert _call(cache, "kvq_decode_attention_noalloc", q, got, scale) == K.KVQ_OK
        torch.cuda.synchronize()
        assert cache.device_errors() == 0
        assert_attention_close(got.cpu().numpy(), ref.cpu().numpy(), f"call {call}")
        if call == 0:  # the second call sees one more token per sequence
            k1 = torch.randn(B, Hkv, 128, generator=gen).to(torch.bfloat16).cuda()
            v1 = torch.randn(B, Hkv, 128, generator=gen).to(torch.bfloat16).cuda()
            cache.append(0, k1, v1, [1] * B)
            # the other cache's decode overwrites the shared array
            Bo, Hqo = other_case[5], other_case[6]
            qo = torch.randn(Bo, Hqo, 128, generator=gen).to(torch.bfloat16).cuda()
            oo = torch.empty(Bo, Hqo, 128, device="cuda")
            assert _call(other, "kvq_decode_attention_noalloc", qo, oo, scale) == K.KVQ_OK
            torch.cuda.synchronize()
            assert float(oo.abs().max()) > 10.0  # values of the other cache are large
    cache.close()
    other.close()


def test_noalloc_rejects_a_call_beyond_the_static_scratch():
    # 512 sequences x 32 query heads with two quantized blocks each need
    # several partial slots per (sequence, head): about 77 MB > 16 MiB
    B, Hq, Hkv, L = 512, 32, 8, 200
    cfg = CacheConfig(1, B, Hq, Hkv, 128, 256, 64, 64, 128, torch.bfloat16, [2], [4])
    cache = KVCache(cfg, "cuda")
    gen = torch.Generator(device="cuda").manual_seed(5)
    k = torch.randn(B * L, Hkv, 128, generator=gen, device="cuda").to(torch.bfloat16)
    cache.append(0, k, k, [L] * B)
    q = torch.randn(B, Hq, 128, generator=gen, device="cuda").to(torch.bfloat16)
    out = torch.zeros(B, Hq, 128, device="cuda")
    st = _call(cache, "kvq_decode_attention_noalloc", q, out, 0.1)
    assert st == K.KVQ_ERR_WORKSPACE
    msg = K.load_library().kvq_last_error().decode()
    assert "static scratch (16777216 bytes)" in msg, msg
    torch.cuda.synchronize()
    assert float(out.abs().max()) == 0.0  # nothing was enqueued
    # a smaller batch of the same cache fits and agrees with the arena path
    ref = torch.empty(8, Hq, 128, device="cuda")
    got = torch.empty(8, Hq, 128, device="cuda")
    assert _call(cache, "kvq_decode_attention", q[:8], ref, 0.1) == K.KVQ_OK
    assert _call(cache, "kvq_decode_attention_noalloc", q[:8], got, 0.1) == K.KVQ_OK
    torch.cuda.synchronize()
    assert_attention_close(got.cpu().numpy(), ref.cpu().numpy(), "batch 8")
    cache.close()
