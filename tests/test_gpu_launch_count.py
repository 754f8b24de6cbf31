"""kvq_cache_kernel_launches: the library's own count of the kernels its
calls enqueue on a cache, which the benchmark reports as its launch count.

Each call must add exactly the kernels it enqueues:
* an append adds the ring write, plus the quantize kernel when a ring flushes;
* a decode adds the decode kernel and the log-sum-exp combine;
* a fused decode step adds, besides those two, the flush kernel on a step
  whose rings are full;
* a dequant adds one.
"""

import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KVCache

pytestmark = pytest.mark.gpu


def _tokens(T, H, dtype, gen):
    k = torch.randn(T, H, 128, generator=gen) * torch.exp(torch.randn(1, H, 128, generator=gen))
    v = torch.randn(T, H, 128, generator=gen)
    return k.to(dtype).cuda(), v.to(dtype).cuda()


def test_launch_count_of_appends_decodes_and_steps():
    B, H, g, G, R = 8, 2, 4, 64, 128
    dtype = torch.bfloat16
    c = KVCache(CacheConfig(1, B, H * g, H, 128, 4096, G, G, R, dtype, [2], [4]))
    assert c.decode_kernel(0) == "tensor_core"
    gen = torch.Generator().manual_seed(9)

    def added(fn):
        n0 = c.kernel_launches()
        fn()
        return c.kernel_launches() - n0

    k, v = _tokens(B * 10, H, dtype, gen)
    assert added(lambda: c.append(0, k, v, [10] * B)) == 1  # rings not full: the ring write only
    k, v = _tokens(B * R, H, dtype, gen)
    assert added(lambda: c.append(0, k, v, [R] * B)) == 2  # past R: the quantize kernel and the ring write
    q = torch.randn(B, H * g, 128, generator=gen).to(dtype).cuda()
    assert added(lambda: c.decode_attention(0, q)) == 2
    assert added(lambda: c.dequant(0, 0, 0, 5)) == 1
    flushes = 0
    for step in range(3 * G):
        kn, vn = _tokens(B, H, dtype, gen)
        q = torch.randn(B, H * g, 128, generator=gen).to(dtype).cuda()
        full = c.lengths(0, 0)[1] == R
        flushes += full
        n = added(lambda: c.decode_step(0, kn, vn, q, out_dtype=torch.float32))
        assert n == (3 if full else 2), f"step {step}: {n} kernels"
    torch.cuda.synchronize()
    assert flushes == 3
    assert c.device_errors() == 0
    # 10 + R + 3G = 330 tokens: one block quantized by the append, three by the steps' flushes
    assert c.lengths(0, 0) == (4 * G, 10 + R + 3 * G - 4 * G)
    c.close()


def test_launch_count_of_the_cuda_core_decode():
    # 4-bit keys in 32-token groups run on the CUDA-core split kernel
    B, H, g = 3, 2, 4
    c = KVCache(CacheConfig(1, B, H * g, H, 128, 1024, 32, 32, 64, torch.float16, [4], [2]))
    assert c.decode_kernel(0) == "cuda_core"
    gen = torch.Generator().manual_seed(3)
    k, v = _tokens(3 * 200, H, torch.float16, gen)
    c.append(0, k, v, [200] * B)
    q = torch.randn(B, H * g, 128, generator=gen).to(torch.float16).cuda()
    n0 = c.kernel_launches()
    c.decode_attention(0, q)
    assert c.kernel_launches() - n0 == 2  # the split kernel and the combine
    torch.cuda.synchronize()
    assert c.device_errors() == 0
    c.close()
