"""Paged block pools on the GPU against the oracle.

A paged cache keeps block records in pages of page_blocks blocks (one
sequence, every KV head) taken from a per-layer pool as sequences grow. Codes,
scales and zero points read back through the page table must equal the
oracle's bit for bit, dequantization too, and decode attention (tensor-core
and CUDA-core kernels, fused decode steps included) must agree with the
oracle within the attention tolerance. A call whose new blocks need more
pages than the pool has free is refused before anything is enqueued;
released sequences return their pages, which later appends reuse.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig
from asymmetric_bit_kv_b200 import kvq as K
from kvq_testutil import Twin, assert_attention_close

pytestmark = pytest.mark.gpu

# (k bits, v bits, group_k, group_v, residual, page_blocks, k_axis, hadamard, sinks)
CASES = [
    (2, 4, 64, 64, 128, 2, 0, 0, 0),    # tensor-core kernel
    (2, 2, 32, 32, 64, 3, 0, 0, 0),     # CUDA-core split kernel
    (2, 2, 64, 128, 128, 1, 1, 1, 4),   # KV1 layout, one block per page
]
IDS = ["tc_k2v4_p2", "split_k2v2_g32_p3", "kv1_p1"]


def _tokens(T, H, dtype, gen):
    k = torch.randn(T, H, 128, generator=gen) * torch.exp(torch.randn(1, H, 128, generator=gen))
    v = torch.randn(T, H, 128, generator=gen)
    return k.to(dtype), v.to(dtype)


def _cfg(case, batch, pool_pages, layers=1):
    kb, vb, G, Gv, R, P, ka, rot, S = case
    return CacheConfig(layers, batch, 8, 2, 128, 4096, G, Gv, R, torch.bfloat16, [kb] * layers, [vb] * layers,
                       sink_tokens=S, k_axis=[ka] * layers, hadamard=rot, page_blocks=P, pool_pages=pool_pages)


def _decode_check(tw, layer, gen, what):
    cfg = tw.cfg
    q = torch.randn(cfg.max_batch, cfg.num_q_heads, 128, generator=gen).to(cfg.kv_dtype)
    out = tw.gpu.decode_attention(layer, q.cuda(), out_dtype=torch.float32, softmax_scale=128 ** -0.5)
    out = out.cpu().numpy()
    for b in range(cfg.max_batch):
        assert_attention_close(out[b], tw.oracle_decode(layer, b, q[b].float().numpy(), 128 ** -0.5), f"{what} seq {b}")


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_paged_codes_dequant_and_decode(case):
    G, R = case[2], case[4]
    cfg = _cfg(case, batch=4, pool_pages=200)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(40 + G)
    plans = [[9 * G + 5, 1, R + 3, 0], [G + 1, 2 * G, 0, 5 * G], [1, 0, 3 * G + 7, G]]
    for step, lens in enumerate(plans):
        k, v = _tokens(sum(lens), 2, cfg.kv_dtype, gen)
        tw.append(0, k, v, lens)
        tw.check_lengths(0, 4)
        _decode_check(tw, 0, gen, f"step {step}")
    for b in range(4):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
    # fused decode steps (one token per sequence), across ring flushes
    for step in range(2 * G + 3):
        k, v = _tokens(4, 2, cfg.kv_dtype, gen)
        q = torch.randn(4, 8, 128, generator=gen).to(cfg.kv_dtype)
        out = tw.gpu.decode_step(0, k.cuda(), v.cuda(), q.cuda(), out_dtype=torch.float32,
                                 softmax_scale=128 ** -0.5)
        for b in range(4):
            tw.ora[(0, b)].append(k[b:b + 1].float().numpy(), v[b:b + 1].float().numpy())
        if step % 37 == 0:
            o = out.cpu().numpy()
            for b in range(4):
                assert_attention_close(o[b], tw.oracle_decode(0, b, q[b].float().numpy(), 128 ** -0.5),
                                       f"decode step {step} seq {b}")
    assert tw.gpu.device_errors() == 0
    for b in range(4):
        tw.check_codes(0, b)


def test_pool_exhaustion_is_refused_and_released_pages_are_reused():
    case = CASES[0]
    G, P = 64, 2
    cfg = _cfg(case, batch=3, pool_pages=6)  # 12 blocks of pool
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(9)
    # sequence 0: 5 blocks (3 pages) + ring; sequence 1: 3 blocks (2 pages)
    lens = [5 * G + 128, 3 * G + 100, 10]
    k, v = _tokens(sum(lens), 2, cfg.kv_dtype, gen)
    tw.append(0, k, v, lens)
    tw.check_lengths(0, 3)
    # sequence 2 asks for 4 blocks = 2 pages with 1 free: refused, nothing changes
    before = [tw.gpu.lengths(0, b) for b in range(3)]
    k2, v2 = _tokens(4 * G + 118, 2, cfg.kv_dtype, gen)
    with pytest.raises(K.KvqError) as ei:
        tw.gpu.append(0, k2.cuda(), v2.cuda(), [0, 0, 4 * G + 118])
    assert ei.value.status == K.KVQ_ERR_CAPACITY
    assert "pages" in str(ei.value)
    assert [tw.gpu.lengths(0, b) for b in range(3)] == before
    _decode_check(tw, 0, gen, "after the refused append")
    # release sequence 0 (3 pages back): the same append now fits
    tw.release_sequence(0)
    assert tw.gpu.lengths(0, 0) == (0, 0)
    tw.append(0, k2, v2, [0, 0, 4 * G + 118])
    tw.check_lengths(0, 3)
    # sequence 0 starts again on the pages left
    k3, v3 = _tokens(G + 130, 2, cfg.kv_dtype, gen)
    tw.append(0, k3, v3, [G + 130, 0, 0])
    tw.check_lengths(0, 3)
    torch.cuda.synchronize()
    for b in range(3):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
    _decode_check(tw, 0, gen, "after reuse")
    assert tw.gpu.device_errors() == 0
