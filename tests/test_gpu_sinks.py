"""Attention sinks on the GPU against the oracle ("KV1-1.2B" card: the first
4 tokens of every sequence keep full-precision K/V).

With sink_tokens = S the first S tokens of each sequence are stored exactly;
quantization, the ring and flushes apply to the tokens after them. Codes,
scales, sink rows, ring rows and dequantized values must match the oracle
bit for bit; attention within the usual tolerance (max-abs 2e-3, max-rel
1e-2 against max(|ref|, 0.2)). Both decode paths are covered: the
tensor-core kernel (group_k >= 64) and the CUDA-core split kernel.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig
from kvq_testutil import Twin, assert_attention_close

pytestmark = pytest.mark.gpu

# (k bits, v bits, group_k, group_v, residual, dtype)
PATHS = [
    (2, 4, 64, 64, 128, torch.bfloat16),   # tensor-core kernel
    (4, 2, 64, 32, 64, torch.float16),     # tensor-core kernel, 4 value groups
    (2, 2, 32, 32, 64, torch.bfloat16),    # CUDA-core split kernel
]


def _cfg(kb, vb, G, Gv, R, dtype, S, batch=4, hq=8, hkv=2):
    return CacheConfig(1, batch, hq, hkv, 128, 4096, G, Gv, R, dtype, [kb], [vb], sink_tokens=S)


def _tokens(T, H, dtype, gen, sink_rows=()):
    k = torch.randn(T, H, 128, generator=gen) * torch.exp(torch.randn(1, H, 128, generator=gen))
    v = torch.randn(T, H, 128, generator=gen)
    for r in sink_rows:  # sink keys far outside the range of the other keys
        k[r] *= 50.0
        v[r] += 3.0
    return k.to(dtype), v.to(dtype)


@pytest.mark.parametrize("S", [4, 8])
@pytest.mark.parametrize("path", PATHS, ids=["tc_k2v4", "tc_k4v2_gv32", "split_k2v2"])
def test_sinks_codes_rows_and_dequant_bit_exact(path, S):
    kb, vb, G, Gv, R, dtype = path
    cfg = _cfg(kb, vb, G, Gv, R, dtype, S)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(70 + S + G)
    # chunks per sequence: some end inside the sinks, some straddle their end,
    # one sequence never gets past them
    plans = [[2, 1, S + 3, R, 2 * G + 5], [S, 0, 1, 3 * G, 1], [1, 1, 1, 0, 0], [0, S + 2 * G + R + 7, 0, 1, 9]]
    for step in range(len(plans[0])):
        lens = [p[step] for p in plans]
        k, v = _tokens(sum(lens), cfg.num_kv_heads, dtype, gen)
        tw.append(0, k, v, lens)
        tw.check_lengths(0, cfg.max_batch)
    torch.cuda.synchronize()
    for b in range(cfg.max_batch):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
    tw.flush_residual(0, cfg.max_batch)
    tw.check_lengths(0, cfg.max_batch)
    for b in range(cfg.max_batch):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)


@pytest.mark.parametrize("g", [1, 4, 8])
@pytest.mark.parametrize("path", PATHS, ids=["tc_k2v4", "tc_k4v2_gv32", "split_k2v2"])
def test_sinks_decode_matches_oracle(path, g):
    kb, vb, G, Gv, R, dtype = path
    S, hkv = 4, 2
    lens = [0, 3, S, S + R // 2, S + 5 * G + R - 3, S + 17 * G + 11]
    cfg = _cfg(kb, vb, G, Gv, R, dtype, S, batch=len(lens), hq=hkv * g, hkv=hkv)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(90 + g + G)
    starts = np.cumsum([0] + lens[:-1])
    sink_rows = [int(s0) + i for s0, n in zip(starts, lens) for i in range(min(S, n))]
    k, v = _tokens(sum(lens), hkv, dtype, gen, sink_rows)
    tw.append(0, k, v, lens)
    q = torch.randn(cfg.max_batch, cfg.num_q_heads, 128, generator=gen).to(dtype)
    scale = 128 ** -0.5
    out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
    torch.cuda.synchronize()
    assert tw.gpu.device_errors() == 0
    out = out.cpu().numpy()
    qn = q.float().numpy()
    for b in range(cfg.max_batch):
        ref = tw.oracle_decode(0, b, qn[b], scale)
        assert_attention_close(out[b], ref, f"seq {b} len {lens[b]}")
    assert np.all(out[0] == 0.0)  # empty sequence


def test_sinks_then_single_token_steps():
    # decode after every one-token append, from an empty cache through the
    # sinks, the ring and several flushes (tensor-core path)
    S, G, R = 4, 64, 128
    cfg = _cfg(2, 4, G, 64, R, torch.bfloat16, S, batch=2, hq=8, hkv=2)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(5)
    scale = 128 ** -0.5
    for step in range(S + R + G + 3):
        k, v = _tokens(2, 2, cfg.kv_dtype, gen, sink_rows=(0, 1) if step < S else ())
        tw.append(0, k, v, [1, 1])
        if step % 17 == 0 or step in (S - 1, S, S + R - 1, S + R, S + R + 1):
            q = torch.randn(2, 8, 128, generator=gen).to(cfg.kv_dtype)
            out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale).cpu().numpy()
            for b in range(2):
                assert_attention_close(out[b], tw.oracle_decode(0, b, q[b].float().numpy(), scale), f"step {step}")
    tw.check_lengths(0, 2)
    for b in range(2):
        tw.check_codes(0, b)
