"""Parity of the CUDA library with the CPU oracle on small and ragged cases.

Codes, scales, zero points, ring contents and dequantized values must match
bit for bit; attention outputs must be within max-abs 2e-3 and max-rel 1e-2
(relative to max(|ref|, 0.2)) of the fp64 oracle.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KvqError
from kvq_testutil import Twin, assert_attention_close, ulp

pytestmark = pytest.mark.gpu


def _cfg(*, batch=3, hq=4, hkv=2, G=32, Gv=32, R=64, kb=2, vb=2, dtype=torch.bfloat16, max_tokens=2048, layers=1):
    return CacheConfig(layers, batch, hq, hkv, 128, max_tokens, G, Gv, R, dtype, [kb] * layers, [vb] * layers)


def _tie_pattern(bits, n, dtype):
    """n values repeating 0, (2^bits - 1) * 0.75 and every half-step
    (k + 1/2) * 0.75: a group holding whole periods has the scale 0.75
    exactly -- whose reciprocal is not exact in fp32 -- and its codes round
    exact ties half to even; None if the pattern is not exact in dtype."""
    qmax = (1 << bits) - 1
    period = [0.0, qmax * 0.75] + [(k + 0.5) * 0.75 for k in range(qmax)]  # every block holds whole periods
    t = torch.tensor([period[i % len(period)] for i in range(n)], dtype=torch.float64)
    return t if torch.equal(t.to(dtype).double(), t) else None


def _adversarial_tokens(T, H, D, dtype, gen, kb=None, vb=None, gv=None):
    """Random tokens with planted edge cases: constant channels, constant
    value groups, signed zeros, exact half-step ties (with a scale of 1 and
    of 0.75) and large magnitudes."""
    k = torch.randn(T, H, D, generator=gen) * torch.exp(torch.randn(1, H, D, generator=gen))
    v = torch.randn(T, H, D, generator=gen)
    k[:, 0, 5] = 0.75                         # constant key channel
    k[:, 1 % H, 9] = -0.0                     # a channel of negative zeros
    v[:, :, 32:64] = 1.25                     # constant value group
    if T >= 5:
        k[:5, 0, 7] = torch.tensor([0.0, 0.5, 1.5, 2.5, 3.0])       # ties at 2 bits
        v[0, 0, :4] = torch.tensor([0.0, 1.0, 1.5, 3.0])
    k[:, 0, 100] = 6.0e4 * torch.sign(torch.randn(T, generator=gen))  # near the fp16 limit
    k[:, 0, 101] = k[:, 0, 101] * 1e-4        # tiny range -> scale floor
    if kb is not None:  # a key channel on exact ties of a scale whose reciprocal is inexact
        t = _tie_pattern(kb, T, dtype)
        if t is not None:
            k[:, 0, 11] = t.float()
    if vb is not None and gv is not None and T >= 2:  # a value group of two tokens on such ties
        t = _tie_pattern(vb, gv, dtype)
        if t is not None:
            v[1, 0, D - gv:D] = t.float()
            v[0, H - 1, 0:gv] = t.flip(0).float()
    return k.to(dtype), v.to(dtype)


CASES = [
    dict(kb=2, vb=2, G=32, Gv=32, R=64, dtype=torch.bfloat16),
    dict(kb=2, vb=4, G=64, Gv=64, R=128, dtype=torch.bfloat16),
    dict(kb=4, vb=2, G=64, Gv=64, R=64, dtype=torch.float16),
    dict(kb=8, vb=4, G=64, Gv=128, R=128, dtype=torch.bfloat16),
    dict(kb=2, vb=8, G=128, Gv=32, R=128, dtype=torch.float16),
    dict(kb=4, vb=4, G=32, Gv=64, R=96, dtype=torch.bfloat16),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"k{c['kb']}v{c['vb']}_G{c['G']}_Gv{c['Gv']}_R{c['R']}_{str(c['dtype'])[6:]}")
def test_append_codes_ring_and_dequant_bit_exact(case):
    G, R = case["G"], case["R"]
    cfg = _cfg(**case)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(G + R + case["kb"])
    H, D = cfg.num_kv_heads, cfg.head_dim
    # chunks per sequence: a long prefill, single tokens, odd chunks that make
    # blocks straddle the ring and the input
    plans = [[3 * G + 5, 1, 1, R - 3, 7, 2 * G + 1], [0, 7, 0, 1, 0, 0], [R + 2 * G + 1, G - 1, 1, 1, 3, 0]]
    for step in range(len(plans[0])):
        lens = [p[step] for p in plans]
        k, v = _adversarial_tokens(sum(lens), H, D, cfg.kv_dtype, gen, case["kb"], case["vb"], case["Gv"])
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


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("case", CASES[:4], ids=lambda c: f"k{c['kb']}v{c['vb']}_G{c['G']}")
def test_decode_matches_oracle(case, g):
    hkv = 2
    cfg = _cfg(batch=5, hq=hkv * g, hkv=hkv, **case)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(100 + g)
    G, R = case["G"], case["R"]
    # empty, residual only, exactly R, ragged tail, long
    lens = [0, R // 2, R, 5 * G + R - 3, 17 * G + 11]
    k = (torch.randn(sum(lens), hkv, 128, generator=gen) * torch.exp(torch.randn(1, hkv, 128, generator=gen))).to(cfg.kv_dtype)
    v = torch.randn(sum(lens), hkv, 128, generator=gen).to(cfg.kv_dtype)
    tw.append(0, k, v, lens)
    q = torch.randn(cfg.max_batch, cfg.num_q_heads, 128, generator=gen).to(cfg.kv_dtype)
    scale = 128 ** -0.5
    out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    qn = q.float().numpy()
    for b in range(cfg.max_batch):
        ref = tw.oracle_decode(0, b, qn[b], scale)
        assert_attention_close(out[b], ref, f"seq {b} len {lens[b]}")
    assert np.all(out[0] == 0.0)  # empty sequence


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_decode_low_precision_output(out_dtype):
    cfg = _cfg(batch=2, hq=8, hkv=2, kb=2, vb=4, G=64, Gv=64, R=128)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(7)
    lens = [1000, 333]
    k = torch.randn(sum(lens), 2, 128, generator=gen).to(cfg.kv_dtype)
    v = (3 * torch.randn(sum(lens), 2, 128, generator=gen)).to(cfg.kv_dtype)
    tw.append(0, k, v, lens)
    q = torch.randn(2, 8, 128, generator=gen).to(cfg.kv_dtype)
    out = tw.gpu.decode_attention(0, q.cuda(), out_dtype=out_dtype).float().cpu().numpy()
    for b in range(2):
        ref = tw.oracle_decode(0, b, q[b].float().numpy(), 128 ** -0.5)
        # the fp32 result is within ATOL of ref; rounding adds at most half a unit
        err = np.abs(out[b] - ref)
        assert np.all(err <= ulp(ref, out_dtype) / 2 + 2e-3), err.max()


def test_decode_after_flush_residual_and_more_appends():
    cfg = _cfg(batch=2, hq=8, hkv=2, kb=4, vb=2, G=32, Gv=32, R=96)
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(9)
    for lens in ([200, 50], [1, 1], [0, 70]):
        k = torch.randn(sum(lens), 2, 128, generator=gen).to(cfg.kv_dtype)
        v = torch.randn(sum(lens), 2, 128, generator=gen).to(cfg.kv_dtype)
        tw.append(0, k, v, lens)
    tw.flush_residual(0, 2)
    k = torch.randn(5, 2, 128, generator=gen).to(cfg.kv_dtype)
    tw.append(0, k, k, [3, 2])
    tw.check_lengths(0, 2)
    q = torch.randn(2, 8, 128, generator=gen).to(cfg.kv_dtype)
    out = tw.gpu.decode_attention(0, q.cuda()).cpu().numpy()
    for b in range(2):
        tw.check_codes(0, b)
        assert_attention_close(out[b], tw.oracle_decode(0, b, q[b].float().numpy(), 128 ** -0.5))


def test_multi_layer_independent_bits():
    cfg = CacheConfig(3, 2, 8, 2, 128, 1024, 64, 64, 64, torch.bfloat16, [8, 4, 2], [4, 2, 2])
    tw = Twin(cfg)
    gen = torch.Generator().manual_seed(11)
    for layer in range(3):
        lens = [300 + 50 * layer, 129]
        k = torch.randn(sum(lens), 2, 128, generator=gen).to(cfg.kv_dtype)
        v = torch.randn(sum(lens), 2, 128, generator=gen).to(cfg.kv_dtype)
        tw.append(layer, k, v, lens)
    q = torch.randn(2, 8, 128, generator=gen).to(cfg.kv_dtype)
    for layer in range(3):
        out = tw.gpu.decode_attention(layer, q.cuda()).cpu().numpy()
        for b in range(2):
            tw.check_codes(layer, b)
            assert_attention_close(out[b], tw.oracle_decode(layer, b, q[b].float().numpy(), 128 ** -0.5))


def test_capacity_and_argument_errors_enqueue_nothing():
    cfg = _cfg(batch=2, max_tokens=256)
    tw = Twin(cfg)
    k = torch.zeros(300, 2, 128, dtype=cfg.kv_dtype)
    with pytest.raises(KvqError) as e:
        tw.gpu.append(0, k.cuda(), k.cuda(), [257, 0])
    assert e.value.status == -3
    assert tw.gpu.lengths(0, 0) == (0, 0)
    with pytest.raises(KvqError) as e:
        tw.gpu.append(1, k.cuda(), k.cuda(), [1, 0])
    assert e.value.status == -1
    with pytest.raises(KvqError):
        tw.gpu.dequant(0, 0, 0, 1)          # beyond the (empty) sequence
    tw.append(0, k[:256], k[:256], [256, 0])
    tw.check_lengths(0, 2)
