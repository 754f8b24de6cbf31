"""kvq_decode_step: one token appended per sequence and decode attention in
one call, against the oracle and against kvq_append + kvq_decode_attention.

Most steps run fused (the new tokens are written and attended to inside the
decode launch); a step where some sequence's ring is full (a flush) or its
sinks are not complete takes the append-then-decode path. Either way the
cache contents must equal the oracle's bit for bit, the outputs must agree
with the oracle within the attention tolerance, and -- since the fused
kernel reads the same values in the same order -- bit for bit with a second
cache driven by kvq_append + kvq_decode_attention.
"""

import numpy as np
import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KVCache
from kvq_testutil import Twin, assert_attention_close

pytestmark = pytest.mark.gpu

# (k bits, v bits, group_k, group_v, residual, dtype, sinks)
CASES = [
    (2, 4, 64, 64, 128, torch.bfloat16, 0),   # tensor-core kernel: fused steps
    (4, 2, 64, 32, 64, torch.float16, 4),     # fused, sinks filled by the first steps
    (2, 2, 32, 32, 64, torch.bfloat16, 0),    # CUDA-core split kernel: append-then-decode
]


@pytest.mark.parametrize("case", CASES, ids=["tc_k2v4", "tc_k4v2_sinks", "split_k2v2"])
def test_decode_step_matches_oracle_and_two_call_path(case):
    kb, vb, G, Gv, R, dtype, S = case
    H, g = 2, 4
    init = [0, 5, R - 1, R, 3 * G + R - 2]
    B = len(init)
    cfg = CacheConfig(1, B, H * g, H, 128, 4096, G, Gv, R, dtype, [kb], [vb], sink_tokens=S)
    tw = Twin(cfg)
    ref = KVCache(cfg, "cuda")
    gen = torch.Generator().manual_seed(123 + G + S)
    k0 = (torch.randn(sum(init), H, 128, generator=gen) * torch.exp(torch.randn(1, H, 128, generator=gen))).to(dtype)
    v0 = torch.randn(sum(init), H, 128, generator=gen).to(dtype)
    tw.append(0, k0, v0, init)
    ref.append(0, k0.cuda(), v0.cuda(), init)
    scale = 128 ** -0.5
    steps = R + G + 5  # every sequence crosses at least one flush
    for step in range(steps):
        k = torch.randn(B, H, 128, generator=gen).to(dtype)
        v = torch.randn(B, H, 128, generator=gen).to(dtype)
        q = torch.randn(B, H * g, 128, generator=gen).to(dtype)
        out = tw.gpu.decode_step(0, k.cuda(), v.cuda(), q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
        for b in range(B):  # the oracle side of the Twin
            tw.ora[(0, b)].append(k[b:b + 1].float().numpy(), v[b:b + 1].float().numpy())
        ref.append(0, k.cuda(), v.cuda(), [1] * B)
        want = ref.decode_attention(0, q.cuda(), out_dtype=torch.float32, softmax_scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(out, want), f"step {step}: fused and two-call outputs differ"
        if step % 23 == 0 or step == steps - 1:
            o = out.cpu().numpy()
            for b in range(B):
                assert_attention_close(o[b], tw.oracle_decode(0, b, q[b].float().numpy(), scale), f"step {step} seq {b}")
    assert tw.gpu.device_errors() == 0
    tw.check_lengths(0, B)
    for b in range(B):
        tw.check_codes(0, b)
        tw.check_dequant(0, b)
        assert ref.lengths(0, b) == tw.gpu.lengths(0, b)
    ref.close()


def test_decode_step_checks_before_enqueueing():
    cfg = CacheConfig(1, 2, 8, 2, 128, 130, 64, 64, 128, torch.bfloat16, [2], [4])
    c = KVCache(cfg, "cuda")
    k = torch.zeros(2, 2, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16, device="cuda")
    c.append(0, torch.zeros(260, 2, 128, dtype=torch.bfloat16, device="cuda"), torch.zeros(260, 2, 128, dtype=torch.bfloat16, device="cuda"), [130, 130])
    before = [c.lengths(0, b) for b in range(2)]
    with pytest.raises(Exception, match="max_tokens"):
        c.decode_step(0, k, k, q)
    assert [c.lengths(0, b) for b in range(2)] == before  # nothing appended
    c.close()
