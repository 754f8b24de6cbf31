"""Pins for the CPU oracle: hand-worked cases, closed forms, invariants and an
independent attention routine. None of these call the CUDA library."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import kvq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits(h):
    return int(np.asarray(h, dtype=np.float16).view(np.uint16))


# --------------------------------------------------------------------------
# fp16 rounding and the quantizer (KV1-1.2B card, BQ2_0)
# --------------------------------------------------------------------------


def test_fp16_rne_golden():
    for c in _load("fp16_rne.json")["cases"]:
        got = _bits(O.fp16_rn(np.float32(c["x"])))
        assert got == int(c["bits"], 16), (c, hex(got))


def test_quantizer_golden():
    for c in _load("quantizer_cases.json")["cases"]:
        x = np.array(c["x"], dtype=np.float32)
        q, d16, m16 = O.quantize_groups(x, c["bits"])
        assert q.tolist() == c["codes"], c["name"]
        assert _bits(d16) == int(c["d16"], 16), (c["name"], hex(_bits(d16)))
        assert _bits(m16) == int(c["m16"], 16), (c["name"], hex(_bits(m16)))
        if "xhat" in c:
            xh = O.dequantize(q, d16, m16)
            assert xh.tolist() == c["xhat"], c["name"]


def test_dequant_golden():
    for c in _load("quantizer_cases.json")["dequant"]["cases"]:
        d16 = np.array([int(c["d16"], 16)], np.uint16).view(np.float16)
        m16 = np.array([int(c["m16"], 16)], np.uint16).view(np.float16)
        xh = O.dequantize(np.array([c["q"]], np.uint8), d16, m16)
        assert float(xh[0]) == c["xhat"], c


def test_negative_zero_min_bits():
    # A group whose minimum is -0.0 must store +0.0 whatever the scan order.
    for x in ([-0.0, 0.0, 3.0], [0.0, -0.0, 3.0], [3.0, -0.0, -0.0]):
        _, _, m16 = O.quantize_groups(np.array(x, np.float32), 2)
        assert _bits(m16) == 0x0000


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_error_bound_exact_grid(bits):
    # min = 0 and max = (2^b-1) * 2^e make m and d exact in fp16: error <= d/2.
    rng = np.random.default_rng(bits)
    qmax = (1 << bits) - 1
    for e in range(-6, 5):
        d = 2.0 ** e
        x = rng.uniform(0, qmax * d, size=(64, 32)).astype(np.float32)
        x[:, 0] = 0.0
        x[:, 1] = qmax * d
        q, d16, m16 = O.quantize_groups(x, bits)
        assert np.all(d16.astype(np.float64) == d) and np.all(m16 == 0)
        err = np.abs(O.dequantize(q, d16[:, None], m16[:, None]).astype(np.float64) - x)
        assert err.max() <= d / 2 * (1 + 2 ** -20)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_error_bound_general(bits):
    rng = np.random.default_rng(10 + bits)
    qmax = (1 << bits) - 1
    x = (rng.standard_normal((512, 64)) * np.exp(rng.standard_normal((512, 1)))).astype(np.float32)
    q, d16, m16 = O.quantize_groups(x, bits)
    mn = x.min(axis=1).astype(np.float64)
    d = (x.max(axis=1).astype(np.float64) - mn) / qmax
    d16f, m16f = d16.astype(np.float64), m16.astype(np.float64)
    bound = d16f / 2 + np.abs(mn - m16f) + qmax * np.abs(d - d16f) + 4 * np.abs(x).max(axis=1) * 2.0 ** -23
    xh = O.dequantize(q, d16[:, None], m16[:, None]).astype(np.float64)
    assert np.all(np.abs(xh - x).max(axis=1) <= bound)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_code_is_nearest_level(bits):
    # Brute force: the code is the nearest of the 2^b levels m + k d (exact
    # arithmetic), except within a hair of a midpoint where fp32 rounding of
    # t may legitimately go either way.
    rng = np.random.default_rng(20 + bits)
    qmax = (1 << bits) - 1
    x = rng.standard_normal((256, 32)).astype(np.float32) * 3
    q, d16, m16 = O.quantize_groups(x, bits)
    levels = m16.astype(np.float64)[:, None, None] + d16.astype(np.float64)[:, None, None] * np.arange(qmax + 1)[None, None, :]
    dist = np.abs(x.astype(np.float64)[:, :, None] - levels)
    best = dist.argmin(axis=2)
    t = (x.astype(np.float64) - m16.astype(np.float64)[:, None]) / d16.astype(np.float64)[:, None]
    near_tie = np.abs(t - np.floor(t) - 0.5) < 1e-4
    ok = (best == q) | near_tie
    assert ok.all()
    assert (np.abs(best.astype(int) - q.astype(int)) <= 1).all()


# --------------------------------------------------------------------------
# Packing (BQ2_0 bit order)
# --------------------------------------------------------------------------


def test_pack_golden():
    for c in _load("pack_cases.json")["cases"]:
        w = O.pack_codes(np.array(c["codes"], np.uint8), c["bits"])
        assert w.tolist() == [int(c["word"], 16)], c


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_pack_roundtrip_and_positions(bits):
    rng = np.random.default_rng(bits)
    per = 32 // bits
    codes = rng.integers(0, 1 << bits, size=(7, 5, per * 3)).astype(np.uint8)
    words = O.pack_codes(codes, bits)
    assert words.shape == (7, 5, 3)
    assert np.array_equal(O.unpack_codes(words, bits), codes)
    # each code read back with an explicit shift and mask
    for i in range(per * 3):
        w = words[..., i // per].astype(np.uint64)
        assert np.array_equal((w >> np.uint64((i % per) * bits)) & np.uint64((1 << bits) - 1), codes[..., i])


def test_block_word_arrangement():
    # Key words run along tokens for a fixed channel; value words along channels
    # for a fixed token.
    G, H, D, b = 32, 2, 32, 2
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 4, size=(G, H, D)).astype(np.uint8)
    kw = O.pack_key_block(codes, b)
    assert kw.shape == (H, D, G * b // 32)
    for h, w, d in [(0, 0, 0), (1, 1, 31), (0, 1, 7)]:
        assert np.array_equal(O.unpack_codes(kw[h, d, w][None], b), codes[w * 16:(w + 1) * 16, h, d])
    vw = O.pack_value_block(codes, b)
    assert vw.shape == (H, G, D * b // 32)
    for h, t, w in [(0, 0, 0), (1, 31, 1), (1, 5, 0)]:
        assert np.array_equal(O.unpack_codes(vw[h, t, w][None], b), codes[t, h, w * 16:(w + 1) * 16])


# --------------------------------------------------------------------------
# KIVI axes: keys per channel, values per token
# --------------------------------------------------------------------------


def test_key_axis_is_per_channel():
    # An outlier channel must not degrade the other channels of the same tokens.
    rng = np.random.default_rng(3)
    k = rng.standard_normal((64, 2, 16)).astype(np.float32)
    k[:, :, 5] *= 1000.0
    codes, d16, m16 = O.quantize_key_block(k, 2)
    err = np.abs(O.dequantize_key_block(codes, d16, m16) - k)
    normal = np.delete(err, 5, axis=2)
    assert normal.max() < 2.0          # ~range/6 of an N(0,1) channel, not ~1000/6
    assert d16.shape == (2, 16) and codes.shape == k.shape


def test_value_axis_is_per_token():
    rng = np.random.default_rng(4)
    v = rng.standard_normal((8, 2, 64)).astype(np.float32)
    v[3] *= 1000.0
    codes, d16, m16 = O.quantize_value_block(v, 4, 32)
    err = np.abs(O.dequantize_value_block(codes, d16, m16) - v)
    assert np.delete(err, 3, axis=0).max() < 0.5
    assert d16.shape == (8, 2, 2)


# --------------------------------------------------------------------------
# Cache state machine (residual ring, flush of group_k tokens)
# --------------------------------------------------------------------------


def _expected_split(L, R, G):
    q = 0 if L <= R else G * math.ceil((L - R) / G)
    return q, L - q


@pytest.mark.parametrize("R,G", [(32, 32), (128, 32), (128, 64), (128, 128), (64, 64), (96, 32)])
def test_state_machine_counts(R, G):
    H, D = 1, 16
    c = O.SequenceCache(H, D, 2, 2, G, 16, R)
    rng = np.random.default_rng(R + G)
    for L in range(1, 3 * R + 5):
        c.append_token(rng.standard_normal((H, D)), rng.standard_normal((H, D)))
        q, n = _expected_split(L, R, G)
        assert (c.quantized_tokens, c.residual_tokens) == (q, n), L
        assert c.quantized_tokens % G == 0 and 0 < c.residual_tokens <= R


@pytest.mark.parametrize("L,R,G,expect", [(1024, 32, 32, (992, 32)), (4096, 128, 32, (3968, 128)),
                                          (4352, 128, 32, (4224, 128)), (8192, 128, 64, (8064, 128)),
                                          (131072, 128, 128, (130944, 128)), (4096, 128, 128, (3968, 128))])
def test_state_machine_table(L, R, G, expect):
    assert _expected_split(L, R, G) == expect
    # and the oracle agrees on a cheap instance (single head, 16 channels)
    c = O.SequenceCache(1, 16, 2, 2, G, 16, R)
    z = np.zeros((L, 1, 16), np.float32)
    c.append(z, z)
    assert (c.quantized_tokens, c.residual_tokens) == expect


def test_ring_and_blocks_hold_the_right_tokens():
    H, D, G, R = 2, 32, 32, 64
    rng = np.random.default_rng(7)
    L = 5 * G + 17
    k = rng.standard_normal((L, H, D)).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    c = O.SequenceCache(H, D, 2, 4, G, 32, R)
    c.append(k, v)
    Q = c.quantized_tokens
    assert np.array_equal(np.stack(c.ring_k), k[Q:]) and np.array_equal(np.stack(c.ring_v), v[Q:])
    K, V = c.dequantized()
    assert K.shape == (L, H, D)
    for j in range(Q // G):
        blk = slice(j * G, (j + 1) * G)
        kr = k[blk]
        rngk = kr.max(axis=0) - kr.min(axis=0)
        assert np.all(np.abs(K[blk] - kr) <= rngk / 6 * 1.01 + 1e-3)
        vr = v[blk].reshape(G, H, 1, 32)
        rngv = (vr.max(axis=3) - vr.min(axis=3))[..., None]
        assert np.all(np.abs(V[blk].reshape(G, H, 1, 32) - vr) <= rngv / 30 * 1.01 + 1e-3)


def test_chunked_append_equals_single_call():
    H, D, G, R = 2, 32, 32, 64
    rng = np.random.default_rng(8)
    L = 300
    k = rng.standard_normal((L, H, D)).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    a = O.SequenceCache(H, D, 2, 2, G, 32, R)
    a.append(k, v)
    b = O.SequenceCache(H, D, 2, 2, G, 32, R)
    pos = 0
    for n in [1, 63, 2, 100, 1, 1, 132]:
        b.append(k[pos:pos + n], v[pos:pos + n])
        pos += n
    assert pos == L
    Ka, Va = a.dequantized()
    Kb, Vb = b.dequantized()
    assert np.array_equal(Ka, Kb) and np.array_equal(Va, Vb)


def test_flush_residual():
    H, D, G, R = 1, 16, 32, 128
    c = O.SequenceCache(H, D, 2, 2, G, 16, R)
    z = np.ones((100, H, D), np.float32)
    c.append(z, z)
    assert (c.quantized_tokens, c.residual_tokens) == (0, 100)
    c.flush_residual()
    assert (c.quantized_tokens, c.residual_tokens) == (96, 4)
    c.flush_residual()
    assert (c.quantized_tokens, c.residual_tokens) == (96, 4)


# --------------------------------------------------------------------------
# Separate residual lengths for keys and values ("Quantize What Counts", KV
# Cache Quantization: residual_length {"k", "v"}); reading 9 of the oracle
# --------------------------------------------------------------------------


def _single_window_counts(L, R, G):
    """(quantized, exact) tokens of one tensor after L single-token appends
    to a ring of R slots that flushes G tokens when full, in closed form."""
    if L <= R:
        return 0, L
    n = R - G + 1 + (L - R - 1) % G
    return L - n, n


@pytest.mark.parametrize("Rk,Rv,G,S", [(64, 128, 32, 0), (128, 64, 32, 0), (32, 96, 32, 2), (128, 256, 64, 0),
                                       (256, 128, 128, 1), (64, 64, 32, 0)])
def test_split_residual_counts_closed_form(Rk, Rv, G, S):
    H, D = 1, 16
    c = O.SequenceCache(H, D, 2, 2, G, 16, Rk, sinks=S, residual_v=Rv)
    rng = np.random.default_rng(Rk + 3 * Rv + G)
    for L in range(1, 3 * max(Rk, Rv) + G + 3):
        c.append_token(rng.standard_normal((H, D)), rng.standard_normal((H, D)))
        s = min(L, S)
        assert c.sink_tokens == s
        assert (c.quantized_tokens, c.residual_tokens) == _single_window_counts(L - s, Rk, G), L
        assert (c.quantized_tokens_v, c.residual_tokens_v) == _single_window_counts(L - s, Rv, G), L
        assert c.length == L


def test_single_window_closed_form_agrees_with_the_table():
    # the closed form above and the ceil form of the single-window test are one rule
    for R, G in [(32, 32), (128, 32), (128, 64), (96, 32)]:
        for L in range(1, 4 * R):
            assert _single_window_counts(L, R, G) == _expected_split(L, R, G), (L, R, G)


def _tensor_state(c, key):
    if key:
        return c.key_blocks, c.ring_k
    return c.value_blocks, c.ring_v


def _same_tensor(a, b, key):
    ba, ra = _tensor_state(a, key)
    bb, rb = _tensor_state(b, key)
    if len(ba) != len(bb) or len(ra) != len(rb):
        return False
    for x, y in zip(ba, bb):
        if not all(np.array_equal(np.asarray(u).view(np.uint8), np.asarray(w).view(np.uint8)) for u, w in zip(x, y)):
            return False
    return all(np.array_equal(u, w) for u, w in zip(ra, rb))


@pytest.mark.parametrize("k_axis,rot", [(0, False), (1, True)])
def test_split_residual_tensors_equal_single_window_caches(k_axis, rot):
    # keys depend only on the key window and values only on the value window:
    # a (Rk, Rv) cache holds the keys of an (Rk, Rk) cache and the values of
    # an (Rv, Rv) cache, bit for bit, after appends and after flush_residual
    H, D, G, Rk, Rv, gv = 2, 32, 32, 64, 160, 32 if k_axis == 0 else 32
    rng = np.random.default_rng(31 + k_axis)
    L = 7 * G + 13
    k = rng.standard_normal((L, H, D)).astype(np.float32) * np.exp(rng.standard_normal(D)).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    mk = lambda r, rv: O.SequenceCache(H, D, 2, 4, G, gv, r, sinks=1, k_axis=k_axis, hadamard=rot, residual_v=rv)
    split, kref, vref = mk(Rk, Rv), mk(Rk, Rk), mk(Rv, Rv)
    pos = 0
    for n in [1, 40, 3, 97, 1, 1, 80, L - 223]:
        for c in (split, kref, vref):
            c.append(k[pos:pos + n], v[pos:pos + n])
        pos += n
        assert _same_tensor(split, kref, True) and _same_tensor(split, vref, False), pos
    assert pos == L
    assert split.quantized_tokens != split.quantized_tokens_v  # the windows really differ here
    for c in (split, kref, vref):
        c.flush_residual()
    assert _same_tensor(split, kref, True) and _same_tensor(split, vref, False)
    assert split.residual_tokens == split.residual_tokens_v == (L - 1) % G


def test_split_residual_exact_tokens_are_the_appended_ones():
    # token i's key is exact iff i >= sinks + quantized keys, its value iff
    # i >= sinks + quantized values; the exact ones are the appended values
    H, D, G, Rk, Rv, S = 2, 32, 32, 128, 64, 2
    rng = np.random.default_rng(41)
    L = S + 6 * G + 5
    k = rng.standard_normal((L, H, D)).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    c = O.SequenceCache(H, D, 2, 2, G, 32, Rk, sinks=S, residual_v=Rv)
    c.append(k, v)
    K, V = c.dequantized()
    qk, qv = S + c.quantized_tokens, S + c.quantized_tokens_v
    assert qk < qv
    assert np.array_equal(K[:S], k[:S]) and np.array_equal(V[:S], v[:S])
    assert np.array_equal(K[qk:], k[qk:]) and np.array_equal(V[qv:], v[qv:])
    # a quantized 2-bit token is never exact for N(0,1) data
    assert np.all(np.any(K[S:qk] != k[S:qk], axis=(1, 2))) and np.all(np.any(V[S:qv] != v[S:qv], axis=(1, 2)))


def test_split_residual_attention_matches_sdpa_on_mixed_cache():
    # the attention of a split cache is textbook attention over the keys of
    # the (Rk, Rk) cache and the values of the (Rv, Rv) cache
    H, Hq, D, G, Rk, Rv = 2, 8, 32, 32, 96, 32
    rng = np.random.default_rng(43)
    L = 9 * G + 21
    k = rng.standard_normal((L, H, D)).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    split = O.SequenceCache(H, D, 2, 4, G, 32, Rk, residual_v=Rv)
    kref = O.SequenceCache(H, D, 2, 4, G, 32, Rk)
    vref = O.SequenceCache(H, D, 2, 4, G, 32, Rv)
    for c in (split, kref, vref):
        c.append(k, v)
    Kk, _ = kref.dequantized()
    _, Vv = vref.dequantized()
    q = rng.standard_normal((Hq, D))
    assert np.abs(O.decode_attention(split, q, D ** -0.5) - _sdpa(q, Kk, Vv, D ** -0.5)).max() < 1e-12


# --------------------------------------------------------------------------
# Attention: hand example, closed forms, and an independent library routine
# --------------------------------------------------------------------------


def _sdpa(q, k, v, scale):
    """torch scaled_dot_product_attention in fp64; q [Hq,D], k/v [L,Hkv,D]."""
    Hq = q.shape[0]
    Hkv = k.shape[1]
    kk = torch.from_numpy(np.asarray(k, np.float64)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    vv = torch.from_numpy(np.asarray(v, np.float64)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    qq = torch.from_numpy(np.asarray(q, np.float64))[:, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)
    return o[:, 0, :].numpy()


def test_attention_hand_example():
    # scores ln3 and 0 -> weights 3/4, 1/4 -> o = 3/4 [4,0] + 1/4 [0,8] = [3,2]
    q = np.array([[1.0, 0.0]])
    k = np.array([[[math.log(3.0), 0.0]], [[0.0, 0.0]]])
    v = np.array([[[4.0, 0.0]], [[0.0, 8.0]]])
    o = O.attention(q, k, v, 1.0)
    assert np.allclose(o, [[3.0, 2.0]], atol=1e-14)


def test_attention_closed_forms():
    rng = np.random.default_rng(11)
    k = rng.standard_normal((50, 2, 8))
    v = rng.standard_normal((50, 2, 8))
    o = O.attention(np.zeros((4, 8)), k, v, 0.3)          # uniform weights
    assert np.allclose(o[0], v[:, 0].mean(0), atol=1e-14) and np.allclose(o[3], v[:, 1].mean(0), atol=1e-14)
    o1 = O.attention(rng.standard_normal((2, 8)), k[:1], v[:1], 0.3)   # one token
    assert np.allclose(o1, v[0], atol=1e-15)
    assert np.array_equal(O.attention(np.ones((2, 8)), k[:0], v[:0], 1.0), np.zeros((2, 8)))


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (32, 8)])
def test_attention_matches_sdpa(Hq, Hkv):
    rng = np.random.default_rng(Hq + Hkv)
    D, L = 16, 77
    q = rng.standard_normal((Hq, D))
    k = rng.standard_normal((L, Hkv, D)) * 2
    v = rng.standard_normal((L, Hkv, D))
    assert np.abs(O.attention(q, k, v, 0.25) - _sdpa(q, k, v, 0.25)).max() < 1e-12


def test_residual_only_cache_is_exact_attention():
    H, D, G, R = 2, 32, 32, 128
    rng = np.random.default_rng(12)
    k = rng.standard_normal((90, H, D)).astype(np.float32)
    v = rng.standard_normal((90, H, D)).astype(np.float32)
    c = O.SequenceCache(H, D, 2, 2, G, 32, R)
    c.append(k, v)
    assert c.quantized_tokens == 0
    q = rng.standard_normal((8, D))
    assert np.abs(O.decode_attention(c, q, D ** -0.5) - _sdpa(q, k, v, D ** -0.5)).max() < 1e-12


def test_quantized_cache_attention_matches_sdpa_on_dequantized():
    H, D, G, R = 2, 64, 32, 64
    rng = np.random.default_rng(13)
    L = 333
    k = rng.standard_normal((L, H, D)).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    c = O.SequenceCache(H, D, 2, 4, G, 32, R)
    c.append(k, v)
    K, V = c.dequantized()
    q = rng.standard_normal((8, D))
    o = O.decode_attention(c, q, D ** -0.5)
    assert np.abs(o - _sdpa(q, K, V, D ** -0.5)).max() < 1e-12
    # and the quantized result stays near exact attention on the raw inputs
    assert np.abs(o - _sdpa(q, k, v, D ** -0.5)).max() < 0.5


# --------------------------------------------------------------------------
# Attention sinks (KV1-1.2B card: the first 4 tokens keep full precision)
# --------------------------------------------------------------------------


def _blocks_equal(a, b):
    return len(a) == len(b) and all(
        np.array_equal(getattr(x, f), getattr(y, f)) for x, y in zip(a, b) for f in ("kc", "kd", "km", "vc", "vd", "vm"))


@pytest.mark.parametrize("S", [1, 4, 8])
def test_sinks_shift_the_quantized_stream(S):
    # the tokens after the sinks are cached exactly as a sink-free cache
    # caches the same tokens: same blocks (codes, scales) and the same ring
    H, D, G, R = 2, 32, 32, 64
    rng = np.random.default_rng(40 + S)
    L = S + 5 * G + 17
    k = (rng.standard_normal((L, H, D)) * 3).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    k[:S] *= 100.0  # outlier sink keys must not reach any key group
    a = O.SequenceCache(H, D, 2, 4, G, 32, R, sinks=S)
    b = O.SequenceCache(H, D, 2, 4, G, 32, R)
    for t in range(L):
        a.append_token(k[t], v[t])
    b.append(k[S:], v[S:])
    assert a.sink_tokens == S and a.length == L
    assert _blocks_equal(a.blocks, b.blocks)
    assert all(np.array_equal(x, y) for x, y in zip(a.ring_k, b.ring_k)) and len(a.ring_k) == len(b.ring_k)
    assert all(np.array_equal(x, k[t]) for t, x in enumerate(a.sink_k))
    a.flush_residual()
    b.flush_residual()
    assert _blocks_equal(a.blocks, b.blocks) and a.sink_tokens == S  # sinks are never flushed


def test_sinks_are_read_exactly_in_token_order():
    H, D, G, R, S = 2, 32, 32, 64, 4
    rng = np.random.default_rng(44)
    L = 200
    k = rng.standard_normal((L, H, D)).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    a = O.SequenceCache(H, D, 4, 2, G, 32, R, sinks=S)
    a.append(k, v)
    K, V = a.dequantized()
    assert K.shape[0] == L
    assert np.array_equal(K[:S], k[:S]) and np.array_equal(V[:S], v[:S])
    b = O.SequenceCache(H, D, 4, 2, G, 32, R)
    b.append(k[S:], v[S:])
    Kb, Vb = b.dequantized()
    assert np.array_equal(K[S:], Kb) and np.array_equal(V[S:], Vb)
    q = rng.standard_normal((8, D))
    o = O.decode_attention(a, q, 0.2)
    assert np.abs(o - _sdpa(q, K, V, 0.2)).max() < 1e-12


def test_short_sequence_is_all_sinks_and_exact():
    # a sequence no longer than S holds only sinks: plain softmax attention
    H, D, S = 1, 4, 4
    k = np.array([[[1.0, 0, 0, 0]], [[0, 2.0, 0, 0]], [[0, 0, 0, 0]]], np.float32)
    v = np.array([[[1.0, 2, 3, 4]], [[5.0, 6, 7, 8]], [[9.0, 10, 11, 12]]], np.float32)
    c = O.SequenceCache(H, D, 2, 2, 32, 32, 64, sinks=S)
    c.append(k, v)
    assert (c.sink_tokens, c.quantized_tokens, c.residual_tokens) == (3, 0, 0)
    q = np.array([[math.log(2.0), math.log(3.0) / 2, 0, 0]])
    # scores ln2, ln3, 0 -> weights 2/6, 3/6, 1/6
    want = (2 * v[0, 0] + 3 * v[1, 0] + 1 * v[2, 0]) / 6
    assert np.allclose(O.decode_attention(c, q, 1.0)[0], want, atol=1e-12)


# --------------------------------------------------------------------------
# BQ2_0: Hadamard rotation and per-token keys (KV1-1.2B card, BQ2_0)
# --------------------------------------------------------------------------


def test_rotation_hand_example_and_basis_columns():
    # [1, 2, 3, 4] . H4 = [10, -2, -4, 0] / 2 (H4 symmetric)
    assert np.array_equal(O.rotate_fp32(np.array([1, 2, 3, 4], np.float32)), np.array([5, -1, -2, 0], np.float32))
    D = 128
    H = O.sylvester(D)
    assert np.allclose(H @ H, np.eye(D), atol=1e-12) and np.array_equal(H, H.T)
    s = np.float32(1.0 / np.sqrt(D))
    for i in (0, 1, 37, 127):
        e = np.zeros(D, np.float32)
        e[i] = 1.0
        # butterflies of a basis vector give exactly +-1: one rounding, by s
        assert np.array_equal(O.rotate_fp32(e), (np.sign(H[i]) * s).astype(np.float32))


def test_rotation_is_the_matrix_product_and_an_involution():
    D = 128
    rng = np.random.default_rng(50)
    x = rng.standard_normal((7, 3, D)).astype(np.float32)
    H = O.sylvester(D)
    y = O.rotate_fp32(x)
    ref = x.astype(np.float64) @ H
    assert np.abs(y - ref).max() <= 1e-5 * np.abs(x).max()   # 7 fp32 roundings of partial sums
    assert np.abs(O.rotate_fp32(y) - x).max() <= 2e-5 * np.abs(x).max()


def test_per_token_key_blocks_use_the_value_quantizer():
    H, D, G, Gv, R = 2, 64, 32, 64, 64
    rng = np.random.default_rng(51)
    k = (rng.standard_normal((G + 3, H, D)) * 2).astype(np.float32)
    v = rng.standard_normal((G + 3, H, D)).astype(np.float32)
    c = O.SequenceCache(H, D, 2, 2, G, Gv, R, k_axis=1)
    c.append(k, v)
    c.flush_residual()
    blk = c.blocks[0]
    kc, kd, km = O.quantize_groups(k[:G].reshape(G, H, 1, D), 2)  # one group per (token, head) over 64 channels
    assert np.array_equal(blk.kc, kc.reshape(G, H, D)) and np.array_equal(blk.kd, kd) and np.array_equal(blk.km, km)
    # BQ2_0 size: 2-bit codes of 64 values + fp16 scale and zero = 20 bytes
    assert O.quantized_bytes_per_token(1, 64, 2, 2, 32, 64, k_axis=1) == 40.0


def test_hadamard_cache_quantizes_rotated_vectors_and_attends_in_the_original_basis():
    H, D, G, Gv, R = 2, 128, 32, 64, 64
    rng = np.random.default_rng(52)
    L = 3 * G + 40
    k = (rng.standard_normal((L, H, D)) * np.exp(rng.standard_normal((1, H, D)))).astype(np.float32)
    v = rng.standard_normal((L, H, D)).astype(np.float32)
    c = O.SequenceCache(H, D, 2, 4, G, Gv, R, k_axis=1, hadamard=True)
    c.append(k, v)
    # the stored blocks are the quantizer applied to the rotated tokens
    kc, kd, km = O.quantize_value_block(O.rotate_fp32(k[:G]), 2, Gv)
    assert np.array_equal(c.blocks[0].kc, kc) and np.array_equal(c.blocks[0].kd, kd)
    vc, vd, vm = O.quantize_value_block(O.rotate_fp32(v[:G]), 4, Gv)
    assert np.array_equal(c.blocks[0].vc, vc) and np.array_equal(c.blocks[0].vm, vm)
    # attention computed independently in the rotated basis: scores of
    # quantized tokens from Hq, their values' contribution multiplied by H
    Hm = O.sylvester(D)
    q = rng.standard_normal((8, D))
    Ks, Vs = c.dequantized()            # stored basis
    Q = c.quantized_tokens
    scale = D ** -0.5
    out = np.zeros((8, D))
    for h in range(8):
        kv = h // 4
        s_q = scale * (Ks[:Q, kv].astype(np.float64) @ (Hm @ q[h]))
        s_r = scale * (Ks[Q:, kv].astype(np.float64) @ q[h])
        s_all = np.concatenate([s_q, s_r])
        p = np.exp(s_all - s_all.max())
        o_rot = p[:Q] @ Vs[:Q, kv].astype(np.float64)
        out[h] = (Hm @ o_rot + p[Q:] @ Vs[Q:, kv].astype(np.float64)) / p.sum()
    assert np.abs(O.decode_attention(c, q, scale) - out).max() < 1e-12
    # with 8-bit codes the rotated cache stays close to exact attention on the
    # raw tokens (a missing or transposed rotation would not)
    c8 = O.SequenceCache(H, D, 8, 8, G, Gv, R, k_axis=1, hadamard=True)
    c8.append(k, v)
    assert np.abs(O.decode_attention(c8, q, scale) - _sdpa(q, k, v, scale)).max() < 0.05


# --------------------------------------------------------------------------
# Sizes (KV1-1.2B card, Memory)
# --------------------------------------------------------------------------


def test_kv1_memory_table():
    t = _load("kv1_memory_table.json")
    m = t["model"]
    per_value = O.quantized_bytes_per_token(1, 64, 2, 2, 64, 64) * 8 / 128
    assert per_value == t["bits_per_value_bq2_0"]
    for row in t["rows"]:
        if row["bits"] == 16:
            per_tok = m["attention_layers"] * m["kv_heads"] * m["head_dim"] * 2 * 2
        else:
            per_tok = m["attention_layers"] * O.quantized_bytes_per_token(
                m["kv_heads"], m["head_dim"], row["bits"], row["bits"], m["group"], m["group"])
        assert round(per_tok / 1024, 1) == row["per_token_kib"], row
        assert round(per_tok * 8192 / 2 ** 20) == row["ctx_8k_mib"], row
        assert round(per_tok * 32768 / 2 ** 20) == row["ctx_32k_mib"], row


# ---------------------------------------------------------------------------
# Several query tokens per sequence (oracle reading 8)
# ---------------------------------------------------------------------------


def _cache(seed, L, R=64, G=32, kb=2, vb=4, H=2, S=0):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((L, H, 16)) * np.exp(rng.standard_normal((1, H, 16)))).astype(np.float16).astype(np.float32)
    v = rng.standard_normal((L, H, 16)).astype(np.float16).astype(np.float32)
    c = O.SequenceCache(H, 16, kb, vb, G, 16, R, sinks=S)
    c.append(k, v)
    return c, k, v


def test_multi_query_is_causal_sdpa_over_the_effective_cache():
    c, _, _ = _cache(3, 150)
    K, V = c.dequantized(effective=True)
    L, T = K.shape[0], 5
    q = np.random.default_rng(4).standard_normal((T, 4, 16))
    o = O.decode_attention_multi(c, q, 0.25)
    # torch SDPA with an explicit mask: query t sees keys j <= L - T + t
    mask = torch.from_numpy(np.arange(L)[None, :] <= (L - T + np.arange(T))[:, None])
    kk = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(2, 0)   # [Hq, L, D]
    vv = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(2, 0)
    qq = torch.from_numpy(q).permute(1, 0, 2)                          # [Hq, T, D]
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=0.25)
    assert np.abs(o - ref.permute(1, 0, 2).numpy()).max() < 1e-12


def test_multi_query_rows_equal_single_decodes_of_the_prefixes():
    # no flush among the last T appends (the ring had room): the cache of the
    # first L - T + t + 1 tokens holds the same blocks, so query t equals a
    # single-token decode of that shorter cache
    L, T = 150, 4            # R 64, G 32: 96 quantized + 54 in the ring, also for 147..149 tokens
    full, k, v = _cache(8, L)
    assert full.residual_tokens >= T + 32
    q = np.random.default_rng(9).standard_normal((T, 4, 16))
    o = O.decode_attention_multi(full, q, 0.3)
    for t in range(T):
        part = O.SequenceCache(2, 16, 2, 4, 32, 16, 64)
        part.append(k[:L - T + t + 1], v[:L - T + t + 1])
        assert part.quantized_tokens == full.quantized_tokens
        assert np.array_equal(o[t], O.decode_attention(part, q[t], 0.3))


def test_multi_query_single_token_is_decode_and_sinks_stay_visible():
    c, _, _ = _cache(5, 90, S=3)
    q = np.random.default_rng(6).standard_normal((1, 4, 16))
    assert np.array_equal(O.decode_attention_multi(c, q, 0.2)[0], O.decode_attention(c, q[0], 0.2))
    # uniform scores (q = 0): query t averages the values of tokens 0 .. L - T + t
    _, V = c.dequantized(effective=True)
    o = O.decode_attention_multi(c, np.zeros((3, 4, 16)), 0.2)
    for t in range(3):
        assert np.allclose(o[t, 0], V[:90 - 3 + t + 1, 0].mean(0), atol=1e-12)


def test_multi_query_prefixes_with_sinks_and_rotation():
    # the prefix property on the KV1 layout: per-token keys, rotation, sinks
    rng = np.random.default_rng(21)
    L, T, H = 4 + 96 + 40, 3, 2   # 4 sinks, 3 blocks of 32, ring of 40 (R 64, G 32)
    k = rng.standard_normal((L, H, 16)).astype(np.float16).astype(np.float32)
    v = rng.standard_normal((L, H, 16)).astype(np.float16).astype(np.float32)

    def cache(n):
        c = O.SequenceCache(H, 16, 2, 2, 32, 16, 64, sinks=4, k_axis=1, hadamard=True)
        c.append(k[:n], v[:n])
        return c

    full = cache(L)
    assert full.sink_tokens == 4 and full.quantized_tokens == 96 and full.residual_tokens == 40
    q = rng.standard_normal((T, 4, 16))
    o = O.decode_attention_multi(full, q, 0.25)
    for t in range(T):
        part = cache(L - T + t + 1)
        assert part.quantized_tokens == full.quantized_tokens
        assert np.array_equal(o[t], O.decode_attention(part, q[t], 0.25))
