"""Plain CPU oracle for the asymmetric 2/4/8-bit KV cache and decode attention.

TEST INFRASTRUCTURE ONLY. This module is a slow, literal restatement of the
method so that the CUDA library can be checked against it. Only the test
suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it; the library itself never does, and it shares no code, table or
constant with the CUDA sources.

Sources (web pages, cited by title and section):

* "KV1-1.2B" model card, section "Quantization Format: KV1.cpp BQ2_0":
  the affine quantizer -- scale ``d = fp16(max((max - min) / 3, 1e-6))``,
  zero ``m = fp16(min)``, code ``q = clamp(round_half_to_even((x - m) / d), 0, 3)``
  computed in fp32 with the fp16-rounded ``m`` and ``d``; dequantization
  ``x_hat = q * d + m``; codes packed lowest bits first (``q0 | q1<<2 | ...``);
  20 bytes per 64 values = 2.5 bits/value. Section "Memory": the per-token and
  32K-context sizes.
* "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache" (README),
  sections "Overview" and "Example": keys quantized per channel, values per
  token, 2 or 4 bits (``k_bits``, ``v_bits``), ``group_size``, and a window of
  ``residual_length`` recent tokens kept in full precision; GQA support
  (update of 2025.01.18).
* "Quantize What Counts: More For Keys, Less For Values", section "KV Cache
  Quantization": independent key and value bit widths, residual length and
  group size per tensor; bit range up to 8.

Readings taken where the pages are silent (each is listed with its reason in
the design notes of the repository):

1. The b-bit quantizer generalises the 2-bit rule by replacing 3 with 2^b - 1;
   the 1e-6 floor on the scale applies at every width.
2. The zero point is formed from ``min + 0.0`` so that a minimum of -0.0 is
   stored as +0.0.
3. Keys are grouped per (KV head, channel) over ``group_k`` consecutive tokens;
   values per (token, KV head) over ``group_v`` consecutive channels.
4. The residual window is a ring of exactly R slots. Appending a token to a
   full ring first quantizes the oldest ``group_k`` tokens of the ring (keys
   and values together). A multi-token append is the same sequence of
   single-token appends. ``flush_residual`` quantizes every complete block of
   ``group_k`` tokens still in the ring.
5. Decode attention is ``softmax(scale * q K~^T) V~`` over every cached token
   (no mask: the decode query is the newest position), where K~, V~ are the
   dequantized values for quantized tokens and the exact stored values for the
   residual window. Query head h reads KV head ``h // (Hq / Hkv)`` (GQA).
   A sequence with no cached tokens yields a zero output.
6. Attention sinks ("KV1-1.2B" card: the first 4 tokens of every sequence
   keep fp16 K/V; BQ2_0 section: positions 0-3 keep full-precision K/V): with
   ``sinks = S`` the first S tokens appended to a sequence are stored exactly
   and never quantized; everything above (ring, flushes, key groups) applies
   to the tokens after them, so key group j covers tokens S + jG .. S + jG +
   G - 1. Decode attention reads the sinks exactly, like the ring.
7. BQ2_0 ("KV1-1.2B" card, Quantization Format): keys quantized per token
   (``k_axis = 1``) are grouped like values, over ``group_v`` channels of one
   (token, KV head). The Hadamard rotation (``hadamard``) multiplies every
   stored K and V head vector by the normalized Sylvester matrix H (H.H = I)
   before it is quantized; here it is applied when a block is quantized, so
   the ring and the sinks keep the exact tokens. Scores of quantized tokens
   use Hq and their values' contribution is multiplied by H again, i.e.
   attention sees the effective keys and values (dequantized) . H. In fp32 the
   product x.H is the radix-2 butterfly (stages of half-width 1, 2, 4, ...;
   a pair (a, b) becomes (a + b, a - b), each one fp32 rounding) followed by
   one fp32 multiplication by fp32(1/sqrt(D)).

8. Several query tokens per sequence (verifying T drafted tokens in one
   pass, a serving pattern none of the pages describes; the plainest reading
   of their decoding rule): the T tokens' keys and values are appended first,
   and query t, at position L - T + t, attends causally to the tokens up to
   its own position. T = 1 is reading 5.

9. Separate residual lengths for keys and values ("Quantize What Counts",
   KV Cache Quantization: ``residual_length`` and ``group_size`` are given
   per tensor): each tensor keeps its own ring -- ``residual`` keys and
   ``residual_v`` values -- and applies reading 4 on its own, flushing its
   oldest ``group_k`` tokens when its ring is full. A token's key and value
   may then be one quantized and one exact. Values are flushed in blocks of
   ``group_k`` tokens too (their groups run along channels, so any block
   length would do; this one keeps the blocks of both tensors aligned). Equal
   lengths give exactly the single-window cache.

Floating point: the quantizer runs in IEEE fp32 (the precision the KV1 card
fixes); numpy evaluates each fp32 operation with one rounding and never
contracts a multiply-add. Attention runs in fp64.
"""

from __future__ import annotations

import numpy as np

F32 = np.float32
F16 = np.float16

# ---------------------------------------------------------------------------
# Quantizer ("KV1-1.2B", Quantization Format: KV1.cpp BQ2_0)
# ---------------------------------------------------------------------------

SCALE_FLOOR = F32(1e-6)


def fp16_rn(x) -> np.ndarray:
    """Round fp32 values to fp16, round-to-nearest-even (IEEE binary16)."""
    return np.asarray(x, dtype=F32).astype(F16)


def quantize_groups(x: np.ndarray, bits: int):
    """Asymmetric min/max quantization of every group along the last axis.

    ``x`` is fp32 with groups along its last axis. Returns ``(codes, d16, m16)``:
    codes (uint8, same shape as ``x``) and the fp16 scale and zero point of
    each group (shape ``x.shape[:-1]``).

    Follows the BQ2_0 rule of the KV1 card with 3 replaced by ``2**bits - 1``:
    ``d = fp16(max((max-min)/(2^b-1), 1e-6))``, ``m = fp16(min)``,
    ``q = clamp(rint((x - m) / d), 0, 2^b-1)``, all in fp32, using the
    fp16-rounded ``m`` and ``d``.
    """
    assert bits in (2, 4, 8)
    x = np.asarray(x, dtype=F32)
    qmax = (1 << bits) - 1
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    d = (mx - mn) / F32(qmax)                       # one fp32 division
    d16 = fp16_rn(np.maximum(d, SCALE_FLOOR))
    m16 = fp16_rn(mn + F32(0.0))
    m32 = m16.astype(F32)[..., None]
    d32 = d16.astype(F32)[..., None]
    t = (x - m32) / d32                             # fp32 sub, then fp32 div
    q = np.clip(np.rint(t), 0, qmax).astype(np.uint8)  # rint: ties to even
    return q, d16, m16


def dequantize(codes: np.ndarray, d16: np.ndarray, m16: np.ndarray) -> np.ndarray:
    """``x_hat = q * d + m`` in fp32: a rounded product, then a rounded sum.

    ``d16``/``m16`` must broadcast against ``codes``.
    """
    return codes.astype(F32) * d16.astype(F32) + m16.astype(F32)


# ---------------------------------------------------------------------------
# Bit packing ("KV1-1.2B", BQ2_0 block: q0 | q1<<2 | q2<<4 | q3<<6)
# ---------------------------------------------------------------------------


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes along the last axis into uint32 words, lowest bits first.

    Code i of a run of ``32 // bits`` codes sits at bits ``[i*bits, (i+1)*bits)``.
    """
    per = 32 // bits
    c = np.asarray(codes, dtype=np.uint64)
    assert c.shape[-1] % per == 0
    c = c.reshape(c.shape[:-1] + (c.shape[-1] // per, per))
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    return (c << shifts).sum(axis=-1).astype(np.uint32)


def unpack_codes(words: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    per = 32 // bits
    w = np.asarray(words, dtype=np.uint64)[..., None]
    shifts = (np.arange(per, dtype=np.uint64) * np.uint64(bits))
    c = (w >> shifts) & np.uint64((1 << bits) - 1)
    return c.reshape(words.shape[:-1] + (words.shape[-1] * per,)).astype(np.uint8)


# ---------------------------------------------------------------------------
# KIVI axes: keys per channel over group_k tokens, values per token over
# group_v channels ("KIVI" README, Overview)
# ---------------------------------------------------------------------------


def quantize_key_block(k: np.ndarray, bits: int):
    """Keys of one block: ``k`` is [G, H, D] fp32 (G = group_k tokens).

    Every (head, channel) is one group over the G tokens. Returns
    codes [G, H, D], d16 [H, D], m16 [H, D].
    """
    q, d16, m16 = quantize_groups(np.transpose(k, (1, 2, 0)), bits)
    return np.transpose(q, (2, 0, 1)), d16, m16


def quantize_value_block(v: np.ndarray, bits: int, group_v: int):
    """Values of one block: ``v`` is [G, H, D] fp32.

    Every (token, head, run of ``group_v`` channels) is one group. Returns
    codes [G, H, D], d16 [G, H, D/group_v], m16 [G, H, D/group_v].
    """
    G, H, D = v.shape
    assert D % group_v == 0
    q, d16, m16 = quantize_groups(v.reshape(G, H, D // group_v, group_v), bits)
    return q.reshape(G, H, D), d16, m16


def dequantize_key_block(codes, d16, m16):
    return dequantize(codes, d16[None, :, :], m16[None, :, :])


def dequantize_value_block(codes, d16, m16):
    G, H, D = codes.shape
    ng = d16.shape[-1]
    c = codes.reshape(G, H, ng, D // ng)
    return dequantize(c, d16[..., None], m16[..., None]).reshape(G, H, D)


# Word arrangement of the library's packed block (documented in its header):
# key words [H, D, G*bits/32] (word w of channel d holds tokens w*32/bits ...),
# value words [H, G, D*bits/32] (word w of a token holds channels w*32/bits ...).


def pack_key_block(codes: np.ndarray, bits: int) -> np.ndarray:
    """codes [G, H, D] -> uint32 [H, D, G*bits/32], packed along tokens."""
    return pack_codes(np.transpose(codes, (1, 2, 0)), bits)       # [H, D, W]


def pack_value_block(codes: np.ndarray, bits: int) -> np.ndarray:
    """codes [G, H, D] -> uint32 [H, G, D*bits/32], packed along channels."""
    words = pack_codes(codes, bits)                              # [G, H, W]
    return np.ascontiguousarray(np.transpose(words, (1, 0, 2)))


# ---------------------------------------------------------------------------
# Hadamard rotation ("KV1-1.2B", BQ2_0: normalized Sylvester Hadamard matrix)
# ---------------------------------------------------------------------------


def sylvester(D: int) -> np.ndarray:
    """The normalized D x D Sylvester Hadamard matrix in fp64 (H . H = I)."""
    H = np.array([[1.0]])
    while H.shape[0] < D:
        H = np.block([[H, H], [H, -H]])
    assert H.shape[0] == D, "D must be a power of two"
    return H / np.sqrt(D)


def rotate_fp32(x: np.ndarray) -> np.ndarray:
    """x . H over the last axis in fp32: the butterfly stages of half-width
    1, 2, 4, ... D/2 (pair (a, b) at positions i, i + w with bit w of i clear
    becomes (a + b, a - b)), then one multiplication by fp32(1/sqrt(D))."""
    y = np.array(x, dtype=F32, copy=True)
    D = y.shape[-1]
    w = 1
    while w < D:
        v = y.reshape(y.shape[:-1] + (D // (2 * w), 2, w))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        w *= 2
    return (y * F32(1.0 / np.sqrt(D))).astype(F32)


# ---------------------------------------------------------------------------
# Cache state machine (KIVI README: residual window of recent fp16 tokens)
# ---------------------------------------------------------------------------


class QuantizedBlock:
    __slots__ = ("kc", "kd", "km", "vc", "vd", "vm")

    def __init__(self, kc, kd, km, vc, vd, vm):
        self.kc, self.kd, self.km, self.vc, self.vd, self.vm = kc, kd, km, vc, vd, vm


class SequenceCache:
    """KV cache of one sequence in one layer.

    Token values are fp32 arrays holding values exactly representable in the
    cache's storage type (fp16 or bf16); the rings keep them unchanged.

    Keys and values each keep their own residual window ("Quantize What
    Counts", KV Cache Quantization: ``residual_length`` given per tensor as
    ``{"k": ..., "v": ...}``): ``residual`` recent keys and ``residual_v``
    recent values (default: the same length) stay exact, and each tensor
    flushes its own oldest ``group_k`` tokens when its ring is full (reading
    4 applied to each tensor on its own). With equal lengths both flush
    together, on the same tokens.
    """

    def __init__(self, num_kv_heads, head_dim, k_bits, v_bits, group_k, group_v, residual, sinks=0, k_axis=0,
                 hadamard=False, residual_v=None):
        residual_v = residual if residual_v is None else residual_v
        for r in (residual, residual_v):
            assert r % group_k == 0 and r >= group_k
        assert sinks >= 0 and k_axis in (0, 1)
        self.H, self.D = num_kv_heads, head_dim
        self.k_bits, self.v_bits = k_bits, v_bits
        self.group_k, self.group_v, self.residual = group_k, group_v, residual
        self.residual_v = residual_v
        self.sinks = sinks
        self.k_axis, self.hadamard = k_axis, bool(hadamard)
        self.sink_k: list[np.ndarray] = []  # the first `sinks` tokens, exact, each [H, D]
        self.sink_v: list[np.ndarray] = []
        self.key_blocks: list[tuple] = []    # (codes [G, H, D], scale, zero) per flushed key block
        self.value_blocks: list[tuple] = []  # (codes [G, H, D], scale [G, H, groups], zero) per value block
        self.ring_k: list[np.ndarray] = []   # oldest first, each [H, D]
        self.ring_v: list[np.ndarray] = []

    @property
    def blocks(self) -> list:
        """Blocks whose keys and values are both quantized, as QuantizedBlock
        (every block when the two residual lengths are equal)."""
        return [QuantizedBlock(*kb, *vb) for kb, vb in zip(self.key_blocks, self.value_blocks)]

    @property
    def quantized_tokens(self) -> int:
        """Quantized keys (after the sinks)."""
        return len(self.key_blocks) * self.group_k

    @property
    def quantized_tokens_v(self) -> int:
        """Quantized values (after the sinks)."""
        return len(self.value_blocks) * self.group_k

    @property
    def residual_tokens(self) -> int:
        """Exact keys in the key ring."""
        return len(self.ring_k)

    @property
    def residual_tokens_v(self) -> int:
        """Exact values in the value ring."""
        return len(self.ring_v)

    @property
    def sink_tokens(self) -> int:
        return len(self.sink_k)

    @property
    def length(self) -> int:
        return self.sink_tokens + self.quantized_tokens + self.residual_tokens

    def _flush_keys(self):
        G = self.group_k
        k = np.stack(self.ring_k[:G]).astype(F32)
        del self.ring_k[:G]
        if self.hadamard:
            k = rotate_fp32(k)
        if self.k_axis == 1:  # per-token keys, grouped like values
            self.key_blocks.append(quantize_value_block(k, self.k_bits, self.group_v))
        else:
            self.key_blocks.append(quantize_key_block(k, self.k_bits))

    def _flush_values(self):
        G = self.group_k
        v = np.stack(self.ring_v[:G]).astype(F32)
        del self.ring_v[:G]
        if self.hadamard:
            v = rotate_fp32(v)
        self.value_blocks.append(quantize_value_block(v, self.v_bits, self.group_v))

    def append_token(self, k: np.ndarray, v: np.ndarray):
        """Append one token ([H, D] each): one of the first `sinks` tokens is
        kept as it is; otherwise a full key ring first flushes its oldest G
        keys, and a full value ring its oldest G values."""
        if len(self.sink_k) < self.sinks:
            self.sink_k.append(np.asarray(k, dtype=F32).copy())
            self.sink_v.append(np.asarray(v, dtype=F32).copy())
            return
        if len(self.ring_k) == self.residual:
            self._flush_keys()
        if len(self.ring_v) == self.residual_v:
            self._flush_values()
        self.ring_k.append(np.asarray(k, dtype=F32).copy())
        self.ring_v.append(np.asarray(v, dtype=F32).copy())

    def append(self, k: np.ndarray, v: np.ndarray):
        """Append T tokens ([T, H, D] each) as T single-token appends."""
        for t in range(k.shape[0]):
            self.append_token(k[t], v[t])

    def flush_residual(self):
        """Quantize every complete block of group_k tokens left in either ring."""
        while len(self.ring_k) >= self.group_k:
            self._flush_keys()
        while len(self.ring_v) >= self.group_k:
            self._flush_values()

    def dequantized(self, effective=False):
        """(K~, V~) as fp32 [L, H, D] in token order: the exact sinks, the
        dequantized blocks (as stored: in the rotated basis for a Hadamard
        cache), then the ring; keys and values each with their own quantized
        and exact parts. effective=True: fp64, with the blocks rotated back
        (. H), the keys and values attention sees."""
        ks, vs = [], []
        if self.sink_k:
            ks.append(np.stack(self.sink_k))
            vs.append(np.stack(self.sink_v))
        Hm = sylvester(self.D) if (effective and self.hadamard) else None
        for kc, kd, km in self.key_blocks:
            if self.k_axis == 1:
                kq = dequantize_value_block(kc, kd, km)
            else:
                kq = dequantize_key_block(kc, kd, km)
            ks.append(kq.astype(np.float64) @ Hm if Hm is not None else kq)
        for vc, vd, vm in self.value_blocks:
            vq = dequantize_value_block(vc, vd, vm)
            vs.append(vq.astype(np.float64) @ Hm if Hm is not None else vq)
        if self.ring_k:
            ks.append(np.stack(self.ring_k))
        if self.ring_v:
            vs.append(np.stack(self.ring_v))
        dt = np.float64 if effective else F32
        if not ks:
            z = np.zeros((0, self.H, self.D), dt)
            return z, z.copy()
        return np.concatenate(ks).astype(dt), np.concatenate(vs).astype(dt)


# ---------------------------------------------------------------------------
# Decode attention (KIVI README: decoding phase; GQA)
# ---------------------------------------------------------------------------


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q k^T) v for one decode query per head, in fp64.

    q [Hq, D]; k, v [L, Hkv, D]. Query head h uses KV head h // (Hq/Hkv).
    Returns fp64 [Hq, D]; zeros when L == 0.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Hq, D = q.shape
    L, Hkv, _ = k.shape
    assert Hq % Hkv == 0
    g = Hq // Hkv
    out = np.zeros((Hq, D), np.float64)
    if L == 0:
        return out
    for h in range(Hq):
        kv = h // g
        s = scale * (k[:, kv, :] @ q[h])
        p = np.exp(s - s.max())
        out[h] = (p @ v[:, kv, :]) / p.sum()
    return out


def decode_attention(cache: SequenceCache, q: np.ndarray, scale: float) -> np.ndarray:
    """Decode attention of one sequence over its sinks, quantized blocks and
    ring (for a Hadamard cache, the effective keys and values)."""
    k, v = cache.dequantized(effective=True)
    return attention(q, k, v, scale)


def decode_attention_multi(cache: SequenceCache, q: np.ndarray, scale: float) -> np.ndarray:
    """Decode attention of T query tokens of one sequence ([T, Hq, D]) whose
    own keys and values are the sequence's T newest cached tokens (reading 8):
    query t sits at position L - T + t and attends to tokens 0 .. L - T + t.
    Returns fp64 [T, Hq, D]."""
    q = np.asarray(q, dtype=np.float64)
    T = q.shape[0]
    k, v = cache.dequantized(effective=True)
    L = k.shape[0]
    assert 1 <= T <= L
    return np.stack([attention(q[t], k[:L - T + t + 1], v[:L - T + t + 1], scale) for t in range(T)])


# ---------------------------------------------------------------------------
# Sizes ("KV1-1.2B", Memory; BQ2_0 block = 20 bytes per 64 values)
# ---------------------------------------------------------------------------


def quantized_bytes_per_token(num_kv_heads, head_dim, k_bits, v_bits, group_k, group_v, k_axis=0) -> float:
    """Bytes per cached token over all KV heads of one layer.

    Codes take ``D*(bk+bv)/8`` bytes; each key group (one channel over group_k
    tokens, or group_v channels of one token with per-token keys) and each
    value group (group_v channels of one token) adds an fp16 scale and an
    fp16 zero point, i.e. 4 bytes.
    """
    D = head_dim
    kgroups = D / group_v if k_axis == 1 else D / group_k
    return num_kv_heads * (D * (k_bits + v_bits) / 8 + 4 * kgroups + 4 * D / group_v)
