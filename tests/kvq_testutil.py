"""Helpers shared by the tests: build a cache and its oracle twin from the same
inputs, read packed block records back from the device, compare results."""

from __future__ import annotations

import numpy as np
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KVCache
from oracle import kvq_oracle as O

ATOL = 2e-3       # max-abs error of attention outputs vs the fp64 oracle
RTOL = 1e-2       # max-rel error, relative to max(|ref|, REL_FLOOR)
REL_FLOOR = ATOL / RTOL


def assert_attention_close(out: np.ndarray, ref: np.ndarray, what: str = ""):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref)
    rel = err / np.maximum(np.abs(ref), REL_FLOOR)
    assert err.max() <= ATOL, f"{what}: max abs err {err.max():.3e} > {ATOL}"
    assert rel.max() <= RTOL, f"{what}: max rel err {rel.max():.3e} > {RTOL}"


def ulp(x: np.ndarray, dtype) -> np.ndarray:
    """Spacing of `dtype` (torch.float16 / torch.bfloat16) at |x|."""
    mant = 10 if dtype == torch.float16 else 7
    emin = -14 if dtype == torch.float16 else -126
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** emin)))
    return 2.0 ** (e - mant)


def chunk_swizzle(row: int, n: int) -> int:
    """Chunk-position permutation of the record layout documented in kvq.h."""
    if n <= 1:
        return 0
    if n >= 8:
        return row & 7
    return (row // (8 // n)) % n


def pair_layout(G: int, kb: int) -> bool:
    """32-token blocks with 2-bit keys: channels d and d + 64 share a 16-byte key row."""
    return G == 32 and kb == 2


def vc_row(t: int, G: int, kb: int) -> int:
    if pair_layout(G, kb):
        a, b = divmod(t, 8)
        return 16 * (b // 4) + 8 * ((b // 2) % 2) + 2 * a + b % 2
    c = 16 // kb
    return (t % c) * (G // c) + t // c


def kc_word_index(d: int, w: int, W: int) -> int:
    if W == 2:  # pair layout (head_dim 128)
        return (d % 64) * 4 + (d // 64) * 2 + w
    if W < 4:
        return d * W + w
    return d * W + (((w >> 2) ^ chunk_swizzle(d, W // 4)) << 2) + (w & 3)


def vc_word_index(t: int, w: int, G: int, kb: int, VW: int) -> int:
    r = vc_row(t, G, kb)
    if VW < 4:
        return r * VW + w
    return r * VW + (((w >> 2) ^ chunk_swizzle(r, VW // 4)) << 2) + (w & 3)


def vsz_half_index(t: int, gg: int, G: int, kb: int, ngrp: int, zero: bool) -> int:
    """Half position of the value scale (or zero point) of token t, group gg,
    in a record's vsz array (layout documented in kvq.h)."""
    if pair_layout(G, kb):
        kst, r = divmod(vc_row(t, G, kb), 16)
        entry = (kst * 4 + ((r & 7) >> 1)) * ngrp + gg
        return entry * 8 + (4 if zero else 0) + 2 * (r >> 3) + (r & 1)
    if G < 64:
        return (t * ngrp + gg) * 2 + (1 if zero else 0)
    cpt16, tokc = 16 // kb, 128 // kb
    jp_count = cpt16 // 2
    tile, tt = divmod(t, 64)
    sg, rem = divmod(tt, tokc)
    col, j = divmod(rem, cpt16)
    mt = sg * jp_count + j // 2
    r = col + 8 * (j & 1)
    entry = ((tile * 4 + mt) * 4 + ((r & 7) >> 1)) * ngrp + gg
    return entry * 8 + (4 if zero else 0) + 2 * (r >> 3) + (r & 1)


class Twin:
    """A device cache and one oracle SequenceCache per (layer, sequence)."""

    def __init__(self, cfg: CacheConfig, device="cuda", oracle_seqs=None, oracle_layers=None):
        self.cfg = cfg
        self.gpu = KVCache(cfg, device)
        self.device = device
        self.oracle_seqs = set(range(cfg.max_batch)) if oracle_seqs is None else set(oracle_seqs)
        self.oracle_layers = set(range(cfg.num_layers)) if oracle_layers is None else set(oracle_layers)
        self.ora = {}
        for layer in self.oracle_layers:
            for b in self.oracle_seqs:
                self.ora[(layer, b)] = self._new_oracle(layer)

    def _new_oracle(self, layer):
        cfg = self.cfg
        return O.SequenceCache(cfg.num_kv_heads, cfg.head_dim, cfg.k_bits[layer], cfg.v_bits[layer], cfg.group_k,
                               cfg.group_v, cfg.residual, sinks=cfg.sink_tokens,
                               k_axis=(cfg.k_axis or [0] * cfg.num_layers)[layer], hadamard=bool(cfg.hadamard),
                               residual_v=cfg.residual_v or None)

    def append(self, layer: int, k: torch.Tensor, v: torch.Tensor, new_lens):
        """k, v: [sum(new_lens), Hkv, D] in the cache dtype (any device)."""
        self.gpu.append(layer, k.to(self.device), v.to(self.device), new_lens)
        if layer in self.oracle_layers:
            off = 0
            for b, n in enumerate(new_lens):
                if b in self.oracle_seqs and n > 0:
                    kk = k[off:off + n].float().cpu().numpy()
                    vv = v[off:off + n].float().cpu().numpy()
                    self.ora[(layer, b)].append(kk, vv)
                off += n

    def release_sequence(self, b: int):
        """Empty sequence b in every layer on both sides."""
        self.gpu.release_sequence(b)
        for layer in self.oracle_layers:
            if (layer, b) in self.ora:
                self.ora[(layer, b)] = self._new_oracle(layer)

    def flush_residual(self, layer: int, batch: int):
        self.gpu.flush_residual(layer, batch)
        for b in range(batch):
            if (layer, b) in self.ora:
                self.ora[(layer, b)].flush_residual()

    def check_lengths(self, layer: int, batch: int):
        for b in range(batch):
            if (layer, b) in self.ora:
                o = self.ora[(layer, b)]
                assert self.gpu.lengths(layer, b) == (o.quantized_tokens, o.residual_tokens), (layer, b)
                assert self.gpu.value_lengths(layer, b) == (o.quantized_tokens_v, o.residual_tokens_v), (layer, b)
                assert self.gpu.sinks(layer, b) == o.sink_tokens, (layer, b, "sinks")

    def read_records(self, layer: int, b: int, h: int, nblk: int):
        """Device block records [0, nblk) of (sequence b, KV head h), split into
        parts, with the documented word placement undone (natural order)."""
        lay = self.gpu.layout(layer)
        cfg = self.cfg
        G, D, Gv = cfg.group_k, cfg.head_dim, cfg.group_v
        kb, vb = lay.k_bits, lay.v_bits
        base = lay.blocks - self.gpu.arena.data_ptr()
        if lay.page_blocks:  # paged: record (page * Hkv + h) * P + j % P, page from the device page table
            P = lay.page_blocks
            pt_off = lay.page_table - self.gpu.arena.data_ptr()
            row = self.gpu.arena[pt_off + b * lay.max_pages * 4:pt_off + (b + 1) * lay.max_pages * 4]
            pages = row.cpu().view(torch.int32).numpy()
            recs = [((int(pages[j // P]) * cfg.num_kv_heads + h) * P + j % P) for j in range(nblk)]
            arena = self.gpu.arena
            raw = np.stack([arena[base + r * lay.record_bytes:base + (r + 1) * lay.record_bytes].cpu().numpy()
                            for r in recs]) if nblk else np.zeros((0, lay.record_bytes), np.uint8)
        else:
            start = base + ((b * cfg.num_kv_heads + h) * lay.max_blocks) * lay.record_bytes
            raw = self.gpu.arena[start:start + nblk * lay.record_bytes].cpu().numpy().reshape(nblk, lay.record_bytes)

        def part(off, nbytes, dtype, shape):
            return np.ascontiguousarray(raw[:, off:off + nbytes]).view(dtype).reshape((nblk,) + shape)

        # a record is a run of tiles of TT tokens (tile i at tile0_offset +
        # i * tile_bytes); per-channel key scales of a multi-tile record sit
        # once at rec_ksz_offset
        TT = lay.tile_tokens
        kcw = TT * kb // 32
        vcw = D * vb // 32
        ng = D // Gv
        vidx = np.array([[vc_word_index(t, w, TT, kb, vcw) for w in range(vcw)] for t in range(TT)])
        kidx = np.array([[kc_word_index(d, w, kcw) for w in range(kcw)] for d in range(D)])
        sidx = np.array([[[vsz_half_index(t, gg, TT, kb, ng, z) for z in (False, True)] for gg in range(ng)]
                         for t in range(TT)])
        kc, vc, vsz, ksz = [], [], [], []
        for i in range(G // TT):
            t0 = lay.tile0_offset + i * lay.tile_bytes
            kc.append(part(t0 + lay.kc_offset, kcw * D * 4, np.uint32, (D * kcw,))[:, kidx])  # [n, D, kcw]
            vc.append(part(t0 + lay.vc_offset, TT * vcw * 4, np.uint32, (TT * vcw,))[:, vidx])
            vsz.append(part(t0 + lay.vsz_offset, TT * ng * 4, np.float16, (TT * ng * 2,))[:, sidx])
            if lay.k_axis == 1:  # per-token keys: (scale, zero) pairs [TT][groups] in every tile
                ksz.append(part(t0 + lay.ksz_offset, TT * ng * 4, np.float16, (TT, ng, 2)))
        if lay.k_axis == 1:
            ksz = np.concatenate(ksz, axis=1)
        elif lay.rec_ksz_offset >= 0:
            ksz = part(lay.rec_ksz_offset, D * 4, np.float16, (D, 2))
        else:
            ksz = part(lay.ksz_offset, D * 4, np.float16, (D, 2))
        return {
            "kc": np.concatenate(kc, axis=2),
            "ksz": ksz,
            "vc": np.concatenate(vc, axis=1),
            "vsz": np.concatenate(vsz, axis=1),
        }

    def read_ring(self, layer: int, b: int):
        """(key ring [H, R, D], value ring [H, RV, D]) of sequence b."""
        lay = self.gpu.layout(layer)
        cfg = self.cfg
        out = []
        for ptr, R in ((lay.ring_k, cfg.residual), (lay.ring_v, cfg.residual_v or cfg.residual)):
            n = cfg.num_kv_heads * R * cfg.head_dim * 2
            start = ptr - self.gpu.arena.data_ptr() + b * n
            raw = self.gpu.arena[start:start + n].cpu()
            out.append(raw.view(cfg.kv_dtype).float().numpy().reshape(cfg.num_kv_heads, R, cfg.head_dim))
        return out

    def read_sinks(self, layer: int, b: int):
        lay = self.gpu.layout(layer)
        cfg = self.cfg
        n = cfg.num_kv_heads * 8 * cfg.head_dim * 2  # KVQ_MAX_SINKS rows per (sequence, KV head)
        out = []
        for ptr in (lay.sink_k, lay.sink_v):
            start = ptr - self.gpu.arena.data_ptr() + b * n
            raw = self.gpu.arena[start:start + n].cpu()
            out.append(raw.view(cfg.kv_dtype).float().numpy().reshape(cfg.num_kv_heads, 8, cfg.head_dim))
        return out

    def check_codes(self, layer: int, b: int):
        """Every packed block part and ring token of sequence b equals the
        oracle's, bit for bit (keys and values each up to their own
        quantized length)."""
        o = self.ora[(layer, b)]
        cfg = self.cfg
        kb, vb = cfg.k_bits[layer], cfg.v_bits[layer]
        nk, nv = len(o.key_blocks), len(o.value_blocks)
        nblk = max(nk, nv)
        for h in range(cfg.num_kv_heads):
            if nblk:
                rec = self.read_records(layer, b, h, nblk)
                for j in range(nk):
                    kc, kd, km = o.key_blocks[j]
                    kw = O.pack_key_block(kc, kb)[h]
                    assert np.array_equal(rec["kc"][j], kw), (layer, b, h, j, "key codes")
                    if o.k_axis == 1:
                        assert np.array_equal(rec["ksz"][j][..., 0].view(np.uint16), kd[:, h].view(np.uint16)), (b, h, j, "key scale")
                        assert np.array_equal(rec["ksz"][j][..., 1].view(np.uint16), km[:, h].view(np.uint16)), (b, h, j, "key zero")
                    else:
                        assert np.array_equal(rec["ksz"][j][:, 0].view(np.uint16), kd[h].view(np.uint16)), (b, h, j, "key scale")
                        assert np.array_equal(rec["ksz"][j][:, 1].view(np.uint16), km[h].view(np.uint16)), (b, h, j, "key zero")
                for j in range(nv):
                    vc, vd, vm = o.value_blocks[j]
                    vw = O.pack_value_block(vc, vb)[h]
                    assert np.array_equal(rec["vc"][j], vw), (layer, b, h, j, "value codes")
                    assert np.array_equal(rec["vsz"][j][..., 0].view(np.uint16), vd[:, h].view(np.uint16)), (b, h, j, "value scale")
                    assert np.array_equal(rec["vsz"][j][..., 1].view(np.uint16), vm[:, h].view(np.uint16)), (b, h, j, "value zero")
        if o.sink_tokens:
            sk, sv = self.read_sinks(layer, b)
            for t in range(o.sink_tokens):
                assert np.array_equal(sk[:, t], o.sink_k[t]), (layer, b, t, "sink key")
                assert np.array_equal(sv[:, t], o.sink_v[t]), (layer, b, t, "sink value")
        if o.residual_tokens or o.residual_tokens_v:
            rk, rv = self.read_ring(layer, b)
            R, RV = cfg.residual, cfg.residual_v or cfg.residual
            for t in range(o.residual_tokens):
                assert np.array_equal(rk[:, (o.quantized_tokens + t) % R], o.ring_k[t]), (layer, b, t, "ring key")
            for t in range(o.residual_tokens_v):
                assert np.array_equal(rv[:, (o.quantized_tokens_v + t) % RV], o.ring_v[t]), (layer, b, t, "ring value")

    def check_dequant(self, layer: int, b: int):
        o = self.ora[(layer, b)]
        L = o.length
        k, v = self.gpu.dequant(layer, b, 0, L)
        K, V = o.dequantized()
        assert np.array_equal(k.cpu().numpy(), K), (layer, b, "dequant keys")
        assert np.array_equal(v.cpu().numpy(), V), (layer, b, "dequant values")

    def oracle_decode(self, layer: int, b: int, q_b: np.ndarray, scale: float):
        return O.decode_attention(self.ora[(layer, b)], q_b, scale)
