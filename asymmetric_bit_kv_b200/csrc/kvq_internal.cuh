// Internal definitions shared by the host entry points and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;  // the decode kernels are specialised for D = 128

// Length table of a layer: int32 [max_batch][kLensStride] per sequence --
// quantized keys, key ring tokens, sink tokens, quantized values (token
// positions after the sinks). The value ring holds the tokens from the
// quantized values up to the end: keys + key ring - quantized values.
constexpr int kLensStride = 4;
constexpr int kLenQ = 0, kLenN = 1, kLenS = 2, kLenQV = 3;

// Per-layer view of the packed cache, passed by value to kernels.
struct LayerView {
  uint8_t* blocks;        // block records [max_batch][Hkv][max_blocks], or the page pool (paged)
  void* ring_k;           // [max_batch][Hkv][R][D] kv dtype
  void* ring_v;
  void* sink_k;           // [max_batch][Hkv][KVQ_MAX_SINKS][D] kv dtype (sink_tokens > 0)
  void* sink_v;
  int32_t* lens;          // [max_batch][kLensStride] length table (see kLensStride)
  int64_t record_bytes;
  int64_t max_blocks;
  // A record is a run of tiles of tile_tokens = min(G, 64) tokens: tile part
  // i at tile0_off + i * tile_bytes, laid out [kc | ksz | vc | vsz] with the
  // byte offsets below; with several tiles and per-channel keys, the key
  // scales are stored once, at rec_ksz_off (else rec_ksz_off = -1).
  int32_t kc_off, ksz_off, vc_off, vsz_off;  // byte offsets inside a tile part
  int32_t tile_tokens, tile_bytes, tile0_off, rec_ksz_off;
  int32_t k_bits, v_bits;
  int32_t num_kv_heads, head_dim, group_k, group_v, residual;
  int32_t residual_v;     // value ring slots (= residual unless the cache sets its own)
  int32_t kv_dtype;       // KVQ_F16 / KVQ_BF16
  int32_t sinks;          // S: sink tokens kept exact at the start of each sequence
  int32_t k_axis;         // 0: keys per channel over G tokens (KIVI); 1: per token over group_v channels (BQ2_0)
  int32_t hadamard;       // 1: K and V rotated by the normalized Sylvester matrix before quantization
  const int32_t* page_table;  // paged: [max_batch][max_pages] page of block run j / page_blocks; else null
  int32_t page_blocks;        // paged: blocks per page (a page holds them for every KV head)
  int32_t max_pages;          // paged: page-table entries per sequence
};

__host__ __device__ inline int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// Byte sizes of the four parts of a block record.
__host__ __device__ inline int64_t kc_bytes(int G, int D, int kb) { return (int64_t)G * kb / 32 * D * 4; }
__host__ __device__ inline int64_t ksz_bytes(int D) { return (int64_t)D * 4; }
// Per-token keys: (scale, zero) pairs [G][D/group_v].
__host__ __device__ inline int64_t ksz_token_bytes(int G, int D, int gv) { return (int64_t)G * (D / gv) * 4; }
__host__ __device__ inline int64_t vc_bytes(int G, int D, int vb) { return (int64_t)G * (D * vb / 32) * 4; }
__host__ __device__ inline int64_t vsz_bytes(int G, int D, int gv) { return (int64_t)G * (D / gv) * 4; }

// ---------------------------------------------------------------------------
// Word placement inside a block record. Both code arrays are stored so that a
// straight copy of the record into shared memory can be read with ldmatrix
// without bank conflicts:
//  * a row of n 16-byte chunks stores chunk c at position c ^ swizzle(row, n),
//    where swizzle spreads 8 consecutive rows over 8 distinct 16-byte bank
//    slots;
//  * value rows are stored in "column-major token order": token t of a block
//    sits in row (t % c) * (G / c) + t / c with c = 16 / k_bits, the number of
//    tokens one 16-bit half of a key word holds (the tokens the decode kernel
//    reads together for one n-tile are then 8 consecutive rows).
//  * Pair layout (32-token blocks with 2-bit keys, W = 2 key words per
//    channel): a channel row is 8 bytes, half of a 16-byte ldmatrix row, so
//    channels d and d + 64 share 16-byte row d % 64 (d first); the decode
//    kernel reads both halves with one ldmatrix and keeps them apart in the
//    columns of its B operand. Token t = 8a + b (b < 8) of such a block
//    sits in value row 16 * (b / 4) + 8 * ((b / 2) % 2) + 2a + b % 2: the
//    16-token k-step b / 4 of its P.V product, at the row whose key score the
//    decode kernel finds on M-tile row (a, b % 2) of key M-tile b / 2.
// ---------------------------------------------------------------------------
__host__ __device__ inline bool pair_layout(int G, int kb) { return G == 32 && kb == 2; }
__host__ __device__ inline int chunk_swizzle(int row, int nchunks) {
  if (nchunks <= 1) return 0;
  if (nchunks >= 8) return row & 7;
  return (row / (8 / nchunks)) % nchunks;
}
// Index (in 32-bit words) of word w of channel d inside the key code array
// of a record; W = G * k_bits / 32 words per channel.
__host__ __device__ inline int kc_word_index(int d, int w, int W) {
  if (W == 2) return (d % (kHeadDim / 2)) * 4 + (d / (kHeadDim / 2)) * 2 + w;  // pair layout
  if (W < 4) return d * W + w;
  const int c = w >> 2;
  return d * W + ((c ^ chunk_swizzle(d, W / 4)) << 2) + (w & 3);
}
// Row of token t (0 <= t < G) in the value code array of a record.
__host__ __device__ inline int vc_row(int t, int G, int kb) {
  if (pair_layout(G, kb)) return 16 * ((t >> 2) & 1) + 8 * ((t >> 1) & 1) + 2 * (t >> 3) + (t & 1);
  const int c = 16 / kb;
  return (t % c) * (G / c) + t / c;
}
// Index (in words) of word w of token t inside the value code array; VW =
// D * v_bits / 32 words per token.
__host__ __device__ inline int vc_word_index(int t, int w, int G, int kb, int VW) {
  const int r = vc_row(t, G, kb);
  if (VW < 4) return r * VW + w;
  const int c = w >> 2;
  return r * VW + ((c ^ chunk_swizzle(r, VW / 4)) << 2) + (w & 3);
}

// Position (in 16-bit halves) of the value scale (zero = false) or zero
// point of token t (0 <= t < G) and value group gg inside the vsz array of a
// record. Blocks of G >= 64 tokens keep them in the order the tensor-core
// decode kernel feeds them to its P.V operands, so that a warp reads one
// 16-byte entry per (k-step, lane quad, group) straight from the staged
// record: a 64-token tile has four k-steps of 16 tokens, k-step mt row r
// (0..15) being the token the key path puts on that row (the inverse of its
// tile_token); entry ((tile*4 + mt)*4 + (r%8)/2, group) holds the scales of
// rows 2q, 2q+1, 8+2q, 9+2q, then their zero points. The pair layout keeps
// the same entries for its two 16-token k-steps, k-step and row being
// vc_row(t) / 16 and vc_row(t) % 16. Other blocks keep the plain [G][groups]
// order of (scale, zero) pairs.
__host__ __device__ inline bool vsz_operand_order(int G, int kb) { return G >= 64 || pair_layout(G, kb); }
__host__ __device__ inline int vsz_half_index(int t, int gg, int G, int kb, int ngrp, bool zero) {
  if (pair_layout(G, kb)) {
    const int row = vc_row(t, G, kb), kst = row >> 4, r = row & 15;
    const int entry = (kst * 4 + ((r & 7) >> 1)) * ngrp + gg;
    return entry * 8 + (zero ? 4 : 0) + 2 * (r >> 3) + (r & 1);
  }
  if (G < 64) return (t * ngrp + gg) * 2 + (zero ? 1 : 0);
  const int CPT16 = 16 / kb, TOKC = 128 / kb, JP = CPT16 / 2;
  const int tile = t / 64, tt = t % 64;
  const int sg = tt / TOKC, rem = tt % TOKC;
  const int col = rem / CPT16, j = rem % CPT16;
  const int mt = sg * JP + j / 2;  // key M-tile of the token
  const int r = col + 8 * (j & 1);  // its row in that M-tile
  const int entry = ((tile * 4 + mt) * 4 + ((r & 7) >> 1)) * ngrp + gg;
  return entry * 8 + (zero ? 4 : 0) + 2 * (r >> 3) + (r & 1);
}

// Byte offsets inside a record of token t's data (t < G, the block's own
// token index): its tile part, the word of key codes holding it for channel
// d (word w of a channel covers tokens w*32/k_bits ...), its key (scale,
// zero) pair for channel d, its value word w and its value scale / zero.
__host__ __device__ inline int64_t tile_base(const LayerView& L, int t) {
  return L.tile0_off + (int64_t)(t / L.tile_tokens) * L.tile_bytes;
}
__host__ __device__ inline int64_t kc_word_byte(const LayerView& L, int d, int w) {
  const int wt = L.tile_tokens * L.k_bits / 32;  // key words per channel per tile
  return L.tile0_off + (int64_t)(w / wt) * L.tile_bytes + L.kc_off + 4 * (int64_t)kc_word_index(d, w % wt, wt);
}
__host__ __device__ inline int64_t ksz_pair_byte(const LayerView& L, int t, int d) {
  if (L.k_axis == 0) return (L.rec_ksz_off >= 0 ? L.rec_ksz_off : L.tile0_off + L.ksz_off) + 4 * (int64_t)d;
  return tile_base(L, t) + L.ksz_off + 4 * (int64_t)((t % L.tile_tokens) * (L.head_dim / L.group_v) + d / L.group_v);
}
__host__ __device__ inline int64_t vc_word_byte(const LayerView& L, int t, int w) {
  return tile_base(L, t) + L.vc_off +
         4 * (int64_t)vc_word_index(t % L.tile_tokens, w, L.tile_tokens, L.k_bits, L.head_dim * L.v_bits / 32);
}
__host__ __device__ inline int64_t vsz_half_byte(const LayerView& L, int t, int g, bool zero) {
  return tile_base(L, t) + L.vsz_off +
         2 * (int64_t)vsz_half_index(t % L.tile_tokens, g, L.tile_tokens, L.k_bits, L.head_dim / L.group_v, zero);
}

// Block record j of (sequence b, KV head h): contiguous per (b, h), or in a
// paged cache record (page * Hkv + h) * page_blocks + j % page_blocks.
__device__ __forceinline__ uint8_t* record_ptr(const LayerView& L, int b, int h, int64_t j) {
  if (L.page_table) {
    const int64_t page = __ldg(L.page_table + (int64_t)b * L.max_pages + j / L.page_blocks);
    return L.blocks + ((page * L.num_kv_heads + h) * L.page_blocks + j % L.page_blocks) * L.record_bytes;
  }
  return L.blocks + (((int64_t)b * L.num_kv_heads + h) * L.max_blocks + j) * L.record_bytes;
}

__device__ __forceinline__ float load_kv(const void* p, int64_t i, int dtype) {
  if (dtype == KVQ_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(reinterpret_cast<const __half*>(p)[i]);
}

// x . H for the 128 channels of one head spread over a warp, channels 4l..4l+3
// in lane l: radix-2 butterflies of half-width 1, 2, 4, ..., 64 (the first two
// inside the lane, the others with the lane at xor distance w/4), then one
// fp32 multiplication by fp32(1/sqrt(128)). The quantizer rotates the keys
// and values and the decode kernel the queries and outputs in this order.
__device__ __forceinline__ void rotate_lane(float (&x)[4], int lane) {
  float a = x[0], c = x[1];
  x[0] = __fadd_rn(a, c);
  x[1] = __fsub_rn(a, c);
  a = x[2], c = x[3];
  x[2] = __fadd_rn(a, c);
  x[3] = __fsub_rn(a, c);
  a = x[0], c = x[2];
  x[0] = __fadd_rn(a, c);
  x[2] = __fsub_rn(a, c);
  a = x[1], c = x[3];
  x[1] = __fadd_rn(a, c);
  x[3] = __fsub_rn(a, c);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const bool upper = lane & o;  // this lane holds the x[i + w] side of its pairs
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, x[e], o);
      x[e] = upper ? __fsub_rn(other, x[e]) : __fadd_rn(x[e], other);
    }
  }
  const float s = (float)(1.0 / sqrt((double)kHeadDim));
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = __fmul_rn(x[e], s);
}

// ---------------------------------------------------------------------------
// The quantizer of the "KV1-1.2B" card (section "Quantization Format: KV1.cpp
// BQ2_0"), widened from 3 to 2^b - 1 levels. Every operation is an explicitly
// rounded fp32 intrinsic so the compiler cannot contract or reassociate it;
// codes, scales and zero points are therefore reproducible bit for bit.
// ---------------------------------------------------------------------------
struct GroupParams {
  __half d16, m16;
  float d, m;  // fp32 copies of the fp16 values, used for the codes
};

__device__ __forceinline__ GroupParams group_params(float mn, float mx, int bits) {
  const float qmax = (float)((1 << bits) - 1);
  const float d = __fdiv_rn(__fsub_rn(mx, mn), qmax);
  GroupParams g;
  g.d16 = __float2half_rn(fmaxf(d, 1e-6f));
  g.m16 = __float2half_rn(__fadd_rn(mn, 0.0f));  // -0.0 min is stored as +0.0
  g.d = __half2float(g.d16);
  g.m = __half2float(g.m16);
  return g;
}

__device__ __forceinline__ uint32_t quant_code(float x, const GroupParams& g, int bits) {
  const float t = __fdiv_rn(__fsub_rn(x, g.m), g.d);
  const float r = fminf(fmaxf(rintf(t), 0.0f), (float)((1 << bits) - 1));  // rint: ties to even
  return (uint32_t)r;
}

// The same code with one multiplication instead of a division: r is 1/d
// rounded to nearest (__frcp_rn, once per group). With a = fl(x - m), the
// product t = fl(a * r) and the quotient fl(a / d) both lie within a
// relative 2^-24 per rounding of a/d (two roundings for t, one for the
// quotient), so they differ by less than |t| * 2^-22. Hence whenever t is
// farther than |t| * 2^-21 from its nearest half-integer (which keeps every
// other half-integer at least 0.5 away) both lie strictly inside the same
// rounding interval and rint(t) = rint(quotient); inside that window (and
// always for |t| >= 2^21) the quotient itself is computed. rint(t) comes
// from one fp32 addition: for |t| < 2^22, t + 1.5 * 2^23 lies in [2^23,
// 2^24), where the spacing is 1, so the sum is rounded to an integer with
// ties to even and its bits minus those of 1.5 * 2^23 are rint(t); e = t -
// rint(t) is exact (Sterbenz), and 0.5 - |e| is the distance to the nearest
// half-integer (exact when it matters, |e| >= 1/4). Only FMA- and ALU-pipe
// instructions on the common path. Bit-exact with quant_code.
__device__ __forceinline__ uint32_t quant_code_rcp(float x, float m, float d, float r, int bits) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float a = __fsub_rn(x, m);
  const float t = __fmul_rn(a, r);
  const float tm = __fadd_rn(t, kRound);
  const float e = __fsub_rn(t, __fsub_rn(tm, kRound));
  int k;
  if (__fsub_rn(0.5f, fabsf(e)) <= fabsf(t) * 0x1p-21f) {
    k = (int)fminf(fmaxf(rintf(__fdiv_rn(a, d)), 0.0f), (float)((1 << bits) - 1));  // rint: ties to even
  } else {
    k = __float_as_int(tm) - __float_as_int(kRound);
  }
  return (uint32_t)min(max(k, 0), (1 << bits) - 1);
}

// A word of N = 32/BITS codes of one group with the reasoning of
// quant_code_rcp, but one branch per word: t is first clamped to
// [-0.49, qmax + 0.49] (every t outside lies beyond a boundary half-integer
// whose both sides clamp to the same code, 0 or qmax, so the code is
// unchanged), which bounds |t| <= qmax + 0.49 and lets one constant
// threshold, (qmax + 0.5) * 2^-21 >= |t| * 2^-21, serve every value: if any
// value of the word falls within it of a half-integer, the whole word is
// recomputed from the exact quotients.
//
// Packing: the bit pattern of tm is that of 1.5 * 2^23 (0x4B400000) plus the
// code, so the word is the sum of the patterns, each shifted to its field
// (one shift-add per code), minus the sum of the constant's shifted copies,
// all modulo 2^32.
template <int BITS, int N>
__host__ __device__ constexpr uint32_t round_bias() {
  uint32_t s = 0;
  for (int i = 0; i < N; ++i) s += 0x4B400000u << (i * BITS);
  return s;
}
// x(i) gives value i of the word (an fp32 conversion of a staged value,
// evaluated where it is used, so only the raw values stay in registers).
template <int BITS, int N, class X>
__device__ __forceinline__ uint32_t quant_word_rcp_fn(X x, float m, float d, float r) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23, bit pattern 0x4B400000
  constexpr int qmax = (1 << BITS) - 1;
  constexpr float lo = -0.49f, hi = (float)qmax + 0.49f;
  constexpr float near = 0.5f - ((float)qmax + 0.5f) * 0x1p-21f;  // |e| above this: within the window
  uint32_t acc = 0;
  float emax = 0.0f;  // the largest |e| of the word
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float t = fminf(fmaxf(__fmul_rn(__fsub_rn(x(i), m), r), lo), hi);
    const float tm = __fadd_rn(t, kRound);
    const float e = __fsub_rn(t, __fsub_rn(tm, kRound));
    emax = fmaxf(emax, fabsf(e));
    acc += __float_as_uint(tm) << (i * BITS);
  }
  uint32_t word = acc - round_bias<BITS, N>();
  if (emax > near) {
    word = 0;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const float q = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x(i), m), d)), 0.0f), (float)qmax);  // ties to even
      word |= (uint32_t)q << (i * BITS);
    }
  }
  return word;
}
template <int BITS, int N>
__device__ __forceinline__ uint32_t quant_word_rcp(const float (&x)[N], float m, float d, float r) {
  return quant_word_rcp_fn<BITS, N>([&](int i) { return x[i]; }, m, d, r);
}

// x_hat = q * d + m with two roundings (no fused multiply-add).
__device__ __forceinline__ float dequant_value(uint32_t q, __half d16, __half m16) {
  return __fadd_rn(__fmul_rn((float)q, __half2float(d16)), __half2float(m16));
}

}  // namespace kvq
