// Append / flush / dequantize kernels.
//
// Method: "KIVI" README, sections "Overview" and "Example" (keys per channel,
// values per token, residual window of recent full-precision tokens), the
// quantizer of the "KV1-1.2B" card, section "Quantization Format: KV1.cpp
// BQ2_0", and per-tensor residual windows ("Quantize What Counts", KV Cache
// Quantization: residual_length {k, v}).
//
// One CTA of kQuantThreads threads quantizes one G-token key block and/or one
// G-token value block of one (sequence, KV head). The G x D rows are staged in
// shared memory with 16-byte loads (all of a thread's loads issued before any
// store). Per-channel keys: every thread takes one channel pair and a slice of
// 32/k_bits tokens (one output word per channel), reduces min/max over its
// slice, the slices of a channel are combined through shared memory, and the
// same thread then packs the slice's codes -- so G*D values are spread over
// D/2 * G*k_bits/32 threads instead of one thread per channel. Values (and the
// scales of per-token keys): one thread per output word of 32/v_bits channels
// of a token, the min/max of a group combined with __shfl_xor. Codes use
// IEEE-rounded fp32 arithmetic (__fsub_rn, __fdiv_rn, rintf), bit-exact with
// the oracle.
#include <algorithm>

#include "kvq_append.cuh"
#include "kvq_decode.cuh"

namespace kvq {

namespace {

// fp32 value (exact) of a 16-bit storage word of kv dtype DT, and of the low
// and high element of a packed pair of them.
template <int DT>
__device__ __forceinline__ float f32_of(uint32_t v) {
  if constexpr (DT == KVQ_BF16) return __uint_as_float(v << 16);
  else return __half2float(__ushort_as_half((unsigned short)v));
}
template <int DT>
__device__ __forceinline__ float f32_lo(uint32_t p) {
  return f32_of<DT>(p & 0xffffu);
}
template <int DT>
__device__ __forceinline__ float f32_hi(uint32_t p) {
  if constexpr (DT == KVQ_BF16) return __uint_as_float(p & 0xffff0000u);
  else return __half2float(__ushort_as_half((unsigned short)(p >> 16)));
}

// Elementwise min / max of two packed pairs of kv-dtype values. Min and max
// are exact in any format, so these equal the fp32 min / max of the
// conversions (up to the sign of a zero, on which no group parameter
// depends: the zero point is min + 0, the scale a difference); one
// instruction per two values.
template <int DT>
__device__ __forceinline__ uint32_t pair_min(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (DT == KVQ_BF16) {
    const __nv_bfloat162 v = __hmin2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                     *reinterpret_cast<const __nv_bfloat162*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  } else {
    const __half2 v = __hmin2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  }
  return r;
}
template <int DT>
__device__ __forceinline__ uint32_t pair_max(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (DT == KVQ_BF16) {
    const __nv_bfloat162 v = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                     *reinterpret_cast<const __nv_bfloat162*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  } else {
    const __half2 v = __hmax2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  }
  return r;
}

// Where row t (0 <= t < G) of a block comes from: the ring (positions before
// `boundary`) or this call's input (row in_row0 + position - boundary).
struct BlockRows {
  const uint16_t* ring;  // ring of (b, h): [R][D]
  const uint16_t* in;    // input [rows][Hkv][D] (null: ring only)
  int64_t in_row0;
  int32_t first;         // position of the block's first token
  int32_t boundary;
  int32_t R, Hkv, h;
  __device__ __forceinline__ const uint16_t* row(int t) const {
    const int i = first + t;
    if (i < boundary) return ring + (int64_t)(i % R) * kHeadDim;
    return in + ((in_row0 + (i - boundary)) * Hkv + h) * kHeadDim;
  }
};

// One CTA quantizes one part of one tensor of a G-token block: per-channel
// keys split by channels (the min/max of a channel runs over all G tokens),
// values and per-token keys split by tokens. The fused step's flush uses
// kStepKeyParts + kStepValueParts CTAs per block (its grid is only batch x
// Hkv blocks); appends use one per tensor.
// (one key CTA and two value CTAs per block: 768 CTAs for 32 x 8 blocks, one
// wave at the kernel's 6 CTAs per SM; two key parts, a second wave, measured
// no faster)
constexpr int kStepKeyParts = 1, kStepValueParts = 2;

struct PartShape {
  bool key;
  int t0, nt;  // staged tokens [t0, t0 + nt) of the block
  int c0, nc;  // quantized channels [c0, c0 + nc) (per-channel keys; else all)
  int sc0, snc;  // staged channels (the rotation needs whole rows)
};
__host__ __device__ inline PartShape part_shape(bool key, int part, int parts, int G, int k_axis, bool rot) {
  PartShape s;
  s.key = key;
  if (key && k_axis == 0) {
    s.t0 = 0, s.nt = G;
    s.nc = kHeadDim / parts, s.c0 = part * s.nc;
  } else {
    s.nt = G / parts, s.t0 = part * s.nt;
    s.c0 = 0, s.nc = kHeadDim;
  }
  s.sc0 = rot ? 0 : s.c0;
  s.snc = rot ? kHeadDim : s.nc;
  return s;
}

// Shared memory of one part CTA (bytes): staged rows [nt][snc] (raw 16-bit,
// or fp32 when rotated), then per-channel keys' slice min/max float2
// [W][nc], then the key groups' fp32 (scale, zero, 1/scale) float4.
struct QuantSmem {
  int rows, red, kpar, total;
};
__host__ __device__ inline QuantSmem part_smem(const PartShape& s, int G, int kb, int gv, int k_axis, bool rot) {
  QuantSmem q;
  q.rows = s.nt * s.snc * (rot ? 4 : 2);
  q.red = (s.key && k_axis == 0) ? (G * kb / 32) * s.nc * 8 : 0;
  q.kpar = !s.key ? 0 : (k_axis == 0 ? s.nc : s.nt * (kHeadDim / gv)) * 16;
  q.total = q.rows + q.red + q.kpar;
  return q;
}
// The largest over the part CTAs of a launch with `parts` parts per tensor.
__host__ __device__ inline int quant_smem_bytes(int G, int kb, int gv, int k_axis, bool rot, int parts) {
  const int a = part_smem(part_shape(true, 0, parts, G, k_axis, rot), G, kb, gv, k_axis, rot).total;
  const int b = part_smem(part_shape(false, 0, parts, G, k_axis, rot), G, kb, gv, k_axis, rot).total;
  return a > b ? a : b;
}

// Stages rows t0 .. t0+nt-1, channels c0 .. c0+nc-1 of a block as raw
// 16-bit values ([nt][nc]) with 16-byte loads. A row has nc/8 chunks (a
// power of two, at most 16, dividing kQuantThreads): each thread keeps one
// chunk column and walks the rows kQuantThreads/(nc/8) apart, four loads in
// flight before their stores (no division per chunk).
__device__ __forceinline__ void stage_raw(const BlockRows& src, int t0, int nt, int c0, int nc, uint16_t* dst) {
  const int lg = __ffs(nc >> 3) - 1;  // log2 of the chunks per row
  const int col = (threadIdx.x & ((1 << lg) - 1)) * 8;
  const int rstep = kQuantThreads >> lg;
  for (int r = threadIdx.x >> lg; r < nt; r += 4 * rstep) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (r + u * rstep < nt) v[u] = *reinterpret_cast<const uint4*>(src.row(t0 + r + u * rstep) + c0 + col);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (r + u * rstep < nt) *reinterpret_cast<uint4*>(dst + (r + u * rstep) * nc + col) = v[u];
  }
}

// Stages rows t0 .. t0+nt-1 rotated (x . H, rotate_lane) as fp32 [nt][D]:
// one warp per row.
template <int DT>
__device__ __forceinline__ void stage_rotated(const BlockRows& src, int t0, int nt, float* dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < nt; t += kQuantThreads / 32) {
    const uint2 raw = *reinterpret_cast<const uint2*>(src.row(t0 + t) + 4 * lane);
    float x[4] = {f32_lo<DT>(raw.x), f32_hi<DT>(raw.x), f32_lo<DT>(raw.y), f32_hi<DT>(raw.y)};
    rotate_lane(x, lane);
    *reinterpret_cast<float4*>(dst + t * kHeadDim + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
  }
}

// Raw packed pairs of channels c .. c+N-1 (N >= 4) of staged 16-bit row t
// (rows of `pitch` channels): N/2 words, 16-byte (N = 4: 8-byte) loads.
template <int N>
__device__ __forceinline__ void row_pairs(const uint8_t* rows, int pitch, int t, int c, uint32_t (&p)[N / 2]) {
  const uint16_t* r = reinterpret_cast<const uint16_t*>(rows) + t * pitch + c;
  if constexpr (N >= 8) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
      const uint4 q = reinterpret_cast<const uint4*>(r)[i];
      p[4 * i] = q.x, p[4 * i + 1] = q.y, p[4 * i + 2] = q.z, p[4 * i + 3] = q.w;
    }
  } else {
    const uint2 q = *reinterpret_cast<const uint2*>(r);
    p[0] = q.x, p[1] = q.y;
  }
}

// Values x[0..N) of channels c .. c+N-1 of staged row t (rows of `pitch`
// channels): fp32 rows when rotated, raw kv-dtype rows otherwise.
template <bool ROT, int DT, int N>
__device__ __forceinline__ void row_values(const uint8_t* rows, int pitch, int t, int c, float (&x)[N]) {
  if constexpr (ROT) {
    const float4* f = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(rows) + t * pitch + c);
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 q = f[i];
      x[4 * i] = q.x, x[4 * i + 1] = q.y, x[4 * i + 2] = q.z, x[4 * i + 3] = q.w;
    }
  } else {
    uint32_t p[N / 2];
    row_pairs<N>(rows, pitch, t, c, p);
#pragma unroll
    for (int i = 0; i < N / 2; ++i) x[2 * i] = f32_lo<DT>(p[i]), x[2 * i + 1] = f32_hi<DT>(p[i]);
  }
}

// One staged value: row t, column c (rows of `pitch` channels).
template <bool ROT, int DT>
__device__ __forceinline__ float staged(const uint8_t* rows, int pitch, int t, int c) {
  if constexpr (ROT) return reinterpret_cast<const float*>(rows)[t * pitch + c];
  else return f32_of<DT>(reinterpret_cast<const uint16_t*>(rows)[t * pitch + c]);
}

// Word index of word w of channel d in a record's key code array (the
// kc_word_index placement) with W = 2^lgW words per channel.
__device__ __forceinline__ int kc_index_p2(int d, int w, int lgW) {
  const int W = 1 << lgW;
  if (lgW == 1) return ((d & (kHeadDim / 2 - 1)) << 2) + ((d / (kHeadDim / 2)) << 1) + w;  // pair layout
  if (lgW < 2) return (d << lgW) + w;
  const int lgn = lgW - 2;  // 16-byte chunks per row: 2^lgn
  const int sw = lgn >= 3 ? (d & 7) : ((d >> (3 - lgn)) & ((1 << lgn) - 1));
  return d * W + ((((w >> 2) ^ sw)) << 2) + (w & 3);
}

// Where a block's parts go inside its record (the tile layout of
// LayerView: tiles of 2^lgT tokens at tile0 + i * tile_bytes).
struct RecOut {
  uint8_t* rec;
  int lgT, tile_bytes, tile0, kc_off, ksz_off, vc_off, vsz_off, rec_ksz;
  __device__ __forceinline__ uint8_t* tile(int t) const { return rec + tile0 + (int64_t)(t >> lgT) * tile_bytes; }
  __device__ __forceinline__ int local(int t) const { return t & ((1 << lgT) - 1); }
};
__device__ __forceinline__ RecOut rec_out(const LayerView& L, uint8_t* rec) {
  return RecOut{rec,         __ffs(L.tile_tokens) - 1, L.tile_bytes, L.tile0_off, L.kc_off,
                L.ksz_off,   L.vc_off,                 L.vsz_off,    L.rec_ksz_off};
}

// Groups of gv channels of staged rows [0, nt) (tokens t0 + row), BITS-wide
// codes: one thread per output word (PER = 32/BITS channels); the gv/PER
// threads of a group combine their min/max with xor shuffles. put_word(t, w,
// word) and put_sz(t, g, params) receive the results (t: token of the block).
// Raw rows take their min/max on packed pairs and convert to fp32 only for
// the codes.
template <bool ROT, int DT, int BITS, bool CODES, class PutWord, class PutSz>
__device__ __forceinline__ void quantize_token_groups(const uint8_t* rows, int t0, int nt, int gv, PutWord put_word,
                                                      PutSz put_sz) {
  constexpr int PER = 32 / BITS;
  constexpr int WPT = kHeadDim / PER;  // words per row
  const int P = gv / PER;              // threads per group: a power of two, <= 32, dividing WPT
  const int lgP = __ffs(P) - 1;
  for (int item = threadIdx.x; item < nt * WPT; item += kQuantThreads) {
    const int t = item / WPT, w = item % WPT;
    float x[PER];        // rotated rows: the values
    uint32_t pr[PER / 2];  // raw rows: the packed pairs
    float mn, mx;
    if constexpr (ROT) {
      row_values<true, DT, PER>(rows, kHeadDim, t, w * PER, x);
      mn = x[0], mx = x[0];
#pragma unroll
      for (int i = 1; i < PER; ++i) {
        mn = fminf(mn, x[i]);
        mx = fmaxf(mx, x[i]);
      }
    } else {
      row_pairs<PER>(rows, kHeadDim, t, w * PER, pr);
      uint32_t lo = pr[0], hi = pr[0];
#pragma unroll
      for (int i = 1; i < PER / 2; ++i) {
        lo = pair_min<DT>(lo, pr[i]);
        hi = pair_max<DT>(hi, pr[i]);
      }
      mn = fminf(f32_lo<DT>(lo), f32_hi<DT>(lo));
      mx = fmaxf(f32_lo<DT>(hi), f32_hi<DT>(hi));
    }
    for (int o = P / 2; o >= 1; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const GroupParams gp = group_params(mn, mx, BITS);
    if constexpr (CODES) {
      const float r = __frcp_rn(gp.d);
      uint32_t word;
      if constexpr (ROT) word = quant_word_rcp<BITS, PER>(x, gp.m, gp.d, r);
      else
        word = quant_word_rcp_fn<BITS, PER>(
            [&](int i) { return (i & 1) ? f32_hi<DT>(pr[i >> 1]) : f32_lo<DT>(pr[i >> 1]); }, gp.m, gp.d, r);
      put_word(t0 + t, w, word);
    }
    if ((w & (P - 1)) == 0) put_sz(t0 + t, w >> lgP, gp);
  }
}

// Key codes packed along the token axis (kc layout, per tile) for channels [c0, c0+nc)
// and token words [w0, w0 + nw): thread item (channel d, word w) packs
// tokens w*PER .. w*PER+PER-1 of channel d (staged row of token t at t - t0,
// column d - sc0) with the fp32 (scale, zero, 1/scale) par(t, d).
template <bool ROT, int DT, int KB, bool PT, class Par>
__device__ __forceinline__ void pack_key_codes(const uint8_t* rows, int pitch, int t0, int sc0, int c0, int nc, int w0,
                                               int nw, const RecOut& ro, Par par) {
  constexpr int LGPER = KB == 2 ? 4 : KB == 4 ? 3 : 2;  // log2 of the tokens per word
  const int lgWt = ro.lgT - LGPER;                        // log2 of the words per channel per tile
  constexpr int PER = 32 / KB;
  const int lgnc = __ffs(nc) - 1;  // nc: a power of two
  for (int item = threadIdx.x; item < nc * nw; item += kQuantThreads) {
    const int d = c0 + (item & (nc - 1)), w = w0 + (item >> lgnc);
    float x[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) x[i] = staged<ROT, DT>(rows, pitch, w * PER + i - t0, d - sc0);
    uint32_t word;
    if constexpr (PT) {  // per-token keys: each token has its own (scale, zero)
      word = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const float4 pr = par(w * PER + i, d);
        float xi[1] = {x[i]};
        word |= quant_word_rcp<KB, 1>(xi, pr.y, pr.x, pr.z) << (i * KB);
      }
    } else {  // per-channel keys: one (scale, zero) for the channel
      const float4 pr = par(0, d);
      word = quant_word_rcp<KB, PER>(x, pr.y, pr.x, pr.z);
    }
    uint8_t* tp = ro.tile(w << LGPER);
    reinterpret_cast<uint32_t*>(tp + ro.kc_off)[kc_index_p2(d, w & ((1 << lgWt) - 1), lgWt)] = word;
  }
}

// Keys per channel (KIVI): channels [c0, c0 + nc) over all G tokens; the
// min/max of every (channels, token word) item, combined through shared
// memory, then the codes (one channel and token word per thread item). Raw
// rows hold exactly the part's channels (sc0 = c0, snc = nc): a min/max
// item is a channel pair, one 32-bit word per staged row, reduced on packed
// pairs. Rotated rows (fp32, all channels staged) take one channel per
// item.
template <bool ROT, int DT, int KB>
__device__ __forceinline__ void quantize_key_channels(const uint8_t* rows, const PartShape& s, int G, const RecOut& ro,
                                                      float2* red, float4* kpar) {
  constexpr int PER = 32 / KB;
  const int W = G / PER;
  const int np = s.nc / 2;  // channel pairs (raw rows: 32-bit words per staged row)
  const int lgnc = __ffs(s.nc) - 1, lgnp = lgnc - 1;  // nc: a power of two
  const uint32_t* r32 = reinterpret_cast<const uint32_t*>(rows);
  if constexpr (ROT) {
    for (int item = threadIdx.x; item < s.nc * W; item += kQuantThreads) {
      const int dl = item & (s.nc - 1), w = item >> lgnc;
      const int col = s.c0 + dl - s.sc0;
      float mn = staged<ROT, DT>(rows, s.snc, w * PER, col), mx = mn;
#pragma unroll 4
      for (int i = 1; i < PER; ++i) {
        const float x = staged<ROT, DT>(rows, s.snc, w * PER + i, col);
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
      red[w * s.nc + dl] = make_float2(mn, mx);
    }
  } else {
    for (int item = threadIdx.x; item < np * W; item += kQuantThreads) {
      const int cp = item & (np - 1), w = item >> lgnp;
      const uint32_t* col = r32 + w * PER * np + cp;
      uint32_t lo = col[0], hi = lo;
#pragma unroll
      for (int i = 1; i < PER; ++i) {
        const uint32_t v = col[i * np];
        lo = pair_min<DT>(lo, v);
        hi = pair_max<DT>(hi, v);
      }
      red[w * s.nc + 2 * cp] = make_float2(f32_lo<DT>(lo), f32_lo<DT>(hi));
      red[w * s.nc + 2 * cp + 1] = make_float2(f32_hi<DT>(lo), f32_hi<DT>(hi));
    }
  }
  __syncthreads();
  __half2* ksz = reinterpret_cast<__half2*>(ro.rec_ksz >= 0 ? ro.rec + ro.rec_ksz : ro.rec + ro.tile0 + ro.ksz_off);
  for (int dl = threadIdx.x; dl < s.nc; dl += kQuantThreads) {
    float mn = INFINITY, mx = -INFINITY;
    for (int w = 0; w < W; ++w) {
      const float2 r = red[w * s.nc + dl];
      mn = fminf(mn, r.x);
      mx = fmaxf(mx, r.y);
    }
    const GroupParams gp = group_params(mn, mx, KB);
    ksz[s.c0 + dl] = __halves2half2(gp.d16, gp.m16);
    kpar[dl] = make_float4(gp.d, gp.m, __frcp_rn(gp.d), 0.f);
  }
  __syncthreads();
  pack_key_codes<ROT, DT, KB, false>(rows, s.snc, 0, s.sc0, s.c0, s.nc, 0, W, ro,
                                     [&](int, int d) { return kpar[d - s.c0]; });
}

// Keys per token over group_v channels (BQ2_0), tokens [t0, t0 + nt): the
// token groups' scales and zero points, then the codes of those tokens
// packed along the token axis.
template <bool ROT, int DT, int KB>
__device__ __forceinline__ void quantize_key_tokens(const uint8_t* rows, const PartShape& s, const RecOut& ro, int gv,
                                                    float4* kpar) {
  constexpr int PER = 32 / KB;
  const int ng = kHeadDim / gv;
  quantize_token_groups<ROT, DT, KB, false>(rows, s.t0, s.nt, gv, [](int, int, uint32_t) {},
                                            [&](int t, int g, const GroupParams& gp) {
                                              reinterpret_cast<__half2*>(ro.tile(t) + ro.ksz_off)[ro.local(t) * ng + g] =
                                                  __halves2half2(gp.d16, gp.m16);
                                              kpar[(t - s.t0) * ng + g] = make_float4(gp.d, gp.m, __frcp_rn(gp.d), 0.f);
                                            });
  __syncthreads();
  pack_key_codes<ROT, DT, KB, true>(rows, kHeadDim, s.t0, 0, 0, kHeadDim, s.t0 / PER, s.nt / PER, ro,
                                    [&](int t, int d) { return kpar[(t - s.t0) * ng + d / gv]; });
}

// Values per token over group_v channels (KIVI), tokens [t0, t0 + nt),
// codes packed along head_dim.
template <bool ROT, int DT, int KB, int VB>
__device__ __forceinline__ void quantize_value_tokens(const uint8_t* rows, const PartShape& s, const RecOut& ro,
                                                      int gv) {
  const int ng = kHeadDim / gv, T = 1 << ro.lgT;
  constexpr int VW = kHeadDim * VB / 32;
  quantize_token_groups<ROT, DT, VB, true>(
      rows, s.t0, s.nt, gv,
      [&](int t, int w, uint32_t word) {
        reinterpret_cast<uint32_t*>(ro.tile(t) + ro.vc_off)[vc_word_index(ro.local(t), w, T, KB, VW)] = word;
      },
      [&](int t, int g, const GroupParams& gp) {
        __half* vsz = reinterpret_cast<__half*>(ro.tile(t) + ro.vsz_off);
        vsz[vsz_half_index(ro.local(t), g, T, KB, ng, false)] = gp.d16;
        vsz[vsz_half_index(ro.local(t), g, T, KB, ng, true)] = gp.m16;
      });
}

// One part CTA: stages its rows, then quantizes keys (record jk) or values
// (record jv). ROT: the rows are multiplied by the normalized Sylvester
// Hadamard matrix first (rotate_lane: radix-2 butterflies of half-width 1,
// 2, 4, ..., then one fp32 multiply by fp32(1/sqrt(D)); "KV1-1.2B" card,
// BQ2_0). DT: the kv dtype of the rows.
template <bool ROT, int DT, int KB>
__device__ __forceinline__ void quantize_key_part(const LayerView& L, int b, int h, int64_t jk, const BlockRows& src,
                                                  const PartShape& s, uint8_t* smem) {
  const int G = L.group_k;
  const QuantSmem sm = part_smem(s, G, KB, L.group_v, L.k_axis, ROT);
  if constexpr (ROT) stage_rotated<DT>(src, s.t0, s.nt, reinterpret_cast<float*>(smem));
  else stage_raw(src, s.t0, s.nt, s.sc0, s.snc, reinterpret_cast<uint16_t*>(smem));
  __syncthreads();
  const RecOut ro = rec_out(L, record_ptr(L, b, h, jk));
  float4* kpar = reinterpret_cast<float4*>(smem + sm.rows + sm.red);
  if (L.k_axis == 0) quantize_key_channels<ROT, DT, KB>(smem, s, G, ro, reinterpret_cast<float2*>(smem + sm.rows), kpar);
  else quantize_key_tokens<ROT, DT, KB>(smem, s, ro, L.group_v, kpar);
}

template <bool ROT, int DT, int KB, int VB>
__device__ __forceinline__ void quantize_value_part(const LayerView& L, int b, int h, int64_t jv, const BlockRows& src,
                                                    const PartShape& s, uint8_t* smem) {
  if constexpr (ROT) stage_rotated<DT>(src, s.t0, s.nt, reinterpret_cast<float*>(smem));
  else stage_raw(src, s.t0, s.nt, 0, kHeadDim, reinterpret_cast<uint16_t*>(smem));
  __syncthreads();
  quantize_value_tokens<ROT, DT, KB, VB>(smem, s, rec_out(L, record_ptr(L, b, h, jv)), L.group_v);
}

// Part `part` of `parts` of the key block jk (key) or the value block jv of
// (sequence b, KV head h), rows from src. The kernels are instantiated per
// rotation, kv dtype and bit widths: one kernel holding both dtypes' paths
// needed more than the 42 registers of 6 CTAs per SM, and one holding every
// bit-width pair spent its short flush launches waiting for instruction
// fetch.
template <bool ROT, int DT, int KB, int VB>
__device__ __forceinline__ void quantize_part(const LayerView& L, int b, int h, bool key, int part, int parts,
                                              int64_t j, const BlockRows& src, uint8_t* smem) {
  const PartShape s = part_shape(key, part, parts, L.group_k, L.k_axis, ROT);
  if (key) quantize_key_part<ROT, DT, KB>(L, b, h, j, src, s, smem);
  else quantize_value_part<ROT, DT, KB, VB>(L, b, h, j, src, s, smem);
}

}  // namespace

cudaError_t opt_in_max_smem(const void* kernel, uint64_t& done_mask);

// grid (max flush blocks * 2 * p.parts, batch, Hkv); block kQuantThreads;
// dynamic smem quant_smem_bytes(..., p.parts). x = (2j + tensor) * parts +
// part: key block j of sequence b covers positions q_old[b] + j*G .., value
// block j positions qv_old[b] + j*G ..: ring tokens before the call's first
// new token, this call's input after; part of parts: a slice of its
// channels (per-channel keys) or tokens (otherwise).
template <bool ROT, int DT, int KB, int VB>
__global__ void __launch_bounds__(kQuantThreads, 6) quantize_blocks_kernel(AppendParams p) {
  const int part = blockIdx.x % p.parts, x = blockIdx.x / p.parts;
  const int j = x >> 1, b = blockIdx.y, h = blockIdx.z;
  const bool key = (x & 1) == 0;
  if (j >= (key ? p.flush[b] : p.flush_v[b])) return;
  extern __shared__ __align__(16) uint8_t smem_q[];
  const LayerView& L = p.L;
  const int G = L.group_k;
  const int64_t unit = (int64_t)b * L.num_kv_heads + h;
  const int R = key ? L.residual : L.residual_v;
  const BlockRows src{reinterpret_cast<const uint16_t*>(key ? L.ring_k : L.ring_v) + unit * R * kHeadDim,
                      reinterpret_cast<const uint16_t*>(key ? p.k_in : p.v_in), p.in_off[b],
                      (key ? p.q_old[b] : p.qv_old[b]) + j * G, p.len_old[b], R, L.num_kv_heads, h};
  quantize_part<ROT, DT, KB, VB>(L, b, h, key, part, p.parts, (key ? p.q_old[b] : p.qv_old[b]) / G + j, src,
                                 smem_q);
}

// grid (batch * Hkv * (kStepKeyParts + kStepValueParts)); block
// kQuantThreads. The flush of a fused decode step: for (sequence, KV head)
// whose ring holds R tokens, the oldest G ring tokens become the next block
// record (one ring shared by keys and values); CTA x of unit x / parts takes
// key part x % parts if below kStepKeyParts, else a value part. The
// decode launch that follows is its programmatic dependent and waits for it
// (griddepcontrol.wait) before reading records; the decode kernel records
// the new lengths.
template <bool ROT, int DT, int KB, int VB>
__global__ void __launch_bounds__(kQuantThreads, 6) step_flush_kernel(FlushParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) uint8_t smem_q[];
  const LayerView& L = p.L;
  constexpr int parts = kStepKeyParts + kStepValueParts;
  const int xp = blockIdx.x % parts;
  const bool key = xp < kStepKeyParts;
  const int part = key ? xp : xp - kStepKeyParts;
  const int unit_i = blockIdx.x / parts;
  const int b = unit_i / L.num_kv_heads, h = unit_i % L.num_kv_heads;
  const int32_t* len = L.lens + (int64_t)b * kLensStride;
  const int q = len[kLenQ], n = len[kLenN];
  if (n != L.residual) return;
  const int64_t unit = (int64_t)b * L.num_kv_heads + h;
  const BlockRows src{reinterpret_cast<const uint16_t*>(key ? L.ring_k : L.ring_v) + unit * L.residual * kHeadDim,
                      nullptr, 0, q, q + n, L.residual, L.num_kv_heads, h};
  quantize_part<ROT, DT, KB, VB>(L, b, h, key, part, key ? kStepKeyParts : kStepValueParts, q / L.group_k, src,
                                 smem_q);
}

// One instance of each quantize kernel per (rotation, kv dtype, key bits,
// value bits), chosen on the host; the shared-memory opt-in is recorded per
// instance and device.
template <bool ROT, int DT, int KB, int VB>
cudaError_t launch_flush_t(const FlushParams& p, int grid, int smem, cudaStream_t stream) {
  static uint64_t done = 0;
  const cudaError_t e = opt_in_max_smem(reinterpret_cast<const void*>(step_flush_kernel<ROT, DT, KB, VB>), done);
  if (e != cudaSuccess) return e;
  step_flush_kernel<ROT, DT, KB, VB><<<grid, kQuantThreads, smem, stream>>>(p);
  return cudaGetLastError();
}
template <bool ROT, int DT, int KB, int VB>
cudaError_t launch_quant_t(const AppendParams& p, dim3 grid, int smem, cudaStream_t stream) {
  static uint64_t done = 0;
  const cudaError_t e = opt_in_max_smem(reinterpret_cast<const void*>(quantize_blocks_kernel<ROT, DT, KB, VB>), done);
  if (e != cudaSuccess) return e;
  quantize_blocks_kernel<ROT, DT, KB, VB><<<grid, kQuantThreads, smem, stream>>>(p);
  return cudaGetLastError();
}
// Returns FN<rotation, dtype, key bits, value bits>(P, GRID, SMEM, STREAM)
// for the layer of P (FN: launch_flush_t or launch_quant_t).
#define KVQ_QUANT_DISPATCH(FN, P, GRID, SMEM, STREAM)                                           \
  do {                                                                                          \
    const LayerView& L_ = (P).L;                                                                \
    const bool rot_ = L_.hadamard != 0, bf_ = L_.kv_dtype == KVQ_BF16;                          \
    const int kb_ = L_.k_bits, vb_ = L_.v_bits;                                                 \
    KVQ_QUANT_BITS(FN, true, KVQ_BF16, rot_ && bf_, P, GRID, SMEM, STREAM)                      \
    KVQ_QUANT_BITS(FN, true, KVQ_F16, rot_ && !bf_, P, GRID, SMEM, STREAM)                      \
    KVQ_QUANT_BITS(FN, false, KVQ_BF16, !rot_ && bf_, P, GRID, SMEM, STREAM)                    \
    KVQ_QUANT_BITS(FN, false, KVQ_F16, !rot_ && !bf_, P, GRID, SMEM, STREAM)                    \
    return cudaErrorInvalidValue;                                                               \
  } while (0)
#define KVQ_QUANT_ONE(FN, R, D, K, V, P, GRID, SMEM, STREAM) \
  if (kb_ == K && vb_ == V) return FN<R, D, K, V>(P, GRID, SMEM, STREAM);
#define KVQ_QUANT_BITS(FN, R, D, COND, P, GRID, SMEM, STREAM)                                                    \
  if (COND) {                                                                                                    \
    KVQ_QUANT_ONE(FN, R, D, 2, 2, P, GRID, SMEM, STREAM) KVQ_QUANT_ONE(FN, R, D, 2, 4, P, GRID, SMEM, STREAM)     \
    KVQ_QUANT_ONE(FN, R, D, 2, 8, P, GRID, SMEM, STREAM) KVQ_QUANT_ONE(FN, R, D, 4, 2, P, GRID, SMEM, STREAM)     \
    KVQ_QUANT_ONE(FN, R, D, 4, 4, P, GRID, SMEM, STREAM) KVQ_QUANT_ONE(FN, R, D, 4, 8, P, GRID, SMEM, STREAM)     \
    KVQ_QUANT_ONE(FN, R, D, 8, 2, P, GRID, SMEM, STREAM) KVQ_QUANT_ONE(FN, R, D, 8, 4, P, GRID, SMEM, STREAM)     \
    KVQ_QUANT_ONE(FN, R, D, 8, 8, P, GRID, SMEM, STREAM)                                                         \
  }

cudaError_t launch_step_flush(const FlushParams& p, cudaStream_t stream) {
  const LayerView& L = p.L;
  const bool rot = L.hadamard != 0;
  const int smem = std::max(
      part_smem(part_shape(true, 0, kStepKeyParts, L.group_k, L.k_axis, rot), L.group_k, L.k_bits, L.group_v, L.k_axis,
                rot).total,
      part_smem(part_shape(false, 0, kStepValueParts, L.group_k, L.k_axis, rot), L.group_k, L.k_bits, L.group_v,
                L.k_axis, rot).total);
  const int grid = p.ctas * (kStepKeyParts + kStepValueParts);
  KVQ_QUANT_DISPATCH(launch_flush_t, p, grid, smem, stream);
}

// grid (batch, Hkv, splits); copies this call's sink tokens to the sinks
// and its tokens that stay exact into the key and value rings (CTA z a
// slice of them), and records the new lengths.
__global__ void ring_write_kernel(AppendParams p) {
  const int b = blockIdx.x, h = blockIdx.y;
  const LayerView& L = p.L;
  const int G = L.group_k, D = L.head_dim;
  const int boundary = p.len_old[b];
  const int q_new = p.q_old[b] + p.flush[b] * G;
  const int qv_new = p.qv_old[b] + p.flush_v[b] * G;
  const int end = boundary + p.t_new[b];
  const int vec_per_tok = D / 8;
  const int ns = p.s_take[b];
  const int64_t unit = (int64_t)b * L.num_kv_heads + h;
  const int64_t sink_base = unit * KVQ_MAX_SINKS + p.s_old[b];
  for (int idx = threadIdx.x; blockIdx.z == 0 && idx < ns * vec_per_tok; idx += blockDim.x) {
    const int i = idx / vec_per_tok, c = (idx % vec_per_tok) * 8;
    const int64_t row = (int64_t)p.in_off[b] - ns + i;
    const int64_t src = (row * L.num_kv_heads + h) * D + c;
    const int64_t dst = (sink_base + i) * D + c;
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(L.sink_k) + dst) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.k_in) + src);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(L.sink_v) + dst) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.v_in) + src);
  }
  // keys from max(boundary, q_new), values from max(boundary, qv_new); each
  // thread issues the loads of up to 4 chunks before their stores
  const int first_k = max(boundary, q_new), first_v = max(boundary, qv_new);
  const int first = min(first_k, first_v);
  // CTA z of gridDim.z takes its slice of the 16-byte chunks
  const int all = (end - first) * vec_per_tok;
  const int per = (all + gridDim.z - 1) / gridDim.z;
  const int lo = blockIdx.z * per;
  const int total = min(all, lo + per);
  const uint16_t* kin = reinterpret_cast<const uint16_t*>(p.k_in);
  const uint16_t* vin = reinterpret_cast<const uint16_t*>(p.v_in);
  uint16_t* rk = reinterpret_cast<uint16_t*>(L.ring_k);
  uint16_t* rv = reinterpret_cast<uint16_t*>(L.ring_v);
  for (int base = lo + threadIdx.x; base < total; base += 4 * blockDim.x) {
    uint4 tk[4], tv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * blockDim.x;
      if (idx >= total) break;
      const int i = first + idx / vec_per_tok, c = (idx % vec_per_tok) * 8;
      const int64_t src = (((int64_t)p.in_off[b] + (i - boundary)) * L.num_kv_heads + h) * D + c;
      if (i >= first_k) tk[u] = *reinterpret_cast<const uint4*>(kin + src);
      if (i >= first_v) tv[u] = *reinterpret_cast<const uint4*>(vin + src);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * blockDim.x;
      if (idx >= total) break;
      const int i = first + idx / vec_per_tok, c = (idx % vec_per_tok) * 8;
      if (i >= first_k) *reinterpret_cast<uint4*>(rk + (unit * L.residual + i % L.residual) * D + c) = tk[u];
      if (i >= first_v) *reinterpret_cast<uint4*>(rv + (unit * L.residual_v + i % L.residual_v) * D + c) = tv[u];
    }
  }
  if (h == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
    int32_t* len = L.lens + (int64_t)b * kLensStride;
    len[kLenQ] = q_new;
    len[kLenN] = end - q_new;
    len[kLenS] = p.s_old[b] + ns;
    len[kLenQV] = qv_new;
  }
}

// grid (ceil(n / 8), Hkv); block D threads. Token t0 + i of sequence `seq`,
// whose first `sinks` tokens are its sinks.
__global__ void dequant_kernel(LayerView L, int seq, int sinks, int t0, int n, float* k_out, float* v_out) {
  const int h = blockIdx.y;
  const int d = threadIdx.x;
  const int G = L.group_k, D = L.head_dim;
  const int Q = L.lens[(int64_t)seq * kLensStride + kLenQ];
  const int QV = L.lens[(int64_t)seq * kLensStride + kLenQV];
  const int kb = L.k_bits, vb = L.v_bits;
  const int64_t unit = (int64_t)seq * L.num_kv_heads + h;
  for (int r = 0; r < 8; ++r) {
    const int i = blockIdx.x * 8 + r;
    if (i >= n || d >= D) continue;
    const int64_t o = ((int64_t)i * L.num_kv_heads + h) * D + d;
    if (t0 + i < sinks) {
      const int64_t src = (unit * KVQ_MAX_SINKS + t0 + i) * D + d;
      k_out[o] = load_kv(L.sink_k, src, L.kv_dtype);
      v_out[o] = load_kv(L.sink_v, src, L.kv_dtype);
      continue;
    }
    const int tok = t0 + i - sinks;  // position after the sinks
    const int t = tok % G;
    if (tok < Q) {
      const uint8_t* rec = record_ptr(L, seq, h, tok / G);
      const int kper = 32 / kb;
      const __half2 ksz = *reinterpret_cast<const __half2*>(rec + ksz_pair_byte(L, t, d));
      const uint32_t kw = *reinterpret_cast<const uint32_t*>(rec + kc_word_byte(L, d, t / kper)) >> ((t % kper) * kb);
      k_out[o] = dequant_value(kw & ((1u << kb) - 1), __low2half(ksz), __high2half(ksz));
    } else {
      k_out[o] = load_kv(L.ring_k, (unit * L.residual + tok % L.residual) * D + d, L.kv_dtype);
    }
    if (tok < QV) {
      const uint8_t* rec = record_ptr(L, seq, h, tok / G);
      const int vper = 32 / vb;
      const uint32_t vq =
          (*reinterpret_cast<const uint32_t*>(rec + vc_word_byte(L, t, d / vper)) >> ((d % vper) * vb)) & ((1u << vb) - 1);
      const int gg = d / L.group_v;
      v_out[o] = dequant_value(vq, *reinterpret_cast<const __half*>(rec + vsz_half_byte(L, t, gg, false)),
                               *reinterpret_cast<const __half*>(rec + vsz_half_byte(L, t, gg, true)));
    } else {
      v_out[o] = load_kv(L.ring_v, (unit * L.residual_v + tok % L.residual_v) * D + d, L.kv_dtype);
    }
  }
}

// Opts a kernel in to the device's largest dynamic shared memory, once per
// (kernel, device): launches then pass what they use.
cudaError_t opt_in_max_smem(const void* kernel, uint64_t& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && (done_mask & (1ull << dev))) return cudaSuccess;
  int optin = 0;
  cudaFuncAttributes fa;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kernel);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
  if (e == cudaSuccess && dev < 64) done_mask |= 1ull << dev;
  return e;
}

// Streaming multiprocessors of the current device (0 if unknown).
int device_sm_count() {
  static int memo[64];  // per device, +1 (0: not queried yet)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    (void)cudaGetLastError();
    return 0;
  }
  if (dev < 64 && memo[dev] > 0) return memo[dev] - 1;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  if (dev < 64) memo[dev] = n + 1;
  return n;
}

cudaError_t launch_quantize(AppendParams& p, int max_flush, cudaStream_t stream) {
  const LayerView& L = p.L;
  const bool rot = L.hadamard != 0;
  // A call that quantizes few blocks (a decode step's flush, a prefill
  // chunk) splits each block and tensor into up to 4 parts -- channel slices
  // for per-channel keys, token slices otherwise -- until the grid fills two
  // waves of the kernel's 6 CTAs per SM; a CTA's time is its own latency
  // (staging, then quantizing), so smaller parts finish sooner.
  const int64_t ctas = 2LL * max_flush * p.batch * L.num_kv_heads;
  const int64_t target = 12LL * std::max(1, device_sm_count());
  // A part keeps at least 32 tokens or channels (a 32-token block split into
  // 8-token slices measured slower than whole); per-token key slices then
  // also hold whole code words (32 / k_bits tokens each).
  const int most_parts = std::max(1, std::min(4, L.group_k / 32));
  p.parts = 1;
  while (p.parts < most_parts && ctas * p.parts < target) p.parts *= 2;
  const int smem = quant_smem_bytes(L.group_k, L.k_bits, L.group_v, L.k_axis, rot, p.parts);
  dim3 grid(2 * max_flush * p.parts, p.batch, L.num_kv_heads);
  KVQ_QUANT_DISPATCH(launch_quant_t, p, grid, smem, stream);
}
#undef KVQ_QUANT_DISPATCH
#undef KVQ_QUANT_BITS
#undef KVQ_QUANT_ONE

cudaError_t launch_append(AppendParams& p, int max_flush, cudaStream_t stream) {
  const LayerView& L = p.L;
  if (max_flush > 0) {
    cudaError_t e = launch_quantize(p, max_flush, stream);
    if (e != cudaSuccess) return e;
  }
  // one CTA per (sequence, KV head), or up to 4 splitting the tokens that
  // stay exact when a call leaves many (a prefill: up to R per sequence), so
  // that each thread has one round of loads
  int most = 0;
  for (int b = 0; b < p.batch; ++b) most = std::max(most, std::min(p.t_new[b], std::max(L.residual, L.residual_v)));
  const int chunks = most * (kHeadDim / 8);
  const int splits = std::max(1, std::min(4, (chunks + 4 * 256 - 1) / (4 * 256)));
  dim3 grid2(p.batch, L.num_kv_heads, splits);
  ring_write_kernel<<<grid2, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

__global__ void page_table_kernel(PageTableUpdate u) {
  for (int i = threadIdx.x; i < u.n; i += blockDim.x) u.table[u.idx[i]] = u.page[i];
}

cudaError_t launch_page_table_update(const PageTableUpdate& u, cudaStream_t stream) {
  if (u.n <= 0) return cudaSuccess;
  page_table_kernel<<<1, 256, 0, stream>>>(u);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const LayerView& L, int seq, int sinks, int t0, int t1, float* k_out, float* v_out,
                           cudaStream_t stream) {
  const int n = t1 - t0;
  if (n <= 0) return cudaSuccess;
  dim3 grid((n + 7) / 8, L.num_kv_heads);
  dequant_kernel<<<grid, L.head_dim, 0, stream>>>(L, seq, sinks, t0, n, k_out, v_out);
  return cudaGetLastError();
}

}  // namespace kvq
