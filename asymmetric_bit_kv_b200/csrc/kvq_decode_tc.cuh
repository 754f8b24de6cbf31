// Tensor-core split-KV decode attention over the packed cache (sm_100a):
// the kernel template, instantiated per (key bits, value bits, value groups
// per head, key n-tiles, key axis) in kvq_decode_tc_k{2,4,8}_n{1,2}.cu.
//
// Method: decoding over per-channel-quantized keys and per-token-quantized
// values plus the full-precision residual window ("KIVI" README, Overview;
// GQA update), with x_hat = q*d + m ("KV1-1.2B" card, BQ2_0).
//
// Design (HBM-bound; the tensor cores only take the dot products off the ALUs):
//  * Persistent CTAs of kNC warps. The work items of all (sequence, KV head)
//    units -- a unit's quantized block records, then its ring tokens in
//    chunks of kResChunk -- are concatenated and cut into one contiguous range
//    per CTA; warp w of a CTA takes items w, w + kNC, ... of its range. Each
//    warp streams its own items through a private ring of SPW shared-memory
//    stages: one lane issues one cp.async.bulk (1-D TMA, no multicast) per
//    record, completing on the stage's mbarrier, and refills a stage as soon
//    as the warp is done with it, so no warp ever waits on another.
//  * Quantized keys, tokens on M: S[token][col] = codes x (q*s). ldmatrix
//    .trans over the channel-major key rows gives each thread two channels
//    of 16/kb tokens in one register; one AND leaves the code at bit
//    position p as the fp16 subnormal code * 2^(p-24), exact, the A operand
//    (p depends only on the A row, whose accumulator is scaled back by
//    2^(24-p)). The B operand is q*s per channel, fp16 high and low parts in
//    two columns per head (or two n-tiles for 8 heads), rebuilt per block
//    from the block's fp16 scales.
//  * Probabilities: after the online softmax (log2 units) each thread holds
//    P[token][two heads] in the m8n8 fragment layout; movmatrix.trans turns
//    it into the B operand of P.V (tokens on K, heads on N).
//  * Values: O[channel][head] = sum_t codes * (p*s) + sum_t p*z: value codes
//    of two tokens per register from ldmatrix.trans over token rows (channels
//    on M), as fp16 subnormals like the keys (the channel rows of O are
//    scaled back when the partial is written), the zero-point term one MMA
//    per value group with an all-ones A.
//  * Ring chunks use bf16 (or f16) m16n8k16 directly on the ring values, with
//    the query and the probabilities split into high and low parts, into the
//    same accumulators as the unit's blocks.
//  * Every warp writes one partial (o, m, l) per unit it passes through; the
//    log-sum-exp combine kernel merges them. mbarrier waits are bounded
//    (~2 s) and set the device error word instead of hanging.
//  * Keys quantized per token (KV1 BQ2_0, the PT instances): the same code
//    layout and A operand, the unit's (rotated) query as B, the token scales
//    on the score rows; see unit_query / unrotate_output.
//  * A unit's query rows may span several query tokens (verifying drafted
//    tokens): ring chunks hide from each its later tokens (DecodeParams).
//  * Paged caches: the issuing lane reads a unit's page once per run of
//    page_blocks blocks.
#pragma once

#include "kvq_decode.cuh"

namespace kvq {
namespace tc {

constexpr int kNC = kMmaConsumers;        // warps per CTA
constexpr int kThreads = kNC * 32;
constexpr long long kWaitCycles = 4000000000LL;  // a bounded wait gives up after ~2 s
constexpr int kRowBytes = kHeadDim * 2;  // one ring row (token, KV head)

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete; false after ~2 s.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// The same copy with an L2 cache policy (createpolicy): block records are
// read exactly once, so they are copied with an evict-first policy and do
// not push out of L2 what is read again soon (the unit's ring rows
// prefetched for its ring chunks, the split partials the combine reads).
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
// L2 prefetch of a global range (16-byte multiple), no shared-memory target.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// ldmatrix keeps a memory clobber so that it stays behind the barrier waits
// that publish the shared memory it reads; the arithmetic asm is free to move.
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr)
      : "memory");
}
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Transpose of an m8n8 b16 matrix held in the mma fragment layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// (a & b) | c in one instruction.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// acc + q.lo * z0 + q.hi * z1 (z0, z1: the high halves of sz0, sz1), each
// product of two fp16 exact and added to the fp32 accumulator with one
// rounding (mixed-precision fma).
__device__ __forceinline__ float fma_q_z(uint32_t q, uint32_t sz0, uint32_t sz1, float acc) {
  asm("{\n\t.reg .b16 ql, qh, s0, z0, s1, z1;\n\tmov.b32 {ql, qh}, %1;\n\tmov.b32 {s0, z0}, %2;\n\t"
      "mov.b32 {s1, z1}, %3;\n\tfma.rn.f32.f16 %0, ql, z0, %0;\n\tfma.rn.f32.f16 %0, qh, z1, %0;\n\t}"
      : "+f"(acc)
      : "r"(q), "r"(sz0), "r"(sz1));
  return acc;
}
// a * b - c with one rounding.
__device__ __forceinline__ uint32_t hfms2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("{\n\t.reg .b32 nc;\n\tneg.f16x2 nc, %3;\n\tfma.rn.f16x2 %0, %1, %2, nc;\n\t}" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_f16(uint32_t x) {
  return __half22float2(*reinterpret_cast<__half2*>(&x));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t x) {
  return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
}
__device__ __forceinline__ float2 unpack_kv(uint32_t x, bool bf16) { return bf16 ? unpack_bf16(x) : unpack_f16(x); }
__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Code j (width B bits) of both 16-bit halves of a register, as fp16
// subnormals: masked in place at bit position p (0..7) of its byte, with the
// exponent field zero, the code reads as the exact fp16 value code * 2^(p-24).
// The MMAs thus multiply exact integers scaled by a power of two that depends
// only on the code's index j, i.e. on the row of the A operand; the row's
// accumulator is scaled back by 2^(24-p), exactly, where it is read. x8 =
// x >> 8 serves codes that sit in the upper byte of a half. One instruction
// per two codes.
template <int B>
__device__ __forceinline__ uint32_t code_sub(uint32_t x, uint32_t x8, int j) {
  const int bit = B * j;
  const uint32_t m = ((1u << B) - 1u) << (bit & 7);
  return (bit >= 8 ? x8 : x) & (m | (m << 16));
}
// Bit position p of code j inside its byte, and 2^e as a float constant.
template <int B>
__host__ __device__ constexpr int code_pos(int j) { return (B * j) & 7; }
__host__ __device__ constexpr float pow2f(int e) {
  float r = 1.f;
  for (int i = 0; i < e; ++i) r *= 2.f;
  for (int i = 0; i > e; --i) r *= 0.5f;
  return r;
}
// Row scale 2^(24-p) of the accumulator rows fed by code j.
template <int B>
__host__ __device__ constexpr float code_unscale(int j) { return pow2f(24 - code_pos<B>(j)); }

// Compile-time shape of one instance. A tile is 64 tokens of a block.
template <int KB, int VB, int NGRP, int NKT>
struct Shape {
  static constexpr int D = kHeadDim;
  static constexpr int TT = 64;              // tokens per tile
  static constexpr int CPT16 = 16 / KB;      // key tokens per 16-bit column
  static constexpr int TOKC = 128 / KB;      // key tokens per 16-byte chunk of a channel row
  static constexpr int SIG = TT / TOKC;      // chunks of a channel row per tile
  static constexpr int JP = CPT16 / 2;       // M-tiles per chunk
  static constexpr int MT = SIG * JP;        // M-tiles (16 tokens) per tile
  static constexpr int VRB = D * VB / 8;     // value code bytes per token
  static constexpr int NCH = VRB / 16;       // 16-byte chunks per value row
  static constexpr int VCPC = 16 / VB;       // value channels per 16-bit column
  static constexpr int MT_PER_CH = VCPC / 2; // channel m-tiles per value chunk
  static constexpr int CH_SPAN = 128 / VB;   // channels per value chunk
  static constexpr int GV = D / NGRP;        // value group (channels)
  static_assert(MT == 4, "a 64-token tile is four 16-token M-tiles");
  static_assert(SIG >= 1, "tile too short for the key code width");
  static_assert(CH_SPAN <= GV, "a value chunk must lie inside one value group");
};

// Token (0..63 inside the tile) on row r (0..15) of key M-tile mt: rows 0-7
// take code 2*jp, rows 8-15 code 2*jp+1 of 16-bit column r%8 of chunk sg.
template <int KB>
__device__ __forceinline__ int tile_token(int mt, int r) {
  constexpr int CPT16 = 16 / KB, TOKC = 128 / KB, JP = CPT16 / 2;
  return (mt / JP) * TOKC + (r & 7) * CPT16 + 2 * (mt % JP) + (r >> 3);
}

// ------------------------------------------------------- residual ring chunks
// The ring tokens are exact (kv dtype), so their dot products run on the
// tensor cores in that dtype (bf16 or f16 m16n8k16), with the scaled query
// and the probabilities split into high and low parts, which keeps both at
// about 16 significant bits; the accumulators are the ones the quantized
// blocks of the unit use.
template <bool BF16>
__device__ __forceinline__ void mma_kv(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (BF16) mma_bf16(d, a, b0, b1);
  else mma_f16(d, a, b0, b1);
}
template <bool BF16>
__device__ __forceinline__ uint32_t pack_kv(float lo, float hi) {
  if constexpr (BF16) return pack_bf16(lo, hi);
  else return pack_f16(lo, hi);
}
template <bool BF16>
__device__ __forceinline__ float2 unpack_kv2(uint32_t x) {
  if constexpr (BF16) return unpack_bf16(x);
  else return unpack_f16(x);
}

// --------------------------------------------------------- quantized blocks
// Walks the (sequence, head) units of consecutive global work items.
struct UnitCursor {
  int b = 0, h = 0, start = 0, end = 0;  // current unit and its item range
  __device__ void seek(const DecodeParams& p, int k) {
    int lo = 0, hi = p.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.seq_start[mid] <= k) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    const int nb = p.nitem[b];
    h = (k - p.seq_start[b]) / nb;
    start = p.seq_start[b] + h * nb;
    end = start + nb;
  }
  __device__ void advance(const DecodeParams& p, int k) {
    if (k >= end || k < start) seek(p, k);
  }
};

// Per-consumer-warp scratch (byte offsets in MmaPlan), rebuilt per block
// from its fp16 scales (prep_block); the unit's queries arrive with the
// warp's first item of the unit:
//   bfrag [NKT][8 kk][32 lanes] uint2: key B fragments. Column n of the
//         n-tile holds q*s of head n/2, fp16 high part (n even) or low part
//         (n odd); with 8 heads n-tile 0 holds the high and n-tile 1 the low
//         parts of heads 0-7. Columns of absent heads stay zero.
//   bias  [8] float: sum_d q_d z_d per head (log2 units);
//   qbuf  [nstages][NG][D]: the queries of the warp's last units (one buffer
//         per unit change, round robin), copied in as stored in q and then
//         converted in place to fp16 times q_prescale, the channel pair
//         (2w, 2w+1) of head h at word h*64 + (w%8)*8 + w/8 (q_word), so that
//         the eight pairs prep_block takes per lane are contiguous.
// q (fp16, a power-of-two multiple of the query) times s (fp16) has at most
// 22 significant bits, so the fp16 high part and the fp16 rounding of the
// remainder (one fused multiply-subtract) hold it exactly; the softmax scale
// is applied to the fp32 scores.
__host__ __device__ constexpr int q_word(int h, int w) { return h * 64 + (w & 7) * 8 + (w >> 3); }

template <int NKT>
__device__ __forceinline__ void prep_block(const uint8_t* stage, const MmaPlan& mp, uint8_t* ws, const uint32_t* qw,
                                           int NG, int lane, float score_scale) {
  uint32_t* bk = reinterpret_cast<uint32_t*>(ws + mp.bfrag_off);
  const uint2* ksz2 = reinterpret_cast<const uint2*>(stage + mp.kc_bytes);  // (s, z) of channels 2c, 2c+1
  float* biasw = reinterpret_cast<float*>(ws + mp.bias_off);
  const int q = lane & 7, half = q >> 2, tq = q & 3;
#pragma unroll
  for (int rep = 0; rep < NKT; ++rep) {  // two passes exactly when there are 8 heads
    const int hh = (lane >> 3) + 4 * rep;
    float bp = 0.f;
    if (hh < NG) {
      const uint4* q4 = reinterpret_cast<const uint4*>(qw + q_word(hh, q));  // words of kk = 0..7
      const uint4 qa = q4[0], qb = q4[1];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t q2 = word_of(kk < 4 ? qa : qb, kk & 3);  // channels 16kk + 2q, +1
        const uint2 sz = ksz2[8 * kk + q];
        const uint32_t s2 = __byte_perm(sz.x, sz.y, 0x5410);
        bp = fma_q_z(q2, sz.x, sz.y, bp);
        const uint32_t hi = hmul2(q2, s2);
        const uint32_t lo = hfms2(q2, s2, hi);
        if (NKT == 1) {
          bk[(kk * 32 + (2 * hh) * 4 + tq) * 2 + half] = hi;
          bk[(kk * 32 + (2 * hh + 1) * 4 + tq) * 2 + half] = lo;
        } else {
          bk[(kk * 32 + hh * 4 + tq) * 2 + half] = hi;
          bk[((8 + kk) * 32 + hh * 4 + tq) * 2 + half] = lo;
        }
      }
    }
    bp += __shfl_xor_sync(0xffffffffu, bp, 1);
    bp += __shfl_xor_sync(0xffffffffu, bp, 2);
    bp += __shfl_xor_sync(0xffffffffu, bp, 4);
    if (q == 0 && hh < NG) biasw[hh] = bp * score_scale;
  }
  __syncwarp();
}


// Heads per lane of the score layout. With 8 query heads per KV head (two
// key n-tiles: high parts, low parts) lane (g, t) holds heads 2t and 2t+1;
// with at most 4 (one n-tile, columns 2h / 2h+1 = high / low part of head
// h) it holds head t, both parts in its own two columns.
template <int NKT>
constexpr int heads_per_lane() { return NKT == 2 ? 2 : 1; }

// Online-softmax state of this lane's heads (log2 units).
template <int HPL>
struct SoftState {
  float m[HPL], l[HPL];
};

// Key score of row r (0: g, 1: g+8) and lane head h of an M-tile's
// accumulators: high part + low part.
template <int NKT>
__device__ __forceinline__ float head_score(const float (&d)[NKT][4], int r, int h) {
  if constexpr (NKT == 2) return d[0][2 * r + h] + d[1][2 * r + h];
  else return d[0][2 * r] + d[0][2 * r + 1];
}

// Online-softmax update of this lane's HPL heads with the scores of MTN
// M-tiles, sc[mt][r * HPL + h] for row r (g, g+8) and lane head h; sc becomes
// the probabilities; O and Z (columns = heads 2t, 2t+1) are rescaled when a
// running maximum grows. GUARD: scores may be -inf (absent tokens), a whole
// update may see none, and absent heads (valid false) are zeroed (ring
// chunks); without it every score is finite, and absent heads just compute
// finite values in columns that are never written (quantized tiles). OWN:
// both output columns of a lane belong to the lane's own score head (the
// pair kernel), so the lane rescales them by its own alpha.
template <int MTN, int HPL, int NGRP, bool GUARD, bool OWN = false>
__device__ __forceinline__ void softmax_update(float (&sc)[MTN][2 * HPL], SoftState<HPL>& st,
                                               const bool (&valid)[HPL], float (&O)[8][4], float (&Z)[NGRP][4],
                                               int lane) {
  float n[HPL], a[HPL];
#pragma unroll
  for (int h = 0; h < HPL; ++h) {
    float mx = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < MTN; ++mt) mx = fmaxf(mx, fmaxf(sc[mt][h], sc[mt][HPL + h]));
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if constexpr (GUARD) {
      // a head with no finite score so far keeps m = -inf, alpha = 1, p = 0
      n[h] = valid[h] ? fmaxf(st.m[h], mx) : -INFINITY;
      a[h] = n[h] == -INFINITY ? 1.f : ex2(st.m[h] - n[h]);
    } else {
      n[h] = fmaxf(st.m[h], mx);
      a[h] = ex2(st.m[h] - n[h]);  // 0 on the first tile (m = -inf)
    }
    st.m[h] = n[h];
    float ps = 0.f;
#pragma unroll
    for (int mt = 0; mt < MTN; ++mt)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float& x = sc[mt][r * HPL + h];
        if constexpr (GUARD) x = n[h] == -INFINITY ? 0.f : ex2(x - n[h]);
        else x = ex2(x - n[h]);
        ps += x;
      }
    st.l[h] = st.l[h] * a[h] + ps;
  }
  bool same = true;
#pragma unroll
  for (int h = 0; h < HPL; ++h) same = same && a[h] == 1.f;
  if (!__all_sync(0xffffffffu, same)) {
    // alpha of the output columns (heads 2t, 2t+1) of this lane
    float a0, a1;
    if constexpr (HPL == 2) {
      a0 = a[0];
      a1 = a[1];
    } else if constexpr (OWN) {
      a0 = a1 = a[0];
    } else {
      const int t = lane & 3, base = lane & ~3;
      a0 = __shfl_sync(0xffffffffu, a[0], base + ((2 * t) & 3));
      a1 = __shfl_sync(0xffffffffu, a[0], base + ((2 * t + 1) & 3));
    }
#pragma unroll
    for (int gg = 0; gg < NGRP; ++gg) {
      Z[gg][0] *= a0;
      Z[gg][1] *= a1;
      Z[gg][2] *= a0;
      Z[gg][3] *= a1;
    }
#pragma unroll
    for (int i2 = 0; i2 < 8; ++i2) {
      O[i2][0] *= a0;
      O[i2][1] *= a1;
      O[i2][2] *= a0;
      O[i2][3] *= a1;
    }
  }
}

// The P.V B operand of one M-tile from its probabilities (rows g and g+8 of
// this lane's heads): bt holds tokens 2t, 2t+1 (rows 0-7) and bb tokens
// 8+2t, 9+2t of head g, as two kv-dtype or fp16 values. With two heads per
// lane the rows are transposed by movmatrix; with one, lane (g, t) fetches
// its two tokens from lanes (2t, g) and (2t+1, g) (rows g and g+8 packed in
// one register there).
template <int HPL>
__device__ __forceinline__ void prob_operand(uint32_t row_g, uint32_t row_g8, uint32_t packed, int lane,
                                             uint32_t& bt, uint32_t& bb) {
  if constexpr (HPL == 2) {
    bt = movmatrix_t(row_g);
    bb = movmatrix_t(row_g8);
  } else {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t u = __shfl_sync(0xffffffffu, packed, 8 * t + g);
    const uint32_t v = __shfl_sync(0xffffffffu, packed, 8 * t + 4 + g);
    bt = __byte_perm(u, v, 0x5410);
    bb = __byte_perm(u, v, 0x7632);
  }
}

// prob_operand with one head per lane where the B columns 4-7 repeat columns
// 0-3 (at most 4 heads per KV head leave them free): lane (g, t) takes the
// tokens of head g & 3, so that columns 4-7 can carry the remainders of
// columns 0-3.
__device__ __forceinline__ void prob_operand_dup(uint32_t packed, int lane, uint32_t& bt, uint32_t& bb) {
  const int g = lane >> 2, t = lane & 3;
  const uint32_t u = __shfl_sync(0xffffffffu, packed, 8 * t + (g & 3));
  const uint32_t v = __shfl_sync(0xffffffffu, packed, 8 * t + 4 + (g & 3));
  bt = __byte_perm(u, v, 0x5410);
  bb = __byte_perm(u, v, 0x7632);
}

// Adds O and Z columns 4-7 into columns 0-3 (lane t += lane t ^ 2): the
// remainder columns of prob_operand_dup, folded into their heads.
template <int NGRP>
__device__ __forceinline__ void fold_remainders(float (&O)[8][4], float (&Z)[NGRP][4]) {
#pragma unroll
  for (int i2 = 0; i2 < 8; ++i2)
#pragma unroll
    for (int e = 0; e < 4; ++e) O[i2][e] += __shfl_xor_sync(0xffffffffu, O[i2][e], 2);
#pragma unroll
  for (int gg = 0; gg < NGRP; ++gg)
#pragma unroll
    for (int e = 0; e < 4; ++e) Z[gg][e] += __shfl_xor_sync(0xffffffffu, Z[gg][e], 2);
}

// One chunk of ring tokens (cnt of its kResChunk rows present, cnt <= 0
// for the placeholder chunk of an empty sequence): stage = key rows
// [kResChunk][D] then value rows, in the kv dtype; accumulated into the
// unit's state like a quantized block. Keys, tokens on M: lane (g, t) holds
// token g's words 2(kk%2) and 2(kk%2)+1 of 16-byte chunk t + 4(kk/2) for
// k-step kk (rows 8-15 absent); the B operand is the scaled query split
// into kv-dtype high and low parts in the same channel order, written over
// the warp's key B fragments (bk, same layout) on its first chunk of the unit
// (a unit's ring chunks come after all of its quantized blocks; qw holds the
// fp16 queries times q_prescale, and score_scale = scale_log2 / q_prescale).
// P.V: after movmatrix, lane (g, t) holds the probabilities of tokens 2t,
// 2t+1 for head g; each output m-tile takes the value word of its channels
// (ch0, ch0+1) from both tokens, paired by one byte permute; two MMAs
// (probability high and low parts) into a scratch accumulator, added to O at
// the row scale of the quantized blocks' value codes (2^(p-24)).
template <bool BF16, int VB, int NGRP, int NKT>
__device__ __forceinline__ void ring_chunk(const uint8_t* stage, const uint32_t* qw, uint2* bk,
                                           const int (&cnt)[heads_per_lane<NKT>()], int NG,
                                           int lane, float score_scale, const bool (&valid)[heads_per_lane<NKT>()],
                                           bool& rq_ready, SoftState<heads_per_lane<NKT>()>& sst, float (&O)[8][4],
                                           float (&Z)[NGRP][4]) {
  using S = Shape<2, VB, NGRP, NKT>;  // value-side constants only
  constexpr int HPL = heads_per_lane<NKT>();
  const int g = lane >> 2, t = lane & 3;
  if (!rq_ready) {
    // column g: head g (two n-tiles) or head g/2, high (g even) or low part
    const int head = NKT == 2 ? g : (g >> 1);
    const bool present = head < NG;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t hi[2], lo[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int w = 4 * t + 16 * (kk >> 1) + 2 * (kk & 1) + e;  // channels 2w, 2w+1
        const uint32_t raw = present ? qw[q_word(head, w)] : 0u;
        const float2 f = unpack_f16(raw);
        const float x0 = f.x * score_scale, x1 = f.y * score_scale;
        hi[e] = pack_kv<BF16>(x0, x1);
        const float2 fh = unpack_kv2<BF16>(hi[e]);
        lo[e] = pack_kv<BF16>(x0 - fh.x, x1 - fh.y);
      }
      if constexpr (NKT == 1) {
        bk[kk * 32 + lane] = (g & 1) ? make_uint2(lo[0], lo[1]) : make_uint2(hi[0], hi[1]);
      } else {
        bk[kk * 32 + lane] = make_uint2(hi[0], hi[1]);
        bk[(8 + kk) * 32 + lane] = make_uint2(lo[0], lo[1]);
      }
    }
    __syncwarp();
    rq_ready = true;
  }
  const uint4* K4 = reinterpret_cast<const uint4*>(stage);
  float Dr[NKT][4];
#pragma unroll
  for (int nt = 0; nt < NKT; ++nt) Dr[nt][0] = Dr[nt][1] = Dr[nt][2] = Dr[nt][3] = 0.f;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint4 kv = K4[g * 16 + t + 4 * m];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint32_t a[4] = {word_of(kv, 2 * hf), 0u, word_of(kv, 2 * hf + 1), 0u};
#pragma unroll
      for (int nt = 0; nt < NKT; ++nt) {
        const uint2 bq = bk[(nt * 8 + 2 * m + hf) * 32 + lane];
        mma_kv<BF16>(Dr[nt], a, bq.x, bq.y);
      }
    }
  }
  // rows 8-15 are absent; row g holds ring token g of the chunk
  float sc[1][2 * HPL];
#pragma unroll
  for (int h = 0; h < HPL; ++h) {
    sc[0][h] = g < cnt[h] ? head_score<NKT>(Dr, 0, h) : -INFINITY;
    sc[0][HPL + h] = -INFINITY;
  }
  softmax_update<1, HPL, NGRP, true>(sc, sst, valid, O, Z, lane);
  // probabilities in kv-dtype high and low parts (only tokens 0-7 exist)
  uint32_t bh, bl, dummy;
  if constexpr (HPL == 2) {
    const uint32_t ph = pack_kv<BF16>(sc[0][0], sc[0][1]);
    const float2 fh = unpack_kv2<BF16>(ph);
    prob_operand<HPL>(ph, pack_kv<BF16>(sc[0][0] - fh.x, sc[0][1] - fh.y), 0u, lane, bh, bl);
  } else {
    const uint32_t ph = pack_kv<BF16>(sc[0][0], 0.f);
    const float hf = unpack_kv2<BF16>(ph).x;
    const uint32_t hl = pack_kv<BF16>(sc[0][0], sc[0][0] - hf);  // (high, low) of row g
    prob_operand<HPL>(0u, 0u, hl, lane, bh, dummy);              // bh = high parts of tokens 2t, 2t+1
    bl = dummy;                                                  // bb = low parts
    if (g >= 4) bh = bl = 0u;  // columns 4-7 hold no head here (see prob_operand_dup)
  }
  const uint32_t* V32 = reinterpret_cast<const uint32_t*>(stage + kResChunk * kRowBytes);  // [rows][64 words]
#pragma unroll
  for (int mt2 = 0; mt2 < 8; ++mt2) {
    const int cch = mt2 / S::MT_PER_CH, P = mt2 % S::MT_PER_CH;
    const int w = (cch * S::CH_SPAN + g * S::VCPC) / 2 + P;
    const uint32_t x = V32[(2 * t) * 64 + w], y = V32[(2 * t + 1) * 64 + w];
    const uint32_t a[4] = {__byte_perm(x, y, 0x5410), __byte_perm(x, y, 0x7632), 0u, 0u};
    float r[4] = {0.f, 0.f, 0.f, 0.f};
    mma_kv<BF16>(r, a, bh, 0u);
    mma_kv<BF16>(r, a, bl, 0u);
    const float s0 = pow2f(code_pos<VB>(2 * P) - 24), s1 = pow2f(code_pos<VB>(2 * P + 1) - 24);
    O[mt2][0] = fmaf(r[0], s0, O[mt2][0]);
    O[mt2][1] = fmaf(r[1], s0, O[mt2][1]);
    O[mt2][2] = fmaf(r[2], s1, O[mt2][2]);
    O[mt2][3] = fmaf(r[3], s1, O[mt2][3]);
  }
}

// ------------------------------------------- per-token keys and the rotation
// Keys quantized per token over whole head vectors ("KV1-1.2B" card, BQ2_0)
// keep the per-channel code layout, so the A operand is built the same way;
// only the scales move: S[t][h] = d_t * (codes . q')[t][h] + m_t * sum(q'_h).
// The B operand is then the unit's query itself (fp16 high and low parts,
// the same columns as q*s), built once per unit instead of once per block,
// and d_t, m_t scale the rows of the fp32 scores. With the rotation, q' = H q
// for the quantized tokens; their part of O is in the rotated basis and is
// multiplied by H again (H . H = I) before any exact-token chunk adds to O,
// and before the partial is written.

// Per-token keys: the key B fragments (same columns as prep_block's, every
// column written, absent heads zero) and bias[h] = sum_d q'_hd * score_scale
// of the unit's query q' (rotated when rot), from qw (fp16 x q_prescale).
template <int NKT>
__device__ __forceinline__ void unit_query(const uint32_t* qw, uint8_t* ws, const MmaPlan& mp, int NG, int lane,
                                           float score_scale, bool rot) {
  uint32_t* bk = reinterpret_cast<uint32_t*>(ws + mp.bfrag_off);
  float* biasw = reinterpret_cast<float*>(ws + mp.bias_off);
#pragma unroll 1
  for (int hh = 0; hh < 4 * NKT; ++hh) {
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (hh < NG) {
      const float2 a = unpack_f16(qw[q_word(hh, 2 * lane)]), c = unpack_f16(qw[q_word(hh, 2 * lane + 1)]);
      x[0] = a.x, x[1] = a.y, x[2] = c.x, x[3] = c.y;
      if (rot) rotate_lane(x, lane);
    }
    float sum = (x[0] + x[1]) + (x[2] + x[3]);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int w = 2 * lane + e;  // channels 2w, 2w+1
      const uint32_t hi = pack_f16(x[2 * e], x[2 * e + 1]);
      const float2 fh = unpack_f16(hi);
      const uint32_t lo = pack_f16(x[2 * e] - fh.x, x[2 * e + 1] - fh.y);
      const int kk = w >> 3, q = w & 7, half = q >> 2, tq = q & 3;
      if (NKT == 1) {
        bk[(kk * 32 + (2 * hh) * 4 + tq) * 2 + half] = hi;
        bk[(kk * 32 + (2 * hh + 1) * 4 + tq) * 2 + half] = lo;
      } else {
        bk[(kk * 32 + hh * 4 + tq) * 2 + half] = hi;
        bk[((8 + kk) * 32 + hh * 4 + tq) * 2 + half] = lo;
      }
    }
    if (lane == 0) biasw[hh] = sum * score_scale;
  }
  __syncwarp();
}

// O (with its zero-point terms Z folded in; FOLD: and its remainder columns)
// times H over the channels, in place: each lane's outputs of heads 2t, 2t+1
// go to scr [NG][128] fp32 (the
// warp's key B-fragment area, which the caller rebuilds afterwards), every
// head is rotated by the warp, and O is read back at its rows' code scale
// (2^(p-24), exact), Z cleared.
template <int VB, int NGRP, bool FOLD>
__device__ __forceinline__ void unrotate_output(float (&O)[8][4], float (&Z)[NGRP][4], float* scr, int NG, int lane,
                                                bool v0, bool v1) {
  using S = Shape<2, VB, NGRP, 1>;  // value-side constants only
  const int g = lane >> 2, t = lane & 3;
  if constexpr (FOLD) fold_remainders<NGRP>(O, Z);
  __syncwarp();  // every lane is done with the B fragments
#pragma unroll
  for (int mt2 = 0; mt2 < 8; ++mt2) {
    const int cch = mt2 / S::MT_PER_CH, P = mt2 % S::MT_PER_CH;
    const int gg = (cch * S::CH_SPAN) / S::GV;
    const int ch0 = cch * S::CH_SPAN + g * S::VCPC + 2 * P;
    const float u0 = code_unscale<VB>(2 * P), u1 = code_unscale<VB>(2 * P + 1);
    if (v0) {
      scr[(2 * t) * kHeadDim + ch0] = fmaf(O[mt2][0], u0, Z[gg][0]);
      scr[(2 * t) * kHeadDim + ch0 + 1] = fmaf(O[mt2][2], u1, Z[gg][2]);
    }
    if (v1) {
      scr[(2 * t + 1) * kHeadDim + ch0] = fmaf(O[mt2][1], u0, Z[gg][1]);
      scr[(2 * t + 1) * kHeadDim + ch0 + 1] = fmaf(O[mt2][3], u1, Z[gg][3]);
    }
  }
  __syncwarp();
#pragma unroll 1
  for (int h = 0; h < NG; ++h) {
    float4* row = reinterpret_cast<float4*>(scr + h * kHeadDim);
    const float4 v = row[lane];
    float x[4] = {v.x, v.y, v.z, v.w};
    rotate_lane(x, lane);
    row[lane] = make_float4(x[0], x[1], x[2], x[3]);
  }
  __syncwarp();
#pragma unroll
  for (int mt2 = 0; mt2 < 8; ++mt2) {
    const int cch = mt2 / S::MT_PER_CH, P = mt2 % S::MT_PER_CH;
    const int ch0 = cch * S::CH_SPAN + g * S::VCPC + 2 * P;
    const float r0 = pow2f(code_pos<VB>(2 * P) - 24), r1 = pow2f(code_pos<VB>(2 * P + 1) - 24);
    O[mt2][0] = v0 ? scr[(2 * t) * kHeadDim + ch0] * r0 : 0.f;
    O[mt2][2] = v0 ? scr[(2 * t) * kHeadDim + ch0 + 1] * r1 : 0.f;
    O[mt2][1] = v1 ? scr[(2 * t + 1) * kHeadDim + ch0] * r0 : 0.f;
    O[mt2][3] = v1 ? scr[(2 * t + 1) * kHeadDim + ch0 + 1] * r1 : 0.f;
  }
#pragma unroll
  for (int gg = 0; gg < NGRP; ++gg) Z[gg][0] = Z[gg][1] = Z[gg][2] = Z[gg][3] = 0.f;
  __syncwarp();
}

// Exact-token chunk r of a unit (the items after its quantized blocks): ring
// chunk r while r < ceil(nres / kResChunk), then the sink chunk if the
// sequence has sinks; an empty sequence's one item is a ring chunk with no
// tokens. Returns the tokens present (<= 0 for none) and whether it is the
// sink chunk.
__device__ __forceinline__ int exact_chunk(const DecodeParams& p, int b, int r, bool& sink) {
  const int nres = p.nres[b];
  sink = false;
  if (r < (nres + kResChunk - 1) / kResChunk) return nres - r * kResChunk;
  const int nsink = p.L.sinks > 0 ? p.L.lens[(int64_t)b * kLensStride + kLenS] : 0;
  sink = nsink > 0;
  return sink ? nsink : nres - r * kResChunk;
}

// Fused decode step: the copy of the chunk holding this call's new token
// (ring index nres - 1) took that row from the input (issue_item); the warp
// also stores it into its ring slot for later calls (no other item of this
// call reads that slot), and the unit of KV head 0 records the sequence's new
// lengths.
__device__ __forceinline__ void store_new_token(const DecodeParams& p, int b, int h, int nb, const uint8_t* stage,
                                                int lane) {
  const LayerView& L = p.L;
  const int i = p.nres[b] - 1;
  const int row = i % kResChunk;
  const int slot = (nb * L.tile_tokens + i) % L.residual;
  const int64_t dst = (((int64_t)b * L.num_kv_heads + h) * L.residual + slot) * kRowBytes;
  reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(L.ring_k) + dst)[lane] =
      reinterpret_cast<const uint2*>(stage + row * kRowBytes)[lane];
  reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(L.ring_v) + dst)[lane] =
      reinterpret_cast<const uint2*>(stage + (kResChunk + row) * kRowBytes)[lane];
  if (h == 0 && lane == 0) {  // the step's lengths (a flush of this step moved G tokens to block nb - 1)
    int32_t* len = L.lens + (int64_t)b * kLensStride;
    len[kLenQ] = nb * L.tile_tokens;
    len[kLenN] = p.nres[b];
    len[kLenQV] = nb * L.tile_tokens;
  }
}

// Issue side of a warp's item stream (one lane): the unit of the last issued
// item and the number of unit changes so far.
struct IssueState {
  UnitCursor u;
  uint64_t pol = evict_first_policy();  // L2 policy of the block-record copies
  int unit = -1;
  int qslot = -1;         // query buffer of the unit (round robin over the nstages buffers)
  int ring0 = 0;          // ring slot of the unit's first ring token
  int run = -1;           // paged cache: page-table entry (j / page_blocks) of the unit held in `page`
  int64_t page = 0;
};

// Issues the copy of work item k (a block record, or the key and value rows
// of a ring chunk) into stage `dst`, completing on `bar`; on the first item
// of a unit also the unit's queries, into the next query buffer (qslot).
__device__ __forceinline__ void issue_item(const DecodeParams& p, const MmaPlan& mp, IssueState& is, int k,
                                           uint8_t* dst, uint64_t* bar, uint8_t* qbuf, int NG) {
  const LayerView& L = p.L;
  UnitCursor& u = is.u;
  u.advance(p, k);
  const int j = k - u.start, nb = p.nblk[u.b];
  const int unit = u.b * L.num_kv_heads + u.h;
  const bool newq = unit != is.unit;
  const uint32_t qbytes = NG * kRowBytes;
  if (newq) {
    is.unit = unit;
    is.qslot = is.qslot + 1 == mp.nstages ? 0 : is.qslot + 1;
    is.ring0 = (nb * L.tile_tokens) % L.residual;
  }
  if (j < nb) {
    // tile item j: tile j % NT of block j / NT (NT = 2^lg_nt tiles per block)
    const int jb = j >> mp.lg_nt, jt = j & ((1 << mp.lg_nt) - 1);
    mbar_expect_tx(bar, mp.tx_bytes + (newq ? qbytes : 0u));
    const uint8_t* rec;
    if (L.page_table) {  // one page-table read per run of page_blocks blocks of the unit
      const int run = jb / L.page_blocks;
      if (newq || run != is.run) {
        is.run = run;
        is.page = __ldg(L.page_table + (int64_t)u.b * L.max_pages + run);
      }
      rec = L.blocks + ((is.page * L.num_kv_heads + u.h) * L.page_blocks + jb % L.page_blocks) * L.record_bytes;
    } else {
      rec = record_ptr(L, u.b, u.h, jb);
    }
    if (mp.lg_nt == 0) {
      bulk_g2s_hint(dst, rec, mp.tx_bytes, bar, is.pol);
    } else {
      const uint8_t* tp = rec + L.tile0_off + (int64_t)jt * L.tile_bytes;
      if (L.rec_ksz_off >= 0) {  // the block's per-channel key scales, then the tile's codes and value scales
        bulk_g2s(dst + mp.kc_bytes, rec + L.rec_ksz_off, kHeadDim * 4, bar);  // read by both tiles
        bulk_g2s_hint(dst, tp, mp.kc_bytes, bar, is.pol);
        bulk_g2s_hint(dst + mp.vc_soff, tp + L.vc_off, L.tile_bytes - L.vc_off, bar, is.pol);
      } else {  // a tile part holds all it needs
        bulk_g2s_hint(dst, tp, L.tile_bytes, bar, is.pol);
      }
    }
    if (j == nb - 1 && p.nres[u.b] > 0) {
      // the unit's ring chunks come next: bring its ring rows into L2 so that
      // those short items do not each wait a full HBM round trip
      const int64_t ring = ((int64_t)u.b * L.num_kv_heads + u.h) * L.residual * kRowBytes;
      bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(L.ring_k) + ring, L.residual * kRowBytes);
      bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(L.ring_v) + ring, L.residual * kRowBytes);
    }
  } else {
    // ring chunk: kResChunk consecutive slots of keys, then of values (or
    // the kResChunk sink rows of the unit)
    bool sink;
    (void)exact_chunk(p, u.b, j - nb, sink);
    const void* ksrc = sink ? L.sink_k : L.ring_k;
    const void* vsrc = sink ? L.sink_v : L.ring_v;
    int64_t row;
    if (sink) {
      row = ((int64_t)u.b * L.num_kv_heads + u.h) * KVQ_MAX_SINKS;
    } else {
      int slot = is.ring0 + (j - nb) * kResChunk;  // (j - nb) * kResChunk < residual
      if (slot >= L.residual) slot -= L.residual;
      row = ((int64_t)u.b * L.num_kv_heads + u.h) * L.residual + slot;
    }
    constexpr uint32_t bytes = kResChunk * kRowBytes;
    mbar_expect_tx(bar, 2 * bytes + (newq ? qbytes : 0u));
    const uint8_t* kr = reinterpret_cast<const uint8_t*>(ksrc) + row * kRowBytes;
    const uint8_t* vr = reinterpret_cast<const uint8_t*>(vsrc) + row * kRowBytes;
    if (p.new_k && !sink && j - nb == (p.nres[u.b] - 1) / kResChunk) {
      // fused decode step: row i of this chunk is the new token, from the
      // input; the ring rows around it as they are
      const int i = (p.nres[u.b] - 1) % kResChunk;
      const uint32_t lo = i * kRowBytes, hi = (kResChunk - 1 - i) * kRowBytes;
      const int64_t in = ((int64_t)u.b * L.num_kv_heads + u.h) * kRowBytes;
      if (lo) {
        bulk_g2s(dst, kr, lo, bar);
        bulk_g2s(dst + bytes, vr, lo, bar);
      }
      if (hi) {
        bulk_g2s(dst + lo + kRowBytes, kr + lo + kRowBytes, hi, bar);
        bulk_g2s(dst + bytes + lo + kRowBytes, vr + lo + kRowBytes, hi, bar);
      }
      bulk_g2s(dst + lo, reinterpret_cast<const uint8_t*>(p.new_k) + in, kRowBytes, bar);
      bulk_g2s(dst + bytes + lo, reinterpret_cast<const uint8_t*>(p.new_v) + in, kRowBytes, bar);
    } else {
      bulk_g2s(dst, kr, bytes, bar);
      bulk_g2s(dst + bytes, vr, bytes, bar);
    }
  }
  if (newq) {
    // the unit's query rows: ngr heads of each of the launch's query tokens
    const int ngr = p.q_heads / L.num_kv_heads;
    uint8_t* qdst = qbuf + (size_t)is.qslot * qbytes;
    for (int t = 0; t < p.qtok; ++t)
      bulk_g2s(qdst + (size_t)t * ngr * kRowBytes,
               reinterpret_cast<const uint8_t*>(p.q) +
                   ((int64_t)u.b * p.q_rows + (int64_t)t * p.q_heads + u.h * ngr) * kRowBytes,
               ngr * kRowBytes, bar);
  }
}

// PT: keys per token over whole head vectors, with the rotation when the
// layer has it (see unit_query); otherwise per-channel keys.
template <int KB, int VB, int NGRP, int NKT, bool PT>
__global__ void __launch_bounds__(kThreads, 2) decode_tc_kernel(DecodeParams p, MmaPlan mp) {
  using S = Shape<KB, VB, NGRP, NKT>;
  constexpr int D = S::D;
  extern __shared__ __align__(128) uint8_t smem[];
  const int c = blockIdx.x;
  const LayerView& L = p.L;
  const int Hkv = L.num_kv_heads;
  const int NG = p.num_q_heads / Hkv;  // query rows per unit
  const int ngr = p.q_heads / Hkv;      // query heads per KV head (rows per query token)
  // tokens of one work item's tile: the block, or 64 of a longer block (this
  // kernel serves blocks of >= 64 tokens, so a tile is always 64 tokens)
  constexpr int G = S::TT;
  const int rs = p.cta_start[c], re = p.cta_start[c + 1];
  const bool bf16 = L.kv_dtype == KVQ_BF16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the combine launch that follows may be scheduled from now on; it waits
  // for this grid to complete before reading any partial
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // a fused decode step that flushes launches this kernel as a dependent of
  // the kernel quantizing the flushed blocks: wait for those records (no-op
  // otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // this warp's items: rs + warp + n*kNC, n = 0, 1, ...; item n lands in the
  // warp's own stage n % SPW (phase parity (n / SPW) & 1, both kept
  // incrementally), and the warp issues item n + SPW as soon as it is done
  // with item n
  const int SPW = mp.nstages;  // stages per warp
  uint8_t* stages = smem + (size_t)warp * SPW * mp.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + mp.bar_off) + warp * SPW;
  uint8_t* ws = smem + mp.ws_soff + warp * mp.ws_bytes;
  const int nmine = rs + warp < re ? (re - rs - warp + kNC - 1) / kNC : 0;
  uint8_t* qbuf = ws + mp.qbuf_off;
  IssueState is;  // issue side (lane 0)
  if (lane == 0) {
    for (int i = 0; i < SPW; ++i) mbar_init(full + i, 1);
    fence_mbar_init();
    for (int n = 0; n < SPW && n < nmine; ++n)
      issue_item(p, mp, is, rs + warp + n * kNC, stages + (size_t)n * mp.stage_bytes, full + n, qbuf, NG);
  }
  __syncwarp();
  bool failed = false;
  int n = 0;  // items of this warp consumed so far
  {
    {  // key B-fragment columns and biases of absent heads stay zero
      uint4* z = reinterpret_cast<uint4*>(ws + mp.bfrag_off);
      for (int e = lane; e < (mp.bias_off + 32) / 16; e += 32) z[e] = make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
    }
    const int g = lane >> 2, t = lane & 3;
    const uint32_t ones[4] = {0x3c003c00u, 0x3c003c00u, 0x3c003c00u, 0x3c003c00u};  // fp16 1.0
    constexpr int kc_row = G * KB / 8;  // key code bytes per channel of a tile
    const int mi = lane >> 3, rr = lane & 7;
    // ldmatrix rows of this lane: 8 consecutive rows, so the chunk swizzle of
    // the record layout depends on the lane's row index only
    const int swk = chunk_swizzle(rr, kc_row / 16);
    const int swv = chunk_swizzle(rr, S::VRB / 16);
    const uint2* bkr = reinterpret_cast<const uint2*>(ws + mp.bfrag_off);
    uint2* bkw = reinterpret_cast<uint2*>(ws + mp.bfrag_off);
    const float* biasr = reinterpret_cast<const float*>(ws + mp.bias_off);
    int qslot = -1;  // query buffer of the current unit (matches IssueState::qslot)
    int st = 0;      // stage of item n and its barrier phase parity
    uint32_t ph = 0;
    const bool v0 = 2 * t < NG, v1 = 2 * t + 1 < NG;  // output columns (heads 2t, 2t+1) of this lane exist
    constexpr int HPL = heads_per_lane<NKT>();
    bool valid[HPL];  // score heads of this lane exist
    if constexpr (HPL == 2) {
      valid[0] = v0;
      valid[1] = v1;
    } else {
      valid[0] = t < NG;
    }
    UnitCursor u;
    int k = rs;
    while (k < re && !failed) {
      u.advance(p, k);
      const int hi = min(u.end, re);
      const int nb = p.nblk[u.b];
      SoftState<HPL> sst;
#pragma unroll
      for (int h = 0; h < HPL; ++h) {
        sst.m[h] = -INFINITY;
        sst.l[h] = 0.f;
      }
      float O[8][4], Z[NGRP][4];
#pragma unroll
      for (int i2 = 0; i2 < 8; ++i2) O[i2][0] = O[i2][1] = O[i2][2] = O[i2][3] = 0.f;
#pragma unroll
      for (int gg = 0; gg < NGRP; ++gg) Z[gg][0] = Z[gg][1] = Z[gg][2] = Z[gg][3] = 0.f;
      bool rq_ready = false;  // the key B fragments hold the ring-chunk query (not a block's q*s)
      bool uq_ready = false;  // PT: they hold the unit's query for its quantized blocks
      bool rotated = false;   // PT with the rotation: O holds rotated-basis terms
      // this warp's items of the unit: k' - rs = warp (mod kNC)
      const int first = k + ((warp - (k - rs)) % kNC + kNC) % kNC;
      for (int kb = first; kb < hi; kb += kNC, ++n) {
        if (!mbar_wait(full + st, ph)) {
          failed = true;
          break;
        }
        const uint8_t* stage = stages + (size_t)st * mp.stage_bytes;
        if (kb == first) qslot = qslot + 1 == SPW ? 0 : qslot + 1;
        uint32_t* qw = reinterpret_cast<uint32_t*>(qbuf + (size_t)qslot * NG * kRowBytes);
        if (kb == first) {
          // the warp's first item of the unit brought its queries: to fp16
          // times q_prescale, in place
          // (the permutation stays inside each head: four heads at a time)
          for (int h0 = 0; h0 < NG; h0 += 4) {
            uint32_t cv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int w = h0 * (D / 2) + lane + 32 * i;
              if (w < NG * (D / 2)) {
                const float2 f = bf16 ? unpack_bf16(qw[w]) : unpack_f16(qw[w]);
                cv[i] = pack_f16(f.x * p.q_prescale, f.y * p.q_prescale);
              }
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int w = h0 * (D / 2) + lane + 32 * i;
              if (w < NG * (D / 2)) qw[q_word(w / (D / 2), w % (D / 2))] = cv[i];
            }
            __syncwarp();
          }
        }
        const int j = kb - u.start;
        if (j < nb) {
          // ============ quantized block
          if constexpr (PT) {
            if (!uq_ready) {
              unit_query<NKT>(qw, ws, mp, NG, lane, p.score_scale, L.hadamard != 0);
              uq_ready = true;
              rq_ready = false;
            }
            rotated = L.hadamard != 0;
          } else {
            prep_block<NKT>(stage, mp, ws, qw, NG, lane, p.score_scale);
          }
          float bias[HPL];
#pragma unroll
          for (int h = 0; h < HPL; ++h) bias[h] = biasr[HPL == 2 ? 2 * t + h : t];
          const uint32_t kc_s = smem_u32(stage);
          const uint32_t vc_s = smem_u32(stage + mp.vc_soff);
          const uint4* vsz4 = reinterpret_cast<const uint4*>(stage + mp.vsz_soff);
#pragma unroll
          for (int tile = 0; tile < G / S::TT; ++tile) {  // one tile per item
            // ---- scores: Dk[M-tile][n-tile] = codes x (q*s)
            float Dk[S::MT][NKT][4];
#pragma unroll
            for (int mt = 0; mt < S::MT; ++mt)
#pragma unroll
              for (int nt = 0; nt < NKT; ++nt) Dk[mt][nt][0] = Dk[mt][nt][1] = Dk[mt][nt][2] = Dk[mt][nt][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
              uint2 bfr[2][NKT];
#pragma unroll
              for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int nt = 0; nt < NKT; ++nt) bfr[hf][nt] = bkr[(nt * 8 + 2 * kp + hf) * 32 + lane];
              const int ch = 16 * (2 * kp + (mi >> 1)) + 8 * (mi & 1) + rr;
#pragma unroll
              for (int sg = 0; sg < S::SIG; ++sg) {
                uint32_t rk[4];
                ldsm_x4_t(kc_s + ch * kc_row + (((tile * S::SIG + sg) ^ swk) << 4), rk[0], rk[1], rk[2], rk[3]);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                  const uint32_t xl = rk[2 * hf], xh = rk[2 * hf + 1], xl8 = xl >> 8, xh8 = xh >> 8;
#pragma unroll
                  for (int jp = 0; jp < S::JP; ++jp) {
                    const uint32_t a[4] = {code_sub<KB>(xl, xl8, 2 * jp), code_sub<KB>(xl, xl8, 2 * jp + 1),
                                           code_sub<KB>(xh, xh8, 2 * jp), code_sub<KB>(xh, xh8, 2 * jp + 1)};
#pragma unroll
                    for (int nt = 0; nt < NKT; ++nt)
                      mma_f16(Dk[sg * S::JP + jp][nt], a, bfr[hf][nt].x, bfr[hf][nt].y);
                  }
                }
              }
            }
            // ---- online softmax over the tile; row r of M-tile mt read code
            // 2*(mt % JP) + r/8 of its column
            float sc[S::MT][2 * HPL];
#pragma unroll
            for (int mt = 0; mt < S::MT; ++mt)
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                const float rs = p.score_scale * code_unscale<KB>(2 * (mt % S::JP) + r);
                if constexpr (PT) {
                  // (scale, zero point) of the row's token
                  const __half2 sz = reinterpret_cast<const __half2*>(stage + mp.kc_bytes)[tile * S::TT +
                                                                                         tile_token<KB>(mt, g + 8 * r)];
                  const float2 dz = __half22float2(sz);
                  const float rst = rs * dz.x;
#pragma unroll
                  for (int h = 0; h < HPL; ++h)
                    sc[mt][r * HPL + h] = fmaf(head_score<NKT>(Dk[mt], r, h), rst, dz.y * bias[h]);
                } else {
#pragma unroll
                  for (int h = 0; h < HPL; ++h)
                    sc[mt][r * HPL + h] = fmaf(head_score<NKT>(Dk[mt], r, h), rs, bias[h]);
                }
              }
            softmax_update<S::MT, HPL, NGRP, false>(sc, sst, valid, O, Z, lane);
            // ---- values: O += codes x (p * s), Z += ones x (p * z)
#pragma unroll
            for (int mt = 0; mt < S::MT; ++mt) {
              // P^T of the M-tile: tokens rows 2t, 2t+1 (bt) and 8+2t, 9+2t (bb), head g
              uint32_t bt, bb;
              if constexpr (HPL == 2)
                prob_operand<HPL>(pack_f16(sc[mt][0], sc[mt][1]), pack_f16(sc[mt][2], sc[mt][3]), 0u, lane, bt, bb);
              else if constexpr (PT)
                prob_operand_dup(pack_f16(sc[mt][0], sc[mt][1]), lane, bt, bb);
              else
                prob_operand<HPL>(0u, 0u, pack_f16(sc[mt][0], sc[mt][1]), lane, bt, bb);
              const int kst = tile * S::MT + mt;
              uint32_t B0[NGRP], B1[NGRP];
              uint32_t R0[PT ? NGRP : 1], R1[PT ? NGRP : 1];
#pragma unroll
              for (int gg = 0; gg < NGRP; ++gg) {
                const uint4 v4 = vsz4[(kst * 4 + t) * NGRP + gg];  // (s, s), (s, s), (z, z), (z, z) of rows 2t.. 9+2t
                B0[gg] = hmul2(bt, v4.x);
                B1[gg] = hmul2(bb, v4.y);
                // PT: whole-vector value groups have scales and zero points
                // that are large next to the values they encode, so p*s and
                // p*z also keep their fp16 remainders (exact): in the free
                // columns 4-7 with at most 4 heads, else in one more MMA each
                if constexpr (PT && HPL == 1) {
                  const bool rem = g >= 4;
                  B0[gg] = rem ? hfms2(bt, v4.x, B0[gg]) : B0[gg];
                  B1[gg] = rem ? hfms2(bb, v4.y, B1[gg]) : B1[gg];
                  const uint32_t z0 = hmul2(bt, v4.z), z1 = hmul2(bb, v4.w);
                  mma_f16(Z[gg], ones, rem ? hfms2(bt, v4.z, z0) : z0, rem ? hfms2(bb, v4.w, z1) : z1);
                } else if constexpr (PT) {
                  R0[gg] = hfms2(bt, v4.x, B0[gg]);
                  R1[gg] = hfms2(bb, v4.y, B1[gg]);
                  const uint32_t z0 = hmul2(bt, v4.z), z1 = hmul2(bb, v4.w);
                  mma_f16(Z[gg], ones, z0, z1);
                  mma_f16(Z[gg], ones, hfms2(bt, v4.z, z0), hfms2(bb, v4.w, z1));
                } else {
                  mma_f16(Z[gg], ones, hmul2(bt, v4.z), hmul2(bb, v4.w));
                }
              }
              const int sg = mt / S::JP, jp = mt % S::JP;
              const int vrow_idx = (2 * jp + (mi & 1)) * (G / S::CPT16) + tile * (S::TT / S::CPT16) + sg * 8 + rr;
              const uint32_t vrow = vc_s + vrow_idx * S::VRB;
#pragma unroll
              for (int cc0 = 0; cc0 < S::NCH; cc0 += 2) {
                uint32_t r[4];
                ldsm_x4_t(vrow + (((cc0 + (mi >> 1)) ^ swv) << 4), r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                  const uint32_t xv = r[2 * cc], yv = r[2 * cc + 1], xv8 = xv >> 8, yv8 = yv >> 8;
                  const int gg = ((cc0 + cc) * S::CH_SPAN) / S::GV;
#pragma unroll
                  for (int P = 0; P < S::MT_PER_CH; ++P) {
                    const uint32_t a[4] = {code_sub<VB>(xv, xv8, 2 * P), code_sub<VB>(xv, xv8, 2 * P + 1),
                                           code_sub<VB>(yv, yv8, 2 * P), code_sub<VB>(yv, yv8, 2 * P + 1)};
                    mma_f16(O[(cc0 + cc) * S::MT_PER_CH + P], a, B0[gg], B1[gg]);
                    if constexpr (PT && HPL == 2) mma_f16(O[(cc0 + cc) * S::MT_PER_CH + P], a, R0[gg], R1[gg]);
                  }
                }
              }
            }
          }
        } else {
          if constexpr (PT) {
            if (rotated) {  // exact tokens add in the original basis
              unrotate_output<VB, NGRP, HPL == 1>(O, Z, reinterpret_cast<float*>(ws + mp.bfrag_off), NG, lane, v0,
                                                  v1);
              rotated = false;
              rq_ready = false;
            }
            uq_ready = false;  // ring_chunk writes its own query over the B fragments
          }
          bool sink;
          const int cnt0 = exact_chunk(p, u.b, j - nb, sink);
          // tokens of the chunk each lane head sees: a ring chunk hides its
          // last lag_base - t tokens from query token t (several per sequence)
          int cnt[HPL];
#pragma unroll
          for (int h = 0; h < HPL; ++h)
            cnt[h] = sink ? cnt0 : cnt0 - (p.lag_base - (HPL == 2 ? 2 * t + h : t) / ngr);
          if (p.new_k && !sink && j - nb == (p.nres[u.b] - 1) / kResChunk) store_new_token(p, u.b, u.h, nb, stage, lane);
          if (bf16)
            ring_chunk<true, VB, NGRP, NKT>(stage, qw, bkw, cnt, NG, lane, p.score_scale, valid, rq_ready, sst, O, Z);
          else
            ring_chunk<false, VB, NGRP, NKT>(stage, qw, bkw, cnt, NG, lane, p.score_scale, valid, rq_ready, sst, O, Z);
        }
        // every lane is done with the stage: refill it with item n + SPW
        __syncwarp();
        if (lane == 0 && n + SPW < nmine) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue_item(p, mp, is, rs + warp + (n + SPW) * kNC, stages + (size_t)st * mp.stage_bytes, full + st, qbuf, NG);
        }
        if (++st == SPW) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (failed) break;
      if constexpr (PT) {
        if (rotated)
          unrotate_output<VB, NGRP, HPL == 1>(O, Z, reinterpret_cast<float*>(ws + mp.bfrag_off), NG, lane, v0, v1);
        else if constexpr (HPL == 1)
          fold_remainders<NGRP>(O, Z);
      }
      // ---------------- this warp's partial for the unit
#pragma unroll
      for (int off = 4; off <= 16; off <<= 1)
#pragma unroll
        for (int h = 0; h < HPL; ++h) sst.l[h] += __shfl_xor_sync(0xffffffffu, sst.l[h], off);
      const int c0 = cta_of_item(p.cta_start, p.num_ctas, u.start);
      const int slot = kNC * (c - c0) + warp;
      if (slot == 0 && lane == 0)  // the unit's slot count, for the combine kernel
        p.unit_slots[u.b * Hkv + u.h] = kNC * (cta_of_item(p.cta_start, p.num_ctas, u.end - 1) - c0 + 1);
      const int64_t base0 = ((int64_t)u.b * p.num_q_heads + u.h * NG + 2 * t) * p.slots + slot;
      const int64_t base1 = base0 + p.slots;
#pragma unroll
      for (int mt2 = 0; mt2 < 8; ++mt2) {
        const int cch = mt2 / S::MT_PER_CH, P = mt2 % S::MT_PER_CH;
        const int gg = (cch * S::CH_SPAN) / S::GV;
        const int ch0 = cch * S::CH_SPAN + g * S::VCPC + 2 * P;
        // rows g (channel ch0, code 2P of its column, held at 2^(p-24)) and
        // g+8 (ch0 + 1, code 2P+1); Z holds the zero-point term per row
        const float u0 = code_unscale<VB>(2 * P), u1 = code_unscale<VB>(2 * P + 1);
        if (v0)
          *reinterpret_cast<float2*>(p.ws_o + base0 * D + ch0) =
              make_float2(fmaf(O[mt2][0], u0, Z[gg][0]), fmaf(O[mt2][2], u1, Z[gg][2]));
        if (v1)
          *reinterpret_cast<float2*>(p.ws_o + base1 * D + ch0) =
              make_float2(fmaf(O[mt2][1], u0, Z[gg][1]), fmaf(O[mt2][3], u1, Z[gg][3]));
      }
      if (g == 0) {
        if constexpr (HPL == 2) {
          if (v0) p.ws_ml[base0] = make_float2(sst.m[0], sst.l[0]);
          if (v1) p.ws_ml[base1] = make_float2(sst.m[1], sst.l[1]);
        } else if (valid[0]) {  // head t
          p.ws_ml[((int64_t)u.b * p.num_q_heads + u.h * NG + t) * p.slots + slot] = make_float2(sst.m[0], sst.l[0]);
        }
      }
      k = hi;
    }
  }
  if (failed) {
    // let the copies still in flight land before the CTA may leave
    if (lane == 0)
      for (int i = n; i < n + SPW && i < nmine; ++i) (void)mbar_wait(full + i % SPW, (i / SPW) & 1);
    if (lane == 0) atomicOr(p.err, 1);
  }
}

// Enqueues one instance. Its dynamic shared-memory size was opted in on this
// device by mma_ctas_per_sm, which the host calls before every launch. After
// the flush kernel of a fused decode step (p.after_flush) it is a
// programmatic dependent of that kernel: its CTAs may start while the flush
// runs and wait for it (griddepcontrol.wait) before reading any record.
template <int KB, int VB, int NGRP, int NKT, bool PT>
cudaError_t launch_instance(const DecodeParams& p, const MmaPlan& mp, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = mp.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = p.after_flush ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<KB, VB, NGRP, NKT, PT>, p, mp);
}

template <int KB, int VB, int NGRP, int NKT, bool PT>
const void* instance_fn() {
  return reinterpret_cast<const void*>(decode_tc_kernel<KB, VB, NGRP, NKT, PT>);
}

}  // namespace tc
}  // namespace kvq
