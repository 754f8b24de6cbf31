// Tensor-core split-KV decode attention over the packed cache (sm_100a).
//
// Method: decoding over per-channel-quantized keys and per-token-quantized
// values plus the full-precision residual window ("KIVI" README, Overview;
// GQA update), with x_hat = q*d + m ("KV1-1.2B" card, BQ2_0).
//
// Design (HBM-bound; tensor cores only take the dot products off the ALUs):
//  * One CTA per (split, KV head, sequence); split 0 is the residual ring.
//    Warp 4 is a producer: one lane streams whole block records from HBM into
//    a ring of shared-memory stages with cp.async.bulk (1-D TMA) completing on
//    mbarriers. Warps 0-3 each consume every fourth block.
//  * Keys: per block, q.k_hat = sum_d (q_d s_d) c_d + sum_d q_d z_d. The
//    scaled query (q_d s_d) is split into an fp16 high part and an fp16
//    low part (rows 0-7 and 8-15 of the m16n8k16 A operand), the codes c are
//    the B operand. Codes reach registers with ldmatrix.trans from the
//    channel-major key rows (two channels of the same tokens per register),
//    and become exact fp16 integers with one lop3 (mask | 0x6400 exponent)
//    and one hsub2 (minus 1024). A code taken from bit position p is c * 2^p;
//    the score is rescaled by 2^-p afterwards (exact).
//  * Values: o[ch][head] = sum_t (p_t s_t) c_t,ch + sum_t p_t z_t. The value
//    codes of two tokens per register come from ldmatrix.trans over the
//    token rows (the A operand, channels on M); the probabilities times the
//    token's value scale are the fp16 B operand (tokens on K, heads on N).
//    The zero-point term is accumulated in fp32 on the side.
//  * Online softmax in log2 units per 64-token tile; fp32 partials per split
//    are merged by the log-sum-exp combine kernel.
#include "kvq_decode.cuh"

namespace kvq {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr long long kWaitCycles = 4000000000LL;  // a bounded wait gives up after ~2 s

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
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Codes selected by `mask` in both 16-bit halves of x, as exact fp16 integers
// (times the power of two of their bit position): (x & mask) | 1024.0h, then
// minus 1024.0h.
__device__ __forceinline__ uint32_t codes_to_f16(uint32_t x, uint32_t mask) {
  uint32_t r = (x & mask) | 0x64006400u;
  __half2 h = *reinterpret_cast<__half2*>(&r);
  h = __hsub2(h, __halves2half2(__ushort_as_half((unsigned short)0x6400), __ushort_as_half((unsigned short)0x6400)));
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_f16(uint32_t x) {
  return __half22float2(*reinterpret_cast<__half2*>(&x));
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ------------------------------------------------------- residual ring split
// Exact attention over the ring tokens [Q, Q+n) of (b, h) with CUDA cores;
// warps 0-3 each take every fourth token. Writes partial slot 0.
__device__ void residual_partial(const DecodeParams& p, int b, int h, int NG, int Q, int n, uint8_t* smem) {
  const LayerView& L = p.L;
  constexpr int D = kHeadDim;
  float* sq = reinterpret_cast<float*>(smem);  // [8][D]
  float* so = sq + 8 * D;                      // [4][8][D]
  float* sm = so + 4 * 8 * D;                  // [4][8]
  float* sl = sm + 32;                         // [4][8]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < NG * D; i += blockDim.x)
    sq[i] = load_kv(p.q, ((int64_t)b * p.num_q_heads + h * NG) * D + i, L.kv_dtype) * p.scale_log2;
  __syncthreads();
  float m[8], l[8], o[8][4];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) o[hh][c] = 0.f;
  }
  if (warp < kConsumerWarps) {
    const int64_t base = ((int64_t)b * L.num_kv_heads + h) * L.residual;
    for (int i = Q + warp; i < Q + n; i += kConsumerWarps) {
      const int64_t row = (base + i % L.residual) * D;
      float kv[4], vv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        kv[c] = load_kv(L.ring_k, row + lane + 32 * c, L.kv_dtype);
        vv[c] = load_kv(L.ring_v, row + lane + 32 * c, L.kv_dtype);
      }
#pragma unroll
      for (int hh = 0; hh < 8; ++hh) {
        if (hh < NG) {
          float part = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) part += sq[hh * D + lane + 32 * c] * kv[c];
          const float sc = warp_sum(part);
          const float mn = fmaxf(m[hh], sc);
          const float alpha = ex2(m[hh] - mn);
          const float pe = ex2(sc - mn);
          l[hh] = l[hh] * alpha + pe;
#pragma unroll
          for (int c = 0; c < 4; ++c) o[hh][c] = o[hh][c] * alpha + pe * vv[c];
          m[hh] = mn;
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      if (hh < NG) {
#pragma unroll
        for (int c = 0; c < 4; ++c) so[(warp * 8 + hh) * D + lane + 32 * c] = o[hh][c];
        if (lane == 0) {
          sm[warp * 8 + hh] = m[hh];
          sl[warp * 8 + hh] = l[hh];
        }
      }
    }
  }
  __syncthreads();
  const int d = threadIdx.x;
  if (d < D) {
    for (int hh = 0; hh < NG; ++hh) {
      float M = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm[w * 8 + hh]);
      float acc = 0.f, lsum = 0.f;
      if (M != -INFINITY) {
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float mw = sm[w * 8 + hh];
          const float f = mw == -INFINITY ? 0.f : ex2(mw - M);
          acc += so[(w * 8 + hh) * D + d] * f;
          lsum += sl[w * 8 + hh] * f;
        }
      }
      const int64_t slot = ((int64_t)b * p.num_q_heads + h * NG + hh) * p.slots;
      p.ws_o[slot * D + d] = acc;
      if (d == 0) p.ws_ml[slot] = make_float2(M, lsum);
    }
  }
}

// --------------------------------------------------------- quantized splits
template <int KB, int VB, int TT, int NGRP>
struct Shape {
  static constexpr int D = kHeadDim;
  static constexpr int CPT16 = 16 / KB;         // key tokens per 16-bit column
  static constexpr int SIGMA_TOK = 128 / KB;    // key tokens per 16-byte row chunk
  static constexpr int SIG = TT / SIGMA_TOK;    // 16-byte key chunks per tile
  static constexpr int NT = TT / 8;             // n-tiles (8 tokens) per tile
  static constexpr int KSTEPS = TT / 16;        // PV k-steps per tile
  static constexpr int VRB = D * VB / 8;        // value code bytes per token
  static constexpr int NCH = VRB / 16;          // 16-byte value chunks per token
  static constexpr int VCPC = 16 / VB;          // value channels per 16-bit column
  static constexpr int MT_PER_CH = 8 / VB;      // m-tiles per value chunk
  static constexpr int CH_SPAN = 128 / VB;      // channels per value chunk
  static constexpr int GV = D / NGRP;           // value group (channels)
  static_assert(SIG >= 1, "tile too short for the key code width");
  static_assert(CH_SPAN <= GV, "a value chunk must lie inside one value group");
};

template <int KB, int TT>
__device__ __forceinline__ int tile_token(int idx, int col) {
  constexpr int CPT16 = 16 / KB, SIGMA_TOK = 128 / KB;
  (void)TT;
  return (idx / CPT16) * SIGMA_TOK + col * CPT16 + (idx % CPT16);
}

template <int KB, int VB, int TT, int NGRP>
__global__ void __launch_bounds__(kThreads) decode_mma_kernel(DecodeParams p, MmaPlan mp) {
  using S = Shape<KB, VB, TT, NGRP>;
  constexpr int D = S::D;
  extern __shared__ __align__(128) uint8_t smem[];
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const LayerView& L = p.L;
  const int NG = p.num_q_heads / L.num_kv_heads;
  const int G = L.group_k;
  const int Q = L.lens[2 * b], n = L.lens[2 * b + 1];
  const int nblk = Q / G;
  const int bps = p.blocks_per_split;
  const int nsplit = (nblk + bps - 1) / bps;
  if (s > nsplit) return;
  if (s == 0) {
    residual_partial(p, b, h, NG, Q, n, smem);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = (s - 1) * bps;
  const int nb = min(s * bps, nblk) - j0;
  const int NS = mp.nstages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + mp.bar_off);
  uint64_t* empty = full + NS;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const int g = lane >> 2, t = lane & 3;
  float lsum = 0.f, m_run = (g < NG) ? -INFINITY : 0.f;
  float zacc[NGRP];
#pragma unroll
  for (int gg = 0; gg < NGRP; ++gg) zacc[gg] = 0.f;
  float O[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) O[i][0] = O[i][1] = O[i][2] = O[i][3] = 0.f;
  bool failed = false;

  if (warp == kConsumerWarps) {
    // ---------------- producer: one lane streams the split's block records
    if (lane == 0) {
      const uint8_t* rec0 = record_ptr(L, b, h, j0);
      int issued = 0;
      for (int i = 0; i < nb; ++i) {
        const int st = i % NS;
        if (i >= NS && !mbar_wait(empty + st, ((i / NS) & 1) ^ 1)) {
          failed = true;
          break;
        }
        const uint8_t* rec = rec0 + (int64_t)i * L.record_bytes;
        uint8_t* dst = smem + (size_t)st * mp.stage_bytes;
        mbar_expect_tx(full + st, mp.tx_bytes);
        bulk_g2s(dst, rec, mp.kc_bytes + D * 4, full + st);
        for (int sg = 0; sg < mp.vseg_count; ++sg)
          bulk_g2s(dst + mp.vc_soff + sg * (mp.vseg_bytes + 16), rec + L.vc_off + sg * mp.vseg_bytes, mp.vseg_bytes,
                   full + st);
        bulk_g2s(dst + mp.vsz_soff, rec + L.vsz_off, mp.vsz_bytes, full + st);
        issued = i + 1;
      }
      // Let every copy land before the CTA may leave.
      for (int i = max(0, issued - NS); i < issued; ++i)
        if (!mbar_wait(full + i % NS, (i / NS) & 1)) failed = true;
    }
  } else {
    // ---------------- consumers
    // This thread's query values: head g, channels 16kk + 2t + {0, 1, 8, 9}.
    float qreg[8][4];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int d = 16 * kk + 2 * t + (e & 1) + 8 * (e >> 1);
        qreg[kk][e] = (g < NG) ? load_kv(p.q, ((int64_t)b * p.num_q_heads + h * NG + g) * D + d, L.kv_dtype) *
                                     p.scale_log2
                               : 0.f;
      }
    const int kc_row = G * KB / 8;  // key code bytes per channel
    for (int i = warp; i < nb; i += kConsumerWarps) {
      const int st = i % NS;
      if (!mbar_wait(full + st, (i / NS) & 1)) {
        failed = true;
        break;
      }
      const uint8_t* stage = smem + (size_t)st * mp.stage_bytes;
      const __half2* ksz = reinterpret_cast<const __half2*>(stage + mp.kc_bytes);
      const __half2* vsz = reinterpret_cast<const __half2*>(stage + mp.vsz_soff);
      const uint32_t kc_s = smem_u32(stage);
      const uint32_t vc_s = smem_u32(stage + mp.vc_soff);

      // A operand: (q*s) split into fp16 high (rows g) and low (rows g+8)
      // parts; bias = sum_d q_d z_d of head g.
      uint32_t A[8][4];
      float bias = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if (g < NG) {
          const int c0 = 16 * kk + 2 * t;
          const uint2 pa = *reinterpret_cast<const uint2*>(ksz + c0);      // (s,z) of c0, c0+1
          const uint2 pb = *reinterpret_cast<const uint2*>(ksz + c0 + 8);  // (s,z) of c0+8, c0+9
          const float2 a0 = unpack_f16(pa.x), a1 = unpack_f16(pa.y);
          const float2 b0 = unpack_f16(pb.x), b1 = unpack_f16(pb.y);
          const float x0 = qreg[kk][0] * a0.x, x1 = qreg[kk][1] * a1.x;
          const float x8 = qreg[kk][2] * b0.x, x9 = qreg[kk][3] * b1.x;
          bias += qreg[kk][0] * a0.y + qreg[kk][1] * a1.y + qreg[kk][2] * b0.y + qreg[kk][3] * b1.y;
          const uint32_t h01 = pack_f16(x0, x1), h89 = pack_f16(x8, x9);
          const float2 f01 = unpack_f16(h01), f89 = unpack_f16(h89);
          A[kk][0] = h01;
          A[kk][1] = pack_f16(x0 - f01.x, x1 - f01.y);
          A[kk][2] = h89;
          A[kk][3] = pack_f16(x8 - f89.x, x9 - f89.y);
        } else {
          A[kk][0] = A[kk][1] = A[kk][2] = A[kk][3] = 0u;
        }
      }
      bias += __shfl_xor_sync(0xffffffffu, bias, 1);
      bias += __shfl_xor_sync(0xffffffffu, bias, 2);

      for (int tile = 0; tile < G / TT; ++tile) {
        // ---------------- scores: S[n-tile][.] = A x codes
        float Sacc[S::NT][4];
#pragma unroll
        for (int i2 = 0; i2 < S::NT; ++i2) Sacc[i2][0] = Sacc[i2][1] = Sacc[i2][2] = Sacc[i2][3] = 0.f;
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {
          const int ch = 16 * (kk + (mi >> 1)) + 8 * (mi & 1) + rr;
#pragma unroll
          for (int sg = 0; sg < S::SIG; ++sg) {
            uint32_t r[4];
            ldsm_x4_t(kc_s + ch * kc_row + (tile * S::SIG + sg) * 16, r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              const uint32_t x0 = r[2 * jj], x1 = r[2 * jj + 1];
              const uint32_t x0h = x0 >> 8, x1h = x1 >> 8;
#pragma unroll
              for (int j = 0; j < S::CPT16; ++j) {
                constexpr uint32_t cm = (1u << KB) - 1;
                const int sh = (j * KB) % 8;
                const uint32_t mask = (cm << sh) | (cm << (sh + 16));
                const bool hib = j * KB >= 8;
                const uint32_t b0 = codes_to_f16(hib ? x0h : x0, mask);
                const uint32_t b1 = codes_to_f16(hib ? x1h : x1, mask);
                mma16816(Sacc[sg * S::CPT16 + j], A[kk + jj], b0, b1);
              }
            }
          }
        }
        // ---------------- online softmax over the tile (log2 units)
        float sc[S::NT][2];
        float mt = -INFINITY;
#pragma unroll
        for (int i2 = 0; i2 < S::NT; ++i2) {
          const float ks = 1.0f / (float)(1 << (((i2 % S::CPT16) * KB) % 8));
          sc[i2][0] = (Sacc[i2][0] + Sacc[i2][2]) * ks + bias;
          sc[i2][1] = (Sacc[i2][1] + Sacc[i2][3]) * ks + bias;
          mt = fmaxf(mt, fmaxf(sc[i2][0], sc[i2][1]));
        }
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        float alpha = 1.f;
        if (g < NG) {
          const float mnew = fmaxf(m_run, mt);
          alpha = ex2(m_run - mnew);
          m_run = mnew;
        }
        float pr[S::NT][2];
        float psum = 0.f;
#pragma unroll
        for (int i2 = 0; i2 < S::NT; ++i2) {
          pr[i2][0] = (g < NG) ? ex2(sc[i2][0] - m_run) : 0.f;
          pr[i2][1] = (g < NG) ? ex2(sc[i2][1] - m_run) : 0.f;
          psum += pr[i2][0] + pr[i2][1];
        }
        lsum = lsum * alpha + psum;
#pragma unroll
        for (int gg = 0; gg < NGRP; ++gg) zacc[gg] *= alpha;
        if (!__all_sync(0xffffffffu, alpha == 1.f)) {
          const float a_lo = __shfl_sync(0xffffffffu, alpha, (2 * t) * 4);
          const float a_hi = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) * 4);
#pragma unroll
          for (int i2 = 0; i2 < 8; ++i2) {
            O[i2][0] *= a_lo;
            O[i2][1] *= a_hi;
            O[i2][2] *= a_lo;
            O[i2][3] *= a_hi;
          }
        }
        // ---------------- values: O += codes x (p * s), zacc += p * z
#pragma unroll
        for (int ks2 = 0; ks2 < S::KSTEPS; ++ks2) {
          const int X = 2 * ks2, Y = 2 * ks2 + 1;
          const int tb = tile * TT;
          const int tX0 = tb + tile_token<KB, TT>(X, 2 * t), tX1 = tb + tile_token<KB, TT>(X, 2 * t + 1);
          const int tY0 = tb + tile_token<KB, TT>(Y, 2 * t), tY1 = tb + tile_token<KB, TT>(Y, 2 * t + 1);
          uint32_t B0[NGRP], B1[NGRP];
#pragma unroll
          for (int gg = 0; gg < NGRP; ++gg) {
            {
              const float2 sx0 = __half22float2(vsz[tX0 * NGRP + gg]), sx1 = __half22float2(vsz[tX1 * NGRP + gg]);
              const float2 sy0 = __half22float2(vsz[tY0 * NGRP + gg]), sy1 = __half22float2(vsz[tY1 * NGRP + gg]);
              B0[gg] = pack_f16(pr[X][0] * sx0.x, pr[X][1] * sx1.x);
              B1[gg] = pack_f16(pr[Y][0] * sy0.x, pr[Y][1] * sy1.x);
              zacc[gg] += pr[X][0] * sx0.y + pr[X][1] * sx1.y + pr[Y][0] * sy0.y + pr[Y][1] * sy1.y;
            }
          }
          const int tokl = tb + tile_token<KB, TT>((mi & 1) ? Y : X, rr);
          const uint32_t vrow = vc_s + (tokl / S::CPT16) * (mp.vseg_bytes + 16) + (tokl % S::CPT16) * S::VRB;
#pragma unroll
          for (int c = 0; c < S::NCH; c += 2) {
            uint32_t r[4];
            ldsm_x4_t(vrow + 16 * (c + (mi >> 1)), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const uint32_t xv = r[2 * cc], yv = r[2 * cc + 1];
              const uint32_t xh = xv >> 8, yh = yv >> 8;
              const int gg = ((c + cc) * S::CH_SPAN) / S::GV;
#pragma unroll
              for (int P = 0; P < S::MT_PER_CH; ++P) {
                constexpr uint32_t cm = (1u << VB) - 1;
                const int p0 = 2 * P, p1 = 2 * P + 1;
                const int sh0 = (p0 * VB) % 8, sh1 = (p1 * VB) % 8;
                const bool h0 = p0 * VB >= 8, h1 = p1 * VB >= 8;
                const uint32_t m0 = (cm << sh0) | (cm << (sh0 + 16)), m1 = (cm << sh1) | (cm << (sh1 + 16));
                uint32_t a[4];
                a[0] = codes_to_f16(h0 ? xh : xv, m0);
                a[1] = codes_to_f16(h1 ? xh : xv, m1);
                a[2] = codes_to_f16(h0 ? yh : yv, m0);
                a[3] = codes_to_f16(h1 ? yh : yv, m1);
                mma16816(O[(c + cc) * S::MT_PER_CH + P], a, B0[gg], B1[gg]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + st);
    }
  }
  if (failed) atomicOr(p.err, 1);
  __syncthreads();  // every stage is consumed and every copy has landed

  // ---------------- merge the consumer warps' states through shared memory
  float* so = reinterpret_cast<float*>(smem);  // [4][8][D]
  float* sm = so + 4 * 8 * D;                  // [4][8]
  float* sl = sm + 32;                         // [4][8]
  if (warp < kConsumerWarps) {
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
#pragma unroll
    for (int gg = 0; gg < NGRP; ++gg) {
      zacc[gg] += __shfl_xor_sync(0xffffffffu, zacc[gg], 1);
      zacc[gg] += __shfl_xor_sync(0xffffffffu, zacc[gg], 2);
    }
    const int h_lo = 2 * t, h_hi = 2 * t + 1;
#pragma unroll
    for (int mt2 = 0; mt2 < 8; ++mt2) {
      const int c = mt2 / S::MT_PER_CH, P = mt2 % S::MT_PER_CH;
      const int gg = (c * S::CH_SPAN) / S::GV;
      const float z_lo = __shfl_sync(0xffffffffu, zacc[gg], h_lo * 4);
      const float z_hi = __shfl_sync(0xffffffffu, zacc[gg], h_hi * 4);
      const int p0 = 2 * P, p1 = 2 * P + 1;
      const float rs0 = 1.0f / (float)(1 << ((p0 * VB) % 8)), rs1 = 1.0f / (float)(1 << ((p1 * VB) % 8));
      const int ch0 = c * S::CH_SPAN + g * S::VCPC + p0;
      if (h_lo < NG) {
        so[(warp * 8 + h_lo) * D + ch0] = O[mt2][0] * rs0 + z_lo;
        so[(warp * 8 + h_lo) * D + ch0 + 1] = O[mt2][2] * rs1 + z_lo;
      }
      if (h_hi < NG) {
        so[(warp * 8 + h_hi) * D + ch0] = O[mt2][1] * rs0 + z_hi;
        so[(warp * 8 + h_hi) * D + ch0 + 1] = O[mt2][3] * rs1 + z_hi;
      }
    }
    if (t == 0 && g < NG) {
      sm[warp * 8 + g] = m_run;
      sl[warp * 8 + g] = lsum;
    }
  }
  __syncthreads();
  const int d = threadIdx.x;
  if (d < D) {
    for (int hh = 0; hh < NG; ++hh) {
      float M = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm[w * 8 + hh]);
      float acc = 0.f, ls = 0.f;
      if (M != -INFINITY) {
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float mw = sm[w * 8 + hh];
          if (mw == -INFINITY) continue;
          const float f = ex2(mw - M);
          acc += so[(w * 8 + hh) * D + d] * f;
          ls += sl[w * 8 + hh] * f;
        }
      }
      const int64_t slot = ((int64_t)b * p.num_q_heads + h * NG + hh) * p.slots + s;
      p.ws_o[slot * D + d] = acc;
      if (d == 0) p.ws_ml[slot] = make_float2(M, ls);
    }
  }
}

template <int KB, int VB, int NGRP>
cudaError_t launch_mma_inst(const DecodeParams& p, const MmaPlan& mp, int max_splits, cudaStream_t stream) {
  auto kern = decode_mma_kernel<KB, VB, 64, NGRP>;
  static uint64_t attr_mask = 0;  // shared-memory opt-in per device
  static int attr_bytes[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_mask & (1ull << dev)) || attr_bytes[dev] < mp.smem_bytes) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mp.smem_bytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) {
      attr_mask |= 1ull << dev;
      attr_bytes[dev] = mp.smem_bytes;
    }
  }
  dim3 grid(max_splits + 1, p.L.num_kv_heads, p.batch);
  kern<<<grid, kThreads, mp.smem_bytes, stream>>>(p, mp);
  return cudaGetLastError();
}

// Every supported (key bits, value bits, value groups per head) instance.
#define KVQ_MMA_INSTANCES(X)                                                                    \
  X(2, 2, 1) X(2, 2, 2) X(2, 4, 1) X(2, 4, 2) X(2, 4, 4) X(2, 8, 1) X(2, 8, 2) X(2, 8, 4)     \
  X(4, 2, 1) X(4, 2, 2) X(4, 4, 1) X(4, 4, 2) X(4, 4, 4) X(4, 8, 1) X(4, 8, 2) X(4, 8, 4)     \
  X(8, 2, 1) X(8, 2, 2) X(8, 4, 1) X(8, 4, 2) X(8, 4, 4) X(8, 8, 1) X(8, 8, 2) X(8, 8, 4)

}  // namespace

bool mma_supported(const LayerView& L) {
  if (L.head_dim != kHeadDim) return false;
  if (L.group_k < 64) return false;                     // tiles of 64 tokens
  if (L.v_bits == 2 && L.group_v < 64) return false;    // a value chunk spans 64 channels
  return true;
}

MmaPlan make_mma_plan(const LayerView& L) {
  MmaPlan mp;
  const int G = L.group_k, D = L.head_dim, kb = L.k_bits, vb = L.v_bits;
  mp.kc_bytes = G * kb / 8 * D;
  const int cpt16 = 16 / kb;
  mp.vseg_bytes = cpt16 * (D * vb / 8);
  mp.vseg_count = G / cpt16;
  mp.vsz_bytes = G * (D / L.group_v) * 4;
  mp.vc_soff = mp.kc_bytes + D * 4;
  mp.vsz_soff = mp.vc_soff + mp.vseg_count * (mp.vseg_bytes + 16);
  mp.stage_bytes = mp.vsz_soff + mp.vsz_bytes;
  mp.tx_bytes = mp.kc_bytes + D * 4 + mp.vseg_count * mp.vseg_bytes + mp.vsz_bytes;
  const int merge_bytes = (8 * D + 4 * 8 * D + 64) * 4;  // residual split / final merge
  int ns = (72 * 1024) / mp.stage_bytes;
  if (ns < 4) ns = 4;
  if (ns > 16) ns = 16;
  while (ns * mp.stage_bytes < merge_bytes) ++ns;
  mp.nstages = ns;
  mp.bar_off = ns * mp.stage_bytes;
  mp.smem_bytes = mp.bar_off + 2 * ns * 8;
  return mp;
}

cudaError_t launch_decode_mma(const DecodeParams& p, const MmaPlan& mp, int max_splits, cudaStream_t stream) {
  const int kb = p.L.k_bits, vb = p.L.v_bits, ng = kHeadDim / p.L.group_v;
#define KVQ_CASE(K, V, N) \
  if (kb == K && vb == V && ng == N) return launch_mma_inst<K, V, N>(p, mp, max_splits, stream);
  KVQ_MMA_INSTANCES(KVQ_CASE)
#undef KVQ_CASE
  return cudaErrorInvalidValue;
}

int mma_ctas_per_sm(const LayerView& L, const MmaPlan& mp) {
  int n = 0;
  const void* fn = nullptr;
  const int kb = L.k_bits, vb = L.v_bits, ng = kHeadDim / L.group_v;
#define KVQ_FN(K, V, N) \
  if (kb == K && vb == V && ng == N) fn = (const void*)decode_mma_kernel<K, V, 64, N>;
  KVQ_MMA_INSTANCES(KVQ_FN)
#undef KVQ_FN
  if (!fn) return 1;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, mp.smem_bytes) != cudaSuccess) return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, mp.smem_bytes) != cudaSuccess || n < 1) return 1;
  return n;
}

}  // namespace kvq
