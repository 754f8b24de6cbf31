// Tensor-core split-KV decode attention over the packed cache (sm_100a).
//
// Method: decoding over per-channel-quantized keys and per-token-quantized
// values plus the full-precision residual window ("KIVI" README, Overview;
// GQA update), with x_hat = q*d + m ("KV1-1.2B" card, BQ2_0).
//
// Design (HBM-bound; tensor cores only take the dot products off the ALUs):
//  * One CTA per (split, KV head, sequence); split 0 is the residual ring.
//    Warp roles: a producer warp (one lane) streams each block record from
//    HBM into a ring of shared-memory stages with ONE cp.async.bulk (1-D TMA)
//    completing on an mbarrier -- the record layout is already the
//    bank-conflict-free shared-memory layout, so no per-row copies are
//    needed; a prep warp turns each landed block's fp16 scales into the
//    per-block operands (below) next to the record; NC consumer warps each
//    own NS/NC stages. Stage hand-offs: full (TMA landed) -> ready (operands
//    prepared) -> empty (consumed).
//  * Keys: per block, q.k_hat = sum_d (q_d s_d) c_d + sum_d q_d z_d. The
//    scaled query (q_d s_d) is split into fp16 high and low parts, rows 0-7
//    and 8-15 of the m16n8k16 A operand (the prep warp writes them in
//    fragment order), the codes c are the B operand. Codes reach registers
//    with ldmatrix.trans from the channel-major key rows (two channels of the
//    same tokens per register) and become exact fp16 integers with one lop3
//    (mask | 0x6400 exponent) and one hsub2 (minus 1024). A code taken from
//    bit position p is c * 2^p; the score is rescaled by 2^-p (exact).
//  * Values: o[ch][head] = sum_t (p_t s_t) c_t,ch + sum_t p_t z_t. The value
//    codes of two tokens per register come from ldmatrix.trans over token
//    rows (the A operand, channels on M); p*s in fp16 (one hmul2 of the
//    packed probabilities and the prep warp's packed scales) is the B operand
//    (tokens on K, heads on N) built straight from the score accumulators'
//    registers. The zero-point term sum_t p_t z_t is one more MMA per value
//    group with an all-ones A operand.
//  * Online softmax in log2 units per 64-token tile; fp32 partials per split
//    are merged by the log-sum-exp combine kernel.
#include <mutex>

#include "kvq_decode.cuh"

namespace kvq {

namespace {

constexpr int kNC = 4;                    // consumer warps
constexpr int kProdWarp = kNC;            // warp index of the producer warp
constexpr int kThreads = (kNC + 1) * 32;
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
// Not volatile: the compiler may schedule these freely. ldmatrix keeps a
// memory clobber so that it stays behind the barrier waits that publish the
// shared memory it reads.
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr)
      : "memory");
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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
// Codes selected by `mask` in both 16-bit halves of x, as exact fp16 integers
// (times the power of two of their bit position): (x & mask) | 1024.0h, then
// minus 1024.0h.
__device__ __forceinline__ uint32_t codes_to_f16(uint32_t x, uint32_t mask, uint32_t magic) {
  uint32_t r = and_or(x, mask, magic);
  __half2 h = *reinterpret_cast<__half2*>(&r);
  h = __hsub2(h, *reinterpret_cast<const __half2*>(&magic));
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_f16(uint32_t x) {
  return __half22float2(*reinterpret_cast<__half2*>(&x));
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// ------------------------------------------------------- residual ring split
// Exact attention over the ring tokens [Q, Q+n) of unit (b, h) by the 128
// consumer threads (named barrier 1), in chunks of up to 128 tokens staged
// in shared memory with cp.async (16-byte rows chunks stored at position
// j ^ (row & 15), so per-row reads are bank-conflict-free):
//   q.k: thread tau owns token tau of the chunk; p.v: thread d owns channel d.
// Writes one partial (slot 0). Scratch (bytes): tile [128][256], q [8][128]
// fp32, p [8][128] fp32, red [4][8][2] fp32.
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kNC * 32) : "memory"); }
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void bf16x8_or_f16x8(const uint4& v, int dtype, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (dtype == KVQ_BF16) {
      f[2 * e] = __uint_as_float(w[e] << 16);
      f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    } else {
      const float2 x = unpack_f16(w[e]);
      f[2 * e] = x.x;
      f[2 * e + 1] = x.y;
    }
  }
}
constexpr int kResTile = 128;                       // ring tokens per chunk
constexpr int kResScratch = kResTile * 256 + 2 * 8 * 128 * 4 + 4 * 8 * 2 * 4;

__device__ void residual_unit(const DecodeParams& p, int b, int h, int NG, uint8_t* scratch) {
  const LayerView& L = p.L;
  constexpr int D = kHeadDim;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint4* tile = reinterpret_cast<uint4*>(scratch);                     // [128 rows][16 chunks]
  float* sq = reinterpret_cast<float*>(scratch + kResTile * 256);      // [8][D]
  float* sp = sq + 8 * D;                                              // [8][kResTile]
  float* red = sp + 8 * kResTile;                                      // [4][8][2]
  const int Q = L.lens[2 * b], n = L.lens[2 * b + 1];
  const int dt = L.kv_dtype;
  const int64_t ring = ((int64_t)b * L.num_kv_heads + h) * L.residual;
  consumers_sync();  // scratch is free
  for (int e = tid; e < NG * D; e += kNC * 32)
    sq[e] = load_kv(p.q, ((int64_t)b * p.num_q_heads + h * NG) * D + e, dt) * p.scale_log2;
  float m[8], l[8], o[8];  // per head; o for channel d = tid
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
    o[hh] = 0.f;
  }
  for (int c0 = 0; c0 < n; c0 += kResTile) {
    const int cnt = min(kResTile, n - c0);
    // ---- keys of the chunk
    if (tid < cnt) {
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(L.ring_k) +
                                                        (ring + (Q + c0 + tid) % L.residual) * D);
#pragma unroll
      for (int j = 0; j < 16; ++j) cp_async16(tile + tid * 16 + (j ^ (tid & 15)), src + j);
    }
    cp_async_wait_all();
    consumers_sync();
    float sc[8];
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) sc[hh] = 0.f;
    if (tid < cnt) {
#pragma unroll 4
      for (int j = 0; j < 16; ++j) {
        float kf[8];
        bf16x8_or_f16x8(tile[tid * 16 + (j ^ (tid & 15))], dt, kf);
#pragma unroll
        for (int hh = 0; hh < 8; ++hh) {
          if (hh < NG) {
            const float4 qa = reinterpret_cast<const float4*>(sq + hh * D + 8 * j)[0];
            const float4 qb = reinterpret_cast<const float4*>(sq + hh * D + 8 * j)[1];
            sc[hh] += qa.x * kf[0] + qa.y * kf[1] + qa.z * kf[2] + qa.w * kf[3] + qb.x * kf[4] + qb.y * kf[5] +
                      qb.z * kf[6] + qb.w * kf[7];
          }
        }
      }
    }
    // ---- chunk max and new running max per head
    float cm[8];
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      cm[hh] = (tid < cnt) ? sc[hh] : -INFINITY;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) cm[hh] = fmaxf(cm[hh], __shfl_xor_sync(0xffffffffu, cm[hh], off));
    }
    if (lane == 0)
#pragma unroll
      for (int hh = 0; hh < 8; ++hh) red[(warp * 8 + hh) * 2] = cm[hh];
    consumers_sync();  // keys done (the tile can take the values), maxima visible
    if (tid < cnt) {
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(L.ring_v) +
                                                        (ring + (Q + c0 + tid) % L.residual) * D);
#pragma unroll
      for (int j = 0; j < 16; ++j) cp_async16(tile + tid * 16 + (j ^ (tid & 15)), src + j);
    }
    float alpha[8], ps[8];
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      const float M = fmaxf(fmaxf(red[hh * 2], red[(8 + hh) * 2]), fmaxf(red[(16 + hh) * 2], red[(24 + hh) * 2]));
      const float mn = fmaxf(m[hh], M);
      alpha[hh] = (hh < NG) ? ex2(m[hh] - mn) : 1.f;
      m[hh] = (hh < NG) ? mn : m[hh];
      const float pv = (tid < cnt && hh < NG) ? ex2(sc[hh] - mn) : 0.f;
      if (tid < kResTile && hh < NG) sp[hh * kResTile + tid] = pv;
      ps[hh] = pv;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ps[hh] += __shfl_xor_sync(0xffffffffu, ps[hh], off);
    }
    cp_async_wait_all();
    consumers_sync();  // sums of the previous reads done; reuse red for the sums
    if (lane == 0)
#pragma unroll
      for (int hh = 0; hh < 8; ++hh) red[(warp * 8 + hh) * 2 + 1] = ps[hh];
    consumers_sync();  // values, probabilities and sums visible
    const int d = tid;  // channel owned for p.v
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      if (hh < NG) {
        l[hh] = l[hh] * alpha[hh] + red[hh * 2 + 1] + red[(8 + hh) * 2 + 1] + red[(16 + hh) * 2 + 1] +
                red[(24 + hh) * 2 + 1];
        o[hh] *= alpha[hh];
      }
    }
    const uint16_t* vrow = reinterpret_cast<const uint16_t*>(tile);
    for (int tau = 0; tau < cnt; ++tau) {
      const uint16_t bits = vrow[(tau * 16 + ((d >> 3) ^ (tau & 15))) * 8 + (d & 7)];
      const float vf = (dt == KVQ_BF16) ? __uint_as_float((uint32_t)bits << 16) : __half2float(__ushort_as_half(bits));
#pragma unroll
      for (int hh = 0; hh < 8; ++hh)
        if (hh < NG) o[hh] += sp[hh * kResTile + tau] * vf;
    }
    consumers_sync();  // tile and sp free for the next chunk
  }
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    if (hh < NG) {
      const int64_t slot = ((int64_t)b * p.num_q_heads + h * NG + hh) * p.slots;
      p.ws_o[slot * D + tid] = o[hh];
      if (tid == 0) p.ws_ml[slot] = make_float2(m[hh], l[hh]);
    }
  }
}

// --------------------------------------------------------- quantized blocks
template <int KB, int VB, int NGRP>
struct Shape {
  static constexpr int D = kHeadDim;
  static constexpr int TT = 64;                 // tokens per tile
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

// Token (within the tile) of column `col` of n-tile `idx`.
template <int KB>
__device__ __forceinline__ int tile_token(int idx, int col) {
  constexpr int CPT16 = 16 / KB, SIGMA_TOK = 128 / KB;
  return (idx / CPT16) * SIGMA_TOK + col * CPT16 + (idx % CPT16);
}

// Walks the (sequence, head) units of consecutive global blocks.
struct UnitCursor {
  int b = 0, h = 0, start = 0, end = 0;  // current unit and its block range
  __device__ void seek(const DecodeParams& p, int k) {
    int lo = 0, hi = p.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.seq_start[mid] <= k) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    const int nb = p.nblk[b];
    h = (k - p.seq_start[b]) / nb;
    start = p.seq_start[b] + h * nb;
    end = start + nb;
  }
  __device__ void advance(const DecodeParams& p, int k) {
    if (k >= end || k < start) seek(p, k);
  }
};

// Per-warp scratch, rebuilt from each block's fp16 scales before its MMAs:
//   afrag [8 kk][32 slots] uint4: slot (g*4 + t) ^ kk holds rows g (fp16
//         high) and g+8 (fp16 low) of (q * s) for channels 16kk + 2t +
//         {0,1,8,9} (A-fragment order; the XOR keeps both the writes and the
//         reads of a k-chunk spread over all shared-memory banks);
//   bias  [8] float: sum_d q_d z_d per head;
//   vpair [k-step][4 t][groups] uint4: (s_X, s_Y, z_X, z_Y) fp16 pairs of the
//         tokens thread t feeds into a PV k-step;
//   wq    [8 kk][8 heads][4 x 16 B] float: the unit's queries times
//         softmax_scale*log2(e), k-chunk-major; piece v of row (kk, head) is
//         stored at v ^ (kk & 3) so the prep's reads spread over all banks.
template <int KB, int VB, int NGRP>
__device__ __forceinline__ void prep_block(const uint8_t* stage, const MmaPlan& mp, uint8_t* ws, int NG, int G,
                                           int lane) {
  using S = Shape<KB, VB, NGRP>;
  constexpr int D = S::D;
  const float* wq = reinterpret_cast<const float*>(ws + mp.wq_off);
  uint4* af = reinterpret_cast<uint4*>(ws + mp.afrag_off);
  const __half2* ksz = reinterpret_cast<const __half2*>(stage + mp.kc_bytes);
  // (head, kk) pairs: lanes 8hh..8hh+7 take the 8 kk of head hh
#pragma unroll
  for (int rep = 0; rep < 2; ++rep) {
    const int pr = lane + 32 * rep;
    const int hh = pr >> 3, kk = pr & 7;
    float bp = 0.f;
    if (hh < NG) {
      const float4* q4 = reinterpret_cast<const float4*>(wq + (kk * 8 + hh) * 16);
      const uint4* s4 = reinterpret_cast<const uint4*>(ksz + 16 * kk);
      float x[16];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 qq = q4[v ^ (kk & 3)];  // wq rows are stored XOR-swizzled by kk
        const uint4 ss = s4[v];
        const float qa[4] = {qq.x, qq.y, qq.z, qq.w};
        const uint32_t sa[4] = {ss.x, ss.y, ss.z, ss.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 sz = unpack_f16(sa[e]);  // (scale, zero) of channel 16kk + 4v + e
          x[4 * v + e] = qa[e] * sz.x;
          bp += qa[e] * sz.y;
        }
      }
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const uint32_t h01 = pack_f16(x[2 * tt], x[2 * tt + 1]), h89 = pack_f16(x[2 * tt + 8], x[2 * tt + 9]);
        const float2 f01 = unpack_f16(h01), f89 = unpack_f16(h89);
        af[kk * 32 + ((hh * 4 + tt) ^ kk)] = make_uint4(h01, pack_f16(x[2 * tt] - f01.x, x[2 * tt + 1] - f01.y), h89,
                                                        pack_f16(x[2 * tt + 8] - f89.x, x[2 * tt + 9] - f89.y));
      }
    }
    if (rep == 1 && NG <= 4) break;
    bp += __shfl_xor_sync(0xffffffffu, bp, 1);
    bp += __shfl_xor_sync(0xffffffffu, bp, 2);
    bp += __shfl_xor_sync(0xffffffffu, bp, 4);
    if (kk == 0 && hh < NG) reinterpret_cast<float*>(ws + mp.bias_off)[hh] = bp;
  }
  const __half* vsz = reinterpret_cast<const __half*>(stage + mp.vsz_soff);
  uint4* vp = reinterpret_cast<uint4*>(ws + mp.vpair_off);
  const int nvp = (G / 16) * 4 * NGRP;
  for (int e = lane; e < nvp; e += 32) {
    const int gg = e % NGRP, tq = (e / NGRP) & 3, kst = e / (NGRP * 4);
    const int tile = kst / S::KSTEPS, ks2 = kst % S::KSTEPS;
    const int tb = tile * S::TT;
    const int tx0 = tb + tile_token<KB>(2 * ks2, 2 * tq), tx1 = tb + tile_token<KB>(2 * ks2, 2 * tq + 1);
    const int ty0 = tb + tile_token<KB>(2 * ks2 + 1, 2 * tq), ty1 = tb + tile_token<KB>(2 * ks2 + 1, 2 * tq + 1);
    const uint32_t ax = *reinterpret_cast<const uint32_t*>(vsz + (tx0 * NGRP + gg) * 2);
    const uint32_t bx = *reinterpret_cast<const uint32_t*>(vsz + (tx1 * NGRP + gg) * 2);
    const uint32_t ay = *reinterpret_cast<const uint32_t*>(vsz + (ty0 * NGRP + gg) * 2);
    const uint32_t by = *reinterpret_cast<const uint32_t*>(vsz + (ty1 * NGRP + gg) * 2);
    // (s, z) halves of two tokens -> (s0, s1) and (z0, z1)
    vp[e] = make_uint4(__byte_perm(ax, bx, 0x5410), __byte_perm(ay, by, 0x5410), __byte_perm(ax, bx, 0x7632),
                       __byte_perm(ay, by, 0x7632));
  }
  __syncwarp();
}

template <int KB, int VB, int NGRP>
__global__ void __launch_bounds__(kThreads) decode_mma_kernel(DecodeParams p, MmaPlan mp) {
  using S = Shape<KB, VB, NGRP>;
  constexpr int D = S::D;
  extern __shared__ __align__(128) uint8_t smem[];
  const int c = blockIdx.x;
  const LayerView& L = p.L;
  const int NG = p.num_q_heads / L.num_kv_heads;
  const int G = L.group_k;
  const int T = p.total_blocks;
  const int rs = cta_first_block(T, p.num_ctas, c), re = cta_first_block(T, p.num_ctas, c + 1);
  const int nb = re - rs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NS = mp.nstages;
  const int stage_bytes = mp.stage_bytes;
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
  bool failed = false;

  if (warp == kProdWarp) {
    // ---------------- producer: one lane streams this CTA's block records
    if (lane == 0) {
      UnitCursor u;
      int issued = 0;
      for (int i = 0; i < nb; ++i) {
        const int st = i % NS;
        if (i >= NS && !mbar_wait(empty + st, ((i / NS) & 1) ^ 1)) {
          failed = true;
          break;
        }
        const int k = rs + i;
        u.advance(p, k);
        mbar_expect_tx(full + st, mp.tx_bytes);
        bulk_g2s(smem + (size_t)st * stage_bytes, record_ptr(L, u.b, u.h, k - u.start), mp.tx_bytes, full + st);
        issued = i + 1;
      }
      // Let every copy land before the CTA may leave.
      for (int i = max(0, issued - NS); i < issued; ++i)
        if (!mbar_wait(full + i % NS, (i / NS) & 1)) failed = true;
    }
  } else {
    // ---------------- consumers
    uint8_t* ws = smem + mp.ws_soff + warp * mp.ws_bytes;
    float* wq = reinterpret_cast<float*>(ws + mp.wq_off);
    auto stage_q = [&](int b, int h) {  // the unit's scaled queries into wq
      __syncwarp();
      // NG*D 16-bit values = NG*16 16-byte vectors; at most 4 per lane, all
      // loads issued before any is used
      const uint4* src =
          reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.q) + ((int64_t)b * p.num_q_heads + h * NG) * D);
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (lane + 32 * i < NG * 16) v[i] = src[lane + 32 * i];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (lane + 32 * i < NG * 16) {
          const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
          float f[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (L.kv_dtype == KVQ_BF16) {
              f[2 * e] = __uint_as_float(w[e] << 16);
              f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
            } else {
              const float2 x = unpack_f16(w[e]);
              f[2 * e] = x.x;
              f[2 * e + 1] = x.y;
            }
          }
          const int e16 = lane + 32 * i;  // 8 channels: head e16/16, channels (e16%16)*8..
          const int hh = e16 >> 4, kk = (e16 & 15) >> 1, v0 = (e16 & 1) * 2;
          float4* row = reinterpret_cast<float4*>(wq + (kk * 8 + hh) * 16);
          row[v0 ^ (kk & 3)] =
              make_float4(f[0] * p.scale_log2, f[1] * p.scale_log2, f[2] * p.scale_log2, f[3] * p.scale_log2);
          row[(v0 + 1) ^ (kk & 3)] =
              make_float4(f[4] * p.scale_log2, f[5] * p.scale_log2, f[6] * p.scale_log2, f[7] * p.scale_log2);
        }
      }
      __syncwarp();
    };
    // residual units of this CTA first (the producer already streams); the
    // consumer scratch areas, contiguous, serve as the ring tile buffer
    for (int r = c; r < p.batch * L.num_kv_heads; r += p.num_ctas)
      residual_unit(p, r / L.num_kv_heads, r % L.num_kv_heads, NG, smem + mp.ws_soff);
    __syncwarp();
    consumers_sync();  // the scratch areas are per warp again
    {  // rows of heads >= NG stay zero
      uint4* af = reinterpret_cast<uint4*>(ws + mp.afrag_off);
      for (int e = lane; e < 8 * 8 * 4; e += 32)  // e = kk*32 + physical slot
        if (((((e & 31) ^ (e >> 5)) >> 2) & 7) >= NG) af[e] = make_uint4(0u, 0u, 0u, 0u);
    }

    const int g = lane >> 2, t = lane & 3;
    const uint32_t magic = 0x64006400u;
    const uint32_t ones[4] = {0x3c003c00u, 0x3c003c00u, 0x3c003c00u, 0x3c003c00u};  // fp16 1.0
    const int kc_row = G * KB / 8;  // key code bytes per channel
    const int ncol = G / S::CPT16;  // value rows per key-column position
    const int mi = lane >> 3, rr = lane & 7;
    // ldmatrix rows of this lane: 8 consecutive rows, so the chunk swizzle of
    // the record layout depends on the lane's row index only
    const int swk = chunk_swizzle(rr, kc_row / 16);
    const int swv = chunk_swizzle(rr, S::VRB / 16);
    const uint4* afr = reinterpret_cast<const uint4*>(ws + mp.afrag_off);
    const uint4* vpr = reinterpret_cast<const uint4*>(ws + mp.vpair_off);
    const float* biasr = reinterpret_cast<const float*>(ws + mp.bias_off);
    UnitCursor u;
    int k = rs;
    while (k < re && !failed) {
      u.advance(p, k);
      const int hi = min(u.end, re);
      stage_q(u.b, u.h);
      float lsum = 0.f, m_run = (g < NG) ? -INFINITY : 0.f;
      float O[8][4], Z[NGRP][4];
#pragma unroll
      for (int i2 = 0; i2 < 8; ++i2) O[i2][0] = O[i2][1] = O[i2][2] = O[i2][3] = 0.f;
#pragma unroll
      for (int gg = 0; gg < NGRP; ++gg) Z[gg][0] = Z[gg][1] = Z[gg][2] = Z[gg][3] = 0.f;
      // this warp's blocks of the unit: i = kb - rs with i % kNC == warp
      const int first = k + ((warp - (k - rs)) % kNC + kNC) % kNC;
      for (int kb = first; kb < hi; kb += kNC) {
        const int i = kb - rs;
        const int st = i % NS;
        if (!mbar_wait(full + st, (i / NS) & 1)) {
          failed = true;
          break;
        }
        const uint8_t* stage = smem + (size_t)st * stage_bytes;
        prep_block<KB, VB, NGRP>(stage, mp, ws, NG, G, lane);
        const float bias = (g < NG) ? biasr[g] : 0.f;
        const uint32_t kc_s = smem_u32(stage);
        const uint32_t vc_s = smem_u32(stage + mp.vc_soff);

        for (int tile = 0; tile < G / S::TT; ++tile) {
          // ---------------- scores: S[n-tile][.] = A x codes
          float Sacc[S::NT][4];
#pragma unroll
          for (int i2 = 0; i2 < S::NT; ++i2) Sacc[i2][0] = Sacc[i2][1] = Sacc[i2][2] = Sacc[i2][3] = 0.f;
          // all key code loads of the tile first (one ldmatrix.x4 per k-chunk
          // pair and 16-byte chunk), then the conversions and MMAs
          uint32_t rk[4][S::SIG][4];
#pragma unroll
          for (int kp = 0; kp < 4; ++kp) {
            const int ch = 16 * (2 * kp + (mi >> 1)) + 8 * (mi & 1) + rr;
#pragma unroll
            for (int sg = 0; sg < S::SIG; ++sg)
              ldsm_x4_t(kc_s + ch * kc_row + (((tile * S::SIG + sg) ^ swk) << 4), rk[kp][sg][0], rk[kp][sg][1],
                        rk[kp][sg][2], rk[kp][sg][3]);
          }
#pragma unroll
          for (int kk = 0; kk < 8; kk += 2) {
#pragma unroll
            for (int sg = 0; sg < S::SIG; ++sg) {
              const uint32_t* r = rk[kk / 2][sg];
#pragma unroll
              for (int jj = 0; jj < 2; ++jj) {
                const uint4 av = afr[(kk + jj) * 32 + ((g * 4 + t) ^ (kk + jj))];
                const uint32_t A[4] = {av.x, av.y, av.z, av.w};
                const uint32_t x0 = r[2 * jj], x1 = r[2 * jj + 1];
                const uint32_t x0h = x0 >> 8, x1h = x1 >> 8;
#pragma unroll
                for (int j = 0; j < S::CPT16; ++j) {
                  constexpr uint32_t cm = (1u << KB) - 1;
                  const int sh = (j * KB) % 8;
                  const uint32_t mask = (cm << sh) | (cm << (sh + 16));
                  const bool hib = j * KB >= 8;
                  const uint32_t b0 = codes_to_f16(hib ? x0h : x0, mask, magic);
                  const uint32_t b1 = codes_to_f16(hib ? x1h : x1, mask, magic);
                  mma16816(Sacc[sg * S::CPT16 + j], A, b0, b1);
                }
              }
            }
          }
          // ---------------- online softmax over the tile (log2 units)
          float pr[S::NT][2];
          float mt = -INFINITY;
#pragma unroll
          for (int i2 = 0; i2 < S::NT; ++i2) {
            const float ks = 1.0f / (float)(1 << (((i2 % S::CPT16) * KB) % 8));
            pr[i2][0] = (Sacc[i2][0] + Sacc[i2][2]) * ks + bias;
            pr[i2][1] = (Sacc[i2][1] + Sacc[i2][3]) * ks + bias;
            mt = fmaxf(mt, fmaxf(pr[i2][0], pr[i2][1]));
          }
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
          float alpha = 1.f;
          if (g < NG) {
            const float mnew = fmaxf(m_run, mt);
            alpha = ex2(m_run - mnew);
            m_run = mnew;
          }
          float psum = 0.f;
#pragma unroll
          for (int i2 = 0; i2 < S::NT; ++i2) {
            pr[i2][0] = (g < NG) ? ex2(pr[i2][0] - m_run) : 0.f;
            pr[i2][1] = (g < NG) ? ex2(pr[i2][1] - m_run) : 0.f;
            psum += pr[i2][0] + pr[i2][1];
          }
          lsum = lsum * alpha + psum;
          if (!__all_sync(0xffffffffu, alpha == 1.f)) {
            const float a_lo = __shfl_sync(0xffffffffu, alpha, (2 * t) * 4);
            const float a_hi = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) * 4);
#pragma unroll
            for (int gg = 0; gg < NGRP; ++gg) {
              Z[gg][0] *= a_lo;
              Z[gg][1] *= a_hi;
              Z[gg][2] *= a_lo;
              Z[gg][3] *= a_hi;
            }
#pragma unroll
            for (int i2 = 0; i2 < 8; ++i2) {
              O[i2][0] *= a_lo;
              O[i2][1] *= a_hi;
              O[i2][2] *= a_lo;
              O[i2][3] *= a_hi;
            }
          }
          // ---------------- values: O += codes x (p * s), Z += ones x (p * z)
#pragma unroll
          for (int ks2 = 0; ks2 < S::KSTEPS; ++ks2) {
            const int X = 2 * ks2, Y = 2 * ks2 + 1;
            const int tb = tile * S::TT;
            const uint32_t pX = pack_f16(pr[X][0], pr[X][1]), pY = pack_f16(pr[Y][0], pr[Y][1]);
            uint32_t B0[NGRP], B1[NGRP];
#pragma unroll
            for (int gg = 0; gg < NGRP; ++gg) {
              const uint4 v4 = vpr[((tile * S::KSTEPS + ks2) * 4 + t) * NGRP + gg];
              B0[gg] = hmul2(pX, v4.x);
              B1[gg] = hmul2(pY, v4.y);
              mma16816(Z[gg], ones, hmul2(pX, v4.z), hmul2(pY, v4.w));
            }
            const int tokl = tb + tile_token<KB>((mi & 1) ? Y : X, rr);
            const uint32_t vrow = vc_s + ((tokl % S::CPT16) * ncol + tokl / S::CPT16) * S::VRB;
#pragma unroll
            for (int cc0 = 0; cc0 < S::NCH; cc0 += 2) {
              uint32_t r[4];
              ldsm_x4_t(vrow + (((cc0 + (mi >> 1)) ^ swv) << 4), r[0], r[1], r[2], r[3]);
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                const uint32_t xv = r[2 * cc], yv = r[2 * cc + 1];
                const uint32_t xh = xv >> 8, yh = yv >> 8;
                const int gg = ((cc0 + cc) * S::CH_SPAN) / S::GV;
#pragma unroll
                for (int P = 0; P < S::MT_PER_CH; ++P) {
                  constexpr uint32_t cm = (1u << VB) - 1;
                  const int p0 = 2 * P, p1 = 2 * P + 1;
                  const int sh0 = (p0 * VB) % 8, sh1 = (p1 * VB) % 8;
                  const bool h0 = p0 * VB >= 8, h1 = p1 * VB >= 8;
                  const uint32_t m0 = (cm << sh0) | (cm << (sh0 + 16)), m1 = (cm << sh1) | (cm << (sh1 + 16));
                  uint32_t a[4];
                  a[0] = codes_to_f16(h0 ? xh : xv, m0, magic);
                  a[1] = codes_to_f16(h1 ? xh : xv, m1, magic);
                  a[2] = codes_to_f16(h0 ? yh : yv, m0, magic);
                  a[3] = codes_to_f16(h1 ? yh : yv, m1, magic);
                  mma16816(O[(cc0 + cc) * S::MT_PER_CH + P], a, B0[gg], B1[gg]);
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + st);
      }
      // ---------------- this warp's partial for the unit
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
      const int slot = kResidualSlots + 4 * (c - cta_of_block(T, p.num_ctas, u.start)) + warp;
      const int h_lo = 2 * t, h_hi = 2 * t + 1;
      const int64_t base_lo = ((int64_t)u.b * p.num_q_heads + u.h * NG + h_lo) * p.slots + slot;
      const int64_t base_hi = ((int64_t)u.b * p.num_q_heads + u.h * NG + h_hi) * p.slots + slot;
#pragma unroll
      for (int mt2 = 0; mt2 < 8; ++mt2) {
        const int cch = mt2 / S::MT_PER_CH, P = mt2 % S::MT_PER_CH;
        const int gg = (cch * S::CH_SPAN) / S::GV;
        const int p0 = 2 * P, p1 = 2 * P + 1;
        const float rs0 = 1.0f / (float)(1 << ((p0 * VB) % 8)), rs1 = 1.0f / (float)(1 << ((p1 * VB) % 8));
        const int ch0 = cch * S::CH_SPAN + g * S::VCPC + p0;
        if (h_lo < NG) {
          p.ws_o[base_lo * D + ch0] = O[mt2][0] * rs0 + Z[gg][0];
          p.ws_o[base_lo * D + ch0 + 1] = O[mt2][2] * rs1 + Z[gg][0];
        }
        if (h_hi < NG) {
          p.ws_o[base_hi * D + ch0] = O[mt2][1] * rs0 + Z[gg][1];
          p.ws_o[base_hi * D + ch0 + 1] = O[mt2][3] * rs1 + Z[gg][1];
        }
      }
      if (t == 0 && g < NG)
        p.ws_ml[((int64_t)u.b * p.num_q_heads + u.h * NG + g) * p.slots + slot] = make_float2(m_run, lsum);
      k = hi;
    }
  }
  if (failed) atomicOr(p.err, 1);
  __syncthreads();  // every stage is consumed and every copy has landed
}

template <int KB, int VB, int NGRP>
cudaError_t launch_mma_inst(const DecodeParams& p, const MmaPlan& mp, int max_splits, cudaStream_t stream) {
  auto kern = decode_mma_kernel<KB, VB, NGRP>;
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
  (void)max_splits;
  kern<<<p.num_ctas, kThreads, mp.smem_bytes, stream>>>(p, mp);
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
  const int G = L.group_k, D = L.head_dim;
  const int ngrp = D / L.group_v;
  mp.tx_bytes = L.vsz_off + G * ngrp * 4;          // kc | ksz | vc | vsz, one copy
  mp.kc_bytes = L.ksz_off;
  mp.vc_soff = L.vc_off;
  mp.vsz_soff = L.vsz_off;
  mp.stage_bytes = (int32_t)round_up(mp.tx_bytes, 128);
  // per-consumer-warp scratch
  mp.afrag_off = 0;
  mp.bias_off = 8 * 8 * 4 * 16;
  mp.vpair_off = mp.bias_off + 64;
  mp.wq_off = (int32_t)round_up(mp.vpair_off + (G / 16) * 4 * ngrp * 16, 16);
  mp.ws_bytes = (int32_t)round_up(mp.wq_off + 8 * D * 4, 128);
  // the four scratch areas together also hold the residual ring tile
  if (kNC * mp.ws_bytes < kResScratch) mp.ws_bytes = (int32_t)round_up((kResScratch + kNC - 1) / kNC, 128);
  // The stage count is a multiple of the consumer-warp count, so stage st is
  // always consumed by warp st % kNC: every waiter of a stage's barriers then
  // waits for its phases in order and never one phase too early (a parity
  // wait two phases ahead would alias a completed phase).
  int ns = (80 * 1024) / mp.stage_bytes;
  ns -= ns % kNC;
  if (ns < kNC) ns = kNC;
  if (ns > 16) ns = 16;
  mp.nstages = ns;
  mp.ws_soff = ns * mp.stage_bytes;
  mp.bar_off = mp.ws_soff + kNC * mp.ws_bytes;
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
  if (kb == K && vb == V && ng == N) fn = (const void*)decode_mma_kernel<K, V, N>;
  KVQ_MMA_INSTANCES(KVQ_FN)
#undef KVQ_FN
  if (!fn) return 1;
  // one occupancy query per (device, instance, shared-memory size)
  struct Entry {
    int dev;
    const void* fn;
    int smem;
    int n;
  };
  static Entry memo[64];
  static int nmemo = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < nmemo; ++i)
    if (memo[i].dev == dev && memo[i].fn == fn && memo[i].smem == mp.smem_bytes) return memo[i].n;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, mp.smem_bytes) != cudaSuccess) return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, mp.smem_bytes) != cudaSuccess || n < 1) return 1;
  if (nmemo < 64) memo[nmemo++] = Entry{dev, fn, mp.smem_bytes, n};
  return n;
}

}  // namespace kvq
