// Tensor-core decode attention for 32-token key groups with 2-bit keys (the
// pair layout of kvq_internal.cuh) and at most two query rows per KV head --
// multi-head attention and the 2-bit/32-token KIVI setting ("KIVI" README,
// Overview and Example: group_size 32, residual_length 128). Instantiated
// per (value bits, value groups per head) in kvq_decode_pair_v{2,4,8}.cu.
//
// Same pipeline as decode_tc_kernel (persistent CTA ranges of work items,
// one private ring of copy stages per warp, ring chunks of exact tokens,
// one partial per warp and unit, the log-sum-exp combine); what differs is
// how a 32-token block meets the m16n8k16 shapes:
//  * Keys. A channel's codes of one block are 8 bytes, so channels d and
//    d + 64 share one 16-byte row and one ldmatrix.trans reads both: in a
//    key M-tile, rows 0-3 and 8-11 hold tokens over channels 0-63 (set A)
//    and rows 4-7 and 12-15 the same tokens over channels 64-127 (set B).
//    The B operand has room for both because a KV head has at most two query
//    rows here: column n is query row n / 4, channel set (n / 2) % 2, fp16
//    high (n even) or low part of q*s. A token's score is then its set-A row
//    in one lane plus its set-B row in another (one shuffle); M-tile jp of a
//    block holds tokens 8a + 2jp + r (rows a and a + 8, a < 4).
//  * Values. A value chunk of 2-bit codes spans 64 channels, two 32-channel
//    groups, so one M-tile's rows need different scales. The B operand of
//    P.V carries them in its columns: column n = 4 * (query row) + value
//    group, p*s of that group, and each output row is read from the column
//    of its own group; the zero points are one all-ones MMA for all groups.
//  * Softmax state: lane (g, t) keeps the state of query row t / 2, so both
//    output columns of the lane (2t, 2t + 1) belong to its own row.
#pragma once

#include "kvq_decode_tc.cuh"

namespace kvq {
namespace tc {

template <int VB, int NGRP>
struct PairShape {
  static constexpr int D = kHeadDim;
  static constexpr int TT = 32;              // tokens per block
  static constexpr int VRB = D * VB / 8;     // value code bytes per token
  static constexpr int NCH = VRB / 16;       // 16-byte chunks per value row
  static constexpr int VCPC = 16 / VB;       // value channels per 16-bit column
  static constexpr int MT_PER_CH = VCPC / 2; // channel M-tiles per value chunk
  static constexpr int CH_SPAN = 128 / VB;   // channels per value chunk
  static constexpr int GV = D / NGRP;        // value group (channels)
  static_assert(NCH * MT_PER_CH == 8, "eight output M-tiles of 16 channels");
  static_assert(NGRP <= 4, "value groups are columns 0-3 of a query row");
};

// The query words a lane needs for the key B fragments of every block of a
// unit (loaded once per unit): lane (g, t) holds column g -- query row g / 4,
// channel set (g / 2) % 2, high (g even) or low part -- for k rows 2t, 2t+1
// (e = 0) and 8+2t, 9+2t (e = 1) of paired-row k-step kk, i.e. channels
// 64*set + 16kk + 8e + 2t and the next (qk), and for the bias the channels
// 2l, 2l+1 and 64+2l, 65+2l of lane l of both query rows (qb).
struct PairQuery {
  uint32_t qk[4][2];
  uint32_t qb[2][2];
};
__device__ __forceinline__ void pair_query(const uint32_t* qw, int NG, int lane, PairQuery& pq) {
  const int g = lane >> 2, t = lane & 3;
  const int row = g >> 2, set = (g >> 1) & 1;
  const bool present = row < NG;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int e = 0; e < 2; ++e) pq.qk[kk][e] = present ? qw[q_word(row, 32 * set + 8 * kk + 4 * e + t)] : 0u;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    pq.qb[r][0] = r < NG ? qw[q_word(r, lane)] : 0u;
    pq.qb[r][1] = r < NG ? qw[q_word(r, 32 + lane)] : 0u;
  }
}

// Key B fragments of one block (registers, the columns of pair_query): q*s
// of fp16 q (times q_prescale) and fp16 s has at most 22 significant bits,
// so the high part and the rounded remainder hold it. bias[r] = sum_d q_rd
// z_d times score_scale.
__device__ __forceinline__ void pair_prep(const uint8_t* stage, int kc_bytes, const PairQuery& pq, int NG, int lane,
                                          float score_scale, uint32_t (&bq)[4][2], float (&bias)[2]) {
  const uint2* ksz2 = reinterpret_cast<const uint2*>(stage + kc_bytes);  // (s, z) of channels 2w, 2w+1
  const int g = lane >> 2, t = lane & 3;
  const int set = (g >> 1) & 1;
  const bool low = g & 1;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const uint2 sz = ksz2[32 * set + 8 * kk + 4 * e + t];
      const uint32_t s2 = __byte_perm(sz.x, sz.y, 0x5410);
      const uint32_t hi = hmul2(pq.qk[kk][e], s2);
      bq[kk][e] = low ? hfms2(pq.qk[kk][e], s2, hi) : hi;
    }
  const uint2 sa = ksz2[lane], sb = ksz2[32 + lane];
  bias[0] = bias[1] = 0.f;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (r < NG) {  // warp-uniform
      float bp = fma_q_z(pq.qb[r][0], sa.x, sa.y, 0.f);
      bp = fma_q_z(pq.qb[r][1], sb.x, sb.y, bp);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) bp += __shfl_xor_sync(0xffffffffu, bp, o);
      bias[r] = bp * score_scale;
    }
  }
}

// One chunk of exact tokens (ring or sinks; cnt of its rows present): keys
// with the query split into kv-dtype high and low parts in the columns of
// this kernel (column n: query row n / 4, high part for n even), so that
// lane (g, t) reads the score of row t / 2 for token g; P.V with column n
// carrying the probabilities of row n / 4 (every value group of the row gets
// the same exact product), added to O at the row scale of the value codes.
template <bool BF16, int VB>
__device__ __forceinline__ void pair_ring_chunk(const uint8_t* stage, const uint32_t* qw, uint2* bk, int cnt, int NG,
                                                int lane, float score_scale, const bool (&valid)[1],
                                                bool& rq_ready, SoftState<1>& sst, float (&O)[8][4],
                                                float (&Z)[1][4]) {
  using S = PairShape<VB, 1>;  // value-side constants only
  const int g = lane >> 2, t = lane & 3;
  if (!rq_ready) {
    const int row = g >> 2;
    const bool present = row < NG;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t hi[2], lo[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int w = 4 * t + 16 * (kk >> 1) + 2 * (kk & 1) + e;  // channels 2w, 2w+1
        const uint32_t raw = present ? qw[q_word(row, w)] : 0u;
        const float2 f = unpack_f16(raw);
        const float x0 = f.x * score_scale, x1 = f.y * score_scale;
        hi[e] = pack_kv<BF16>(x0, x1);
        const float2 fh = unpack_kv2<BF16>(hi[e]);
        lo[e] = pack_kv<BF16>(x0 - fh.x, x1 - fh.y);
      }
      bk[kk * 32 + lane] = (g & 1) ? make_uint2(lo[0], lo[1]) : make_uint2(hi[0], hi[1]);
    }
    __syncwarp();
    rq_ready = true;
  }
  const uint4* K4 = reinterpret_cast<const uint4*>(stage);
  float Dr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint4 kv = K4[g * 16 + t + 4 * m];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint32_t a[4] = {word_of(kv, 2 * hf), 0u, word_of(kv, 2 * hf + 1), 0u};
      const uint2 bq = bk[(2 * m + hf) * 32 + lane];
      mma_kv<BF16>(Dr, a, bq.x, bq.y);
    }
  }
  // rows 8-15 are absent; row g holds token g of the chunk
  float sc[1][2];
  sc[0][0] = g < cnt ? Dr[0] + Dr[1] : -INFINITY;
  sc[0][1] = -INFINITY;
  softmax_update<1, 1, 1, true, true>(sc, sst, valid, O, Z, lane);
  const uint32_t ph = pack_kv<BF16>(sc[0][0], 0.f);
  const float hf = unpack_kv2<BF16>(ph).x;
  const uint32_t hl = pack_kv<BF16>(sc[0][0], sc[0][0] - hf);  // (high, low) of token g
  const int src = 2 * (g >> 2);                                // a lane of query row g / 4
  const uint32_t u = __shfl_sync(0xffffffffu, hl, 8 * t + src);
  const uint32_t v = __shfl_sync(0xffffffffu, hl, 8 * t + 4 + src);
  const bool col = (g >> 2) < NG;
  const uint32_t bh = col ? __byte_perm(u, v, 0x5410) : 0u;  // high parts of tokens 2t, 2t+1
  const uint32_t bl = col ? __byte_perm(u, v, 0x7632) : 0u;  // low parts
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

template <int VB, int NGRP>
__global__ void __launch_bounds__(kThreads, 2) decode_pair_kernel(DecodeParams p, MmaPlan mp) {
  using S = PairShape<VB, NGRP>;
  constexpr int D = S::D;
  extern __shared__ __align__(128) uint8_t smem[];
  const int c = blockIdx.x;
  const LayerView& L = p.L;
  const int Hkv = L.num_kv_heads;
  const int NG = p.num_q_heads / Hkv;  // query rows per unit (1 or 2)
  const int ngr = p.q_heads / Hkv;      // query heads per KV head (rows per query token)
  const int rs = p.cta_start[c], re = p.cta_start[c + 1];
  const bool bf16 = L.kv_dtype == KVQ_BF16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int SPW = mp.nstages;
  uint8_t* stages = smem + (size_t)warp * SPW * mp.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + mp.bar_off) + warp * SPW;
  uint8_t* ws = smem + mp.ws_soff + warp * mp.ws_bytes;
  const int nmine = rs + warp < re ? (re - rs - warp + kNC - 1) / kNC : 0;
  uint8_t* qbuf = ws + mp.qbuf_off;
  IssueState is;
  if (lane == 0) {
    for (int i = 0; i < SPW; ++i) mbar_init(full + i, 1);
    fence_mbar_init();
    for (int n = 0; n < SPW && n < nmine; ++n)
      issue_item(p, mp, is, rs + warp + n * kNC, stages + (size_t)n * mp.stage_bytes, full + n, qbuf, NG);
  }
  __syncwarp();
  bool failed = false;
  int n = 0;
  const int g = lane >> 2, t = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  const int qrow = t >> 1;  // this lane's query row (softmax state and output columns)
  const bool valid[1] = {qrow < NG};
  const uint32_t ones[4] = {0x3c003c00u, 0x3c003c00u, 0x3c003c00u, 0x3c003c00u};  // fp16 1.0
  const int swv = chunk_swizzle(rr, S::NCH);
  // a token's set-A and set-B score rows meet in lanes (g < 4, t even) and
  // (g >= 4, t odd), one xor-17 shuffle apart; both hold its full score
  const bool score_lane = (g < 4) == ((t & 1) == 0);
  const int psrc = 4 * t + 2 * (g >> 2);                      // probabilities of B column g (query row g / 4)
  const bool pcol = (g >> 2) < NG;
  const int vgrp = min(g & 3, NGRP - 1);                      // value group of B column g
  uint2* bkw = reinterpret_cast<uint2*>(ws + mp.bfrag_off);
  int qslot = -1;  // query buffer of the current unit (matches IssueState::qslot)
  int st = 0;      // stage of item n and its barrier phase parity
  uint32_t ph = 0;
  PairQuery pq;  // the unit's query words for the key B fragments
  UnitCursor u;
  int k = rs;
  while (k < re && !failed) {
    u.advance(p, k);
    const int hi = min(u.end, re);
    const int nb = p.nblk[u.b];
    SoftState<1> sst;
    sst.m[0] = -INFINITY;
    sst.l[0] = 0.f;
    float O[8][4], Z[1][4];
#pragma unroll
    for (int i2 = 0; i2 < 8; ++i2) O[i2][0] = O[i2][1] = O[i2][2] = O[i2][3] = 0.f;
    Z[0][0] = Z[0][1] = Z[0][2] = Z[0][3] = 0.f;
    bool rq_ready = false;
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
        // the unit's queries, to fp16 times q_prescale in the q_word order
        uint32_t cv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int w = lane + 32 * i;
          if (w < NG * (D / 2)) {
            const float2 f = bf16 ? unpack_bf16(qw[w]) : unpack_f16(qw[w]);
            cv[i] = pack_f16(f.x * p.q_prescale, f.y * p.q_prescale);
          }
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int w = lane + 32 * i;
          if (w < NG * (D / 2)) qw[q_word(w / (D / 2), w % (D / 2))] = cv[i];
        }
        __syncwarp();
        pair_query(qw, NG, lane, pq);
      }
      const int j = kb - u.start;
      if (j < nb) {
        // ============ quantized block of 32 tokens
        uint32_t bq[4][2];
        float bias[2];
        pair_prep(stage, mp.kc_bytes, pq, NG, lane, p.score_scale, bq, bias);
        const float bias_l = qrow ? bias[1] : bias[0];
        const uint32_t kc_s = smem_u32(stage);
        const uint32_t vc_s = smem_u32(stage + mp.vc_soff);
        const uint4* vsz4 = reinterpret_cast<const uint4*>(stage + mp.vsz_soff);
        // ---- scores: Dk[jp] = codes x (q*s), both channel sets
        float Dk[4][4];
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) Dk[jp][0] = Dk[jp][1] = Dk[jp][2] = Dk[jp][3] = 0.f;
#pragma unroll
        for (int kp = 0; kp < 2; ++kp) {
          uint32_t rk[4];
          ldsm_x4_t(kc_s + (32 * kp + 8 * mi + rr) * 16, rk[0], rk[1], rk[2], rk[3]);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t xl = rk[2 * hf], xh = rk[2 * hf + 1], xl8 = xl >> 8, xh8 = xh >> 8;
#pragma unroll
            for (int jp = 0; jp < 4; ++jp) {
              const uint32_t a[4] = {code_sub<2>(xl, xl8, 2 * jp), code_sub<2>(xl, xl8, 2 * jp + 1),
                                     code_sub<2>(xh, xh8, 2 * jp), code_sub<2>(xh, xh8, 2 * jp + 1)};
              mma_f16(Dk[jp], a, bq[2 * kp + hf][0], bq[2 * kp + hf][1]);
            }
          }
        }
        // ---- a token's score: its set-A row plus its set-B row (M-tile jp,
        // rows g and g + 8: tokens 8(g % 4) + 2jp and 8(g % 4) + 2jp + 1)
        float sc[4][2];
#pragma unroll
        for (int jp = 0; jp < 4; ++jp)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float x = Dk[jp][2 * r] + Dk[jp][2 * r + 1];
            const float s = x + __shfl_xor_sync(0xffffffffu, x, 17);
            sc[jp][r] = score_lane ? fmaf(s, p.score_scale * code_unscale<2>(2 * jp + r), bias_l) : -INFINITY;
          }
        softmax_update<4, 1, 1, false, true>(sc, sst, valid, O, Z, lane);
        // ---- values: O += codes x (p * s), Z += ones x (p * z)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          // k rows 2t, 2t+1 of k-step i: tokens 8t + 4i, +1 (M-tile 2i);
          // rows 8+2t, 9+2t: tokens 8t + 4i + 2, +3 (M-tile 2i + 1)
          const uint32_t pk0 = pack_f16(sc[2 * i][0], sc[2 * i][1]), pk1 = pack_f16(sc[2 * i + 1][0], sc[2 * i + 1][1]);
          uint32_t bt = __shfl_sync(0xffffffffu, pk0, psrc), bb = __shfl_sync(0xffffffffu, pk1, psrc);
          if (!pcol) bt = bb = 0u;
          const uint4 v4 = vsz4[(i * 4 + t) * NGRP + vgrp];  // (s, s), (s, s), (z, z), (z, z)
          const uint32_t B0 = hmul2(bt, v4.x), B1 = hmul2(bb, v4.y);
          mma_f16(Z[0], ones, hmul2(bt, v4.z), hmul2(bb, v4.w));
          const uint32_t vrow = vc_s + (16 * i + 8 * (mi & 1) + rr) * S::VRB;
#pragma unroll
          for (int cc0 = 0; cc0 < S::NCH; cc0 += 2) {
            uint32_t r[4];
            ldsm_x4_t(vrow + (((cc0 + (mi >> 1)) ^ swv) << 4), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const uint32_t xv = r[2 * cc], yv = r[2 * cc + 1], xv8 = xv >> 8, yv8 = yv >> 8;
#pragma unroll
              for (int P = 0; P < S::MT_PER_CH; ++P) {
                const uint32_t a[4] = {code_sub<VB>(xv, xv8, 2 * P), code_sub<VB>(xv, xv8, 2 * P + 1),
                                       code_sub<VB>(yv, yv8, 2 * P), code_sub<VB>(yv, yv8, 2 * P + 1)};
                mma_f16(O[(cc0 + cc) * S::MT_PER_CH + P], a, B0, B1);
              }
            }
          }
        }
      } else {
        bool sink;
        const int cnt0 = exact_chunk(p, u.b, j - nb, sink);
        const int cnt = sink ? cnt0 : cnt0 - (p.lag_base - qrow / ngr);
        if (p.new_k && !sink && j - nb == (p.nres[u.b] - 1) / kResChunk) store_new_token(p, u.b, u.h, nb, stage, lane);
        if (bf16)
          pair_ring_chunk<true, VB>(stage, qw, bkw, cnt, NG, lane, p.score_scale, valid, rq_ready, sst, O, Z);
        else
          pair_ring_chunk<false, VB>(stage, qw, bkw, cnt, NG, lane, p.score_scale, valid, rq_ready, sst, O, Z);
      }
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
    // ---------------- this warp's partial for the unit
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) sst.l[0] += __shfl_xor_sync(0xffffffffu, sst.l[0], off);
    const int c0 = cta_of_item(p.cta_start, p.num_ctas, u.start);
    const int slot = kNC * (c - c0) + warp;
    if (slot == 0 && lane == 0)
      p.unit_slots[u.b * Hkv + u.h] = kNC * (cta_of_item(p.cta_start, p.num_ctas, u.end - 1) - c0 + 1);
    if (valid[0]) {
      const int64_t base = ((int64_t)u.b * p.num_q_heads + u.h * NG + qrow) * p.slots + slot;
      // output row g of M-tile mt2 (channel ch0; row g + 8: ch0 + 1) sits in
      // column 4 * qrow + its value group: this lane's column 2t + e when
      // the group is 2 (t % 2) + e
#pragma unroll
      for (int mt2 = 0; mt2 < 8; ++mt2) {
        const int cch = mt2 / S::MT_PER_CH, P = mt2 % S::MT_PER_CH;
        const int ch0 = cch * S::CH_SPAN + g * S::VCPC + 2 * P;
        const int grp = ch0 / S::GV;
        if ((grp >> 1) == (t & 1)) {
          const bool e = grp & 1;
          const float u0 = code_unscale<VB>(2 * P), u1 = code_unscale<VB>(2 * P + 1);
          *reinterpret_cast<float2*>(p.ws_o + base * D + ch0) =
              make_float2(fmaf(e ? O[mt2][1] : O[mt2][0], u0, e ? Z[0][1] : Z[0][0]),
                          fmaf(e ? O[mt2][3] : O[mt2][2], u1, e ? Z[0][3] : Z[0][2]));
        }
      }
      if (g == 0 && (t & 1) == 0) p.ws_ml[base] = make_float2(sst.m[0], sst.l[0]);
    }
    k = hi;
  }
  if (failed) {
    if (lane == 0)
      for (int i = n; i < n + SPW && i < nmine; ++i) (void)mbar_wait(full + i % SPW, (i / SPW) & 1);
    if (lane == 0) atomicOr(p.err, 1);
  }
}

template <int VB, int NGRP>
cudaError_t launch_pair_instance(const DecodeParams& p, const MmaPlan& mp, cudaStream_t stream) {
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
  return cudaLaunchKernelEx(&cfg, decode_pair_kernel<VB, NGRP>, p, mp);
}

template <int VB, int NGRP>
const void* pair_instance_fn() {
  return reinterpret_cast<const void*>(decode_pair_kernel<VB, NGRP>);
}

}  // namespace tc
}  // namespace kvq
