// Split-KV decode attention over the packed cache, and the log-sum-exp combine.
//
// Method: "KIVI" README (decoding over per-channel-quantized keys, per-token-
// quantized values and the full-precision residual window; GQA update) with
// the dequantization x_hat = q*d + m of the "KV1-1.2B" card (BQ2_0).
// The key-side dequantization is folded per block: since every channel of a
// G-token block has one (scale, zero), q.k_hat = sum_d (q_d s_d) c_d + sum_d q_d z_d,
// so the per-token work is a dot product of the scaled query with raw codes.
#include "kvq_decode.cuh"

namespace kvq {

namespace {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int NG>
struct SoftmaxState {
  float m[NG], l[NG], o[NG][4];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int hh = 0; hh < NG; ++hh) {
      m[hh] = -INFINITY;
      l[hh] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) o[hh][c] = 0.f;
    }
  }
  // score in log2 units; v: this lane's 4 channels of the token's value
  __device__ __forceinline__ void update(int hh, float score, const float* v) {
    const float mn = fmaxf(m[hh], score);
    const float alpha = exp2f(m[hh] - mn);
    const float pe = exp2f(score - mn);
    l[hh] = l[hh] * alpha + pe;
#pragma unroll
    for (int c = 0; c < 4; ++c) o[hh][c] = o[hh][c] * alpha + pe * v[c];
    m[hh] = mn;
  }
};

// Value of token tb of a block record at this lane's channels lane + 32c,
// dequantized (x_hat = q*d + m, two roundings): the record's word placement
// and its (scale, zero) order are resolved once per token, not per channel.
__device__ __forceinline__ void token_values(const LayerView& L, const uint8_t* rec, int tb, int lane,
                                             float (&vv)[4]) {
  constexpr int D = kHeadDim;
  const int G = L.tile_tokens, kb = L.k_bits, vb = L.v_bits, Gv = L.group_v;
  const int vper = 32 / vb, VW = D / vper, ng = D / Gv;
  const uint8_t* tp = rec + tile_base(L, tb);  // the token's tile and its index there
  const int t = tb % G;
  const uint32_t* vc = reinterpret_cast<const uint32_t*>(tp + L.vc_off);
  const __half* vsz = reinterpret_cast<const __half*>(tp + L.vsz_off);
  const int row = vc_row(t, G, kb);
  const int sw = VW >= 4 ? chunk_swizzle(row, VW / 4) : 0;
  // (scale, zero) of group gg at vsz[zi(gg)] / vsz[zi(gg) + zoff]
  int zbase, zstride, zoff;
  if (!vsz_operand_order(G, kb)) {
    zbase = t * ng * 2;
    zstride = 2;
    zoff = 1;
  } else {
    const int i0 = vsz_half_index(t, 0, G, kb, ng, false);
    zstride = ng > 1 ? vsz_half_index(t, 1, G, kb, ng, false) - i0 : 0;
    zbase = i0;
    zoff = 4;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int d = lane + 32 * c, w = d / vper, gg = d / Gv;
    const int wi = VW < 4 ? row * VW + w : row * VW + (((w >> 2) ^ sw) << 2) + (w & 3);
    const uint32_t vq = (vc[wi] >> ((d % vper) * vb)) & ((1u << vb) - 1);
    const int zi = zbase + gg * zstride;
    vv[c] = dequant_value(vq, vsz[zi], vsz[zi + zoff]);
  }
}

// One CTA = one split of one (sequence, KV head); 4 warps, each warp walks a
// quarter of the split's tokens with its own online-softmax state; lane owns
// channels lane + 32c, c = 0..3.
template <int NG>
__global__ void __launch_bounds__(128) decode_split_simple_kernel(DecodeParams p) {
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const LayerView& L = p.L;
  const int G = L.group_k, R = L.residual, RV = L.residual_v;
  const int32_t* len = L.lens + (int64_t)b * kLensStride;
  const int Q = len[kLenQ], n = len[kLenN], nsink = len[kLenS], QV = len[kLenQV];
  // blocks with a quantized key or value part; a block below one boundary
  // and above the other reads that tensor's tokens from its ring (separate
  // residual lengths for keys and values)
  const int QM = max(Q, QV), nblk = QM / G;
  const int bps = p.blocks_per_split;
  const int S = (nblk + bps - 1) / bps;
  if (s > S) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int D = kHeadDim;

  __shared__ float sq[NG][D];
  __shared__ float sqs[NG][D];
  __shared__ float sbias[4][NG];
  __shared__ float sm[4][NG], sl[4][NG];
  __shared__ float so[4][NG][D];

  const int ngr = p.q_heads / L.num_kv_heads;  // query rows hh: token hh / ngr, head h * ngr + hh % ngr
  for (int i = threadIdx.x; i < NG * D; i += blockDim.x) {
    const int hh = i / D, d = i % D;
    const int64_t row = (int64_t)b * p.q_rows + (hh / ngr) * p.q_heads + h * ngr + hh % ngr;
    sq[hh][d] = load_kv(p.q, row * D + d, L.kv_dtype) * p.scale_log2;
  }
  __syncthreads();
  if (L.hadamard && s > 0) {
    // quantized tokens live in the rotated basis: score them against Hq
    // (radix-2 butterflies, then 1/sqrt(D)); their partial is rotated back by
    // the combine
    for (int w = 1; w < D; w *= 2) {
      for (int i = threadIdx.x; i < NG * (D / 2); i += blockDim.x) {
        const int hh = i / (D / 2), pi = i % (D / 2);
        const int c = (pi / w) * 2 * w + pi % w;
        const float a = sq[hh][c], e = sq[hh][c + w];
        sq[hh][c] = a + e;
        sq[hh][c + w] = a - e;
      }
      __syncthreads();
    }
    const float rs = (float)(1.0 / sqrt((double)D));
    for (int i = threadIdx.x; i < NG * D; i += blockDim.x) sq[i / D][i % D] *= rs;
    __syncthreads();
  }

  SoftmaxState<NG> st;
  st.init();

  if (s == 0) {
    // Sinks and the residual ring: exact stored values.
    const int64_t unit = (int64_t)b * L.num_kv_heads + h;
    const int nx = Q + n - QM;  // tokens exact in both tensors
    for (int e = warp; e < nsink + nx; e += 4) {
      // e < nsink: sink e; otherwise the token at position QM + e - nsink
      const bool sink = e < nsink;
      const int i = QM + e - nsink;
      const int64_t krow = sink ? (unit * KVQ_MAX_SINKS + e) * D : (unit * R + i % R) * D;
      const int64_t vrow = sink ? (unit * KVQ_MAX_SINKS + e) * D : (unit * RV + i % RV) * D;
      const void* ksrc = sink ? L.sink_k : L.ring_k;
      const void* vsrc = sink ? L.sink_v : L.ring_v;
      float kv[4], vv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        kv[c] = load_kv(ksrc, krow + lane + 32 * c, L.kv_dtype);
        vv[c] = load_kv(vsrc, vrow + lane + 32 * c, L.kv_dtype);
      }
#pragma unroll
      for (int hh = 0; hh < NG; ++hh) {
        // query token hh / ngr does not see the sequence's last lag_base - hh / ngr tokens
        if (!sink && i - Q >= n - (p.lag_base - hh / ngr)) continue;
        float part = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) part += sq[hh][lane + 32 * c] * kv[c];
        st.update(hh, warp_sum(part), vv);
      }
    }
  } else {
    const int kb = L.k_bits, Gv = L.group_v;
    const int kper = 32 / kb;
    const uint32_t kmask = (1u << kb) - 1;
    const int j0 = (s - 1) * bps, j1 = min(s * bps, nblk);
    const int64_t unit = (int64_t)b * L.num_kv_heads + h;
    for (int j = j0; j < j1; ++j) {
      const uint8_t* rec = record_ptr(L, b, h, j);
      if (j * G >= Q || j * G >= QV) {
        // keys or values of this block still exact, in their ring (never
        // with the rotation: a rotated cache has one residual length)
        const bool kq = j * G < Q, vq = j * G < QV;
#pragma unroll 1
        for (int t = warp; t < G; t += 4) {
          const int i = j * G + t;
          float kv[4], vv[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int d = lane + 32 * c;
            if (kq) {
              const __half2 sz = *reinterpret_cast<const __half2*>(rec + ksz_pair_byte(L, t, d));
              const uint32_t kq2 =
                  (*reinterpret_cast<const uint32_t*>(rec + kc_word_byte(L, d, t / kper)) >> ((t % kper) * kb)) & kmask;
              kv[c] = dequant_value(kq2, __low2half(sz), __high2half(sz));
            } else {
              kv[c] = load_kv(L.ring_k, (unit * R + i % R) * D + d, L.kv_dtype);
            }
          }
          if (vq) {
            token_values(L, rec, t, lane, vv);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) vv[c] = load_kv(L.ring_v, (unit * RV + i % RV) * D + lane + 32 * c, L.kv_dtype);
          }
#pragma unroll
          for (int hh = 0; hh < NG; ++hh) {
            // a multi-token launch hides the newest tokens from earlier query tokens
            if (i - Q >= n - (p.lag_base - hh / ngr)) continue;
            float part = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) part += sq[hh][lane + 32 * c] * kv[c];
            st.update(hh, warp_sum(part), vv);
          }
        }
        continue;
      }
      if (L.k_axis == 1) {
        // per-token keys (BQ2_0): dequantize each key and dot it with q
        const int ng = D / Gv, TT = L.tile_tokens;
#pragma unroll 2
        for (int t = warp; t < G; t += 4) {
          float kv[4], vv[4];
          const uint8_t* tp = rec + tile_base(L, t);
          const uint32_t* kc = reinterpret_cast<const uint32_t*>(tp + L.kc_off);
          const __half2* ksz = reinterpret_cast<const __half2*>(tp + L.ksz_off);
          const int tl = t % TT;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int d = lane + 32 * c;
            const __half2 sz = ksz[tl * ng + d / Gv];
            const uint32_t kq = (kc[kc_word_index(d, tl / kper, TT / kper)] >> ((tl % kper) * kb)) & kmask;
            kv[c] = dequant_value(kq, __low2half(sz), __high2half(sz));
          }
          token_values(L, rec, t, lane, vv);
#pragma unroll
          for (int hh = 0; hh < NG; ++hh) {
            float part = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) part += sq[hh][lane + 32 * c] * kv[c];
            st.update(hh, warp_sum(part), vv);
          }
        }
        continue;
      }
      {
        const int d = threadIdx.x;
        const __half2 sz = *reinterpret_cast<const __half2*>(rec + ksz_pair_byte(L, 0, d));
        const float sc = __low2float(sz), z = __high2float(sz);
#pragma unroll
        for (int hh = 0; hh < NG; ++hh) {
          sqs[hh][d] = sq[hh][d] * sc;
          const float bsum = warp_sum(sq[hh][d] * z);
          if (lane == 0) sbias[warp][hh] = bsum;
        }
      }
      __syncthreads();
      float bias[NG];
#pragma unroll
      for (int hh = 0; hh < NG; ++hh) bias[hh] = sbias[0][hh] + sbias[1][hh] + sbias[2][hh] + sbias[3][hh];
      const int TT = L.tile_tokens;
      for (int t = warp; t < G; t += 4) {
        float kcode[4], vv[4];
        const uint32_t* kc = reinterpret_cast<const uint32_t*>(rec + tile_base(L, t) + L.kc_off);
        const int tl = t % TT, kw = tl / kper, ksh = (tl % kper) * kb;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int d = lane + 32 * c;
          kcode[c] = (float)((kc[kc_word_index(d, kw, TT / kper)] >> ksh) & kmask);
        }
        token_values(L, rec, t, lane, vv);
#pragma unroll
        for (int hh = 0; hh < NG; ++hh) {
          float part = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) part += sqs[hh][lane + 32 * c] * kcode[c];
          st.update(hh, warp_sum(part) + bias[hh], vv);
        }
      }
      __syncthreads();
    }
  }

  // Merge the four warps' states and write this split's partial.
#pragma unroll
  for (int hh = 0; hh < NG; ++hh) {
#pragma unroll
    for (int c = 0; c < 4; ++c) so[warp][hh][lane + 32 * c] = st.o[hh][c];
    if (lane == 0) {
      sm[warp][hh] = st.m[hh];
      sl[warp][hh] = st.l[hh];
    }
  }
  __syncthreads();
  const int d = threadIdx.x;
#pragma unroll
  for (int hh = 0; hh < NG; ++hh) {
    const float M = fmaxf(fmaxf(sm[0][hh], sm[1][hh]), fmaxf(sm[2][hh], sm[3][hh]));
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = sm[w][hh] == -INFINITY ? 0.f : exp2f(sm[w][hh] - M);
        acc += so[w][hh][d] * f;
        lsum += sl[w][hh] * f;
      }
    }
    const int64_t slot = ((int64_t)b * p.num_q_heads + h * NG + hh) * p.slots + s;
    p.ws_o[slot * D + d] = acc;
    if (d == 0) p.ws_ml[slot] = make_float2(M, lsum);
  }
}

// Log-sum-exp merge of the partial slots of one (sequence, query head):
// M = max_s m_s over slots with l_s > 0, out = sum_s 2^(m_s-M) o_s / sum_s
// 2^(m_s-M) l_s, rounded to the output dtype (nearest even); a sequence with
// no tokens gives zeros. WPH warps per (sequence, query head), lane L owning
// channels 4L..4L+3 (one 16-byte load per slot): warp w of a head merges
// slots w, w + WPH, ... online, issuing the loads of 16 of its slots at once
// (one round trip to L2 per 16 slots), and the head's warps then merge their
// states through shared memory. CTAs of max(4, WPH) warps, grid
// (ceil(Hq * WPH / warps), batch).
struct MergeState {
  float M, l;
  float4 acc, acc0;  // acc0: hadamard split mode, the exact-token slot 0 (kept apart)
};

__device__ __forceinline__ void merge_into(MergeState& a, const MergeState& b) {
  const float M = fmaxf(a.M, b.M);
  if (M == -INFINITY) return;
  const float ra = a.M == -INFINITY ? 0.f : exp2f(a.M - M), rb = b.M == -INFINITY ? 0.f : exp2f(b.M - M);
  a.acc = make_float4(a.acc.x * ra + b.acc.x * rb, a.acc.y * ra + b.acc.y * rb, a.acc.z * ra + b.acc.z * rb,
                      a.acc.w * ra + b.acc.w * rb);
  a.acc0 = make_float4(a.acc0.x * ra + b.acc0.x * rb, a.acc0.y * ra + b.acc0.y * rb, a.acc0.z * ra + b.acc0.z * rb,
                       a.acc0.w * ra + b.acc0.w * rb);
  a.l = a.l * ra + b.l * rb;
  a.M = M;
}

template <int WPH>
__global__ void __launch_bounds__(32 * (WPH > 4 ? WPH : 4)) combine_kernel(CombineParams p) {
  constexpr int kWarps = WPH > 4 ? WPH : 4, kHeads = kWarps / WPH;
  __shared__ MergeState s_st[kWarps][32];
  // wait for the decode grid this launch depends on (no-op without one)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hw = warp / WPH, wi = warp % WPH;  // head of the CTA, warp within the head
  const int hq = blockIdx.x * kHeads + hw, b = blockIdx.y;
  const bool active = hq < p.num_q_heads;
  constexpr int D = kHeadDim;
  constexpr int C = 16;  // slots per batch of loads
  int S = 0;  // slots of this (sequence, head)
  if (active) {
    if (p.persistent) {
      const int h = hq / (p.num_q_heads / p.num_kv_heads);
      S = __ldcg(p.unit_slots + b * p.num_kv_heads + h);
    } else {
      const int32_t* len = p.lens + (int64_t)b * kLensStride;
      const int nblk = max(len[kLenQ], len[kLenQV]) / p.group_k;
      S = (nblk + p.blocks_per_split - 1) / p.blocks_per_split + 1;
    }
  }
  const int64_t base = ((int64_t)b * p.num_q_heads + hq) * p.slots;
  const float2* ml_p = p.ws_ml + base;
  const float4* o_p = reinterpret_cast<const float4*>(p.ws_o + base * D) + lane;  // slot s at o_p[s * D / 4]
  MergeState st{-INFINITY, 0.f, make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
  const bool rot = p.hadamard && !p.persistent;
  for (int s0 = wi; s0 < S; s0 += C * WPH) {
    float2 ml[C];
    float4 v[C];
#pragma unroll
    for (int e = 0; e < C; ++e) {
      const int s = s0 + e * WPH;
      const bool in = s < S;
      ml[e] = in ? __ldcg(ml_p + s) : make_float2(-INFINITY, 0.f);
      v[e] = in ? __ldcg(o_p + (int64_t)s * (D / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mc = st.M;
#pragma unroll
    for (int e = 0; e < C; ++e)
      if (ml[e].y > 0.f) mc = fmaxf(mc, ml[e].x);
    if (mc == -INFINITY) continue;  // nothing yet
    const float r = st.M == -INFINITY ? 0.f : exp2f(st.M - mc);
    st.acc = make_float4(st.acc.x * r, st.acc.y * r, st.acc.z * r, st.acc.w * r);
    st.acc0 = make_float4(st.acc0.x * r, st.acc0.y * r, st.acc0.z * r, st.acc0.w * r);
    st.l *= r;
    st.M = mc;
#pragma unroll
    for (int e = 0; e < C; ++e) {
      if (ml[e].y > 0.f) {
        const float w = exp2f(ml[e].x - st.M);
        float4& a = (rot && s0 + e * WPH == 0) ? st.acc0 : st.acc;
        a.x += w * v[e].x;
        a.y += w * v[e].y;
        a.z += w * v[e].z;
        a.w += w * v[e].w;
        st.l += w * ml[e].y;
      }
    }
  }
  if constexpr (WPH > 1) {
    // the head's warps merge their states pairwise in shared memory
    s_st[warp][lane] = st;
    __syncthreads();
#pragma unroll
    for (int half = WPH / 2; half >= 1; half >>= 1) {
      if (wi < half) {
        merge_into(st, s_st[warp + half][lane]);
        if (half > 1) s_st[warp][lane] = st;
      }
      if (half > 1) __syncthreads();
    }
    if (wi != 0) return;
  }
  if (!active) return;
  float4 acc = st.acc;
  const float lsum = st.l;
  if (rot) {
    // the quantized part back to the original basis: acc . H over the warp's
    // 128 channels (lane L holds 4L..4L+3): butterflies of half-width 1 and 2
    // inside the lane, 4..64 across lanes, then 1/sqrt(D)
    float x[4] = {acc.x, acc.y, acc.z, acc.w};
    float a0 = x[0], a1 = x[1];
    x[0] = a0 + a1;
    x[1] = a0 - a1;
    a0 = x[2];
    a1 = x[3];
    x[2] = a0 + a1;
    x[3] = a0 - a1;
    a0 = x[0];
    a1 = x[1];
    x[0] = a0 + x[2];
    x[1] = a1 + x[3];
    x[2] = a0 - x[2];
    x[3] = a1 - x[3];
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float y = __shfl_xor_sync(0xffffffffu, x[e], m);
        x[e] = upper ? y - x[e] : x[e] + y;
      }
    }
    const float rs = (float)(1.0 / sqrt((double)D));
    acc = make_float4(x[0] * rs + st.acc0.x, x[1] * rs + st.acc0.y, x[2] * rs + st.acc0.z, x[3] * rs + st.acc0.w);
  }
  float r[4] = {0.f, 0.f, 0.f, 0.f};
  if (lsum > 0.f) {
    r[0] = __fdiv_rn(acc.x, lsum);
    r[1] = __fdiv_rn(acc.y, lsum);
    r[2] = __fdiv_rn(acc.z, lsum);
    r[3] = __fdiv_rn(acc.w, lsum);
  }
  // output row of query row hq: query token jv / ngr, head h * ngr + jv % ngr
  const int ngv = p.num_q_heads / p.num_kv_heads, ngr = p.q_heads / p.num_kv_heads;
  const int jv = hq % ngv;
  const int64_t o = ((int64_t)b * p.q_rows + (jv / ngr) * p.q_heads + (hq / ngv) * ngr + jv % ngr) * D + 4 * lane;
  if (p.out_dtype == KVQ_F32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + o) = make_float4(r[0], r[1], r[2], r[3]);
  } else if (p.out_dtype == KVQ_BF16) {
    __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(p.out) + o;
    *reinterpret_cast<__nv_bfloat162*>(d) = __floats2bfloat162_rn(r[0], r[1]);
    *reinterpret_cast<__nv_bfloat162*>(d + 2) = __floats2bfloat162_rn(r[2], r[3]);
  } else {
    __half* d = reinterpret_cast<__half*>(p.out) + o;
    *reinterpret_cast<__half2*>(d) = __floats2half2_rn(r[0], r[1]);
    *reinterpret_cast<__half2*>(d + 2) = __floats2half2_rn(r[2], r[3]);
  }
}

template <int NG>
cudaError_t launch_simple(const DecodeParams& p, int max_splits, cudaStream_t stream) {
  dim3 grid(max_splits + 1, p.L.num_kv_heads, p.batch);
  decode_split_simple_kernel<NG><<<grid, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

int split_ctas_per_sm(int num_q_heads, int num_kv_heads) {
  const int g = num_q_heads / num_kv_heads;
  const void* fn = g == 1   ? reinterpret_cast<const void*>(decode_split_simple_kernel<1>)
                   : g == 2 ? reinterpret_cast<const void*>(decode_split_simple_kernel<2>)
                   : g == 4 ? reinterpret_cast<const void*>(decode_split_simple_kernel<4>)
                            : reinterpret_cast<const void*>(decode_split_simple_kernel<8>);
  static int memo[9] = {0};  // per head ratio (one device type per process)
  if (memo[g] > 0) return memo[g];
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, 128, 0) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    return 4;
  }
  memo[g] = n;
  return n;
}

cudaError_t launch_decode(const DecodeParams& p, int max_splits, cudaStream_t stream) {
  if (p.batch <= 0) return cudaSuccess;
  const int g = p.num_q_heads / p.L.num_kv_heads;
  cudaError_t e;
  switch (g) {
    case 1: e = launch_simple<1>(p, max_splits, stream); break;
    case 2: e = launch_simple<2>(p, max_splits, stream); break;
    case 4: e = launch_simple<4>(p, max_splits, stream); break;
    case 8: e = launch_simple<8>(p, max_splits, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_combine(p, stream);
}

cudaError_t launch_combine(const DecodeParams& p, cudaStream_t stream) {
  if (p.batch <= 0) return cudaSuccess;
  // Warps per (sequence, query head): enough that each merges at most 16
  // slots (one round of loads), from the most slots a unit can use.
  const int most = p.persistent ? p.max_unit_slots : p.slots;
  int wph = 1;
  while (wph < 32 && wph * 16 < most) wph *= 2;
  const int warps = wph > 4 ? wph : 4, heads = warps / wph;
  // Programmatic dependent launch: the combine grid may be scheduled while
  // the decode grid (which allows it at its start) is still running; each
  // combine CTA waits for the decode grid to complete before it reads.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.num_q_heads + heads - 1) / heads, p.batch);
  cfg.blockDim = dim3(32 * warps);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = p.persistent ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const CombineParams cp{p.ws_o,         p.ws_ml,          p.out,           p.unit_slots,
                         p.L.lens,       p.out_dtype,      p.num_q_heads,   p.L.num_kv_heads,
                         p.slots,        p.L.group_k,      p.blocks_per_split, p.persistent, p.L.hadamard,
                         p.q_heads,      p.q_rows};
  switch (wph) {
    case 1: return cudaLaunchKernelEx(&cfg, combine_kernel<1>, cp);
    case 2: return cudaLaunchKernelEx(&cfg, combine_kernel<2>, cp);
    case 4: return cudaLaunchKernelEx(&cfg, combine_kernel<4>, cp);
    case 8: return cudaLaunchKernelEx(&cfg, combine_kernel<8>, cp);
    case 16: return cudaLaunchKernelEx(&cfg, combine_kernel<16>, cp);
    default: return cudaLaunchKernelEx(&cfg, combine_kernel<32>, cp);
  }
}

}  // namespace kvq
