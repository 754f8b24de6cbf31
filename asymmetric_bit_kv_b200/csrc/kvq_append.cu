// Append / flush / dequantize kernels.
//
// Method: "KIVI" README, sections "Overview" and "Example" (keys per channel,
// values per token, residual window of recent full-precision tokens) and the
// quantizer of the "KV1-1.2B" card, section "Quantization Format: KV1.cpp
// BQ2_0". One CTA quantizes one G-token block of one (sequence, KV head):
// the block is staged in shared memory as raw 16-bit values, keys are reduced
// per channel (one thread per channel), values per group_v channels of a token
// with warp __shfl_xor min/max reductions, and codes are packed into 32-bit
// words lowest bits first.
#include "kvq_append.cuh"

namespace kvq {

namespace {

__device__ __forceinline__ float bits_to_float(uint16_t v, int dtype) {
  if (dtype == KVQ_BF16) return __uint_as_float((uint32_t)v << 16);
  return __half2float(__ushort_as_half(v));
}

}  // namespace

// One group quantizer pass over rows of D values: every (row, run of gv
// channels) is one group; each thread owns one output word (32/bits
// channels) and the gv/(32/bits) threads of a group combine their min/max
// with xor shuffles. val(t, d) reads value d of row t; put_word(t, w, word)
// and put_sz(t, g, d16, m16) store the codes and the group's scale and zero.
template <class Val, class PutWord, class PutSz>
__device__ __forceinline__ void quantize_rows(int rows, int D, int bits, int gv, Val val, PutWord put_word,
                                              PutSz put_sz) {
  const int per = 32 / bits;
  const int wpt = D / per;  // words per row
  const int P = gv / per;   // threads per group, a power of two <= 32
  for (int widx = threadIdx.x; widx < rows * wpt; widx += blockDim.x) {
    const int t = widx / wpt, w = widx % wpt;
    float mn = val(t, w * per), mx = mn;
    for (int i = 1; i < per; ++i) {
      const float x = val(t, w * per + i);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    for (int o = P / 2; o >= 1; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const GroupParams gp = group_params(mn, mx, bits);
    uint32_t word = 0;
    for (int i = 0; i < per; ++i) word |= quant_code(val(t, w * per + i), gp, bits) << (i * bits);
    put_word(t, w, word);
    if ((w % P) == 0) put_sz(t, w / P, gp.d16, gp.m16);
  }
}

// grid (max flush blocks, batch, Hkv); block kQuantThreads; dynamic smem
// 2*G*D*2 bytes (ROT: 2*G*D*4). ROT: every token's key and value head vector
// is multiplied by the normalized Sylvester Hadamard matrix (rotate_lane:
// radix-2 butterflies of half-width 1, 2, 4, ..., then one fp32
// multiplication by fp32(1/sqrt(D))) and staged as fp32 before the block is
// quantized ("KV1-1.2B" card, BQ2_0).
template <bool ROT>
__global__ void __launch_bounds__(kQuantThreads) quantize_blocks_kernel(AppendParams p) {
  const int j = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  if (j >= p.flush[b]) return;
  const LayerView& L = p.L;
  const int G = L.group_k, D = L.head_dim, R = L.residual;
  const int kb = L.k_bits, vb = L.v_bits, Gv = L.group_v;
  const int dt = L.kv_dtype;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* sk = reinterpret_cast<uint16_t*>(smem_raw);  // [G][D] raw (not ROT)
  uint16_t* sv = sk + G * D;
  float* fk = reinterpret_cast<float*>(smem_raw);  // [G][D] fp32 (ROT)
  float* fv = fk + G * D;

  const int first = p.q_old[b] + j * G;  // position of the block's first token (after the sinks)
  const int boundary = p.q_old[b] + p.n_old[b];
  const int64_t ring_base = ((int64_t)b * L.num_kv_heads + h) * R;
  // Row t of the block (token first + t) of the keys or the values: in the
  // ring, or in this call's input.
  auto row_ptr = [&](int t, bool value) -> const uint16_t* {
    const int i = first + t;
    if (i < boundary)
      return reinterpret_cast<const uint16_t*>(value ? L.ring_v : L.ring_k) + (ring_base + i % R) * D;
    const int64_t row = (int64_t)p.in_off[b] + (i - boundary);
    return reinterpret_cast<const uint16_t*>(value ? p.v_in : p.k_in) + (row * L.num_kv_heads + h) * D;
  };
  if constexpr (ROT) {
    // one warp per row of G keys then G values, 4 channels per lane, rotated
    // in registers (D = 128)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int row = warp; row < 2 * G; row += kQuantThreads / 32) {
      const bool value = row >= G;
      const int t = value ? row - G : row;
      const uint2 raw = *reinterpret_cast<const uint2*>(row_ptr(t, value) + 4 * lane);
      float x[4] = {bits_to_float(raw.x & 0xffffu, dt), bits_to_float(raw.x >> 16, dt),
                    bits_to_float(raw.y & 0xffffu, dt), bits_to_float(raw.y >> 16, dt)};
      rotate_lane(x, lane);
      *reinterpret_cast<float4*>((value ? fv : fk) + t * D + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
    }
  } else {
    // Stage the G x D block, 8 values (16 bytes) per load.
    const int vec_per_tok = D / 8;
    for (int idx = threadIdx.x; idx < G * vec_per_tok; idx += blockDim.x) {
      const int t = idx / vec_per_tok, c = (idx % vec_per_tok) * 8;
      *reinterpret_cast<uint4*>(sk + t * D + c) = *reinterpret_cast<const uint4*>(row_ptr(t, false) + c);
      *reinterpret_cast<uint4*>(sv + t * D + c) = *reinterpret_cast<const uint4*>(row_ptr(t, true) + c);
    }
  }
  __syncthreads();
  auto kval = [&](int t, int d) -> float {
    if constexpr (ROT) return fk[t * D + d];
    else return bits_to_float(sk[t * D + d], dt);
  };
  auto vval = [&](int t, int d) -> float {
    if constexpr (ROT) return fv[t * D + d];
    else return bits_to_float(sv[t * D + d], dt);
  };

  uint8_t* rec = record_ptr(L, b, h, p.q_old[b] / G + j);
  uint32_t* kc = reinterpret_cast<uint32_t*>(rec + L.kc_off);
  __half2* ksz = reinterpret_cast<__half2*>(rec + L.ksz_off);
  uint32_t* vc = reinterpret_cast<uint32_t*>(rec + L.vc_off);
  __half* vsz = reinterpret_cast<__half*>(rec + L.vsz_off);

  if (L.k_axis == 0) {
    // Keys: one group per channel over the G tokens (KIVI: per-channel keys).
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float mn = kval(0, d), mx = mn;
      for (int t = 1; t < G; ++t) {
        const float x = kval(t, d);
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
      }
      const GroupParams gp = group_params(mn, mx, kb);
      ksz[d] = __halves2half2(gp.d16, gp.m16);
      const int per = 32 / kb;
      const int nw = G / per;  // words per channel, stored contiguously
      for (int w = 0; w < nw; ++w) {
        uint32_t word = 0;
        for (int i = 0; i < per; ++i) word |= quant_code(kval(w * per + i, d), gp, kb) << (i * kb);
        kc[kc_word_index(d, w, nw)] = word;
      }
    }
  } else {
    // Keys per token (BQ2_0), grouped like values over group_v channels:
    // (scale, zero) pairs [G][D/group_v] row-major, then the codes packed
    // along the token axis in the per-channel key layout, so that the decode
    // kernels read both key axes' codes the same way.
    __shared__ __half2 s_ksz[128 * 4];  // G <= 128 tokens x D/group_v <= 4 groups
    const int ng = D / Gv;
    quantize_rows(G, D, kb, Gv, kval, [](int, int, uint32_t) {}, [&](int t, int g, __half d16, __half m16) {
      ksz[t * ng + g] = s_ksz[t * ng + g] = __halves2half2(d16, m16);
    });
    __syncthreads();  // the pairs just stored are read back below
    const int per = 32 / kb, nw = G / per;
    for (int idx = threadIdx.x; idx < D * nw; idx += blockDim.x) {
      const int d = idx / nw, w = idx % nw;
      uint32_t word = 0;
      for (int i = 0; i < per; ++i) {
        const int t = w * per + i;
        const __half2 sz = s_ksz[t * ng + d / Gv];
        GroupParams gp;
        gp.d16 = __low2half(sz);
        gp.m16 = __high2half(sz);
        gp.d = __half2float(gp.d16);
        gp.m = __half2float(gp.m16);
        word |= quant_code(kval(t, d), gp, kb) << (i * kb);
      }
      kc[kc_word_index(d, w, nw)] = word;
    }
  }

  // Values: one group per group_v channels of a token (KIVI: per-token values).
  const int vwpt = D * vb / 32;
  quantize_rows(G, D, vb, Gv, vval,
                [&](int t, int w, uint32_t word) { vc[vc_word_index(t, w, G, kb, vwpt)] = word; },
                [&](int t, int g, __half d16, __half m16) {
                  vsz[vsz_half_index(t, g, G, kb, D / Gv, false)] = d16;
                  vsz[vsz_half_index(t, g, G, kb, D / Gv, true)] = m16;
                });
}

// grid (batch, Hkv); copies this call's sink tokens to the sinks and its
// unflushed new tokens into the ring, and records the new lengths.
__global__ void ring_write_kernel(AppendParams p) {
  const int b = blockIdx.x, h = blockIdx.y;
  const LayerView& L = p.L;
  const int G = L.group_k, D = L.head_dim, R = L.residual;
  const int boundary = p.q_old[b] + p.n_old[b];
  const int q_new = p.q_old[b] + p.flush[b] * G;
  const int end = boundary + p.t_new[b];
  const int first = max(boundary, q_new);
  const int vec_per_tok = D / 8;
  const int ns = p.s_take[b];
  const int64_t sink_base = ((int64_t)b * L.num_kv_heads + h) * KVQ_MAX_SINKS + p.s_old[b];
  for (int idx = threadIdx.x; idx < ns * vec_per_tok; idx += blockDim.x) {
    const int i = idx / vec_per_tok, c = (idx % vec_per_tok) * 8;
    const int64_t row = (int64_t)p.in_off[b] - ns + i;
    const int64_t src = (row * L.num_kv_heads + h) * D + c;
    const int64_t dst = (sink_base + i) * D + c;
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(L.sink_k) + dst) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.k_in) + src);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(L.sink_v) + dst) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.v_in) + src);
  }
  const int64_t ring_base = ((int64_t)b * L.num_kv_heads + h) * R;
  for (int idx = threadIdx.x; idx < (end - first) * vec_per_tok; idx += blockDim.x) {
    const int i = first + idx / vec_per_tok, c = (idx % vec_per_tok) * 8;
    const int64_t row = (int64_t)p.in_off[b] + (i - boundary);
    const int64_t src = (row * L.num_kv_heads + h) * D + c;
    const int64_t dst = (ring_base + i % R) * D + c;
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(L.ring_k) + dst) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.k_in) + src);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(L.ring_v) + dst) =
        *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.v_in) + src);
  }
  if (h == 0 && threadIdx.x == 0) {
    L.lens[3 * b] = q_new;
    L.lens[3 * b + 1] = end - q_new;
    L.lens[3 * b + 2] = p.s_old[b] + ns;
  }
}

// grid (ceil(n / 8), Hkv); block D threads. Token t0 + i of sequence `seq`,
// whose first `sinks` tokens are its sinks.
__global__ void dequant_kernel(LayerView L, int seq, int sinks, int t0, int n, float* k_out, float* v_out) {
  const int h = blockIdx.y;
  const int d = threadIdx.x;
  const int G = L.group_k, D = L.head_dim, R = L.residual;
  const int Q = L.lens[3 * seq];
  const int kb = L.k_bits, vb = L.v_bits;
  for (int r = 0; r < 8; ++r) {
    const int i = blockIdx.x * 8 + r;
    if (i >= n || d >= D) continue;
    const int64_t o = ((int64_t)i * L.num_kv_heads + h) * D + d;
    if (t0 + i < sinks) {
      const int64_t src = (((int64_t)seq * L.num_kv_heads + h) * KVQ_MAX_SINKS + t0 + i) * D + d;
      k_out[o] = load_kv(L.sink_k, src, L.kv_dtype);
      v_out[o] = load_kv(L.sink_v, src, L.kv_dtype);
      continue;
    }
    const int tok = t0 + i - sinks;  // position after the sinks
    if (tok < Q) {
      const uint8_t* rec = record_ptr(L, seq, h, tok / G);
      const int t = tok % G;
      const uint32_t* kc = reinterpret_cast<const uint32_t*>(rec + L.kc_off);
      const int kper = 32 / kb;
      __half2 ksz;
      uint32_t kw;
      if (L.k_axis == 0) {
        ksz = reinterpret_cast<const __half2*>(rec + L.ksz_off)[d];
        kw = kc[kc_word_index(d, t / kper, G / kper)] >> ((t % kper) * kb);
      } else {  // per-token keys: (scale, zero) per (token, channel group), codes as above
        ksz = reinterpret_cast<const __half2*>(rec + L.ksz_off)[t * (D / L.group_v) + d / L.group_v];
        kw = kc[kc_word_index(d, t / kper, G / kper)] >> ((t % kper) * kb);
      }
      k_out[o] = dequant_value(kw & ((1u << kb) - 1), __low2half(ksz), __high2half(ksz));
      const uint32_t* vc = reinterpret_cast<const uint32_t*>(rec + L.vc_off);
      const int vper = 32 / vb;
      const uint32_t vq = (vc[vc_word_index(t, d / vper, G, kb, D / vper)] >> ((d % vper) * vb)) & ((1u << vb) - 1);
      const __half* vsz = reinterpret_cast<const __half*>(rec + L.vsz_off);
      const int ng = D / L.group_v, gg = d / L.group_v;
      v_out[o] = dequant_value(vq, vsz[vsz_half_index(t, gg, G, kb, ng, false)], vsz[vsz_half_index(t, gg, G, kb, ng, true)]);
    } else {
      const int64_t src = (((int64_t)seq * L.num_kv_heads + h) * R + tok % R) * D + d;
      k_out[o] = load_kv(L.ring_k, src, L.kv_dtype);
      v_out[o] = load_kv(L.ring_v, src, L.kv_dtype);
    }
  }
}

cudaError_t launch_append(const AppendParams& p, int max_flush, cudaStream_t stream) {
  const LayerView& L = p.L;
  if (max_flush > 0) {
    const bool rot = L.hadamard != 0;
    const size_t smem = (size_t)2 * L.group_k * L.head_dim * (rot ? sizeof(float) : sizeof(uint16_t));
    // The shared-memory opt-in is per function and per device.
    static uint64_t attr_set_mask[2] = {0, 0};
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) return e0;
    if (dev >= 64 || !(attr_set_mask[rot] & (1ull << dev))) {
      e0 = rot ? cudaFuncSetAttribute(quantize_blocks_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      2 * 128 * kHeadDim * (int)sizeof(float))
               : cudaFuncSetAttribute(quantize_blocks_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      2 * 128 * kHeadDim * (int)sizeof(uint16_t));
      if (e0 != cudaSuccess) return e0;
      if (dev < 64) attr_set_mask[rot] |= 1ull << dev;
    }
    dim3 grid(max_flush, p.batch, L.num_kv_heads);
    if (rot) quantize_blocks_kernel<true><<<grid, kQuantThreads, smem, stream>>>(p);
    else quantize_blocks_kernel<false><<<grid, kQuantThreads, smem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dim3 grid2(p.batch, L.num_kv_heads);
  ring_write_kernel<<<grid2, 128, 0, stream>>>(p);
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
