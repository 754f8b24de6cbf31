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

// grid (max flush blocks, batch, Hkv); block kQuantThreads; dynamic smem 2*G*D*2 bytes.
__global__ void __launch_bounds__(kQuantThreads) quantize_blocks_kernel(AppendParams p) {
  const int j = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  if (j >= p.flush[b]) return;
  const LayerView& L = p.L;
  const int G = L.group_k, D = L.head_dim, R = L.residual;
  const int kb = L.k_bits, vb = L.v_bits, Gv = L.group_v;
  extern __shared__ uint16_t smem[];
  uint16_t* sk = smem;              // [G][D]
  uint16_t* sv = smem + G * D;      // [G][D]

  const int first = p.q_old[b] + j * G;  // absolute index of the block's first token
  const int boundary = p.q_old[b] + p.n_old[b];
  const int64_t ring_base = ((int64_t)b * L.num_kv_heads + h) * R;
  // Stage the G x D block, 8 values (16 bytes) per load.
  const int vec_per_tok = D / 8;
  for (int idx = threadIdx.x; idx < G * vec_per_tok; idx += blockDim.x) {
    const int t = idx / vec_per_tok, c = (idx % vec_per_tok) * 8;
    const int i = first + t;
    const uint4* ksrc;
    const uint4* vsrc;
    if (i < boundary) {
      const int64_t off = (ring_base + i % R) * D + c;
      ksrc = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(L.ring_k) + off);
      vsrc = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(L.ring_v) + off);
    } else {
      const int64_t row = (int64_t)p.in_off[b] + (i - boundary);
      const int64_t off = (row * L.num_kv_heads + h) * D + c;
      ksrc = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.k_in) + off);
      vsrc = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.v_in) + off);
    }
    *reinterpret_cast<uint4*>(sk + t * D + c) = *ksrc;
    *reinterpret_cast<uint4*>(sv + t * D + c) = *vsrc;
  }
  __syncthreads();

  uint8_t* rec = record_ptr(L, b, h, p.q_old[b] / G + j);
  uint32_t* kc = reinterpret_cast<uint32_t*>(rec + L.kc_off);
  __half2* ksz = reinterpret_cast<__half2*>(rec + L.ksz_off);
  uint32_t* vc = reinterpret_cast<uint32_t*>(rec + L.vc_off);
  __half* vsz = reinterpret_cast<__half*>(rec + L.vsz_off);
  const int dt = L.kv_dtype;

  // Keys: one group per channel over the G tokens (KIVI: per-channel keys).
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float mn = bits_to_float(sk[d], dt), mx = mn;
    for (int t = 1; t < G; ++t) {
      const float x = bits_to_float(sk[t * D + d], dt);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    const GroupParams gp = group_params(mn, mx, kb);
    ksz[d] = __halves2half2(gp.d16, gp.m16);
    const int per = 32 / kb;
    const int nw = G / per;  // words per channel, stored contiguously
    for (int w = 0; w < nw; ++w) {
      uint32_t word = 0;
      for (int i = 0; i < per; ++i)
        word |= quant_code(bits_to_float(sk[(w * per + i) * D + d], dt), gp, kb) << (i * kb);
      kc[kc_word_index(d, w, nw)] = word;
    }
  }

  // Values: one group per group_v channels of a token (KIVI: per-token
  // values). Each thread owns one output word (32/vb channels); the P threads
  // of a group combine their min/max with xor shuffles.
  const int per = 32 / vb;
  const int wpt = D / per;      // words per token
  const int P = Gv / per;       // threads per group, a power of two <= 32
  for (int widx = threadIdx.x; widx < G * wpt; widx += blockDim.x) {
    const int t = widx / wpt, w = widx % wpt;
    const uint16_t* xs = sv + t * D + w * per;
    float mn = bits_to_float(xs[0], dt), mx = mn;
    for (int i = 1; i < per; ++i) {
      const float x = bits_to_float(xs[i], dt);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    for (int o = P / 2; o >= 1; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const GroupParams gp = group_params(mn, mx, vb);
    uint32_t word = 0;
    for (int i = 0; i < per; ++i) word |= quant_code(bits_to_float(xs[i], dt), gp, vb) << (i * vb);
    vc[vc_word_index(t, w, G, kb, wpt)] = word;
    if ((w % P) == 0) {
      vsz[vsz_half_index(t, w / P, G, kb, D / Gv, false)] = gp.d16;
      vsz[vsz_half_index(t, w / P, G, kb, D / Gv, true)] = gp.m16;
    }
  }
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
      const __half2 ksz = reinterpret_cast<const __half2*>(rec + L.ksz_off)[d];
      const int kper = 32 / kb;
      const uint32_t kq = (kc[kc_word_index(d, t / kper, G / kper)] >> ((t % kper) * kb)) & ((1u << kb) - 1);
      k_out[o] = dequant_value(kq, __low2half(ksz), __high2half(ksz));
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
    const size_t smem = (size_t)2 * L.group_k * L.head_dim * sizeof(uint16_t);
    // The shared-memory opt-in is per function and per device.
    static uint64_t attr_set_mask = 0;
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) return e0;
    if (dev >= 64 || !(attr_set_mask & (1ull << dev))) {
      e0 = cudaFuncSetAttribute(quantize_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                2 * 128 * kHeadDim * (int)sizeof(uint16_t));
      if (e0 != cudaSuccess) return e0;
      if (dev < 64) attr_set_mask |= 1ull << dev;
    }
    dim3 grid(max_flush, p.batch, L.num_kv_heads);
    quantize_blocks_kernel<<<grid, kQuantThreads, smem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  dim3 grid2(p.batch, L.num_kv_heads);
  ring_write_kernel<<<grid2, 128, 0, stream>>>(p);
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
