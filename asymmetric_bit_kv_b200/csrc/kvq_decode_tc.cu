// Host side of the tensor-core decode kernel (kvq_decode_tc.cuh): which
// layers it serves, its shared-memory plan, its occupancy and the dispatch to
// the instance of a layer's (key bits, value bits, value groups, key n-tiles).
#include <algorithm>
#include <mutex>

#include "kvq_decode_tc.cuh"

namespace kvq {
namespace tc {
#define KVQ_TC_DECL(K, N)                                                                                   \
  cudaError_t launch_tc_k##K##_##N(int vb, int ngrp, bool pt, const DecodeParams& p, const MmaPlan& mp,           \
                                   cudaStream_t s);                                                              \
  const void* fn_tc_k##K##_##N(int vb, int ngrp, bool pt);
KVQ_TC_DECL(2, 1)
KVQ_TC_DECL(2, 2)
KVQ_TC_DECL(4, 1)
KVQ_TC_DECL(4, 2)
KVQ_TC_DECL(8, 1)
KVQ_TC_DECL(8, 2)
#undef KVQ_TC_DECL
#define KVQ_PAIR_DECL(V)                                                                                   \
  cudaError_t launch_pair_v##V(int ngrp, const DecodeParams& p, const MmaPlan& mp, cudaStream_t s);            \
  const void* fn_pair_v##V(int ngrp);
KVQ_PAIR_DECL(2)
KVQ_PAIR_DECL(4)
KVQ_PAIR_DECL(8)
#undef KVQ_PAIR_DECL
}  // namespace tc

namespace {

int key_ntiles(const LayerView& L, int num_q_heads) { return num_q_heads / L.num_kv_heads > 4 ? 2 : 1; }

// 32-token blocks with 2-bit keys (the pair layout): decode_pair_kernel.
bool pair_path(const LayerView& L) { return pair_layout(L.group_k, L.k_bits); }

const void* instance_for(const LayerView& L, int num_q_heads) {
  const int vb = L.v_bits, ng = kHeadDim / L.group_v, nkt = key_ntiles(L, num_q_heads);
  if (pair_path(L)) return vb == 2 ? tc::fn_pair_v2(ng) : vb == 4 ? tc::fn_pair_v4(ng) : tc::fn_pair_v8(ng);
#define KVQ_TC_PICK(K, N) \
  if (L.k_bits == K && nkt == N) return tc::fn_tc_k##K##_##N(vb, ng, L.k_axis == 1);
  KVQ_TC_PICK(2, 1) KVQ_TC_PICK(2, 2) KVQ_TC_PICK(4, 1) KVQ_TC_PICK(4, 2) KVQ_TC_PICK(8, 1) KVQ_TC_PICK(8, 2)
#undef KVQ_TC_PICK
  return nullptr;
}

}  // namespace

// Largest dynamic shared memory a CTA of the current device may opt in to,
// less 1 KB for the kernel's static shared memory; 0 if unknown.
int smem_limit() {
  static int memo[64];  // per device, +1 (0: not queried yet)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    (void)cudaGetLastError();
    return 0;
  }
  if (dev < 64 && memo[dev] > 0) return memo[dev] - 1;
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  const int lim = std::max(0, optin - 1024);
  if (dev < 64) memo[dev] = lim + 1;
  return lim;
}

bool mma_supported(const LayerView& L, int num_q_heads) {
  if (L.head_dim != kHeadDim) return false;
  if (L.residual_v != L.residual) return false;  // one ring for keys and values
  if (pair_path(L)) {
    // per-channel keys, no rotation, at most two query rows per KV head
    // (they share the B operand with the second channel set and the value
    // groups)
    if (L.k_axis != 0 || L.hadamard || num_q_heads > 2 * L.num_kv_heads) return false;
    return make_mma_plan(L, num_q_heads).smem_bytes <= smem_limit();
  }
  // per-token keys with one group per head vector (BQ2_0), with or without
  // the rotation; the rotation with per-channel keys runs on the CUDA-core
  // kernel
  if (L.k_axis == 1 && L.group_v != kHeadDim) return false;
  if (L.hadamard && L.k_axis != 1) return false;
  if (L.group_k < 64) return false;                   // tiles of 64 tokens (blocks of 128 are two of them)
  if (L.v_bits == 2 && L.group_v < 64) return false;  // a 2-bit value chunk spans 64 channels
  // two stages per warp must fit
  return make_mma_plan(L, num_q_heads).smem_bytes <= smem_limit();
}

MmaPlan make_mma_plan(const LayerView& L, int num_q_heads) {
  MmaPlan mp;
  const int G = L.group_k;
  const int NG = num_q_heads / L.num_kv_heads;
  const int nkt = key_ntiles(L, num_q_heads);
  // a stage holds one tile item as [kc | ksz | vc | vsz]: the record itself
  // (one tile), or a tile part of a longer block (plus the block's
  // per-channel key scales, when it stores them once for all its tiles)
  const int NT = G / L.tile_tokens;
  mp.lg_nt = NT == 4 ? 2 : NT == 2 ? 1 : 0;  // G / tile_tokens: 1, 2 (or 4)
  const int ksz_stage = L.rec_ksz_off >= 0 ? kHeadDim * 4 : L.vc_off - L.ksz_off;
  mp.kc_bytes = L.ksz_off;
  mp.vc_soff = mp.kc_bytes + ksz_stage;
  mp.vsz_soff = mp.vc_soff + (L.vsz_off - L.vc_off);
  mp.tx_bytes = NT == 1 ? L.tile_bytes : (L.rec_ksz_off >= 0 ? kHeadDim * 4 : 0) + L.tile_bytes;
  const int ring_bytes = 2 * kResChunk * tc::kRowBytes;  // key and value rows of a ring chunk
  mp.stage_bytes = (int32_t)round_up(std::max(mp.tx_bytes, ring_bytes), 128);
  // per-consumer-warp scratch
  mp.bfrag_off = 0;
  mp.bias_off = nkt * 8 * 32 * 8;
  mp.qbuf_off = (int32_t)round_up(mp.bias_off + 32, 128);
  // Stages (and query buffers) per warp: two (one being read, one landing)
  // when two CTAs then fit an SM, else up to four with one CTA per SM.
  auto smem_for = [&](int spw) {
    const int ws = (int)round_up(mp.qbuf_off + spw * NG * tc::kRowBytes, 128);
    return tc::kNC * (spw * (mp.stage_bytes + 8) + ws);
  };
  int spw = 2;
  if (smem_for(2) > 113 * 1024)
    while (spw < 4 && smem_for(spw + 1) <= 226 * 1024) ++spw;
  mp.nstages = spw;
  mp.ws_bytes = (int32_t)round_up(mp.qbuf_off + spw * NG * tc::kRowBytes, 128);
  mp.ws_soff = tc::kNC * spw * mp.stage_bytes;
  mp.bar_off = mp.ws_soff + tc::kNC * mp.ws_bytes;
  mp.smem_bytes = mp.bar_off + tc::kNC * spw * 8;
  return mp;
}

int mma_ctas_per_sm(const LayerView& L, const MmaPlan& mp, int num_q_heads) {
  const void* fn = instance_for(L, num_q_heads);
  if (!fn) return 1;
  // Once per (device, instance): opt the instance in to the device's largest
  // dynamic shared memory (so that no plan can exceed what was opted in);
  // then one occupancy query per (device, instance, shared-memory size).
  struct Entry {
    int dev;
    const void* fn;
    int smem;  // -1: the opt-in record of (dev, fn)
    int n;
  };
  static Entry memo[256];
  static int nmemo = 0;
  static std::mutex mu;
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> lock(mu);
  bool opted = false;
  for (int i = 0; i < nmemo; ++i) {
    if (memo[i].dev != dev || memo[i].fn != fn) continue;
    if (memo[i].smem == mp.smem_bytes) return memo[i].n;
    if (memo[i].smem == -1) opted = true;
  }
  if (nmemo + 2 > 256) return 1;
  if (!opted) {
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, fn) != cudaSuccess ||
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes) !=
            cudaSuccess) {
      (void)cudaGetLastError();  // the launch reports its own error, not this one
      return 1;
    }
    memo[nmemo++] = Entry{dev, fn, -1, 0};
  }
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, tc::kThreads, mp.smem_bytes) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    return 1;
  }
  memo[nmemo++] = Entry{dev, fn, mp.smem_bytes, n};
  return n;
}

int mma_max_rows(const LayerView& L) { return pair_path(L) ? 2 : 8; }

cudaError_t launch_decode_mma(const DecodeParams& p, const MmaPlan& mp, cudaStream_t stream) {
  const LayerView& L = p.L;
  const int vb = L.v_bits, ng = kHeadDim / L.group_v, nkt = key_ntiles(L, p.num_q_heads);
  if (pair_path(L))
    return vb == 2 ? tc::launch_pair_v2(ng, p, mp, stream)
                   : vb == 4 ? tc::launch_pair_v4(ng, p, mp, stream) : tc::launch_pair_v8(ng, p, mp, stream);
#define KVQ_TC_GO(K, N) \
  if (L.k_bits == K && nkt == N) return tc::launch_tc_k##K##_##N(vb, ng, L.k_axis == 1, p, mp, stream);
  KVQ_TC_GO(2, 1) KVQ_TC_GO(2, 2) KVQ_TC_GO(4, 1) KVQ_TC_GO(4, 2) KVQ_TC_GO(8, 1) KVQ_TC_GO(8, 2)
#undef KVQ_TC_GO
  return cudaErrorInvalidValue;
}

}  // namespace kvq
