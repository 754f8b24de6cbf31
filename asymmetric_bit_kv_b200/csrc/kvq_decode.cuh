// Parameters and launchers of the split-KV decode attention kernels.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Split-KV decode over one layer. Two ways of cutting the work, each with
// its own partial-slot numbering per (sequence, query head):
//  * split mode (CUDA-core kernel): slot 0 is the residual ring; slot s >= 1
//    covers quantized blocks [(s-1)*blocks_per_split, min(s*blocks_per_split,
//    nblk));
//  * persistent mode (tensor-core kernel): the quantized blocks of all
//    (sequence, KV head) units, concatenated in (sequence, head, block) order,
//    are cut into num_ctas contiguous ranges (CTA c takes
//    [c*T/num_ctas, (c+1)*T/num_ctas)); slot 0 holds the residual ring,
//    slot 1 + 4*(c - c0) + w the blocks that warp w of CTA c processed for
//    the unit, c0 being the unit's first CTA.
struct DecodeParams {
  LayerView L;
  const void* q;        // [batch][Hq][D], kv dtype
  void* out;            // [batch][Hq][D], out dtype
  float* ws_o;          // [max_batch][Hq][slots][D] unnormalised partial outputs
  float2* ws_ml;        // [max_batch][Hq][slots]: (running max in log2 units, sum)
  float scale_log2;     // softmax scale * log2(e)
  int32_t out_dtype;
  int32_t batch;
  int32_t num_q_heads;
  int32_t blocks_per_split;
  int32_t slots;        // partial slots per (sequence, query head)
  int32_t* err;         // device word: a kernel sets bit 0 when a bounded wait gave up
  int32_t persistent;   // 1: persistent-mode slots (see above)
  int32_t total_blocks; // T, persistent mode
  int32_t num_ctas;     // persistent mode
  int32_t nblk[KVQ_MAX_BATCH];       // quantized blocks per sequence (host mirror)
  int32_t seq_start[KVQ_MAX_BATCH];  // first global block of sequence b: sum_{b'<b} nblk*Hkv
};

constexpr int kResidualSlots = 1;  // persistent mode: the residual ring's partial

// Persistent mode: first global block of CTA c, and the CTA holding block k.
__host__ __device__ inline int32_t cta_first_block(int64_t T, int32_t nctas, int32_t c) {
  return (int32_t)((int64_t)c * T / nctas);
}
__host__ __device__ inline int32_t cta_of_block(int64_t T, int32_t nctas, int32_t k) {
  int32_t c = (int32_t)((int64_t)k * nctas / T);
  while (c + 1 < nctas && cta_first_block(T, nctas, c + 1) <= k) ++c;
  while (c > 0 && cta_first_block(T, nctas, c) > k) --c;
  return c;
}
// Number of partial slots a (sequence, head) unit uses in persistent mode.
__host__ __device__ inline int32_t persistent_slots(int64_t T, int32_t nctas, int32_t unit_start, int32_t nblk) {
  if (nblk <= 0) return kResidualSlots;
  const int32_t c0 = cta_of_block(T, nctas, unit_start);
  const int32_t c1 = cta_of_block(T, nctas, unit_start + nblk - 1);
  return kResidualSlots + 4 * (c1 - c0 + 1);
}

// Shared-memory plan of the tensor-core decode kernel: NS stages, each one
// block record exactly as stored (its layout is bank-conflict-free for
// ldmatrix), then one scratch area per consumer warp.
struct MmaPlan {
  int32_t tx_bytes;     // bytes of one record copy (kc | ksz | vc | vsz)
  int32_t kc_bytes;     // key codes (then 4*D bytes of key scale/zero)
  int32_t vc_soff;      // value codes
  int32_t vsz_soff;     // value scale/zero
  int32_t stage_bytes;
  int32_t nstages;
  int32_t ws_soff;      // first consumer-warp scratch
  int32_t ws_bytes;     // bytes per consumer-warp scratch
  int32_t afrag_off;    // scratch: A fragments (scaled query, fp16 high/low)
  int32_t bias_off;     // scratch: per-head sum_d q_d z_d
  int32_t vpair_off;    // scratch: value scale/zero of token pairs (fp16)
  int32_t wq_off;       // scratch: the unit's scaled queries (fp32)
  int32_t bar_off;      // offset of the mbarriers
  int32_t smem_bytes;   // dynamic shared memory per CTA
};

bool mma_supported(const LayerView& L);
MmaPlan make_mma_plan(const LayerView& L);
int mma_ctas_per_sm(const LayerView& L, const MmaPlan& mp);
cudaError_t launch_decode_mma(const DecodeParams& p, const MmaPlan& mp, int max_splits, cudaStream_t stream);

// Enqueue the CUDA-core split kernel (any supported shape) and the
// log-sum-exp combine. max_splits is the largest quantized split count of any
// sequence (from the host mirror).
cudaError_t launch_decode(const DecodeParams& p, int max_splits, cudaStream_t stream);

// The log-sum-exp combine alone (after launch_decode_mma).
cudaError_t launch_combine(const DecodeParams& p, cudaStream_t stream);

// Device memory for the split partials other than the arena's workspace.
struct StaticScratch {
  uint8_t* base;   // device address, 256-byte aligned
  int64_t bytes;
};

// Host side of kvq_decode_attention (kvq_api.cu): validation, split plan and
// launches; the partials go to `scratch` when it is not null.
kvq_status enqueue_decode(kvq_cache* c, int32_t layer, const void* q, void* out, int32_t out_dtype,
                          float softmax_scale, int32_t batch, void* stream, const StaticScratch* scratch);
void clear_last_error();
kvq_status report_cuda_error(cudaError_t e, const char* what);

}  // namespace kvq
