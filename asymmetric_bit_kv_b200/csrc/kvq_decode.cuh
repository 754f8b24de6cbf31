// Parameters and launchers of the split-KV decode attention kernels.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Split-KV decode over one layer. Split 0 of every (sequence, KV head) is the
// residual ring; split s >= 1 covers quantized blocks
// [(s-1)*blocks_per_split, min(s*blocks_per_split, nblk)).
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
};

// Shared-memory plan of the tensor-core decode kernel (one stage = one block
// record; value codes land in segments padded by 16 bytes).
struct MmaPlan {
  int32_t kc_bytes;     // key codes of a record (then 4*D bytes of key scale/zero)
  int32_t vseg_bytes;   // value codes of one segment of 16/k_bits tokens
  int32_t vseg_count;   // segments per block
  int32_t vsz_bytes;    // value scale/zero of a record
  int32_t vc_soff;      // stage offset of the first value segment
  int32_t vsz_soff;     // stage offset of the value scale/zero
  int32_t stage_bytes;
  int32_t tx_bytes;     // bytes one stage receives
  int32_t nstages;
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

}  // namespace kvq
