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
};

// Enqueue the split kernel and the log-sum-exp combine. max_splits is the
// largest quantized split count of any sequence (from the host mirror).
cudaError_t launch_decode(const DecodeParams& p, int max_splits, cudaStream_t stream);

}  // namespace kvq
