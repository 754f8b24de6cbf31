// Parameters and launchers of the append / flush / dequantize kernels.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

constexpr int kQuantThreads = 256;

// Per-call append plan, passed by value (kernel parameter space up to 32 KB).
// Lengths are the host mirror's values before the call, as token positions
// after the sinks. Keys and values flush on their own (each tensor has its
// own ring); with one residual length their plans coincide.
struct AppendParams {
  LayerView L;
  const void* k_in;  // [sum t_new][Hkv][D], kv dtype
  const void* v_in;
  int32_t batch;
  int32_t parts;                   // CTAs per block and tensor of the quantize kernel (set by launch_append)
  int32_t q_old[KVQ_MAX_BATCH];    // quantized keys before the call
  int32_t qv_old[KVQ_MAX_BATCH];   // quantized values before the call
  int32_t len_old[KVQ_MAX_BATCH];  // tokens before the call (quantized keys + key ring)
  int32_t t_new[KVQ_MAX_BATCH];    // tokens appended by the call after the sinks
  int32_t in_off[KVQ_MAX_BATCH];   // first input row of each sequence after its sinks
  int32_t flush[KVQ_MAX_BATCH];    // G-token key blocks quantized by the call
  int32_t flush_v[KVQ_MAX_BATCH];  // G-token value blocks quantized by the call
  int32_t s_old[KVQ_MAX_BATCH];    // sink tokens before the call
  int32_t s_take[KVQ_MAX_BATCH];   // sink tokens taken by the call (input rows in_off - s_take ..)
};

// Enqueues the quantize kernel (max_flush = the largest key or value block
// count of any sequence; none if 0) and the ring / sink / length-table write.
// p.parts is chosen here.
cudaError_t launch_append(AppendParams& p, int max_flush, cudaStream_t stream);

// Paged caches: page-table entries set by one launch (table[idx[i]] =
// page[i]), enqueued before the append kernels that write the new pages.
constexpr int kMaxPageUpdates = 1536;
struct PageTableUpdate {
  int32_t* table;
  int32_t n;
  int32_t idx[kMaxPageUpdates];
  int32_t page[kMaxPageUpdates];
};
cudaError_t launch_page_table_update(const PageTableUpdate& u, cudaStream_t stream);
cudaError_t launch_dequant(const LayerView& L, int seq, int sinks, int t0, int t1, float* k_out, float* v_out,
                           cudaStream_t stream);

}  // namespace kvq
