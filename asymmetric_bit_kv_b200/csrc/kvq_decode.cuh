// Parameters and launchers of the split-KV decode attention kernels.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Split-KV decode over one layer. Two ways of cutting the work, each with
// its own partial-slot numbering per (sequence, query head):
//  * split mode (CUDA-core kernel): slot 0 is the residual ring; slot s >= 1
//    covers quantized blocks [(s-1)*blocks_per_split, min(s*blocks_per_split,
//    nblk));
//  * persistent mode (tensor-core kernel): the work of a (sequence, KV head)
//    unit is its quantized blocks followed by its ring tokens in chunks of
//    kResChunk (one chunk even for an empty sequence); the work items of all
//    units, concatenated in (sequence, head, item) order, are cut into
//    num_ctas contiguous ranges of equal cost (CTA c takes [cta_start[c],
//    cta_start[c+1]), every range non-empty; see plan_cta_starts), and slot
//    kMmaConsumers*(c - c0) + w holds what warp w of CTA c processed for the
//    unit, c0 being the unit's first CTA; every warp writes its slot of every
//    unit its CTA's range touches (zero weight if it had no items).
constexpr int kMaxCtas = 1024;  // persistent mode: CTAs of one decode launch

struct DecodeParams {
  LayerView L;
  const void* q;        // [batch][Hq][D], kv dtype
  void* out;            // [batch][Hq][D], out dtype
  float* ws_o;          // [batch][Hq][slots][D] unnormalised partial outputs
  float2* ws_ml;        // [batch][Hq][slots]: (running max in log2 units, sum)
  const void* new_k;    // fused decode step: this call's new token per sequence, [batch][Hkv][D]
  const void* new_v;    //   (ring index nres[b] - 1; null: no new token)
  float scale_log2;     // softmax scale * log2(e)
  float q_prescale;     // tensor-core kernel: power of two the queries are scaled by in fp16
  float score_scale;    // scale_log2 / q_prescale
  int32_t out_dtype;
  int32_t batch;
  int32_t num_q_heads;
  int32_t blocks_per_split;
  int32_t slots;        // partial slots per (sequence, query head): the slot stride
  int32_t* err;         // device word: a kernel sets bit 0 when a bounded wait gave up
  int32_t* unit_slots;  // persistent mode: [batch][Hkv] slot count of each unit, written by the decode kernel
  int32_t persistent;   // 1: persistent-mode slots (see above)
  int32_t total_blocks; // T, persistent mode: work items of all units
  int32_t num_ctas;     // persistent mode
  int32_t after_flush;  // persistent mode: launched after the flush kernel of a fused decode step
  int32_t max_unit_slots;  // persistent mode: a bound on the slots any unit uses (sizes the combine)
  // Query rows. A unit (sequence b, KV head h) has num_q_heads / Hkv rows:
  // row j is query token t = j / (q_heads / Hkv) of this launch and head
  // h * (q_heads / Hkv) + j % (q_heads / Hkv), read from row
  // b * q_rows + t * q_heads + that head of q (written to the same row of
  // out). Query token t attends to the ring except its last lag_base - t
  // tokens (several query tokens per sequence; one token: q_rows = q_heads,
  // lag_base = 0).
  int32_t q_heads;      // Hq of the q and out arrays
  int32_t q_rows;       // rows of q and out per sequence
  int32_t qtok;         // query tokens of this launch
  int32_t lag_base;
  int32_t nblk[KVQ_MAX_BATCH];       // quantized blocks per sequence (host mirror)
  int32_t nres[KVQ_MAX_BATCH];       // ring tokens per sequence (host mirror)
  int32_t nitem[KVQ_MAX_BATCH];      // persistent mode: work items per unit of sequence b
  int32_t seq_start[KVQ_MAX_BATCH];  // first global item (block in split mode) of sequence b
  int32_t cta_start[kMaxCtas + 1];   // persistent mode: first global item of CTA c
};

constexpr int kMmaConsumers = 6;   // warps per CTA of the tensor-core kernel
constexpr int kResChunk = 8;       // ring tokens per work item, persistent mode
static_assert(KVQ_MAX_SINKS == kResChunk, "the sink rows of a unit are one exact-token chunk");

// Work items of one unit: quantized blocks, then ring chunks, then one chunk
// of sink tokens if the sequence has any (at least one item: an empty
// sequence gets one ring chunk with no tokens).
__host__ __device__ inline int32_t unit_items(int32_t nblk, int32_t nres, int32_t nsink) {
  const int32_t items = nblk + (nres + kResChunk - 1) / kResChunk + (nsink > 0 ? 1 : 0);
  return items > 0 ? items : 1;
}

// Persistent mode: the CTA whose item range [starts[c], starts[c+1]) holds
// item k (starts strictly increasing, starts[0] = 0).
__host__ __device__ inline int32_t cta_of_item(const int32_t* starts, int32_t nctas, int32_t k) {
  int32_t lo = 0, hi = nctas - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (starts[mid] <= k) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Cost of a unit's items in half units: a quantized block 2, an exact-token
// chunk 1. CTA c of N starts at the item whose cost interval holds c*C/N (C:
// the total cost), so N <= C / (largest item cost) keeps every range
// non-empty, and a unit of cost u overlaps at most floor(u*N/C) + 2 ranges.
__host__ __device__ inline int64_t unit_cost(int32_t nblk, int32_t nitem) { return 2 * (int64_t)nblk + (nitem - nblk); }

// Parameters of the flush kernel of a fused decode step: CTA i quantizes,
// for (sequence i / Hkv, KV head i % Hkv) whose ring holds R tokens, the
// oldest G ring tokens into the next block record.
struct FlushParams {
  LayerView L;
  int32_t ctas;  // batch * Hkv
};
cudaError_t launch_step_flush(const FlushParams& p, cudaStream_t stream);

// Shared-memory plan of the tensor-core decode kernel: per warp nstages
// stages (a block record exactly as stored, or the key and value rows of a
// ring chunk), then one scratch area per warp, then the stage barriers.
struct MmaPlan {
  int32_t tx_bytes;     // bytes of one record copy (kc | ksz | vc | vsz)
  int32_t kc_bytes;     // key codes (then 4*D bytes of key scale/zero)
  int32_t vc_soff;      // value codes
  int32_t vsz_soff;     // value scale/zero
  int32_t stage_bytes;
  int32_t nstages;      // stages per warp
  int32_t lg_nt;        // log2 of the tile items per block record
  int32_t ws_soff;      // first consumer-warp scratch
  int32_t ws_bytes;     // bytes per consumer-warp scratch
  int32_t bfrag_off;    // scratch: key B fragments (q*s, fp16 high/low)
  int32_t bias_off;     // scratch: per-head sum_d q_d z_d
  int32_t qbuf_off;     // scratch: the queries of the warp's current units (kv dtype)
  int32_t bar_off;      // offset of the mbarriers
  int32_t smem_bytes;   // dynamic shared memory per CTA
};

bool mma_supported(const LayerView& L, int num_q_heads);
int mma_max_rows(const LayerView& L);  // query rows per KV head one tensor-core launch takes
MmaPlan make_mma_plan(const LayerView& L, int num_q_heads);
int mma_ctas_per_sm(const LayerView& L, const MmaPlan& mp, int num_q_heads);
cudaError_t launch_decode_mma(const DecodeParams& p, const MmaPlan& mp, cudaStream_t stream);

// Enqueue the CUDA-core split kernel (any supported shape) and the
// log-sum-exp combine. max_splits is the largest quantized split count of any
// sequence (from the host mirror).
cudaError_t launch_decode(const DecodeParams& p, int max_splits, cudaStream_t stream);
// Resident CTAs per SM of the CUDA-core split kernel for this head ratio.
int split_ctas_per_sm(int num_q_heads, int num_kv_heads);

// Parameters of the log-sum-exp combine (small: no per-sequence tables).
struct CombineParams {
  const float* ws_o;
  const float2* ws_ml;
  void* out;
  const int32_t* unit_slots;  // persistent mode: slots per unit
  const int32_t* lens;        // split mode: the layer's length table (kLensStride per sequence)
  int32_t out_dtype, num_q_heads, num_kv_heads, slots, group_k, blocks_per_split, persistent;
  int32_t hadamard;  // split mode: slots >= 1 (quantized tokens) hold rotated partials
  int32_t q_heads, q_rows;  // output row of query row j of a unit: see DecodeParams
};

// The log-sum-exp combine of the partial slots (after the decode kernel).
cudaError_t launch_combine(const DecodeParams& p, cudaStream_t stream);

// Device memory for the split partials other than the arena's workspace.
struct StaticScratch {
  uint8_t* base;   // device address, 256-byte aligned
  int64_t bytes;
};

// Several query tokens per sequence, one launch's share (see DecodeParams):
// q and out point at the group's first query token.
struct QueryGroup {
  int32_t q_rows, qtok, lag_base;
};

// Host side of kvq_decode_attention (kvq_api.cu): validation, split plan and
// launches; the partials (and the slot table) go to `scratch` when it is not
// null; qg: a group of query tokens (null: one query token per sequence);
// new_k/new_v: a fused decode step's new tokens; after_flush: the step's
// flush kernel was enqueued just before.
kvq_status enqueue_decode(kvq_cache* c, int32_t layer, const void* new_k, const void* new_v, const void* q, void* out,
                          int32_t out_dtype, float softmax_scale, int32_t batch, void* stream,
                          const StaticScratch* scratch, const QueryGroup* qg = nullptr, bool after_flush = false);
void clear_last_error();
kvq_status report_cuda_error(cudaError_t e, const char* what);
kvq_status report_status(kvq_status s, const char* what);
int cache_device(const kvq_cache* c);  // the device current when the cache was created

}  // namespace kvq
