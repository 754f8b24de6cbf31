/*
 * kvq.h -- C ABI of a B200 (sm_100a) library for an asymmetric 2/4/8-bit
 * KV cache and decode attention over it.
 *
 * The method (web pages, cited by title and section):
 *  - "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache" (README),
 *    sections "Overview" and "Example": keys are quantized per channel and
 *    values per token, at 2 or 4 bits (k_bits, v_bits) with a group size, and
 *    the residual_length most recent tokens stay in full precision; the GQA
 *    update (2025.01.18) adds grouped-query attention.
 *  - "KV1-1.2B" model card, section "Quantization Format: KV1.cpp BQ2_0":
 *    the quantizer itself -- in fp32, d = fp16(max((max-min)/(2^b-1), 1e-6)),
 *    m = fp16(min), q = clamp(round_half_to_even((x - m) / d), 0, 2^b-1) with
 *    the fp16-rounded m and d, dequantization x_hat = q*d + m, and codes packed
 *    lowest bits first.
 *  - "Quantize What Counts: More For Keys, Less For Values", section "KV Cache
 *    Quantization": key and value bit widths chosen independently and per
 *    layer (bit range up to 8); residual length, group size and axis given
 *    per tensor ({"k": ..., "v": ...}).
 *
 * Ownership. The caller allocates one device arena per cache (size from
 * kvq_cache_required_bytes) and owns it, every input and output buffer and
 * every stream. The library never allocates device memory. A kvq_cache handle
 * is host memory owned by the library (freed by kvq_cache_destroy) and must
 * not outlive its arena.
 *
 * Errors. Every entry point validates its arguments on the host before it
 * enqueues anything; on failure it returns a negative kvq_status, enqueues no
 * work and leaves the cache unchanged. kvq_last_error() gives a one-line
 * reason. KVQ_ERR_CUDA reports a failed launch. Work is asynchronous on the
 * given stream (a cudaStream_t; NULL = legacy default stream); faults during
 * execution surface at the caller's next synchronisation, as for any CUDA
 * kernel. Calls on one cache must be ordered on one stream: they share the
 * arena's length table, decode plan and split-partial workspace.
 *
 * Threading. A handle is not thread-safe; distinct handles are independent.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = -1, /* null pointer, bad index, bad shape or size  */
  KVQ_ERR_UNSUPPORTED = -2, /* valid but not built: bits, dims, dtype      */
  KVQ_ERR_CAPACITY = -3,    /* a sequence would exceed max_tokens, or a
                               paged layer's pool has too few free pages   */
  KVQ_ERR_WORKSPACE = -4,   /* arena smaller than kvq_cache_required_bytes,
                               or a call's split partials do not fit the
                               memory they go to (arena workspace or the
                               static scratch of the no-alloc decode)      */
  KVQ_ERR_CUDA = -5         /* a CUDA launch or call failed                */
} kvq_status;

typedef enum kvq_dtype { KVQ_F16 = 0, KVQ_BF16 = 1, KVQ_F32 = 2 } kvq_dtype;

#define KVQ_MAX_BATCH 512  /* sequences per cache                        */
#define KVQ_MAX_LAYERS 512 /* layers per cache                           */
#define KVQ_MAX_SPLITS 256 /* quantized splits per (sequence, KV head)   */
#define KVQ_MAX_SINKS 8    /* sink tokens per sequence                   */

/* Cache shape. Names follow the KIVI README "Example" (k_bits, v_bits,
 * group_size, residual_length) with the group size and residual length
 * given per tensor as in "Quantize What Counts", KV Cache Quantization
 * (group_size {"k", "v"}, residual_length {"k", "v"}).                     */
typedef struct kvq_config {
  int32_t num_layers;   /* 1 .. KVQ_MAX_LAYERS                              */
  int32_t max_batch;    /* sequences, 1 .. KVQ_MAX_BATCH                    */
  int32_t num_q_heads;  /* Hq, a multiple of num_kv_heads                   */
  int32_t num_kv_heads; /* Hkv; Hq/Hkv in {1, 2, 4, 8}                      */
  int32_t head_dim;     /* D = 128                                          */
  int32_t max_tokens;   /* per-sequence capacity: sinks + quantized + residual */
  int32_t group_k;      /* G: tokens per key group (one group per channel);
                           32, 64 or 128. Flushes move G tokens at a time.  */
  int32_t group_v;      /* channels per value group (one group per token);
                           32, 64 or 128, dividing head_dim                 */
  int32_t residual;     /* R: full-precision key ring slots (and value ring
                           slots unless residual_v is set); a multiple of G */
  int32_t kv_dtype;     /* KVQ_F16 or KVQ_BF16: keys, values, ring, queries */
  const int8_t* k_bits; /* host [num_layers], each 2, 4 or 8 (copied)       */
  const int8_t* v_bits; /* host [num_layers], each 2, 4 or 8 (copied)       */
  int32_t sink_tokens;  /* S, 0..KVQ_MAX_SINKS: the first S tokens of every
                           sequence are kept exact and never quantized
                           (KV1-1.2B card: attention sinks, 4 in KV1);
                           quantization and the ring start at token S      */
  const int8_t* k_axis; /* host [num_layers] or null (all 0), copied: 0 keys
                           per channel over G tokens (KIVI), 1 keys per token
                           over group_v channels like values (KV1 BQ2_0)    */
  int32_t hadamard;     /* 1: every K and V head vector is multiplied by the
                           normalized Sylvester Hadamard matrix H before it
                           is quantized, queries by H for quantized tokens
                           and their output contribution by H again (KV1
                           BQ2_0); sinks and ring stay exact. 0: none       */
  int32_t page_blocks;  /* 0: every (sequence, KV head) owns max_tokens/G
                           block records up front (contiguous). >= 1: block
                           records live in pages of page_blocks blocks of
                           one sequence (all its KV heads), drawn per layer
                           from a pool of pool_pages pages as the sequence's
                           quantized part grows and returned by
                           kvq_release_sequence / kvq_cache_reset, so a
                           ragged batch holds only the pages it uses        */
  int32_t pool_pages;   /* pages per layer when page_blocks >= 1            */
  int32_t residual_v;   /* 0: values share R. Else the value ring's slots, a
                           multiple of G: keys and values then keep their own
                           full-precision windows and each flushes its own
                           oldest G tokens when its ring is full ("Quantize
                           What Counts": residual_length {"k", "v"}). Not
                           with hadamard. Layers run on the CUDA-core
                           decode kernel when it differs from residual.     */
} kvq_config;

typedef struct kvq_cache kvq_cache;

/* Where one layer's packed cache lives, for tests and tools that read it.
 * Token positions below are counted after the sequence's s sink tokens
 * (s = min(S, tokens appended so far)): position i is token s + i.
 * Block records: for sequence b, KV head h and key block j (positions
 * [j*G, (j+1)*G) of that sequence) the record starts at
 *   blocks + ((b * num_kv_heads + h) * max_blocks + j) * record_bytes
 * (a paged cache: see page_table below). A record is a run of tiles of
 * T = min(G, 64) tokens: tile i (tokens i*T ..) starts at tile0_offset +
 * i*tile_bytes, and holds at the given byte offsets from its start
 * (t below: the token's index inside the tile):
 *   kc  uint32 [D][W], W = T*k_bits/32: channel d's row holds W words; word
 *       w packs the codes of tokens w*(32/k_bits) + i, i = 0.., code i at
 *       bits [i*k_bits, ...) (per-channel keys packed along the token axis);
 *   ksz half2 [D]: (scale d, zero point m) of each channel's key group --
 *       when G = 128 these pairs are stored once per record, at
 *       rec_ksz_offset (a block has one key group per channel), and the tile
 *       holds none (rec_ksz_offset = -1 otherwise);
 *   (k_axis 1: kc exactly as above, codes of each channel packed along the
 *   token axis; ksz half2 [T][D/group_v], (scale, zero point) per (token,
 *   channel group), row-major, in every tile);
 *   vc  uint32 [T][V], V = D*v_bits/32: one row of V words per token; word w
 *       packs the codes of channels w*(32/v_bits) + i, code i at bits
 *       [i*v_bits, ...) (per-token values packed along head_dim);
 *   vsz fp16 scale and zero point of each (token, value group): for
 *       T = 64, and for the pair layout below, 16-byte entries in the order
 *       the decode kernel reads them (see kvq_internal.cuh:
 *       vsz_half_index); otherwise the pairs [T][D/group_v] of (scale, zero
 *       point).
 * Placement inside kc and vc (so that one copy of a tile is readable with
 * ldmatrix without shared-memory bank conflicts): in a row of n >= 2
 * 16-byte chunks (4 words each), chunk c of row r is stored at chunk
 * position c ^ s(r, n), with s(r, n) = r & 7 for n >= 8 and
 * (r / (8/n)) % n otherwise; rows of fewer than 4 words are not permuted.
 * Value rows are stored in token order t -> (t % c) * (T/c) + t / c, with
 * c = 16/k_bits. Pair layout (T = 32 with 2-bit keys, W = 2): the key rows
 * of channels d and d + 64 (d < 64) share 16 bytes, words 4d, 4d+1 (channel
 * d) and 4d+2, 4d+3 (channel d + 64); token t = 8a + b (b < 8) sits in value
 * row 16*(b/4) + 8*((b/2) % 2) + 2a + b % 2.
 * (kvq_internal.cuh: kc_word_index, vc_word_index,
 * kc_word_byte, ksz_pair_byte, vc_word_byte, vsz_half_byte.)
 * Rings: keys [max_batch][num_kv_heads][R][D] and values
 * [max_batch][num_kv_heads][RV][D] in kv_dtype (RV = residual_v, or R);
 * position i of a sequence whose key (value) is exact sits in slot i % R
 * (i % RV). With separate residual lengths a block record may hold only its
 * key part or only its value part (the other tensor's tokens are still in
 * their ring); kvq_seq_lengths / kvq_seq_value_lengths tell which.
 * Sinks: [max_batch][num_kv_heads][KVQ_MAX_SINKS][D] in kv_dtype; sink
 * token i (< s) in row i, the other rows zero.                             */
typedef struct kvq_layout {
  void* blocks;
  int64_t record_bytes;
  int64_t max_blocks;
  int64_t kc_offset, ksz_offset, vc_offset, vsz_offset;  /* inside a tile */
  void* ring_k;
  void* ring_v;
  int32_t k_bits, v_bits;
  void* sink_k;
  void* sink_v;
  int32_t k_axis, hadamard;
  /* paged caches (page_blocks >= 1): block j of (b, h) is record
   * (page * num_kv_heads + h) * page_blocks + j % page_blocks of `blocks`,
   * page = page_table[b * max_pages + j / page_blocks] (int32, device);
   * max_blocks is then the per-sequence capacity in blocks.               */
  void* page_table;
  int32_t page_blocks, max_pages;
  /* tiles of a record (see above)                                          */
  int32_t tile_tokens, tile_bytes, tile0_offset, rec_ksz_offset;
} kvq_layout;

/* Device bytes the arena must hold for cfg: all layers' block records and
 * rings, the length table, the decode plan and the split-partial workspace.
 * Sizes follow from the method's layout (KV1-1.2B card, Quantization Format:
 * b-bit codes plus an fp16 scale and zero point per group; KIVI README,
 * Overview: keys grouped per channel, values per token, R exact tokens).   */
KVQ_API kvq_status kvq_cache_required_bytes(const kvq_config* cfg, size_t* bytes);

/* Validate cfg and bind a cache to dev_arena (device pointer, 256-byte
 * aligned, arena_bytes >= required), with the arena's device current. Every
 * sequence starts empty: the call zeroes the arena's length table and
 * residual rings, and waits for that to finish before it returns. The cache
 * is the KIVI README's quantized KV cache ("Overview": per-channel keys,
 * per-token values, a full-precision residual window; "Example": k_bits,
 * v_bits, group_size, residual_length), one per model, all layers.         */
KVQ_API kvq_status kvq_cache_create(const kvq_config* cfg, void* dev_arena, size_t arena_bytes,
                            kvq_cache** out);

/* Free the host handle. Does not touch the arena.                          */
KVQ_API kvq_status kvq_cache_destroy(kvq_cache* cache);

/* Empty every sequence of every layer (stream-ordered).                    */
KVQ_API kvq_status kvq_cache_reset(kvq_cache* cache, void* stream);

/* Empty sequence `seq` in every layer (stream-ordered) and, in a paged
 * cache, return its pages to the pools. Calls that use the pages again are
 * ordered after this one on the same stream.                              */
KVQ_API kvq_status kvq_release_sequence(kvq_cache* cache, int32_t seq, void* stream);

/* Append new_lens[b] tokens to sequence b of `layer`, b < batch.
 * k, v: device, token-major [sum(new_lens)][num_kv_heads][head_dim] in
 * kv_dtype, sequences in order. new_lens: host [batch], each >= 0.
 * Semantics (KIVI README: residual window of recent full-precision tokens;
 * KV1 card: each token quantized once when it enters the cache, the first
 * S kept exact): tokens are appended one by one; each of a sequence's first
 * S tokens goes to its sinks as it is; a later token that finds the ring
 * full (R tokens) first
 * causes the oldest G ring tokens to be quantized -- keys per channel over
 * the G tokens, values per token over group_v channels -- into one block
 * record. Blocks that a long append would quantize straight away are read
 * from k, v directly. Fails with KVQ_ERR_CAPACITY if a sequence would exceed
 * max_tokens (sinks included) or, in a paged cache, if the layer's pool has
 * fewer free pages than the call's new blocks need; nothing is enqueued
 * then. A paged cache takes the pages in this call (and in
 * kvq_flush_residual and kvq_decode_step).                                 */
KVQ_API kvq_status kvq_append(kvq_cache* cache, int32_t layer, const void* k, const void* v,
                      const int32_t* new_lens, int32_t batch, void* stream);

/* Quantize every complete group of G tokens left in the rings of sequences
 * 0..batch-1 of `layer`: a ring of n tokens keeps n % G (KIVI README,
 * Overview: tokens leave the full-precision window in groups; the
 * end-of-prefill flush of its "Example"). Keys and values each flush their
 * own ring.                                                                */
KVQ_API kvq_status kvq_flush_residual(kvq_cache* cache, int32_t layer, int32_t batch, void* stream);

/* One decode query per sequence: out[b][h] = softmax(scale * q[b][h] K~^T) V~
 * over all cached tokens of sequence b (no mask), K~/V~ the exact sinks, the
 * dequantized blocks and the exact ring tokens; query head h reads KV head
 * h / (Hq/Hkv) (GQA). q: device [batch][Hq][D] in kv_dtype. out: device
 * [batch][Hq][D] in out_dtype (F32, F16 or BF16; round to nearest even).
 * A sequence with no tokens gives zeros. Uses the arena's decode plan and
 * workspace. This is the KIVI README's decoding over the quantized cache
 * ("Overview": attention over quantized keys and values plus the
 * full-precision recent tokens; GQA per its 2025.01.18 update), with
 * x_hat = q*d + m of the KV1-1.2B card (Quantization Format).              */
KVQ_API kvq_status kvq_decode_attention(kvq_cache* cache, int32_t layer, const void* q, void* out,
                                int32_t out_dtype, float softmax_scale, int32_t batch,
                                void* stream);

/* Size of the library's own device scratch for kvq_decode_attention_noalloc:
 * 16 MiB, held on every GPU that loads the library until the process exits. */
#define KVQ_STATIC_SCRATCH_BYTES (16u << 20)

/* Decode attention of num_tokens query tokens per sequence (verifying
 * drafted tokens in one pass). q: device [batch][num_tokens][Hq][D] in
 * kv_dtype; out: device [batch][num_tokens][Hq][D] in out_dtype. The query
 * tokens' keys and values must already be the sequence's num_tokens newest
 * cached tokens (kvq_append first): query token t, at position L - T + t,
 * attends to tokens 0 .. L - T + t (causal among the T). Those tokens must
 * still be in the ring: a sequence with fewer than num_tokens ring tokens is
 * refused with KVQ_ERR_UNSUPPORTED before anything is enqueued;
 * 1 <= num_tokens <= residual. num_tokens = 1 is kvq_decode_attention.
 * Runs as ceil(num_tokens * Hq / Hkv / 8) or a few more decode passes over
 * the cache (at most 8 query rows per KV head per pass); a launch failure in
 * a later pass leaves the earlier passes' rows of out written. The pages do
 * not describe several query tokens per sequence: this is the plainest
 * extension of their decoding rule (causal, like prefill).                 */
KVQ_API kvq_status kvq_decode_attention_multi(kvq_cache* cache, int32_t layer, const void* q, void* out,
                                              int32_t out_dtype, float softmax_scale, int32_t batch,
                                              int32_t num_tokens, void* stream);

/* Same result as kvq_decode_attention, for callers that cannot allocate
 * device memory at the point of the call, for example an engine whose device
 * memory is all handed to its own pool at start-up, or code running under a
 * fixed memory budget where a cudaMalloc could fail or stall the device.
 * This call allocates nothing. Its decode plan, per-unit slot counts and
 * split partials go to a static device array of KVQ_STATIC_SCRATCH_BYTES
 * that the library holds, not to the arena, whose workspace, plan and slot
 * table it leaves untouched; it still writes the cache's device error word
 * if a bounded wait gives up (kvq_device_errors). The pages have no
 * counterpart: this is an interface choice of this library.
 * - Size limit: after the plan (about 32 * batch bytes) and the slot table
 *   (4 * batch * Hkv bytes), each partial slot takes batch * Hq *
 *   (4*head_dim + 8) bytes; the call plans its split so that the slots a
 *   (sequence, query head) uses fit what remains, down to one CTA per unit.
 *   A call for which even that does not fit (fewer than 6 slots on the
 *   tensor-core kernel, 2 on the CUDA-core one) returns KVQ_ERR_WORKSPACE,
 *   enqueues nothing, and kvq_last_error() gives the sizes.
 * - Device: the current device must be the one the cache was created on
 *   (else KVQ_ERR_INVALID_ARG): the array is per device.
 * - Set-up: the first call on each device looks up the array's device
 *   address (cudaGetSymbolAddress, with that device current) and keeps it
 *   for the process. Make that first call before any stream capture. A
 *   cudaDeviceReset invalidates the kept address: do not call this entry
 *   point after one.
 * - Sharing: every call on a device uses the same array and leaves the last
 *   call's contents in it. Each call writes every plan entry, slot count and
 *   partial it reads before reading it, so nothing has to start at zero.
 *   Calls that may overlap on the GPU race on the array (different streams,
 *   or several caches): order them.                                        */
KVQ_API kvq_status kvq_decode_attention_noalloc(kvq_cache* cache, int32_t layer, const void* q, void* out,
                                        int32_t out_dtype, float softmax_scale, int32_t batch,
                                        void* stream);

/* One decode step: append one token to each sequence b < batch (k, v:
 * device [batch][num_kv_heads][head_dim] in kv_dtype, as kvq_append with
 * new_lens all 1), then decode attention for q over every token including
 * the new one (as kvq_decode_attention). Same results as those two calls.
 * When the layer runs on the tensor-core kernel, keys and values share one
 * residual length and every sequence's sinks are complete, the step is
 * fused: a small prep launch quantizes the oldest G tokens of every full
 * ring (only in steps where some ring is full) and plans the decode, and
 * the decode launch attends to the new tokens and writes them into their
 * ring slots -- no separate append kernels (the decode loop of the KV1-1.2B
 * card, Quickstart, where each token is quantized once as it enters the
 * cache; KIVI README, Overview, for the window). All checks run before
 * anything is enqueued.                                                   */
KVQ_API kvq_status kvq_decode_step(kvq_cache* cache, int32_t layer, const void* k, const void* v, const void* q,
                                   void* out, int32_t out_dtype, float softmax_scale, int32_t batch, void* stream);

/* Reconstruct tokens [t0, t1) of sequence `seq` as fp32: x_hat = q*d + m
 * (an fp32 product, then an fp32 sum; KV1 card, BQ2_0) for quantized tokens
 * (in the rotated basis for a hadamard cache: as stored) and the exact
 * stored value for sink and ring tokens (t counts every token of the
 * sequence, sinks first). k_out, v_out: device
 * [t1-t0][num_kv_heads][head_dim] fp32. 0 <= t0 <= t1 <= sequence length.  */
KVQ_API kvq_status kvq_dequant(kvq_cache* cache, int32_t layer, int32_t seq, int32_t t0, int32_t t1,
                       float* k_out, float* v_out, void* stream);

/* Device-side failures recorded since the last call, then cleared: bit 0 =
 * a decode kernel gave up a bounded wait on its copy pipeline (its partial
 * results are invalid); bit 1 = a decode CTA found an empty work range in
 * its plan (results invalid; not expected). Synchronous: waits for the
 * device to finish its work. No counterpart on the pages: a diagnostic of
 * this library.                                                           */
KVQ_API kvq_status kvq_device_errors(kvq_cache* cache, int32_t* flags);

/* Kernels enqueued so far by the calls on this cache, counted on the host
 * when each call enqueues them: one per launch, whatever the kernel (append:
 * ring write, plus the quantize kernel when a ring flushes, plus a page-table
 * update when pages are taken; decode: the decode kernel and the combine
 * kernel; a fused step's flush kernel on a step whose rings are full;
 * dequant). For accounting, e.g. a benchmark that reads it
 * around a timed region. No counterpart on the pages.
 * - cache, count: non-null (else KVQ_ERR_INVALID_ARG). Host only.          */
KVQ_API kvq_status kvq_cache_kernel_launches(const kvq_cache* cache, uint64_t* count);

/* Layer layout (see kvq_layout): where the packed codes, scales and zero
 * points of the KV1-1.2B card's format (Quantization Format) and the
 * KIVI README's full-precision window live. For tests and tools that read
 * the cache; no counterpart on the pages beyond the format itself.         */
KVQ_API kvq_status kvq_get_layout(const kvq_cache* cache, int32_t layer, kvq_layout* out);

/* Host mirror of a sequence's key lengths: quantized keys (a multiple of G)
 * and key ring tokens (the sink tokens come on top: kvq_seq_sinks). The
 * split of the KIVI README's Overview (quantized tokens, full-precision
 * window); a test accessor, no counterpart on the pages otherwise.          */
KVQ_API kvq_status kvq_seq_lengths(const kvq_cache* cache, int32_t layer, int32_t seq,
                           int32_t* quantized, int32_t* residual);

/* The same for the values: quantized values and value ring tokens (equal to
 * the key lengths unless residual_v differs from residual; "Quantize What
 * Counts", residual_length {"k", "v"}). A test accessor.                   */
KVQ_API kvq_status kvq_seq_value_lengths(const kvq_cache* cache, int32_t layer, int32_t seq,
                                 int32_t* quantized, int32_t* residual);

/* Host mirror of a sequence's sink tokens, min(S, tokens appended). No
 * counterpart on the pages beyond the sinks themselves (KV1 card).         */
KVQ_API kvq_status kvq_seq_sinks(const kvq_cache* cache, int32_t layer, int32_t seq, int32_t* sinks);

/* Which decode kernel kvq_decode_attention runs for one layer when a KV
 * head has rows_per_kv_head query rows (num_q_heads / num_kv_heads for one
 * query token per sequence): the general CUDA-core split kernel, the
 * tensor-core kernel (key blocks of 64 or more tokens), or its variant for
 * 32-token blocks with 2-bit keys (at most two rows per KV head). The
 * choice depends on the device's shared memory: call with the cache's
 * device current. A test and tuning accessor; no counterpart on the pages. */
typedef enum kvq_kernel {
  KVQ_KERNEL_CUDA_CORE = 0,
  KVQ_KERNEL_TENSOR_CORE = 1,
  KVQ_KERNEL_TENSOR_CORE_PAIR = 2
} kvq_kernel;
KVQ_API kvq_status kvq_decode_kernel(const kvq_cache* cache, int32_t layer, int32_t rows_per_kv_head,
                                     int32_t* kernel);

/* Static description of a status code.                                     */
KVQ_API const char* kvq_status_string(kvq_status status);

/* Reason for the last failure on this thread ("" if none).                 */
KVQ_API const char* kvq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
