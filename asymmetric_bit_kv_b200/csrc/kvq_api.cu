// Host side of the C ABI declared in include/kvq.h: argument validation, the
// arena plan, the host mirror of sequence lengths, the flush planner and the
// split planner. All device work is enqueued by the launchers of
// kvq_append.cu and kvq_decode.cu.
#include <algorithm>
#include <cstddef>
#include <cmath>
#include <cstdint>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "kvq_append.cuh"
#include "kvq_decode.cuh"

struct kvq_cache {
  kvq_config cfg;                 // k_bits / v_bits / k_axis point at the vectors below
  std::vector<int8_t> k_bits, v_bits, k_axis;
  uint8_t* arena;
  size_t arena_bytes;
  int device;
  // per layer
  std::vector<int64_t> blocks_off, ring_k_off, ring_v_off, sink_k_off, sink_v_off, record_bytes;
  int64_t max_blocks;
  int64_t lens_off;               // int32 [num_layers][max_batch][kLensStride]
  int64_t ws_o_off, ws_ml_off;    // split partials
  int64_t err_off;                // int32 device error word
  int64_t uslots_off;             // int32 [max_batch][num_kv_heads] slots per unit (decode -> combine)
  int32_t slots;                  // partial slots per (sequence, query head)
  int32_t sm_count;
  uint64_t launches = 0;          // kernels enqueued by calls on this cache (kvq_cache_kernel_launches)
  // host mirror [num_layers][max_batch]: quantized keys, key ring tokens,
  // sinks, quantized values (the value ring holds q_len + n_len - qv_len)
  std::vector<int32_t> q_len, n_len, s_len, qv_len;
  // paged block pools (cfg.page_blocks >= 1)
  std::vector<int64_t> pt_off;                   // per layer: int32 page table [max_batch][max_pages]
  int32_t max_pages = 0;                         // page-table entries per sequence
  std::vector<std::vector<int32_t>> free_pages;  // per layer: free page ids (a stack)
  std::vector<int32_t> pt_host;                  // [num_layers][max_batch][max_pages] mirror
  std::vector<int32_t> pages_held;               // [num_layers][max_batch]
};

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

kvq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool is_group(int g) { return g == 32 || g == 64 || g == 128; }
bool is_bits(int b) { return b == 2 || b == 4 || b == 8; }

kvq_status validate_config(const kvq_config* c) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "config is null");
  if (c->num_layers < 1 || c->num_layers > KVQ_MAX_LAYERS)
    return fail(KVQ_ERR_INVALID_ARG, "num_layers %d outside 1..%d", c->num_layers, KVQ_MAX_LAYERS);
  if (c->max_batch < 1 || c->max_batch > KVQ_MAX_BATCH)
    return fail(KVQ_ERR_INVALID_ARG, "max_batch %d outside 1..%d", c->max_batch, KVQ_MAX_BATCH);
  if (c->num_kv_heads < 1 || c->num_q_heads < 1 || c->num_q_heads % c->num_kv_heads != 0)
    return fail(KVQ_ERR_INVALID_ARG, "num_q_heads %d must be a positive multiple of num_kv_heads %d",
                c->num_q_heads, c->num_kv_heads);
  const int g = c->num_q_heads / c->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8)
    return fail(KVQ_ERR_UNSUPPORTED, "query heads per KV head %d not in {1,2,4,8}", g);
  if (c->head_dim != kvq::kHeadDim)
    return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d: only %d is built", c->head_dim, kvq::kHeadDim);
  if (!is_group(c->group_k)) return fail(KVQ_ERR_UNSUPPORTED, "group_k %d not in {32,64,128}", c->group_k);
  if (!is_group(c->group_v) || c->head_dim % c->group_v != 0)
    return fail(KVQ_ERR_UNSUPPORTED, "group_v %d not in {32,64,128} or not dividing head_dim", c->group_v);
  if (c->residual < c->group_k || c->residual % c->group_k != 0)
    return fail(KVQ_ERR_INVALID_ARG, "residual %d must be a positive multiple of group_k %d", c->residual,
                c->group_k);
  if (c->residual_v != 0 && (c->residual_v < c->group_k || c->residual_v % c->group_k != 0))
    return fail(KVQ_ERR_INVALID_ARG, "residual_v %d must be 0 or a positive multiple of group_k %d", c->residual_v,
                c->group_k);
  if (c->residual_v != 0 && c->residual_v != c->residual && c->hadamard)
    return fail(KVQ_ERR_UNSUPPORTED, "separate key and value residual lengths with the Hadamard rotation");
  if (c->max_tokens < 1) return fail(KVQ_ERR_INVALID_ARG, "max_tokens %d < 1", c->max_tokens);
  if (c->sink_tokens < 0 || c->sink_tokens > KVQ_MAX_SINKS)
    return fail(KVQ_ERR_INVALID_ARG, "sink_tokens %d outside 0..%d", c->sink_tokens, KVQ_MAX_SINKS);
  if (c->kv_dtype != KVQ_F16 && c->kv_dtype != KVQ_BF16)
    return fail(KVQ_ERR_UNSUPPORTED, "kv_dtype %d: only F16 and BF16", c->kv_dtype);
  if (!c->k_bits || !c->v_bits) return fail(KVQ_ERR_INVALID_ARG, "k_bits / v_bits is null");
  for (int l = 0; l < c->num_layers; ++l)
    if (!is_bits(c->k_bits[l]) || !is_bits(c->v_bits[l]))
      return fail(KVQ_ERR_UNSUPPORTED, "layer %d bits k=%d v=%d not in {2,4,8}", l, c->k_bits[l], c->v_bits[l]);
  if (c->k_axis)
    for (int l = 0; l < c->num_layers; ++l)
      if (c->k_axis[l] != 0 && c->k_axis[l] != 1)
        return fail(KVQ_ERR_INVALID_ARG, "layer %d k_axis %d not 0 or 1", l, c->k_axis[l]);
  if (c->hadamard != 0 && c->hadamard != 1) return fail(KVQ_ERR_INVALID_ARG, "hadamard %d not 0 or 1", c->hadamard);
  if (c->page_blocks < 0) return fail(KVQ_ERR_INVALID_ARG, "page_blocks %d < 0", c->page_blocks);
  if (c->page_blocks > 0) {
    if (c->pool_pages < 1) return fail(KVQ_ERR_INVALID_ARG, "pool_pages %d < 1 with page_blocks %d", c->pool_pages,
                                       c->page_blocks);
    if ((int64_t)c->pool_pages * c->num_kv_heads * c->page_blocks > INT32_MAX)
      return fail(KVQ_ERR_UNSUPPORTED, "more than 2^31 block records in one layer's pool");
  }
  // the work items of one decode launch are counted in int32
  const int64_t items = (int64_t)c->max_batch * c->num_kv_heads *
                        ((int64_t)c->max_tokens / c->group_k + std::max(c->residual, c->residual_v) / 8 + 2);
  if (items > INT32_MAX / 2) return fail(KVQ_ERR_UNSUPPORTED, "max_batch x num_kv_heads x max_tokens too large");
  return KVQ_OK;
}

int residual_v_of(const kvq_config& c) { return c.residual_v > 0 ? c.residual_v : c.residual; }

// Byte geometry of a layer's block records: runs of tiles of min(G, 64)
// tokens, each tile part [kc | ksz | vc | vsz]; a block of several tiles with
// per-channel keys stores its key scales once, before its tiles.
struct RecordGeometry {
  int32_t tile_tokens, tile_bytes, tile0_off, rec_ksz_off, kc_off, ksz_off, vc_off, vsz_off;
  int64_t record_bytes;
};
RecordGeometry record_geometry(int G, int D, int kb, int vb, int gv, int k_axis) {
  using kvq::round_up;
  RecordGeometry g;
  g.tile_tokens = std::min(G, 64);
  const int nt = G / g.tile_tokens;
  const bool shared_ksz = k_axis == 0 && nt > 1;
  const int64_t ksz = k_axis == 1 ? kvq::ksz_token_bytes(g.tile_tokens, D, gv) : (shared_ksz ? 0 : kvq::ksz_bytes(D));
  g.kc_off = 0;
  g.ksz_off = (int32_t)kvq::kc_bytes(g.tile_tokens, D, kb);
  g.vc_off = g.ksz_off + (int32_t)ksz;
  g.vsz_off = g.vc_off + (int32_t)kvq::vc_bytes(g.tile_tokens, D, vb);
  g.tile_bytes = (int32_t)round_up(g.vsz_off + kvq::vsz_bytes(g.tile_tokens, D, gv), 16);
  g.rec_ksz_off = shared_ksz ? 0 : -1;
  g.tile0_off = shared_ksz ? (int32_t)round_up(kvq::ksz_bytes(D), 16) : 0;
  g.record_bytes = round_up(g.tile0_off + (int64_t)nt * g.tile_bytes, 16);
  return g;
}

struct Plan {
  std::vector<int64_t> blocks_off, ring_k_off, ring_v_off, sink_k_off, sink_v_off, record_bytes, pt_off;
  int64_t max_blocks, lens_off, err_off, uslots_off, ws_o_off, ws_ml_off, total;
  int32_t slots, max_pages;
};

Plan make_plan(const kvq_config* c) {
  using kvq::round_up;
  Plan p;
  const int G = c->group_k, D = c->head_dim;
  const int64_t seqheads = (int64_t)c->max_batch * c->num_kv_heads;
  p.max_blocks = c->max_tokens / G;
  const bool paged = c->page_blocks > 0;
  p.max_pages = paged ? (int32_t)((p.max_blocks + c->page_blocks - 1) / c->page_blocks) : 0;
  // block records per layer: every sequence's capacity, or the page pool
  const int64_t records = paged ? (int64_t)c->pool_pages * c->num_kv_heads * c->page_blocks : seqheads * p.max_blocks;
  int64_t off = 0;
  for (int l = 0; l < c->num_layers; ++l) {
    const int kb = c->k_bits[l], vb = c->v_bits[l];
    const int64_t rec = record_geometry(G, D, kb, vb, c->group_v, c->k_axis ? c->k_axis[l] : 0).record_bytes;
    p.record_bytes.push_back(rec);
    p.blocks_off.push_back(off);
    off = round_up(off + records * rec, 256);
    p.ring_k_off.push_back(off);
    off = round_up(off + seqheads * c->residual * D * 2, 256);
    p.ring_v_off.push_back(off);
    off = round_up(off + seqheads * residual_v_of(*c) * D * 2, 256);
    const int64_t sink = c->sink_tokens > 0 ? seqheads * KVQ_MAX_SINKS * D * 2 : 0;
    p.sink_k_off.push_back(off);
    off = round_up(off + sink, 256);
    p.sink_v_off.push_back(off);
    off = round_up(off + sink, 256);
    p.pt_off.push_back(off);
    off = round_up(off + (paged ? (int64_t)c->max_batch * p.max_pages * 4 : 0), 256);
  }
  p.lens_off = off;
  off = round_up(off + (int64_t)c->num_layers * c->max_batch * kvq::kLensStride * 4, 256);
  p.err_off = off;
  off = round_up(off + 4, 256);
  p.uslots_off = off;
  off = round_up(off + seqheads * 4, 256);
  // partial slots per (sequence, query head): enough for the split kernel
  // (one per split + the ring) and for the persistent kernel (one per
  // consumer warp of each CTA range overlapping the unit's work items, at
  // most 65 such ranges)
  p.slots = (int32_t)std::max<int64_t>(
      std::min<int64_t>(p.max_blocks, KVQ_MAX_SPLITS) + 1,
      kvq::kMmaConsumers *
          (std::min<int64_t>(p.max_blocks + (c->residual + kvq::kResChunk - 1) / kvq::kResChunk + 1, 64) + 2));
  const int64_t partials = (int64_t)c->max_batch * c->num_q_heads * p.slots;
  p.ws_o_off = off;
  off = round_up(off + partials * D * 4, 256);
  p.ws_ml_off = off;
  off = round_up(off + partials * 8, 256);
  p.total = off;
  return p;
}

kvq::LayerView layer_view(const kvq_cache* c, int layer) {
  kvq::LayerView v;
  const kvq_config& cfg = c->cfg;
  const int G = cfg.group_k, D = cfg.head_dim;
  const int kb = c->k_bits[layer], vb = c->v_bits[layer];
  v.blocks = c->arena + c->blocks_off[layer];
  v.ring_k = c->arena + c->ring_k_off[layer];
  v.ring_v = c->arena + c->ring_v_off[layer];
  v.sink_k = c->arena + c->sink_k_off[layer];
  v.sink_v = c->arena + c->sink_v_off[layer];
  v.sinks = cfg.sink_tokens;
  v.lens = reinterpret_cast<int32_t*>(c->arena + c->lens_off) + (int64_t)layer * cfg.max_batch * kvq::kLensStride;
  v.record_bytes = c->record_bytes[layer];
  v.max_blocks = c->max_blocks;
  v.k_axis = c->k_axis[layer];
  v.hadamard = cfg.hadamard;
  const RecordGeometry rg = record_geometry(G, D, kb, vb, cfg.group_v, v.k_axis);
  v.kc_off = rg.kc_off;
  v.ksz_off = rg.ksz_off;
  v.vc_off = rg.vc_off;
  v.vsz_off = rg.vsz_off;
  v.tile_tokens = rg.tile_tokens;
  v.tile_bytes = rg.tile_bytes;
  v.tile0_off = rg.tile0_off;
  v.rec_ksz_off = rg.rec_ksz_off;
  v.k_bits = kb;
  v.v_bits = vb;
  v.num_kv_heads = cfg.num_kv_heads;
  v.head_dim = D;
  v.group_k = G;
  v.group_v = cfg.group_v;
  v.residual = cfg.residual;
  v.residual_v = residual_v_of(cfg);
  v.kv_dtype = cfg.kv_dtype;
  const bool paged = cfg.page_blocks > 0;
  v.page_table = paged ? reinterpret_cast<const int32_t*>(c->arena + c->pt_off[layer]) : nullptr;
  v.page_blocks = paged ? cfg.page_blocks : 0;
  v.max_pages = c->max_pages;
  return v;
}

kvq_status check_cache_layer(const kvq_cache* c, int layer) {
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is null");
  if (layer < 0 || layer >= c->cfg.num_layers)
    return fail(KVQ_ERR_INVALID_ARG, "layer %d outside 0..%d", layer, c->cfg.num_layers - 1);
  return KVQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Paged caches: gives each sequence b < batch the pages that its
// blocks_after[b] block records need (taken from the layer's pool) and
// enqueues the page-table update; fails before changing anything if the
// pool is short.
kvq_status take_pages(kvq_cache* c, int layer, const int32_t* blocks_after, int batch, cudaStream_t stream) {
  const kvq_config& cfg = c->cfg;
  const int P = cfg.page_blocks;
  int32_t* held = &c->pages_held[(size_t)layer * cfg.max_batch];
  std::vector<int32_t>& pool = c->free_pages[layer];
  auto pages_after = [&](int b) { return (int32_t)(((int64_t)blocks_after[b] + P - 1) / P); };
  int64_t need = 0;
  for (int b = 0; b < batch; ++b) need += std::max<int64_t>(0, pages_after(b) - held[b]);
  if (need == 0) return KVQ_OK;
  if (need > (int64_t)pool.size())
    return fail(KVQ_ERR_CAPACITY, "layer %d: the call needs %lld new pages; the pool has %zu free of %d", layer,
                (long long)need, pool.size(), cfg.pool_pages);
  kvq::PageTableUpdate* u = new (std::nothrow) kvq::PageTableUpdate;
  if (!u) return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
  u->table = reinterpret_cast<int32_t*>(c->arena + c->pt_off[layer]);
  u->n = 0;
  cudaError_t e = cudaSuccess;
  for (int b = 0; b < batch && e == cudaSuccess; ++b) {
    const int32_t want = pages_after(b);
    int32_t* row = &c->pt_host[((size_t)layer * cfg.max_batch + b) * c->max_pages];
    while (held[b] < want && e == cudaSuccess) {
      const int32_t page = pool.back();
      pool.pop_back();
      row[held[b]] = page;
      u->idx[u->n] = b * c->max_pages + held[b];
      u->page[u->n] = page;
      ++held[b];
      if (++u->n == kvq::kMaxPageUpdates) {
        e = kvq::launch_page_table_update(*u, stream);
        if (e == cudaSuccess) ++c->launches;
        u->n = 0;
      }
    }
  }
  if (e == cudaSuccess && u->n > 0) {
    e = kvq::launch_page_table_update(*u, stream);
    if (e == cudaSuccess) ++c->launches;
  }
  delete u;
  if (e != cudaSuccess) return cuda_fail(e, "page-table update");
  return KVQ_OK;
}

// Key or value blocks that a ring holding n of its R slots flushes when T
// tokens arrive one by one (a token that finds the ring full first moves
// its oldest G tokens to a block), or every complete group (flush_all).
int ring_flushes(int n, int T, int R, int G, bool flush_all) {
  if (flush_all) return n / G;
  return n + T <= R ? 0 : (n + T - R + G - 1) / G;
}

// Shared by kvq_append (t_new from the caller) and kvq_flush_residual
// (t_new = 0, every complete group of each ring flushed). Keys and values
// each follow their own ring.
kvq_status enqueue_append(kvq_cache* c, int layer, const void* k, const void* v, const int32_t* new_lens,
                          int batch, bool flush_all, cudaStream_t stream) {
  const kvq_config& cfg = c->cfg;
  const int G = cfg.group_k, R = cfg.residual, RV = residual_v_of(cfg);
  kvq::AppendParams* p = new (std::nothrow) kvq::AppendParams;
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
  std::memset(p, 0, sizeof *p);
  p->L = layer_view(c, layer);
  p->k_in = k;
  p->v_in = v;
  p->batch = batch;
  const size_t base = (size_t)layer * cfg.max_batch;
  int32_t* ql = &c->q_len[base];
  int32_t* nl = &c->n_len[base];
  int32_t* sl = &c->s_len[base];
  int32_t* qvl = &c->qv_len[base];
  int max_flush = 0;
  int64_t off = 0;
  thread_local std::vector<int32_t> blocks_after;
  blocks_after.resize(batch);
  for (int b = 0; b < batch; ++b) {
    // the sequence's first sink_tokens tokens go to its sinks
    const int all = flush_all ? 0 : new_lens[b];
    const int take = std::min(all, cfg.sink_tokens - sl[b]);
    p->s_old[b] = sl[b];
    p->s_take[b] = take;
    off += take;
    const int T = all - take;
    const int len = ql[b] + nl[b];
    const int fk = ring_flushes(nl[b], T, R, G, flush_all);
    const int fv = ring_flushes(len - qvl[b], T, RV, G, flush_all);
    p->q_old[b] = ql[b];
    p->qv_old[b] = qvl[b];
    p->len_old[b] = len;
    p->t_new[b] = T;
    p->in_off[b] = (int32_t)off;
    p->flush[b] = fk;
    p->flush_v[b] = fv;
    off += T;
    max_flush = std::max(max_flush, std::max(fk, fv));
    blocks_after[b] = std::max(ql[b] + fk * G, qvl[b] + fv * G) / G;
  }
  if (cfg.page_blocks > 0) {
    const kvq_status ps = take_pages(c, layer, blocks_after.data(), batch, stream);
    if (ps != KVQ_OK) {
      delete p;
      return ps;
    }
  }
  cudaError_t e = kvq::launch_append(*p, max_flush, stream);
  if (e == cudaSuccess) {
    c->launches += max_flush > 0 ? 2 : 1;  // the quantize kernel on a flush, the ring write
    for (int b = 0; b < batch; ++b) {
      const int qn = p->q_old[b] + p->flush[b] * G;
      const int end = p->len_old[b] + p->t_new[b];
      ql[b] = qn;
      nl[b] = end - qn;
      qvl[b] = p->qv_old[b] + p->flush_v[b] * G;
      sl[b] += p->s_take[b];
    }
  }
  delete p;
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return KVQ_OK;
}

// Persistent-mode plan of a decode launch from p.nblk, p.nres, p.nitem
// (batch sequences, Hkv units each): p.seq_start, the number of CTAs and
// their item ranges p.cta_start, cut at equal cost (a quantized block costs 2,
// an exact-token chunk 1, in half units): CTA c starts at the item whose cost
// interval [P(k), P(k+1)) holds c*C/N, compared in exact integer arithmetic
// as P*N against c*C. N is at most max_ctas and max(units, items / 4); at
// most C / (largest item cost), so that no range is empty; and small enough
// that no unit overlaps more than slot_cap / kMmaConsumers ranges (a unit of
// cost u overlaps at most floor(u*N/C) + 2 of them). One pass over the
// sequences and the CTAs.
void plan_cta_starts(kvq::DecodeParams& p, int batch, int hkv, int64_t max_ctas, int32_t slot_cap) {
  int64_t T = 0, C = 0, cu_max = 0;
  bool blocks = false;
  for (int b = 0; b < batch; ++b) {
    p.seq_start[b] = (int32_t)T;
    T += (int64_t)hkv * p.nitem[b];
    const int64_t cu = kvq::unit_cost(p.nblk[b], p.nitem[b]);
    C += (int64_t)hkv * cu;
    cu_max = std::max(cu_max, cu);
    blocks = blocks || p.nblk[b] > 0;
  }
  int64_t N = std::min<int64_t>(max_ctas, std::max<int64_t>((int64_t)batch * hkv, (T + 3) / 4));
  N = std::min<int64_t>(N, C / (blocks ? 2 : 1));
  const int64_t kmax = slot_cap / kvq::kMmaConsumers - 2;
  N = kmax < 0 ? 1 : std::min<int64_t>(N, ((kmax + 1) * C + cu_max - 1) / cu_max - 1);
  N = std::max<int64_t>(1, std::min<int64_t>(N, kvq::kMaxCtas));
  p.total_blocks = (int32_t)T;
  p.num_ctas = (int32_t)N;
  p.max_unit_slots = (int32_t)std::min<int64_t>(slot_cap, kvq::kMmaConsumers * (cu_max * N / C + 2));
  p.cta_start[0] = 0;
  int b = 0;
  int64_t cost0 = 0;  // cost before sequence b
  for (int64_t c = 1; c < N; ++c) {
    const int64_t x = c * C;  // threshold, scaled by N
    int64_t cs = (int64_t)hkv * kvq::unit_cost(p.nblk[b], p.nitem[b]);
    while ((cost0 + cs) * N <= x) {
      cost0 += cs;
      ++b;
      cs = (int64_t)hkv * kvq::unit_cost(p.nblk[b], p.nitem[b]);
    }
    const int64_t cu = kvq::unit_cost(p.nblk[b], p.nitem[b]);
    const int64_t r = x - cost0 * N;
    const int64_t h = r / (cu * N);
    const int64_t r2 = r - h * cu * N;
    const int64_t nb = p.nblk[b];
    const int64_t j = r2 < 2 * nb * N ? r2 / (2 * N) : nb + (r2 - 2 * nb * N) / N;
    p.cta_start[c] = (int32_t)(p.seq_start[b] + h * p.nitem[b] + j);
  }
  p.cta_start[N] = (int32_t)T;
}

}  // namespace

namespace kvq {

// Decode attention of kvq_decode_attention and its variants. The split
// partials live in the arena's workspace (slot stride: the arena's slot
// count, or what the workspace holds for a group of query tokens), or, with
// `scratch`, in that memory together with the unit slot counts (the slot
// stride then cut to what fits; a call for which no split fits is rejected
// before anything is enqueued). new_k/new_v: a fused decode step's new
// tokens, already counted in the host mirror; after_flush: that step's flush
// kernel was enqueued just before.
kvq_status enqueue_decode(kvq_cache* c, int32_t layer, const void* new_k, const void* new_v, const void* q, void* out,
                          int32_t out_dtype, float softmax_scale, int32_t batch, void* stream,
                          const StaticScratch* scratch, const QueryGroup* qg, bool after_flush) {
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (batch < 0 || batch > c->cfg.max_batch)
    return fail(KVQ_ERR_INVALID_ARG, "batch %d outside 0..%d", batch, c->cfg.max_batch);
  if (out_dtype != KVQ_F32 && out_dtype != KVQ_F16 && out_dtype != KVQ_BF16)
    return fail(KVQ_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  if (!std::isfinite(softmax_scale)) return fail(KVQ_ERR_INVALID_ARG, "softmax_scale is not finite");
  if (batch == 0) return KVQ_OK;
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "q or out is null");
  if (!aligned16(q) || !aligned16(out)) return fail(KVQ_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  const kvq_config& cfg = c->cfg;
  const int G = cfg.group_k;
  const kvq::LayerView L = layer_view(c, layer);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // query rows per launch: the query heads of each of the group's tokens
  const int qtok = qg ? qg->qtok : 1;
  const int Hv = cfg.num_q_heads * qtok;
  const bool use_mma = kvq::mma_supported(L, Hv);
  // partial slots per (sequence, query row) that fit the arena's workspace
  // (sized for num_q_heads rows): all of them for one query token, fewer for
  // a group, whose slot stride is then cut to what the launch uses
  int32_t slot_cap =
      qg ? (int32_t)std::min<int64_t>(c->slots, (int64_t)cfg.max_batch * cfg.num_q_heads * c->slots /
                                                    ((int64_t)batch * Hv))
         : c->slots;
  thread_local DecodeParams params;  // large (per-sequence tables): one per thread, not on the stack
  DecodeParams& p = params;
  std::memset(&p, 0, offsetof(DecodeParams, nblk));  // the per-sequence tables are written below
  p.L = L;
  p.new_k = new_k;
  p.new_v = new_v;
  p.q = q;
  p.out = out;
  p.ws_o = reinterpret_cast<float*>(c->arena + c->ws_o_off);
  p.ws_ml = reinterpret_cast<float2*>(c->arena + c->ws_ml_off);
  p.unit_slots = reinterpret_cast<int32_t*>(c->arena + c->uslots_off);
  if (scratch) {
    // unit slot counts, then the partials (o, then (m, l)), 256-byte aligned
    const int64_t plan_b = 0;
    const int64_t us_b = kvq::round_up((int64_t)batch * cfg.num_kv_heads * 4, 256);
    const int64_t per_slot = (int64_t)batch * Hv * (kHeadDim * 4 + 8);
    const int64_t room = scratch->bytes - plan_b - us_b - 256;
    const int64_t fit = room > 0 ? room / per_slot : 0;
    slot_cap = (int32_t)std::min<int64_t>(fit, c->slots);
    if (slot_cap < (use_mma ? kMmaConsumers : 2))
      return fail(KVQ_ERR_WORKSPACE,
                  "the static scratch (%lld bytes) holds %d partial slots per query row for batch %d x %d query rows; "
                  "this decode needs at least %d",
                  (long long)scratch->bytes, slot_cap, batch, Hv, use_mma ? kMmaConsumers : 2);
    uint8_t* base = scratch->base;
    p.unit_slots = reinterpret_cast<int32_t*>(base + plan_b);
    p.ws_o = reinterpret_cast<float*>(base + plan_b + us_b);
    p.ws_ml = reinterpret_cast<float2*>(base + plan_b + us_b +
                                        kvq::round_up((int64_t)batch * Hv * slot_cap * kHeadDim * 4, 256));
  }
  if (use_mma && slot_cap < kMmaConsumers)
    return fail(KVQ_ERR_WORKSPACE, "the workspace holds %d partial slots per query row for %d query rows; need %d",
                slot_cap, Hv, kMmaConsumers);
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  // the tensor-core kernel multiplies fp16 queries by fp16 key scales: a power
  // of two near scale_log2 keeps those products as far from the fp16 limit as
  // the scaled query would, exactly; the rest of the scale is applied to the
  // fp32 scores
  int scale_exp = 0;  // |scale_log2| in [2^scale_exp, 2^(scale_exp+1))
  if (p.scale_log2 != 0.f) {
    (void)std::frexp(std::fabs(p.scale_log2), &scale_exp);
    scale_exp -= 1;
  }
  p.q_prescale = std::ldexp(1.f, std::min(0, std::max(-8, scale_exp)));
  p.score_scale = p.scale_log2 / p.q_prescale;
  p.out_dtype = out_dtype;
  p.batch = batch;
  p.num_q_heads = Hv;
  p.q_heads = cfg.num_q_heads;
  p.q_rows = qg ? qg->q_rows : cfg.num_q_heads;
  p.qtok = qtok;
  p.lag_base = qg ? qg->lag_base : 0;
  p.err = reinterpret_cast<int32_t*>(c->arena + c->err_off);
  cudaError_t e;
  if (use_mma) {
    // Persistent plan from the host mirror: the work items of every
    // (sequence, KV head) unit (quantized blocks, ring chunks, sinks),
    // concatenated and cut into one contiguous range of equal cost per CTA,
    // one CTA per resident slot (fewer if there is little work).
    const kvq::MmaPlan mp = kvq::make_mma_plan(L, Hv);
    const int per_sm = kvq::mma_ctas_per_sm(L, mp, Hv);
    for (int b = 0; b < batch; ++b) {
      const size_t i = (size_t)layer * cfg.max_batch + b;
      p.nblk[b] = c->q_len[i] / L.tile_tokens;  // tile items of the quantized blocks
      p.nres[b] = c->n_len[i];
      p.nitem[b] = kvq::unit_items(p.nblk[b], p.nres[b], c->s_len[i]);
    }
    p.persistent = 1;
    p.slots = slot_cap;
    p.after_flush = after_flush ? 1 : 0;
    plan_cta_starts(p, batch, cfg.num_kv_heads, (int64_t)std::max(1, c->sm_count) * per_sm, slot_cap);
    e = kvq::launch_decode_mma(p, mp, st);
    if (e == cudaSuccess) e = kvq::launch_combine(p, st);
    if (e == cudaSuccess) c->launches += 2;  // the decode kernel and the combine
  } else {
    // Split plan (host mirror): blocks per split chosen to minimise (waves
    // of CTAs) x (blocks per CTA + a fixed per-CTA overhead), with at most
    // slot_cap - 1 splits.
    const int per_sm = kvq::split_ctas_per_sm(Hv, cfg.num_kv_heads);
    thread_local std::vector<int> nblk;
    nblk.resize(batch);
    int max_blk = 0;
    for (int b = 0; b < batch; ++b) {
      const size_t i = (size_t)layer * cfg.max_batch + b;
      nblk[b] = std::max(c->q_len[i], c->qv_len[i]) / G;
      max_blk = std::max(max_blk, nblk[b]);
    }
    const int64_t slots_gpu = (int64_t)std::max(1, c->sm_count) * per_sm;
    const int64_t min_bps = std::max<int64_t>(1, (max_blk + (slot_cap - 1) - 1) / (slot_cap - 1));
    int64_t bps = std::max<int64_t>(min_bps, max_blk);
    double best = 1e300;
    for (int64_t cand = min_bps; cand <= std::max<int64_t>(min_bps, max_blk); ++cand) {
      int64_t ctas = 0;
      for (int b = 0; b < batch; ++b) ctas += (nblk[b] + cand - 1) / cand;
      ctas *= cfg.num_kv_heads;
      const double waves = (double)((ctas + slots_gpu - 1) / slots_gpu);
      const double cost = waves * (double)(cand + 2);
      if (cost < best) {
        best = cost;
        bps = cand;
      }
    }
    p.blocks_per_split = (int32_t)bps;
    const int nsplits = (int)((max_blk + bps - 1) / bps);
    p.slots = slot_cap;
    e = kvq::launch_decode(p, nsplits, st);
    if (e == cudaSuccess) c->launches += 2;  // the split kernel and the combine
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return KVQ_OK;
}

void clear_last_error() { g_last_error.clear(); }
kvq_status report_cuda_error(cudaError_t e, const char* what) { return cuda_fail(e, what); }
kvq_status report_status(kvq_status s, const char* what) { return fail(s, "%s", what); }
int cache_device(const kvq_cache* c) { return c->device; }

}  // namespace kvq

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "sequence capacity exceeded";
    case KVQ_ERR_WORKSPACE: return "arena or static scratch too small";
    case KVQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* kvq_last_error(void) { return g_last_error.c_str(); }

kvq_status kvq_cache_required_bytes(const kvq_config* cfg, size_t* bytes) {
  g_last_error.clear();
  kvq_status s = validate_config(cfg);
  if (s != KVQ_OK) return s;
  if (!bytes) return fail(KVQ_ERR_INVALID_ARG, "bytes is null");
  *bytes = (size_t)make_plan(cfg).total;
  return KVQ_OK;
}

kvq_status kvq_cache_create(const kvq_config* cfg, void* dev_arena, size_t arena_bytes, kvq_cache** out) {
  g_last_error.clear();
  kvq_status s = validate_config(cfg);
  if (s != KVQ_OK) return s;
  if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is null");
  if (!dev_arena) return fail(KVQ_ERR_INVALID_ARG, "arena is null");
  if (reinterpret_cast<uintptr_t>(dev_arena) & 255u) return fail(KVQ_ERR_INVALID_ARG, "arena not 256-byte aligned");
  Plan plan = make_plan(cfg);
  if ((int64_t)arena_bytes < plan.total)
    return fail(KVQ_ERR_WORKSPACE, "arena %zu bytes < required %lld", arena_bytes, (long long)plan.total);
  kvq_cache* c = new (std::nothrow) kvq_cache;
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "out of host memory");
  c->cfg = *cfg;
  c->k_bits.assign(cfg->k_bits, cfg->k_bits + cfg->num_layers);
  c->v_bits.assign(cfg->v_bits, cfg->v_bits + cfg->num_layers);
  if (cfg->k_axis) c->k_axis.assign(cfg->k_axis, cfg->k_axis + cfg->num_layers);
  else c->k_axis.assign(cfg->num_layers, 0);
  c->cfg.k_bits = c->k_bits.data();
  c->cfg.v_bits = c->v_bits.data();
  c->cfg.k_axis = c->k_axis.data();
  c->arena = static_cast<uint8_t*>(dev_arena);
  c->arena_bytes = arena_bytes;
  c->blocks_off = plan.blocks_off;
  c->ring_k_off = plan.ring_k_off;
  c->ring_v_off = plan.ring_v_off;
  c->sink_k_off = plan.sink_k_off;
  c->sink_v_off = plan.sink_v_off;
  c->record_bytes = plan.record_bytes;
  c->max_blocks = plan.max_blocks;
  c->lens_off = plan.lens_off;
  c->ws_o_off = plan.ws_o_off;
  c->ws_ml_off = plan.ws_ml_off;
  c->err_off = plan.err_off;
  c->uslots_off = plan.uslots_off;
  c->slots = plan.slots;
  c->pt_off = plan.pt_off;
  c->max_pages = plan.max_pages;
  if (cfg->page_blocks > 0) {
    c->free_pages.assign(cfg->num_layers, {});
    for (auto& f : c->free_pages)
      for (int32_t i = cfg->pool_pages - 1; i >= 0; --i) f.push_back(i);
    c->pt_host.assign((size_t)cfg->num_layers * cfg->max_batch * c->max_pages, 0);
    c->pages_held.assign((size_t)cfg->num_layers * cfg->max_batch, 0);
  }
  c->q_len.assign((size_t)cfg->num_layers * cfg->max_batch, 0);
  c->n_len.assign((size_t)cfg->num_layers * cfg->max_batch, 0);
  c->s_len.assign((size_t)cfg->num_layers * cfg->max_batch, 0);
  c->qv_len.assign((size_t)cfg->num_layers * cfg->max_batch, 0);
  const size_t lens_bytes = (size_t)cfg->num_layers * cfg->max_batch * kvq::kLensStride * 4;
  cudaError_t e = cudaGetDevice(&c->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device);
  if (e == cudaSuccess) e = cudaMemset(c->arena + c->lens_off, 0, lens_bytes);
  if (e == cudaSuccess) e = cudaMemset(c->arena + c->err_off, 0, 4);
  // Ring slots and sink rows that no token has reached yet hold zeros, never
  // stale bit patterns: the decode kernel reads whole chunks of ring slots
  // and sink rows and masks the scores of those past the sequence, so their
  // values must be finite.
  const size_t ring_bytes = (size_t)cfg->max_batch * cfg->num_kv_heads * cfg->residual * cfg->head_dim * 2;
  const size_t ring_v_bytes = (size_t)cfg->max_batch * cfg->num_kv_heads * residual_v_of(*cfg) * cfg->head_dim * 2;
  const size_t sink_bytes =
      cfg->sink_tokens > 0 ? (size_t)cfg->max_batch * cfg->num_kv_heads * KVQ_MAX_SINKS * cfg->head_dim * 2 : 0;
  for (int l = 0; l < cfg->num_layers && e == cudaSuccess; ++l) {
    e = cudaMemset(c->arena + c->ring_k_off[l], 0, ring_bytes);
    if (e == cudaSuccess) e = cudaMemset(c->arena + c->ring_v_off[l], 0, ring_v_bytes);
    if (e == cudaSuccess && sink_bytes) e = cudaMemset(c->arena + c->sink_k_off[l], 0, sink_bytes);
    if (e == cudaSuccess && sink_bytes) e = cudaMemset(c->arena + c->sink_v_off[l], 0, sink_bytes);
    if (e == cudaSuccess && cfg->page_blocks > 0)  // entries not yet given out name page 0 (valid memory)
      e = cudaMemset(c->arena + c->pt_off[l], 0, (size_t)cfg->max_batch * c->max_pages * 4);
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    delete c;
    return cuda_fail(e, "zeroing the length table");
  }
  *out = c;
  return KVQ_OK;
}

kvq_status kvq_cache_destroy(kvq_cache* c) {
  g_last_error.clear();
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is null");
  delete c;
  return KVQ_OK;
}

kvq_status kvq_cache_reset(kvq_cache* c, void* stream) {
  g_last_error.clear();
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is null");
  cudaError_t e = cudaMemsetAsync(c->arena + c->lens_off, 0,
                                  (size_t)c->cfg.num_layers * c->cfg.max_batch * kvq::kLensStride * 4,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reset");
  std::fill(c->q_len.begin(), c->q_len.end(), 0);
  std::fill(c->n_len.begin(), c->n_len.end(), 0);
  std::fill(c->s_len.begin(), c->s_len.end(), 0);
  std::fill(c->qv_len.begin(), c->qv_len.end(), 0);
  if (c->cfg.page_blocks > 0) {
    for (auto& f : c->free_pages) {
      f.clear();
      for (int32_t i = c->cfg.pool_pages - 1; i >= 0; --i) f.push_back(i);
    }
    std::fill(c->pages_held.begin(), c->pages_held.end(), 0);
  }
  return KVQ_OK;
}

kvq_status kvq_release_sequence(kvq_cache* c, int32_t seq, void* stream) {
  g_last_error.clear();
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is null");
  const kvq_config& cfg = c->cfg;
  if (seq < 0 || seq >= cfg.max_batch) return fail(KVQ_ERR_INVALID_ARG, "seq %d outside 0..%d", seq, cfg.max_batch - 1);
  for (int l = 0; l < cfg.num_layers; ++l) {
    cudaError_t e = cudaMemsetAsync(c->arena + c->lens_off + ((size_t)l * cfg.max_batch + seq) * kvq::kLensStride * 4,
                                    0, kvq::kLensStride * 4, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "release");
  }
  for (int l = 0; l < cfg.num_layers; ++l) {
    const size_t i = (size_t)l * cfg.max_batch + seq;
    c->q_len[i] = c->n_len[i] = c->s_len[i] = c->qv_len[i] = 0;
    if (cfg.page_blocks > 0) {
      const int32_t* row = &c->pt_host[i * c->max_pages];
      for (int32_t k = c->pages_held[i] - 1; k >= 0; --k) c->free_pages[l].push_back(row[k]);
      c->pages_held[i] = 0;
    }
  }
  return KVQ_OK;
}

kvq_status kvq_append(kvq_cache* c, int32_t layer, const void* k, const void* v, const int32_t* new_lens,
                      int32_t batch, void* stream) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (batch < 0 || batch > c->cfg.max_batch)
    return fail(KVQ_ERR_INVALID_ARG, "batch %d outside 0..%d", batch, c->cfg.max_batch);
  if (batch > 0 && !new_lens) return fail(KVQ_ERR_INVALID_ARG, "new_lens is null");
  int64_t total = 0;
  for (int b = 0; b < batch; ++b) {
    if (new_lens[b] < 0) return fail(KVQ_ERR_INVALID_ARG, "new_lens[%d] = %d < 0", b, new_lens[b]);
    const size_t i = (size_t)layer * c->cfg.max_batch + b;
    const int64_t L = (int64_t)c->s_len[i] + c->q_len[i] + c->n_len[i] + new_lens[b];
    if (L > c->cfg.max_tokens)
      return fail(KVQ_ERR_CAPACITY, "sequence %d would hold %lld tokens > max_tokens %d", b, (long long)L,
                  c->cfg.max_tokens);
    total += new_lens[b];
  }
  if (total > INT32_MAX) return fail(KVQ_ERR_INVALID_ARG, "more than 2^31-1 tokens in one call");
  if (total > 0) {
    if (!k || !v) return fail(KVQ_ERR_INVALID_ARG, "k or v is null");
    if (!aligned16(k) || !aligned16(v)) return fail(KVQ_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
  }
  if (batch == 0) return KVQ_OK;
  return enqueue_append(c, layer, k, v, new_lens, batch, false, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_flush_residual(kvq_cache* c, int32_t layer, int32_t batch, void* stream) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (batch < 0 || batch > c->cfg.max_batch)
    return fail(KVQ_ERR_INVALID_ARG, "batch %d outside 0..%d", batch, c->cfg.max_batch);
  if (batch == 0) return KVQ_OK;
  return enqueue_append(c, layer, nullptr, nullptr, nullptr, batch, true, static_cast<cudaStream_t>(stream));
}

kvq_status kvq_decode_attention(kvq_cache* c, int32_t layer, const void* q, void* out, int32_t out_dtype,
                                float softmax_scale, int32_t batch, void* stream) {
  g_last_error.clear();
  return kvq::enqueue_decode(c, layer, nullptr, nullptr, q, out, out_dtype, softmax_scale, batch, stream, nullptr);
}

kvq_status kvq_decode_attention_multi(kvq_cache* c, int32_t layer, const void* q, void* out, int32_t out_dtype,
                                      float softmax_scale, int32_t batch, int32_t num_tokens, void* stream) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (batch < 0 || batch > c->cfg.max_batch)
    return fail(KVQ_ERR_INVALID_ARG, "batch %d outside 0..%d", batch, c->cfg.max_batch);
  if (num_tokens < 1 || num_tokens > c->cfg.residual)
    return fail(KVQ_ERR_INVALID_ARG, "num_tokens %d outside 1..%d (the residual window)", num_tokens,
                c->cfg.residual);
  if (out_dtype != KVQ_F32 && out_dtype != KVQ_F16 && out_dtype != KVQ_BF16)
    return fail(KVQ_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  if (batch == 0) return KVQ_OK;
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "q or out is null");
  const kvq_config& cfg = c->cfg;
  // the query tokens' own keys and values are the newest cached tokens,
  // still in the ring, where the causal mask applies
  for (int b = 0; b < batch; ++b) {
    const size_t i = (size_t)layer * cfg.max_batch + b;
    const int n = std::min(c->n_len[i], c->q_len[i] + c->n_len[i] - c->qv_len[i]);
    if (n < num_tokens)
      return fail(KVQ_ERR_UNSUPPORTED,
                  "sequence %d has %d ring tokens: its %d query tokens must be its newest tokens, in the ring", b,
                  n, num_tokens);
  }
  // groups of query tokens, at most 8 query rows per KV head per launch
  // (2 where the tensor-core kernel of the layer takes no more)
  const int ngr = cfg.num_q_heads / cfg.num_kv_heads;
  const kvq::LayerView lv = layer_view(c, layer);
  const int max_rows = kvq::mma_supported(lv, cfg.num_q_heads) ? kvq::mma_max_rows(lv) : 8;
  const int64_t qrow = (int64_t)cfg.num_q_heads * cfg.head_dim;  // elements per query token of a sequence
  const int out_size = out_dtype == KVQ_F32 ? 4 : 2;
  for (int t0 = 0; t0 < num_tokens;) {
    int tp = 1;
    while (2 * tp * ngr <= max_rows && t0 + 2 * tp <= num_tokens) tp *= 2;
    const kvq::QueryGroup g{num_tokens * cfg.num_q_heads, tp, num_tokens - 1 - t0};
    s = kvq::enqueue_decode(c, layer, nullptr, nullptr, static_cast<const uint8_t*>(q) + t0 * qrow * 2,
                            static_cast<uint8_t*>(out) + t0 * qrow * out_size, out_dtype, softmax_scale, batch,
                            stream, nullptr, &g);
    if (s != KVQ_OK) return s;
    t0 += tp;
  }
  return KVQ_OK;
}

kvq_status kvq_decode_step(kvq_cache* c, int32_t layer, const void* k, const void* v, const void* q, void* out,
                           int32_t out_dtype, float softmax_scale, int32_t batch, void* stream) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (batch < 0 || batch > c->cfg.max_batch)
    return fail(KVQ_ERR_INVALID_ARG, "batch %d outside 0..%d", batch, c->cfg.max_batch);
  if (out_dtype != KVQ_F32 && out_dtype != KVQ_F16 && out_dtype != KVQ_BF16)
    return fail(KVQ_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  if (!std::isfinite(softmax_scale)) return fail(KVQ_ERR_INVALID_ARG, "softmax_scale is not finite");
  if (batch == 0) return KVQ_OK;
  if (!k || !v || !q || !out) return fail(KVQ_ERR_INVALID_ARG, "k, v, q or out is null");
  if (!aligned16(k) || !aligned16(v) || !aligned16(q) || !aligned16(out))
    return fail(KVQ_ERR_INVALID_ARG, "k, v, q and out must be 16-byte aligned");
  const kvq_config& cfg = c->cfg;
  const size_t base = (size_t)layer * cfg.max_batch;
  // The new tokens ride along with the decode when the layer runs on the
  // tensor-core kernel, every sequence's sinks are complete and keys and
  // values share one ring: the prep kernel then quantizes the oldest G
  // tokens of every full ring (one block per such sequence and KV head),
  // its plan counts the new tokens, and the decode kernel writes them into
  // their ring slots. Otherwise: append, then decode.
  bool fused = kvq::mma_supported(layer_view(c, layer), c->cfg.num_q_heads) && residual_v_of(cfg) == cfg.residual;
  bool flush = false;
  for (int b = 0; b < batch; ++b) {
    const int64_t L = (int64_t)c->s_len[base + b] + c->q_len[base + b] + c->n_len[base + b] + 1;
    if (L > cfg.max_tokens)
      return fail(KVQ_ERR_CAPACITY, "sequence %d would hold %lld tokens > max_tokens %d", b, (long long)L,
                  cfg.max_tokens);
    if (c->s_len[base + b] < cfg.sink_tokens) fused = false;
    flush = flush || c->n_len[base + b] == cfg.residual;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!fused) {
    thread_local std::vector<int32_t> ones;
    ones.assign(batch, 1);
    s = enqueue_append(c, layer, k, v, ones.data(), batch, false, st);
    if (s != KVQ_OK) return s;
    return kvq::enqueue_decode(c, layer, nullptr, nullptr, q, out, out_dtype, softmax_scale, batch, stream, nullptr);
  }
  const int G = cfg.group_k;
  if (flush && cfg.page_blocks > 0) {
    thread_local std::vector<int32_t> blocks_after;
    blocks_after.resize(batch);
    for (int b = 0; b < batch; ++b)
      blocks_after[b] = (c->q_len[base + b] + (c->n_len[base + b] == cfg.residual ? G : 0)) / G;
    s = take_pages(c, layer, blocks_after.data(), batch, st);
    if (s != KVQ_OK) return s;
  }
  thread_local std::vector<int32_t> flushed;
  flushed.assign(batch, 0);
  for (int b = 0; b < batch; ++b) {
    if (c->n_len[base + b] == cfg.residual) {
      flushed[b] = 1;
      c->q_len[base + b] += G;
      c->qv_len[base + b] += G;
      c->n_len[base + b] -= G;
    }
    ++c->n_len[base + b];
  }
  if (flush) {
    kvq::FlushParams fp;
    fp.L = layer_view(c, layer);
    fp.ctas = batch * cfg.num_kv_heads;
    const cudaError_t e = kvq::launch_step_flush(fp, st);
    if (e != cudaSuccess) s = cuda_fail(e, "flush launch");
    else ++c->launches;
  }
  if (s == KVQ_OK)
    s = kvq::enqueue_decode(c, layer, k, v, q, out, out_dtype, softmax_scale, batch, stream, nullptr, nullptr, flush);
  if (s != KVQ_OK)
    for (int b = 0; b < batch; ++b) {
      --c->n_len[base + b];
      if (flushed[b]) {
        c->q_len[base + b] -= G;
        c->qv_len[base + b] -= G;
        c->n_len[base + b] += G;
      }
    }
  return s;
}

kvq_status kvq_dequant(kvq_cache* c, int32_t layer, int32_t seq, int32_t t0, int32_t t1, float* k_out,
                       float* v_out, void* stream) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (seq < 0 || seq >= c->cfg.max_batch) return fail(KVQ_ERR_INVALID_ARG, "seq %d out of range", seq);
  const size_t i = (size_t)layer * c->cfg.max_batch + seq;
  const int L = c->s_len[i] + c->q_len[i] + c->n_len[i];
  if (t0 < 0 || t0 > t1 || t1 > L)
    return fail(KVQ_ERR_INVALID_ARG, "token range [%d,%d) outside [0,%d]", t0, t1, L);
  if (t1 == t0) return KVQ_OK;
  if (!k_out || !v_out) return fail(KVQ_ERR_INVALID_ARG, "k_out or v_out is null");
  cudaError_t e = kvq::launch_dequant(layer_view(c, layer), seq, c->s_len[i], t0, t1, k_out, v_out,
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
  ++c->launches;
  return KVQ_OK;
}

kvq_status kvq_device_errors(kvq_cache* c, int32_t* flags) {
  g_last_error.clear();
  if (!c || !flags) return fail(KVQ_ERR_INVALID_ARG, "cache or flags is null");
  int32_t v = 0;
  cudaError_t e = cudaMemcpy(&v, c->arena + c->err_off, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && v != 0) e = cudaMemset(c->arena + c->err_off, 0, 4);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  *flags = v;
  return KVQ_OK;
}

kvq_status kvq_cache_kernel_launches(const kvq_cache* c, uint64_t* count) {
  g_last_error.clear();
  if (!c || !count) return fail(KVQ_ERR_INVALID_ARG, "cache or count is null");
  *count = c->launches;
  return KVQ_OK;
}

kvq_status kvq_decode_kernel(const kvq_cache* c, int32_t layer, int32_t rows, int32_t* kernel) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (!kernel) return fail(KVQ_ERR_INVALID_ARG, "kernel is null");
  if (rows < 1 || rows > 64) return fail(KVQ_ERR_INVALID_ARG, "rows_per_kv_head %d outside 1..64", rows);
  const kvq::LayerView v = layer_view(c, layer);
  if (!kvq::mma_supported(v, rows * c->cfg.num_kv_heads)) *kernel = KVQ_KERNEL_CUDA_CORE;
  else *kernel = kvq::pair_layout(v.group_k, v.k_bits) ? KVQ_KERNEL_TENSOR_CORE_PAIR : KVQ_KERNEL_TENSOR_CORE;
  return KVQ_OK;
}

kvq_status kvq_get_layout(const kvq_cache* c, int32_t layer, kvq_layout* out) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (!out) return fail(KVQ_ERR_INVALID_ARG, "out is null");
  const kvq::LayerView v = layer_view(c, layer);
  out->blocks = v.blocks;
  out->record_bytes = v.record_bytes;
  out->max_blocks = v.max_blocks;
  out->kc_offset = v.kc_off;
  out->ksz_offset = v.ksz_off;
  out->vc_offset = v.vc_off;
  out->vsz_offset = v.vsz_off;
  out->ring_k = v.ring_k;
  out->ring_v = v.ring_v;
  out->k_bits = v.k_bits;
  out->v_bits = v.v_bits;
  out->sink_k = v.sink_k;
  out->sink_v = v.sink_v;
  out->k_axis = v.k_axis;
  out->hadamard = v.hadamard;
  out->page_table = const_cast<int32_t*>(v.page_table);
  out->page_blocks = v.page_blocks;
  out->max_pages = v.max_pages;
  out->tile_tokens = v.tile_tokens;
  out->tile_bytes = v.tile_bytes;
  out->tile0_offset = v.tile0_off;
  out->rec_ksz_offset = v.rec_ksz_off;
  return KVQ_OK;
}

kvq_status kvq_seq_lengths(const kvq_cache* c, int32_t layer, int32_t seq, int32_t* quantized,
                           int32_t* residual) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (seq < 0 || seq >= c->cfg.max_batch) return fail(KVQ_ERR_INVALID_ARG, "seq %d out of range", seq);
  if (!quantized || !residual) return fail(KVQ_ERR_INVALID_ARG, "output pointer is null");
  const size_t i = (size_t)layer * c->cfg.max_batch + seq;
  *quantized = c->q_len[i];
  *residual = c->n_len[i];
  return KVQ_OK;
}

kvq_status kvq_seq_value_lengths(const kvq_cache* c, int32_t layer, int32_t seq, int32_t* quantized,
                                 int32_t* residual) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (seq < 0 || seq >= c->cfg.max_batch) return fail(KVQ_ERR_INVALID_ARG, "seq %d out of range", seq);
  if (!quantized || !residual) return fail(KVQ_ERR_INVALID_ARG, "output pointer is null");
  const size_t i = (size_t)layer * c->cfg.max_batch + seq;
  *quantized = c->qv_len[i];
  *residual = c->q_len[i] + c->n_len[i] - c->qv_len[i];
  return KVQ_OK;
}

kvq_status kvq_seq_sinks(const kvq_cache* c, int32_t layer, int32_t seq, int32_t* sinks) {
  g_last_error.clear();
  kvq_status s = check_cache_layer(c, layer);
  if (s != KVQ_OK) return s;
  if (seq < 0 || seq >= c->cfg.max_batch) return fail(KVQ_ERR_INVALID_ARG, "seq %d out of range", seq);
  if (!sinks) return fail(KVQ_ERR_INVALID_ARG, "output pointer is null");
  *sinks = c->s_len[(size_t)layer * c->cfg.max_batch + seq];
  return KVQ_OK;
}

}  // extern "C"
