// Instances of decode_tc_kernel for one key width KVQ_TC_KB and key n-tile
// count KVQ_TC_NKT (defined by the including file): every supported (value
// bits, value groups per head). One file per pair keeps the compile units
// small enough to build in parallel.
#include "kvq_decode_tc.cuh"

#define KVQ_TC_CAT2(a, b, c) a##b##_##c
#define KVQ_TC_CAT(a, b, c) KVQ_TC_CAT2(a, b, c)
#define KVQ_TC_LAUNCH KVQ_TC_CAT(launch_tc_k, KVQ_TC_KB, KVQ_TC_NKT)
#define KVQ_TC_FN KVQ_TC_CAT(fn_tc_k, KVQ_TC_KB, KVQ_TC_NKT)

namespace kvq {
namespace tc {

// (value bits, value groups per head) pairs with a value chunk inside one
// group; per-token keys (pt) take one group per head vector
#define KVQ_TC_VB_NG(X) X(2, 1) X(2, 2) X(4, 1) X(4, 2) X(4, 4) X(8, 1) X(8, 2) X(8, 4)
#define KVQ_TC_VB_PT(X) X(2, 1) X(4, 1) X(8, 1)

cudaError_t KVQ_TC_LAUNCH(int vb, int ngrp, bool pt, const DecodeParams& p, const MmaPlan& mp, cudaStream_t stream) {
#define KVQ_TC_CASE(V, N) \
  if (!pt && vb == V && ngrp == N) return launch_instance<KVQ_TC_KB, V, N, KVQ_TC_NKT, false>(p, mp, stream);
  KVQ_TC_VB_NG(KVQ_TC_CASE)
#undef KVQ_TC_CASE
#define KVQ_TC_CASE(V, N) \
  if (pt && vb == V && ngrp == N) return launch_instance<KVQ_TC_KB, V, N, KVQ_TC_NKT, true>(p, mp, stream);
  KVQ_TC_VB_PT(KVQ_TC_CASE)
#undef KVQ_TC_CASE
  return cudaErrorInvalidValue;
}

const void* KVQ_TC_FN(int vb, int ngrp, bool pt) {
#define KVQ_TC_CASE(V, N) \
  if (!pt && vb == V && ngrp == N) return instance_fn<KVQ_TC_KB, V, N, KVQ_TC_NKT, false>();
  KVQ_TC_VB_NG(KVQ_TC_CASE)
#undef KVQ_TC_CASE
#define KVQ_TC_CASE(V, N) \
  if (pt && vb == V && ngrp == N) return instance_fn<KVQ_TC_KB, V, N, KVQ_TC_NKT, true>();
  KVQ_TC_VB_PT(KVQ_TC_CASE)
#undef KVQ_TC_CASE
  return nullptr;
}

}  // namespace tc
}  // namespace kvq
