// decode_pair_kernel instances with 2-bit values (1, 2 or 4 value groups per head).
#include "kvq_decode_pair.cuh"

namespace kvq {
namespace tc {

cudaError_t launch_pair_v2(int ngrp, const DecodeParams& p, const MmaPlan& mp, cudaStream_t stream) {
  if (ngrp == 1) return launch_pair_instance<2, 1>(p, mp, stream);
  if (ngrp == 2) return launch_pair_instance<2, 2>(p, mp, stream);
  if (ngrp == 4) return launch_pair_instance<2, 4>(p, mp, stream);
  return cudaErrorInvalidValue;
}

const void* fn_pair_v2(int ngrp) {
  if (ngrp == 1) return pair_instance_fn<2, 1>();
  if (ngrp == 2) return pair_instance_fn<2, 2>();
  if (ngrp == 4) return pair_instance_fn<2, 4>();
  return nullptr;
}

}  // namespace tc
}  // namespace kvq
