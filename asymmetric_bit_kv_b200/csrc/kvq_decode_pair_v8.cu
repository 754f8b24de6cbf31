// decode_pair_kernel instances with 8-bit values (1, 2 or 4 value groups per head).
#include "kvq_decode_pair.cuh"

namespace kvq {
namespace tc {

cudaError_t launch_pair_v8(int ngrp, const DecodeParams& p, const MmaPlan& mp, cudaStream_t stream) {
  if (ngrp == 1) return launch_pair_instance<8, 1>(p, mp, stream);
  if (ngrp == 2) return launch_pair_instance<8, 2>(p, mp, stream);
  if (ngrp == 4) return launch_pair_instance<8, 4>(p, mp, stream);
  return cudaErrorInvalidValue;
}

const void* fn_pair_v8(int ngrp) {
  if (ngrp == 1) return pair_instance_fn<8, 1>();
  if (ngrp == 2) return pair_instance_fn<8, 2>();
  if (ngrp == 4) return pair_instance_fn<8, 4>();
  return nullptr;
}

}  // namespace tc
}  // namespace kvq
