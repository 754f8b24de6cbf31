// kvq_decode_attention_noalloc: decode attention whose split partials live in
// a scratch array that this library holds in device memory, so the call needs
// no device memory from its caller beyond the cache, the query and the output.
//
// The array is a file-scope __device__ variable: every GPU on which the
// library's module is loaded holds KVQ_STATIC_SCRATCH_BYTES of it until the
// process exits. Host code cannot use the array's name as a device address (on
// the host it names a stand-in object), so the device address is looked up
// with cudaGetSymbolAddress once per device, with that device current, and
// passed to the kernels.
#include <mutex>

#include "kvq_decode.cuh"

namespace {

static __device__ __align__(256) uint8_t g_decode_scratch[KVQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
uint8_t* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up on the
// first call per device); nullptr and *err on failure.
uint8_t* scratch_address(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = static_cast<uint8_t*>(ptr);
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

kvq_status kvq_decode_attention_noalloc(kvq_cache* c, int32_t layer, const void* q, void* out, int32_t out_dtype,
                                        float softmax_scale, int32_t batch, void* stream) {
  kvq::clear_last_error();
  if (!c) return kvq::report_status(KVQ_ERR_INVALID_ARG, "cache is null");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return kvq::report_cuda_error(e, "cudaGetDevice");
  // the array looked up below belongs to the current device: it must be the
  // device that holds the cache's arena
  if (dev != kvq::cache_device(c))
    return kvq::report_status(KVQ_ERR_INVALID_ARG, "the current device is not the cache's device");
  uint8_t* base = scratch_address(&e);
  if (!base) return kvq::report_cuda_error(e, "looking up the static decode scratch");
  const kvq::StaticScratch scratch{base, (int64_t)KVQ_STATIC_SCRATCH_BYTES};
  return kvq::enqueue_decode(c, layer, nullptr, nullptr, q, out, out_dtype, softmax_scale, batch, stream, &scratch);
}

}  // extern "C"
