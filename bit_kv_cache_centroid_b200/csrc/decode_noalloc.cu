// decode_noalloc.cu — kv2_attention_decode_noalloc: the same decode attention
// as kv2_attention_decode, but its scratch (per-query-head tables and split-K
// partials) lives in a fixed array inside the library instead of a workspace
// the caller allocates.
//
// Who needs this: code that must not allocate device memory itself, for
// example a plugin running inside a host framework that owns the device
// allocator and forbids cudaMalloc, or a latency-critical serving loop where a
// cudaMalloc/cudaFree pair would synchronize the device. Such a caller still
// passes its own inputs and outputs; only the scratch is provided here.
//
// The array is a file-scope __device__ object of kNoallocScratchBytes (8 MiB):
// every GPU that loads the library holds it until the process exits. In host
// code the array's name is only a host-side stand-in, so its device address is
// looked up once per device with cudaGetSymbolAddress (on the first call made
// while that device is current) and cached. That first call per device should
// happen before any stream capture. All calls share the one array, and each
// call leaves its contents behind: calls whose kernels overlap on the GPU (for
// example on two streams) race on it and must be serialized by the caller.
// Nothing needs clearing between calls: every scratch byte a call reads was
// written earlier in the same call.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoallocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once).
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" kv2_status kv2_attention_decode_noalloc(const kv2_cache* cache, int len, const uint16_t* Q,
                                                   int H_q, float sm_scale, void* out, int out_dtype,
                                                   void* stream) {
  // Shapes the library does not support report 0 here; the delegated call
  // below then returns the precise error.
  const size_t need = kv2_decode_workspace_size(cache, H_q, len);
  if (need > kNoallocScratchBytes)
    return kv2::set_last_error(KV2_ERR_WORKSPACE,
                               "decode_noalloc: this shape needs %zu bytes of scratch; the library's "
                               "fixed array holds %zu bytes (use kv2_attention_decode with a workspace)",
                               need, kNoallocScratchBytes);
  void* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess)
    return kv2::set_last_error(KV2_ERR_CUDA, "decode_noalloc: scratch set-up failed: %s", cudaGetErrorString(e));
  return kv2_attention_decode(cache, len, Q, H_q, sm_scale, out, out_dtype, scratch, kNoallocScratchBytes, stream);
}
