// decode_noalloc.cu — kv2_attention_decode_noalloc: the same decode attention
// as kv2_attention_decode, but its scratch (per-query-head tables and split-K
// partials) lives in a fixed array inside the library instead of a workspace
// the caller allocates; and kv2_decode_noalloc_error, which reads (and
// optionally clears) that array's error word.
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
// while that device is current) and cached per device ordinal. That first call
// per device should happen before any stream capture. The cached address
// belongs to the device's primary context (the one the runtime API uses): the
// entry points must not be used from another driver context, nor after
// cudaDeviceReset in the same process.
//
// All calls share the one array, and each call leaves its contents behind:
// calls whose kernels overlap on the GPU (for example on two streams) race on
// it and must be serialized by the caller. Apart from its first 32-bit word,
// every scratch byte a call reads was written earlier in the same call. That
// first word is the decode kernel's sticky error word (set to 1 when a wait
// for its cache tiles runs out of budget; the affected outputs are NaN): the
// array starts zeroed, no decode call clears it, and kv2_decode_noalloc_error
// reads it and, on request, clears it.
#include <mutex>

#include <nvtx3/nvToolsExt.h>

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
  nvtxRangePushA("kv2_attention_decode_noalloc");
  struct Pop { ~Pop() { nvtxRangePop(); } } pop_;
  // every argument check first, so that a bad call neither loads the module
  // nor touches the device
  size_t need = 0;
  if (kv2_status st = kv2::validate_decode(cache, len, Q, H_q, out, out_dtype, &need); st != KV2_OK) return st;
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

extern "C" kv2_status kv2_decode_noalloc_error(int* flag, int clear, void* stream) {
  if (!flag) return kv2::set_last_error(KV2_ERR_INVALID_ARG, "decode_noalloc_error: flag is NULL");
  void* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess)
    return kv2::set_last_error(KV2_ERR_CUDA, "decode_noalloc_error: scratch set-up failed: %s", cudaGetErrorString(e));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  e = cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear && word) {
    e = cudaMemsetAsync(scratch, 0, sizeof(word), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess)
    return kv2::set_last_error(KV2_ERR_CUDA, "decode_noalloc_error: %s", cudaGetErrorString(e));
  *flag = word;
  return kv2::set_last_error(KV2_OK, "");
}
