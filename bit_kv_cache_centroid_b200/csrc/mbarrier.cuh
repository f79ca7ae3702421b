// mbarrier.cuh — shared-memory barriers with bounded waits, and the 1-D bulk
// copy (global -> this CTA's shared memory) that completes on one of them.
#pragma once

#include <cstdint>
#include <cstdlib>

namespace kv2 {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// makes barrier initialisation visible to the other threads and to the bulk-copy unit
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// try_wait suspends the calling thread (it issues nothing) until the phase
// completes or a hardware time limit passes; either way control comes back.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t phase) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}\n"
      : "=r"(done)
      : "r"(bar), "r"(phase)
      : "memory");
  return done != 0;
}
// Bounded wait: until the phase completes or `budget` SM clock cycles pass.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, unsigned long long budget) {
  const unsigned long long t0 = clock64();
  while (!mbar_try(bar, phase)) {
    if (clock64() - t0 > budget) return false;
  }
  return true;
}
// one arrival that also announces `bytes` of bulk-copy traffic for this phase
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// bytes (a multiple of 16) from global src to shared dst (both 16-byte
// aligned); completes as transaction bytes on `bar`
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Host side: the wait budget in SM clock cycles (KV2_WAIT_BUDGET_CYCLES,
// default 2^31, about one second), and KV2_FORCE_WAIT_TIMEOUT=1, under which
// kernels wait on a barrier that nothing completes (tests of the timeout path).
inline unsigned long long env_wait_budget() {
  const char* e = std::getenv("KV2_WAIT_BUDGET_CYCLES");
  return e ? std::strtoull(e, nullptr, 10) : (1ull << 31);
}
inline int env_force_timeout() {
  const char* e = std::getenv("KV2_FORCE_WAIT_TIMEOUT");
  return (e && e[0] == '1') ? 1 : 0;
}

}  // namespace kv2
