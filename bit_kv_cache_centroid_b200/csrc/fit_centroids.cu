// fit_centroids.cu — QSAC-aware centre fitting on the GPU.
//
// Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
// World Models", "1. QSAC": the clustering picks INT2-friendly Key centres.
// The loop is read as Lloyd iterations whose assignment step is the QSAC
// decision (the quantize kernel in its assignment-only mode: weighted-distance
// ranking, C candidates, least estimated perturbation) and whose update step
// moves every centre to the mean of the keys assigned to it (an unchosen
// centre keeps its value).
//
// The mean is made independent of summation order, so that the result does
// not depend on scheduling: each bf16 key value becomes a whole number of
// 2^-24 units (truncated toward zero; exact for |k| >= 2^-17) and the units
// are summed in 64-bit integers; mean = (double)sum / count (one fp64
// rounding) * 2^-24, rounded to fp16 (nearest even). Valid while
// n * max|k| < 2^39.
//
// Kernels:
//   centroid_accumulate  grid (key chunks, d / 32, H): each CTA owns a 32-channel
//                        slice of every centre in shared memory (64-bit integer
//                        atomics), walks its chunk of keys and adds its totals
//                        to the global sums once (and the counts, slice 0);
//   centroid_finalize    one thread per (head, centre, channel): the mean.
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace kv2 {
namespace {

constexpr int kSlice = 32;          // channels per accumulation CTA
constexpr int kAccThreads = 256;    // 8 keys x 32 channels per pass
constexpr int kKeysPerCta = 512;
constexpr double kUnit = 16777216.0;   // 2^24 units per 1.0

__global__ void __launch_bounds__(kAccThreads) centroid_accumulate(const uint16_t* __restrict__ X, int n, int H,
                                                                   int D, int M,
                                                                   const int32_t* __restrict__ assign,
                                                                   unsigned long long* __restrict__ sums,
                                                                   unsigned long long* __restrict__ counts) {
  extern __shared__ unsigned long long acc[];       // [M][kSlice], then [M] counts
  unsigned long long* cnt = acc + size_t(M) * kSlice;
  const int h = blockIdx.z, slice = blockIdx.y;
  const int c = threadIdx.x % kSlice, kk = threadIdx.x / kSlice;
  for (int i = threadIdx.x; i < M * (kSlice + 1); i += kAccThreads) acc[i] = 0ull;
  __syncthreads();
  const int t0 = blockIdx.x * kKeysPerCta, t1 = min(n, t0 + kKeysPerCta);
  for (int t = t0 + kk; t < t1; t += kAccThreads / kSlice) {
    const int j = assign[size_t(t) * H + h];
    const float v = __uint_as_float(uint32_t(X[(size_t(t) * H + h) * D + slice * kSlice + c]) << 16);
    const long long units = __double2ll_rz(double(v) * kUnit);
    atomicAdd(&acc[size_t(j) * kSlice + c], static_cast<unsigned long long>(units));
    if (slice == 0 && c == 0) atomicAdd(&cnt[j], 1ull);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < M * kSlice; i += kAccThreads) {
    const unsigned long long s = acc[i];
    if (s != 0ull) atomicAdd(&sums[(size_t(h) * M + i / kSlice) * D + slice * kSlice + i % kSlice], s);
  }
  if (slice == 0)
    for (int j = threadIdx.x; j < M; j += kAccThreads)
      if (cnt[j] != 0ull) atomicAdd(&counts[size_t(h) * M + j], cnt[j]);
}

__global__ void centroid_finalize(const unsigned long long* __restrict__ sums,
                                  const unsigned long long* __restrict__ counts, int H, int D, int M,
                                  uint16_t* __restrict__ cent) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= size_t(H) * M * D) return;
  const unsigned long long n = counts[i / D];
  if (n == 0ull) return;                              // unchosen: keeps its value
  const double q = __ll2double_rn(static_cast<long long>(sums[i])) / __ull2double_rn(n);
  cent[i] = __half_as_ushort(__double2half(q * (1.0 / kUnit)));
}

}  // namespace

size_t fit_centroids_workspace_bytes(int H, int D, int M) {
  return (size_t(H) * M * D + size_t(H) * M) * sizeof(unsigned long long);
}

cudaError_t launch_fit_centroids(const FitCentroidsArgs& a, cudaStream_t s) {
  unsigned long long* sums = static_cast<unsigned long long*>(a.ws);
  unsigned long long* counts = sums + size_t(a.H) * a.M * a.D;
  const size_t acc_smem = size_t(a.M) * (kSlice + 1) * sizeof(unsigned long long);
  cudaError_t e = cudaFuncSetAttribute(centroid_accumulate, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(acc_smem));
  if (e != cudaSuccess) return e;
  QuantizeArgs q{};
  q.K = a.X;
  q.V = a.X;                      // not read in assignment mode
  q.B = 1;
  q.H = a.H;
  q.d = a.D;
  q.M = a.M;
  q.r = 0;
  q.cap = a.n;
  q.n_new = a.n;
  q.pos = 0;
  q.C = a.C;
  q.cent = a.cent;
  q.P = nullptr;
  q.w = a.w;
  q.Wg = a.Wg;
  q.group = a.group;
  q.assign = a.assign;
  for (int it = 0; it < a.iters; ++it) {
    e = launch_quantize(q, s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(a.ws, 0, fit_centroids_workspace_bytes(a.H, a.D, a.M), s);
    if (e != cudaSuccess) return e;
    const dim3 grid((a.n + kKeysPerCta - 1) / kKeysPerCta, a.D / kSlice, a.H);
    centroid_accumulate<<<grid, kAccThreads, acc_smem, s>>>(a.X, a.n, a.H, a.D, a.M, a.assign, sums, counts);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t total = size_t(a.H) * a.M * a.D;
    centroid_finalize<<<unsigned((total + 255) / 256), 256, 0, s>>>(sums, counts, a.H, a.D, a.M, a.cent);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace kv2
