// Tensor-core fp32 accumulation: the chain of 16 mma.sync m16n8k16 steps
// (fp16 operands, fp32 accumulators) that the quantizer's ranking runs per
// output, on adversarial data, against the exact sum of the products (the
// fp16 x fp16 products are exact; the host sums them in long double).
// Prints, per data law, the largest |error| / sum |products|.
//
// Laws: 0 plain normal values; 1 exponents spread over 2^-12 .. 2^12;
// 2 one dominant product per row (1024) among small ones (1e-3);
// 3 half the products +1, half -1 (cancellation).
#include <cmath>
#include <cstdio>
#include <random>
#include <vector>

#include <cuda_fp16.h>

constexpr int kSteps = 16, kK = 16 * kSteps, kTrials = 4096;

__global__ void chain(const __half* A, const __half* B, float* D) {
  const int lane = threadIdx.x, g = lane >> 2, t = lane & 3;
  for (int tr = blockIdx.x; tr < kTrials; tr += gridDim.x) {
    const __half* a = A + size_t(tr) * 16 * kK;   // [16][kK]
    const __half* b = B + size_t(tr) * 8 * kK;    // [8][kK]
    float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int s = 0; s < kSteps; ++s) {
      const int k0 = 16 * s;
      auto word = [](const __half* p) { return *reinterpret_cast<const unsigned*>(p); };
      const unsigned a0 = word(a + g * kK + k0 + 2 * t), a1 = word(a + (g + 8) * kK + k0 + 2 * t);
      const unsigned a2 = word(a + g * kK + k0 + 2 * t + 8), a3 = word(a + (g + 8) * kK + k0 + 2 * t + 8);
      const unsigned b0 = word(b + g * kK + k0 + 2 * t), b1 = word(b + g * kK + k0 + 2 * t + 8);
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
          "{%0,%1,%2,%3};\n"
          : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
          : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    float* o = D + size_t(tr) * 128;
    o[g * 8 + 2 * t] = d[0];
    o[g * 8 + 2 * t + 1] = d[1];
    o[(g + 8) * 8 + 2 * t] = d[2];
    o[(g + 8) * 8 + 2 * t + 1] = d[3];
  }
}

int main() {
  std::mt19937_64 rng(7);
  std::normal_distribution<double> nrm(0.0, 1.0);
  std::uniform_int_distribution<int> uni(0, 1 << 30);
  std::vector<__half> A(size_t(kTrials) * 16 * kK), B(size_t(kTrials) * 8 * kK);
  std::vector<float> fa(A.size()), fb(B.size());
  for (int tr = 0; tr < kTrials; ++tr) {
    const int law = tr % 4;
    for (int i = 0; i < 16 * kK; ++i) {
      double v;
      if (law == 0) v = nrm(rng);
      else if (law == 1) v = nrm(rng) * std::ldexp(1.0, uni(rng) % 24 - 12);
      else if (law == 2) v = (i % kK == 0) ? 1024.0 : nrm(rng) * 1e-3;
      else v = ((i % kK) < kK / 2 ? 1.0 : -1.0) * (1.0 + 1e-3 * nrm(rng));
      const __half h = __float2half_rn(float(v));
      A[size_t(tr) * 16 * kK + i] = h;
      fa[size_t(tr) * 16 * kK + i] = __half2float(h);
    }
    for (int i = 0; i < 8 * kK; ++i) {
      const double v = (law == 3) ? 1.0 + 1e-3 * nrm(rng)
                                  : nrm(rng) * (law == 1 ? std::ldexp(1.0, uni(rng) % 16 - 8) : 1.0);
      const __half h = __float2half_rn(float(v));
      B[size_t(tr) * 8 * kK + i] = h;
      fb[size_t(tr) * 8 * kK + i] = __half2float(h);
    }
  }
  __half *dA = nullptr, *dB = nullptr;
  float* dD = nullptr;
  if (cudaMalloc(&dA, A.size() * 2) != cudaSuccess || cudaMalloc(&dB, B.size() * 2) != cudaSuccess ||
      cudaMalloc(&dD, size_t(kTrials) * 128 * 4) != cudaSuccess) {
    std::printf("{\"error\": \"cudaMalloc\"}\n");
    return 1;
  }
  cudaMemcpy(dA, A.data(), A.size() * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dB, B.data(), B.size() * 2, cudaMemcpyHostToDevice);
  chain<<<148, 32>>>(dA, dB, dD);
  const cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    std::printf("{\"error\": \"%s\"}\n", cudaGetErrorString(e));
    return 1;
  }
  std::vector<float> D(size_t(kTrials) * 128);
  cudaMemcpy(D.data(), dD, D.size() * 4, cudaMemcpyDeviceToHost);
  double worst[4] = {0.0, 0.0, 0.0, 0.0};
  for (int tr = 0; tr < kTrials; ++tr) {
    for (int m = 0; m < 16; ++m)
      for (int n = 0; n < 8; ++n) {
        long double sum = 0.0L, mag = 0.0L;
        for (int k = 0; k < kK; ++k) {
          const long double p = static_cast<long double>(fa[size_t(tr) * 16 * kK + m * kK + k]) *
                                fb[size_t(tr) * 8 * kK + n * kK + k];
          sum += p;
          mag += fabsl(p);
        }
        if (mag > 0.0L) {
          const double err = std::fabs(double(static_cast<long double>(D[size_t(tr) * 128 + m * 8 + n]) - sum));
          worst[tr % 4] = std::fmax(worst[tr % 4], err / double(mag));
        }
      }
  }
  std::printf("{\"worst_rel\": [%.6e, %.6e, %.6e, %.6e]}\n", worst[0], worst[1], worst[2], worst[3]);
  cudaFree(dA);
  cudaFree(dB);
  cudaFree(dD);
  return 0;
}
