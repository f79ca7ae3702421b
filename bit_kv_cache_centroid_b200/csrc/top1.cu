// top1.cu — the most-attended token of each query (retrieval analysis).
//
// Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
// World Models" analyses how Key quantization shifts which temporal-spatial
// tokens a Query selects (the retrieval shift of its introduction and Table 1).
// The index of the largest attention logit per query, over the packed cache
// (centre + INT2 residual + PSAC term, as decode reads it) or over dense bf16
// keys, lets a caller count how often quantization moves it.
//
//   logit_t = q . khat_t + (q P) . a_t     (packed; fp32, channels in order)
//   logit_t = q . k_t                      (dense)
//
// One thread per token computes its logit for one query head; each CTA keeps
// its best (logit, lowest index) and a second kernel reduces the CTAs of a
// query. Not on the attention hot path: plain CUDA-core arithmetic.
#include <cfloat>
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace kv2 {
namespace {

constexpr int kTopThreads = 256;
constexpr int kTokensPerCta = 4096;

struct Top1Params {
  const uint16_t* Q;        // bf16 [B][nq][H_q][d]
  const uint16_t* K;        // dense bf16 [B][len][H_kv][d] (dense mode) or null
  const uint32_t* k_code;   // packed cache (packed mode)
  const uint32_t* k_sz;
  const void* cidx;
  const uint16_t* psac;
  const uint16_t* psac_scale;
  const uint16_t* cent;
  const float* P;
  const int32_t* table;     // paged cache: block table (null: contiguous)
  int page;
  int group;                // channels per (scale, zero) group
  int B, nq, H_q, H_kv, d, M, r, cap, len, psac_fmt, splits;
  unsigned long long* part;  // [B*nq*H_q][splits]: (order key of the logit << 32) | ~index
};

// larger logit first, then lower index: the 64-bit key's maximum
__device__ __forceinline__ unsigned long long top_key(float logit, int t) {
  return (static_cast<unsigned long long>(float_order(logit)) << 32) | static_cast<unsigned>(~t);
}

__global__ void __launch_bounds__(kTopThreads) top1_split(Top1Params p) {
  extern __shared__ float sh[];                     // q [d], u [r]
  float* q = sh;
  float* u = sh + p.d;
  const int bq = blockIdx.x, split = blockIdx.y;   // query (b, query, head), token range
  const int b = bq / (p.nq * p.H_q), hq = bq % p.H_q;
  const int h = hq / (p.H_q / p.H_kv);
  for (int c = threadIdx.x; c < p.d; c += kTopThreads) q[c] = bf16_to_f32(p.Q[size_t(bq) * p.d + c]);
  __syncthreads();
  if (!p.K)
    for (int i = threadIdx.x; i < p.r; i += kTopThreads) {
      float acc = 0.0f;
      for (int c = 0; c < p.d; ++c) acc = fmaf(q[c], p.P[(size_t(h) * p.d + c) * p.r + i], acc);
      u[i] = acc;
    }
  __syncthreads();
  unsigned long long best = 0ull;
  const int t_end = min(p.len, (split + 1) * kTokensPerCta);
  for (int t = split * kTokensPerCta + threadIdx.x; t < t_end; t += kTopThreads) {
    float acc = 0.0f;
    if (p.K) {
      const uint16_t* kr = p.K + ((size_t(b) * p.len + t) * p.H_kv + h) * p.d;
      for (int c = 0; c < p.d; ++c) acc = fmaf(q[c], bf16_to_f32(kr[c]), acc);
    } else {
      const size_t slot = cache_slot(p.table, p.page, p.H_kv, p.cap, b, h, t);
      const int j = (p.M <= 256) ? int(static_cast<const uint8_t*>(p.cidx)[slot])
                                 : int(static_cast<const uint16_t*>(p.cidx)[slot]);
      const uint16_t* mu = p.cent + (size_t(h) * p.M + min(j, p.M - 1)) * p.d;
      for (int c = 0; c < p.d; ++c) {
        const uint32_t sz = p.k_sz[slot * (p.d / p.group) + c / p.group];
        const float s = f16_to_f32(uint16_t(sz & 0xffff)), z = f16_to_f32(uint16_t(sz >> 16));
        const uint32_t code = (p.k_code[slot * (p.d / 16) + c / 16] >> (2 * (c % 16))) & 3u;
        acc = fmaf(q[c], fmaf(float(code), s, z) + f16_to_f32(mu[c]), acc);
      }
      for (int i = 0; i < p.r; ++i) {
        float a;
        if (p.psac_fmt == 1)
          a = float(reinterpret_cast<const int8_t*>(p.psac)[slot * p.r + i]) * f16_to_f32(p.psac_scale[slot]);
        else
          a = f16_to_f32(p.psac[slot * p.r + i]);
        acc = fmaf(u[i], a, acc);
      }
    }
    const unsigned long long key = top_key(acc, t);
    best = key > best ? key : best;
  }
  // block maximum of the keys
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
    best = other > best ? other : best;
  }
  __shared__ unsigned long long wbest[kTopThreads / 32];
  if ((threadIdx.x & 31) == 0) wbest[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kTopThreads / 32; ++w) best = wbest[w] > best ? wbest[w] : best;
    p.part[size_t(bq) * p.splits + split] = best;
  }
}

__global__ void top1_reduce(const unsigned long long* part, int n, int splits, int32_t* top1) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  unsigned long long best = 0ull;
  for (int s = 0; s < splits; ++s) best = part[size_t(i) * splits + s] > best ? part[size_t(i) * splits + s] : best;
  top1[i] = (best == 0ull) ? -1 : int(~static_cast<unsigned>(best & 0xffffffffu));
}

}  // namespace

size_t top1_workspace_bytes(int B, int nq, int H_q, int len) {
  const int splits = len > 0 ? (len + kTokensPerCta - 1) / kTokensPerCta : 1;
  return size_t(B) * nq * H_q * splits * sizeof(unsigned long long);
}

cudaError_t launch_top1(const Top1Args& a, cudaStream_t s) {
  Top1Params p{};
  p.Q = a.Q;
  p.K = a.K;
  p.B = a.B;
  p.nq = a.nq;
  p.H_q = a.H_q;
  p.H_kv = a.H_kv;
  p.d = a.d;
  p.len = a.len;
  if (a.c) {
    const kv2_cache& c = *a.c;
    p.k_code = c.k_code;
    p.k_sz = c.k_sz;
    p.cidx = c.cidx;
    p.psac = c.psac;
    p.psac_scale = c.psac_scale;
    p.cent = c.centroids;
    p.P = c.P;
    p.M = c.M;
    p.r = c.r;
    p.cap = c.capacity;
    p.psac_fmt = c.psac_fmt;
    p.table = c.block_table;
    p.page = c.page_tokens;
    p.group = cache_group(c);
  }
  p.splits = a.len > 0 ? (a.len + kTokensPerCta - 1) / kTokensPerCta : 1;
  p.part = static_cast<unsigned long long*>(a.ws);
  const int nq = a.B * a.nq * a.H_q;
  cudaError_t e = cudaMemsetAsync(a.ws, 0, top1_workspace_bytes(a.B, a.nq, a.H_q, a.len), s);
  if (e != cudaSuccess) return e;
  if (a.len > 0) {
    top1_split<<<dim3(nq, p.splits), kTopThreads, (a.d + (a.K ? 0 : p.r)) * sizeof(float), s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  top1_reduce<<<(nq + 127) / 128, 128, 0, s>>>(p.part, nq, p.splits, a.top1);
  return cudaGetLastError();
}

}  // namespace kv2
