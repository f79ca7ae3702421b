// quantize.cu — QSAC centroid assignment, INT2 residual / value packing and
// PSAC coefficients for appended tokens (one CTA = up to KT keys of one KV head).
//
// Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
// World Models", section "1. Quantization Sensitivity-Aware Clustering (QSAC)"
// (candidates by a Query-sensitivity-weighted distance, choice by the
// estimated perturbation of the INT2 residual from its dynamic range and the
// channels' sensitivity) and section "2. Principal Subspace Attention
// Compensation (PSAC)" (projection of the Key error on the top Query
// directions). The fp32 operation order of every decision is the one stated in
// include/kv2.h and reproduced bit for bit:
//   ranking  score_j = fmaf(-2, dot_j, nrm_j), dot_j = fmaf chain over c of
//            (w_c*k_c) * mu_jc, nrm_j = fmaf chain over c of (w_c*mu_jc) * mu_jc;
//   choice   E_j = fmaf chain over g of (Wg_g*s_g) * s_g;
//   PSAC     a_i = fmaf chain over c of P_ci * e_c.
//
// Phases of one CTA (256 threads):
//   1. stage the head's centroid table in shared memory as fp16, transposed to
//      [d][M] with centroid j at column (j%32)*CPL + j/32 so that lane l of a
//      warp owns centroids l, l+32, ...; stage w_c*k_c as fp32 [d][KT];
//   2. ranking: a register-tiled fp32 FMA product (KPT keys x CPL centroids
//      per thread), scores written to shared memory (aliasing the table);
//   3. top-C per key (one thread per key, insertion into a sorted list);
//   4. E_j per (key, candidate), least (E, rank) by a 64-bit shared atomicMin;
//   5. encode: per (key, group) K residual and V codecs, then PSAC per (key, i).
// Ranking is the dominant cost (M*d FMAs per key); it runs on the CUDA cores in
// fp32 so that its decisions are exact and reproducible.
#include <cfloat>

#include "common.cuh"
#include "internal.h"

namespace kv2 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int D, int CPL, int KPT>
struct QCfg {
  static constexpr int MP = 32 * CPL;            // padded centroid count
  static constexpr int KT = kWarps * KPT;        // keys per CTA
  static constexpr int SCS = MP + 1;             // score row stride (floats)
  static constexpr size_t mu_bytes = size_t(D) * MP * 2;
  static constexpr size_t sc_bytes = size_t(KT) * SCS * 4;
  static constexpr size_t regionA = mu_bytes > sc_bytes ? mu_bytes : sc_bytes;
  static constexpr size_t wk_bytes = size_t(D) * KT * 4;   // also e_s [KT][D]
  static size_t smem(int C) {
    size_t off = regionA;
    off += wk_bytes;
    off += size_t(MP) * 4;     // nrm_s
    off += size_t(D) * 4;      // w_s
    off += size_t(KT) * 8;     // best_s
    off += size_t(KT) * C * 2; // cand_s
    return (off + 15) & ~size_t(15);
  }
};

__device__ __forceinline__ void load_row_f32(const uint16_t* src, float* dst, int n) {
  // bf16 row -> fp32, n multiple of 8, src 16-byte aligned
  for (int c = 0; c < n; c += 8) {
    uint4 v = *reinterpret_cast<const uint4*>(src + c);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      dst[c + 2 * i] = __uint_as_float(u[i] << 16);
      dst[c + 2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
  }
}

template <int D, int CPL, int KPT>
__global__ void __launch_bounds__(kThreads, 1) quantize_kernel(QuantizeArgs a) {
  using Cfg = QCfg<D, CPL, KPT>;
  constexpr int MP = Cfg::MP, KT = Cfg::KT, SCS = Cfg::SCS;
  constexpr int NG = D / kGroup;
  extern __shared__ __align__(16) unsigned char smem[];
  __half* mu_s = reinterpret_cast<__half*>(smem);                    // [D][MP]
  float* sc_s = reinterpret_cast<float*>(smem);                      // [KT][SCS] (after ranking)
  float* wk_s = reinterpret_cast<float*>(smem + Cfg::regionA);       // [D][KT]
  float* e_s = wk_s;                                                 // [KT][D] (after ranking)
  float* nrm_s = wk_s + D * KT;                                      // [MP]
  float* w_s = nrm_s + MP;                                           // [D]
  unsigned long long* best_s = reinterpret_cast<unsigned long long*>(w_s + D);  // [KT]
  uint16_t* cand_s = reinterpret_cast<uint16_t*>(best_s + KT);       // [KT][C]

  const int tid = threadIdx.x;
  const int h = blockIdx.y;
  const int rows_total = a.B * a.n_new;
  const int row0 = blockIdx.x * KT;
  const int nrows = min(KT, rows_total - row0);
  const int M = a.M, C = a.C;
  const __half* cent = reinterpret_cast<const __half*>(a.cent) + size_t(h) * M * D;

  auto key_ptr = [&](const uint16_t* base, int row) {
    const int b = row / a.n_new, t = row - b * a.n_new;
    return base + ((size_t(b) * a.n_new + t) * a.H + h) * D;
  };
  auto slot_of = [&](int row) {
    const int b = row / a.n_new, t = row - b * a.n_new;
    return (size_t(b) * a.H + h) * a.cap + size_t(a.pos + t);
  };

  // ---- phase 1: stage centroids (fp16, transposed + lane-interleaved), w, w*k
  for (int i = tid; i < D; i += kThreads) w_s[i] = a.w[size_t(h) * D + i];
  for (int idx = tid; idx < MP * (D / 8); idx += kThreads) {
    const int j = idx % MP, c8 = idx / MP;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j < M) v = *reinterpret_cast<const uint4*>(cent + size_t(j) * D + c8 * 8);
    const int col = (j % 32) * CPL + j / 32;
    const __half* hv = reinterpret_cast<const __half*>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) mu_s[(c8 * 8 + i) * MP + col] = hv[i];
  }
  for (int j = tid; j < KT; j += kThreads) best_s[j] = ~0ull;
  __syncthreads();
  for (int idx = tid; idx < KT * (D / 8); idx += kThreads) {
    const int k = idx % KT, c8 = idx / KT;
    float f[8];
    if (k < nrows) {
      uint4 v = *reinterpret_cast<const uint4*>(key_ptr(a.K, row0 + k) + c8 * 8);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(u[i] << 16);
        f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) wk_s[(c8 * 8 + i) * KT + k] = __fmul_rn(w_s[c8 * 8 + i], f[i]);
  }
  for (int j = tid; j < MP; j += kThreads) {
    float acc = 0.0f;
    if (j < M) {
      const __half* row = cent + size_t(j) * D;
      for (int c = 0; c < D; ++c) {
        const float m = __half2float(row[c]);
        acc = __fmaf_rn(__fmul_rn(w_s[c], m), m, acc);
      }
    }
    nrm_s[j] = acc;
  }
  __syncthreads();

  // ---- phase 2: ranking scores, register tile KPT keys x CPL centroids
  const int warp = tid >> 5, lane = tid & 31;
  {
    float acc[KPT][CPL];
#pragma unroll
    for (int k = 0; k < KPT; ++k)
#pragma unroll
      for (int j = 0; j < CPL; ++j) acc[k][j] = 0.0f;
    const float* wk_base = wk_s + warp * KPT;
    const __half* mu_base = mu_s + lane * CPL;
#pragma unroll 2
    for (int c = 0; c < D; ++c) {
      float wk[KPT];
#pragma unroll
      for (int k = 0; k < KPT; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(wk_base + c * KT + k);
        wk[k] = v.x; wk[k + 1] = v.y; wk[k + 2] = v.z; wk[k + 3] = v.w;
      }
      float m[CPL];
      if constexpr (CPL >= 8) {
#pragma unroll
        for (int j = 0; j < CPL; j += 8) {
          const uint4 v = *reinterpret_cast<const uint4*>(mu_base + c * MP + j);
          const __half2* h2 = reinterpret_cast<const __half2*>(&v);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(h2[i]);
            m[j + 2 * i] = f.x; m[j + 2 * i + 1] = f.y;
          }
        }
      } else if constexpr (CPL == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(mu_base + c * MP);
        const __half2* h2 = reinterpret_cast<const __half2*>(&v);
        const float2 f0 = __half22float2(h2[0]), f1 = __half22float2(h2[1]);
        m[0] = f0.x; m[1] = f0.y; m[2] = f1.x; m[3] = f1.y;
      } else if constexpr (CPL == 2) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(mu_base + c * MP));
        m[0] = f.x; m[1] = f.y;
      } else {
        m[0] = __half2float(mu_base[c * MP]);
      }
#pragma unroll
      for (int k = 0; k < KPT; ++k)
#pragma unroll
        for (int j = 0; j < CPL; ++j) acc[k][j] = __fmaf_rn(wk[k], m[j], acc[k][j]);
    }
    __syncthreads();  // every warp is done with mu_s: scores may overwrite it
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int cj = j * 32 + lane;  // centroid id owned by this lane
      const float nrm = nrm_s[cj];
#pragma unroll
      for (int k = 0; k < KPT; ++k) {
        const float s = (cj < M) ? __fmaf_rn(-2.0f, acc[k][j], nrm) : FLT_MAX;
        sc_s[(warp * KPT + k) * SCS + cj] = s;
      }
    }
  }
  __syncthreads();

  // ---- phase 3: the C best-ranked centroids per key (ties -> lower id)
  for (int k = tid; k < nrows; k += kThreads) {
    const float* sc = sc_s + k * SCS;
    uint16_t* list = cand_s + k * C;
    int cnt = 0;
    for (int j = 0; j < M; ++j) {
      const float s = sc[j];
      if (cnt == C && !(s < sc[list[C - 1]])) continue;
      int p = (cnt < C) ? cnt++ : C - 1;
      while (p > 0 && sc[list[p - 1]] > s) {
        list[p] = list[p - 1];
        --p;
      }
      list[p] = static_cast<uint16_t>(j);
    }
  }
  __syncthreads();

  // ---- phase 4: perturbation estimate per (key, candidate); least (E, rank)
  if (C > 1) {
    for (int task = tid; task < nrows * C; task += kThreads) {
      const int k = task / C, i = task - k * C;
      const int j = cand_s[k * C + i];
      const uint16_t* krow = key_ptr(a.K, row0 + k);
      const __half* mrow = cent + size_t(j) * D;
      float E = 0.0f;
#pragma unroll 1
      for (int g = 0; g < NG; ++g) {
        float mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
        for (int c = g * kGroup; c < (g + 1) * kGroup; c += 8) {
          const uint4 kv = *reinterpret_cast<const uint4*>(krow + c);
          const uint4 mv = *reinterpret_cast<const uint4*>(mrow + c);
          const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
          const __half2* mh = reinterpret_cast<const __half2*>(&mv);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 mf = __half22float2(mh[q]);
            const float x0 = __fsub_rn(__uint_as_float(ku[q] << 16), mf.x);
            const float x1 = __fsub_rn(__uint_as_float(ku[q] & 0xffff0000u), mf.y);
            mn = fminf(mn, fminf(x0, x1));
            mx = fmaxf(mx, fmaxf(x0, x1));
          }
        }
        const GroupParams p = group_params(mn, mx);
        E = __fmaf_rn(__fmul_rn(a.Wg[size_t(h) * NG + g], p.s), p.s, E);
      }
      const unsigned long long key = (static_cast<unsigned long long>(float_order(E)) << 32) | unsigned(i);
      atomicMin(&best_s[k], key);
    }
    __syncthreads();
  }

  // ---- phase 5a: K residual and V codecs per (key, group)
  for (int task = tid; task < nrows * NG * 2; task += kThreads) {
    const int which = task / (nrows * NG);   // 0: keys, 1: values
    const int kg = task - which * nrows * NG;
    const int k = kg / NG, g = kg - k * NG;
    const int row = row0 + k;
    const size_t slot = slot_of(row);
    float x[kGroup];
    int j = 0;
    if (which == 0) {
      const int rank = (C > 1) ? int(best_s[k] & 0xffffffffu) : 0;
      j = cand_s[k * C + rank];
      const uint16_t* krow = key_ptr(a.K, row) + g * kGroup;
      const __half* mrow = cent + size_t(j) * D + g * kGroup;
      load_row_f32(krow, x, kGroup);
#pragma unroll
      for (int c = 0; c < kGroup; ++c) x[c] = __fsub_rn(x[c], __half2float(mrow[c]));
    } else {
      load_row_f32(key_ptr(a.V, row) + g * kGroup, x, kGroup);
    }
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int c = 1; c < kGroup; ++c) { mn = fminf(mn, x[c]); mx = fmaxf(mx, x[c]); }
    const GroupParams p = group_params(mn, mx);
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int c = 0; c < kGroup; ++c) {
      const uint32_t q = group_code(x[c], p);
      if (c < 16) w0 |= q << (2 * c); else w1 |= q << (2 * (c - 16));
      if (which == 0) e_s[k * D + g * kGroup + c] = __fsub_rn(x[c], group_dequant(q, p));
    }
    uint32_t* code = (which == 0 ? a.k_code : a.v_code) + slot * (D / 16) + g * 2;
    code[0] = w0;
    code[1] = w1;
    (which == 0 ? a.k_sz : a.v_sz)[slot * NG + g] = uint32_t(p.s_bits) | (uint32_t(p.z_bits) << 16);
    if (which == 0 && g == 0) {
      if (M <= 256) static_cast<uint8_t*>(a.cidx)[slot] = uint8_t(j);
      else static_cast<uint16_t*>(a.cidx)[slot] = uint16_t(j);
    }
  }
  if (a.r == 0) return;
  __syncthreads();

  // ---- phase 5b: PSAC coefficients a_i = sum_c P_ci e_c (ascending c)
  for (int task = tid; task < nrows * a.r; task += kThreads) {
    const int k = task / a.r, i = task - k * a.r;
    const float* Pcol = a.P + size_t(h) * D * a.r + i;
    const float* e = e_s + k * D;
    float acc = 0.0f;
    for (int c = 0; c < D; ++c) acc = __fmaf_rn(Pcol[size_t(c) * a.r], e[c], acc);
    a.psac[slot_of(row0 + k) * a.r + i] = f16_rn(acc);
  }
}

template <int D, int CPL, int KPT>
cudaError_t launch_cfg(const QuantizeArgs& a, cudaStream_t s) {
  using Cfg = QCfg<D, CPL, KPT>;
  const size_t smem = Cfg::smem(a.C);
  auto kern = quantize_kernel<D, CPL, KPT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int rows = a.B * a.n_new;
  dim3 grid((rows + Cfg::KT - 1) / Cfg::KT, a.H);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const QuantizeArgs& a, cudaStream_t s) {
  const int mp = (a.M + 31) / 32;
  if (mp <= 1) return launch_cfg<D, 1, 16>(a, s);
  if (mp <= 2) return launch_cfg<D, 2, 16>(a, s);
  if (mp <= 4) return launch_cfg<D, 4, 16>(a, s);
  if (mp <= 8) return launch_cfg<D, 8, 8>(a, s);
  return launch_cfg<D, 16, 4>(a, s);
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t s) {
  if (a.B * a.n_new == 0) return cudaSuccess;
  return a.d == 64 ? launch_d<64>(a, s) : launch_d<128>(a, s);
}

}  // namespace kv2
