// quantize.cu — QSAC centroid assignment, INT2 residual / value packing and
// PSAC coefficients for appended tokens.
//
// Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
// World Models", section "1. Quantization Sensitivity-Aware Clustering (QSAC)"
// (candidates by a Query-sensitivity-weighted distance, choice by the
// estimated perturbation of the INT2 residual from its dynamic range and the
// channels' sensitivity) and section "2. Principal Subspace Attention
// Compensation (PSAC)" (projection of the Key error on the top Query
// directions). The decisions are those of the definitions below, evaluated in
// fp32 in the stated order, and reproduced bit for bit:
//   ranking  D_j = sum_c w_c (k_c - mu_jc)^2: t = k_c - mu_jc, then
//            acc = fmaf(w_c * t, t, acc) over ascending c; candidates = the set
//            of the C smallest (D_j, j);
//   choice   E_j = fmaf chain over g of (Wg_g*s_g) * s_g; the least (E_j, j)
//            over the candidate set;
//   PSAC     a_i = fmaf chain over c of P_ci * e_c.
//
// Structure: persistent CTAs, each bound to one KV head, stage the head's
// centroid table once (fp16, transposed to [d][M] with centroid j at column
// (j%32)*CPL + j/32, so lane l of a warp owns centroids l, l+32, ...) and the
// centroid norms, then loop over tiles of 8*KPT keys. Within a tile every warp
// runs its own KPT keys through the whole pipeline with warp synchronization
// only: w*k staging, the ranking product, top-C by warp-wide integer
// min-reductions of order-preserving score keys, the perturbation estimate per
// candidate, the K-residual and V codecs and the PSAC coefficients.
//
// Ranking in two steps. The M*d products (the dominant cost) run in the
// expanded form f_j = nrm_j - 2 dot_j, nrm_j = sum_c (w_c mu_jc) mu_jc,
// dot_j = sum_c (w_c k_c) mu_jc (register tile KPT keys x CPL centres per
// lane, one fp32 FMA per product, fma chains over ascending c), which equals
// D_j - sum_c w_c k_c^2 in exact arithmetic. With Ka = sum_c |w_c| k_c^2 and
// Na = max_j sum_c |w_c| mu_jc^2, standard error bounds of fma chains give
// |f_j - (D_j - K)| <= g (Na + 2 sqrt(Ka Na)) (Cauchy-Schwarz bounds
// sum_c |w_c k_c mu_jc|) and |fp32 D_j - D_j| <= g (sqrt(Ka) + sqrt(Na))^2,
// g = gamma_{d+3} = (d+3) 2^-24 / (1 - (d+3) 2^-24). So every centre of the
// exact C smallest has f_j <= c + 2b, where c is the C-th smallest f and
// b = g (Ka + 2 Na + 4 sqrt(Ka Na)). When no centre outside the fast top C
// lies under that threshold (nearly always), the fast top C is the exact set;
// otherwise every centre under it gets its fp32 D_j by the definition and the
// C smallest (D_j, j) are taken from those. The threshold is computed with
// g doubled and upward rounding, so it only ever errs towards the exact path.
// Tensor cores are not used: the exact decisions need the fp32 chains.
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
  static constexpr int KT = kWarps * KPT;        // keys per tile
  static constexpr size_t mu_bytes = size_t(D) * MP * 2;
  static constexpr size_t warp_wk_bytes = size_t(D) * KPT * 4;   // w*k [D][KPT], later e [KPT][D]
  // per warp: w*k / e, best (E, centre id) per key, candidates, and (int8 PSAC
  // format only, r8 = r) the fp32 coefficients [KPT][r8] before quantization
  __host__ __device__ static size_t cand_end(int C) { return (warp_wk_bytes + size_t(KPT) * 8 + size_t(KPT) * C * 2 + 15) & ~size_t(15); }
  __host__ __device__ static size_t warp_bytes(int C, int r8) { return (cand_end(C) + size_t(KPT) * r8 * 4 + 15) & ~size_t(15); }
  __host__ __device__ static size_t head_bytes(int r) { return mu_bytes + size_t(MP) * 4 + size_t(D) * 4 + size_t(D) * r * 4; }
  static size_t smem(int C, int r, int r8) { return head_bytes(r) + size_t(kWarps) * warp_bytes(C, r8); }
};

// Upper end of the fast scores that may belong to a centre of the exact C
// smallest distances (c: the C-th smallest fast score; bound derived in the
// file comment, with gamma_{d+3} doubled and every operation rounded up).
__device__ __forceinline__ float rank_threshold(float c, float ka, float na, int d) {
  const float g = float(2 * (d + 8)) * 0x1p-24f;
  const float cross = __fmul_ru(4.0f, __fsqrt_ru(__fmul_ru(ka, na)));
  const float b = __fmul_ru(g, __fadd_ru(__fadd_ru(ka, __fmul_ru(2.0f, na)), cross));
  return __fadd_ru(c, __fmul_ru(2.0f, b));
}

// D_j = sum_c w_c (k_c - mu_jc)^2 by the definition's fp32 order; krow: the
// key's D bf16 values (16-byte aligned), mu_col: centre j's column of the
// staged [D][MP] table.
template <int D, int MP>
__device__ __forceinline__ float exact_distance(const uint16_t* krow, const __half* mu_col, const float* w_s) {
  float acc = 0.0f;
#pragma unroll 2
  for (int c8 = 0; c8 < D / 8; ++c8) {
    const uint4 kv = *reinterpret_cast<const uint4*>(krow + c8 * 8);
    const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = c8 * 8 + q;
      const float kc = __uint_as_float((q & 1) ? (ku[q / 2] & 0xffff0000u) : (ku[q / 2] << 16));
      const float t = __fsub_rn(kc, __half2float(mu_col[c * MP]));
      acc = __fmaf_rn(__fmul_rn(w_s[c], t), t, acc);
    }
  }
  return acc;
}

// GS: channels per (scale, zero) group (32, 64 or 128); a group is SPG
// sub-groups of 32 channels (one code-word pair each)
template <int D, int CPL, int KPT, int GS>
__global__ void __launch_bounds__(kThreads) quantize_kernel(QuantizeArgs a) {
  using Cfg = QCfg<D, CPL, KPT>;
  constexpr int MP = Cfg::MP, KT = Cfg::KT;
  constexpr int NG = D / GS, NS = D / kGroup, SPG = GS / kGroup;
  static_assert(GS % kGroup == 0 && D % GS == 0, "groups of whole 32-channel sub-groups");
  static_assert(D * KPT >= 32 * KPT + D / 2, "the w*k buffer holds the exact pass's lists and one key row");
  extern __shared__ __align__(16) unsigned char smem[];
  __half* mu_s = reinterpret_cast<__half*>(smem);                            // [D][MP]
  float* nrm_s = reinterpret_cast<float*>(smem + Cfg::mu_bytes);              // [MP]
  float* w_s = nrm_s + MP;                                                    // [D]
  float* P_s = w_s + D;                                                       // [D][r]
  __shared__ uint32_t na_bits;   // Na = max_j sum_c |w_c| mu_jc^2 (non-negative: ordered as its bits)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r8 = (a.psac_fmt == 1) ? a.r : 0;
  unsigned char* wbase = smem + Cfg::head_bytes(a.r) + size_t(warp) * Cfg::warp_bytes(a.C, r8);
  float* wk_w = reinterpret_cast<float*>(wbase);                              // [D][KPT]
  float* e_w = wk_w;                                                          // [KPT][D] after ranking
  unsigned long long* best_w = reinterpret_cast<unsigned long long*>(wbase + Cfg::warp_wk_bytes);  // [KPT]
  uint16_t* cand_w = reinterpret_cast<uint16_t*>(best_w + KPT);              // [KPT][C]
  float* psa_w = reinterpret_cast<float*>(wbase + Cfg::cand_end(a.C));         // [KPT][r8]

  // a decode launched as this kernel's programmatic dependent may start now;
  // it waits for this grid before reading the slots written here
  asm volatile("griddepcontrol.launch_dependents;");
  const int h = blockIdx.y;
  const int rows_total = a.B * a.n_new;
  const int ntiles = (rows_total + KT - 1) / KT;
  const int M = a.M, C = a.C;
  const __half* cent = reinterpret_cast<const __half*>(a.cent) + size_t(h) * M * D;

  auto key_ptr = [&](const uint16_t* base, int row) {
    const int b = row / a.n_new, t = row - b * a.n_new;
    return base + ((size_t(b) * a.n_new + t) * a.H + h) * D;
  };
  auto slot_of = [&](int row) {
    const int b = row / a.n_new, t = row - b * a.n_new;
    return cache_slot(a.table, a.page, a.H, a.cap, b, h, a.pos + t);
  };

  // ---- once per CTA: centroid table (fp16, transposed, lane-interleaved), w,
  // the PSAC basis, norms
  if (tid == 0) na_bits = 0;
  for (int i = tid; i < D; i += kThreads) w_s[i] = a.w[size_t(h) * D + i];
  for (int i = tid; i < D * a.r; i += kThreads) P_s[i] = a.P[size_t(h) * D * a.r + i];
  for (int idx = tid; idx < MP * (D / 8); idx += kThreads) {
    const int j = idx % MP, c8 = idx / MP;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j < M) v = *reinterpret_cast<const uint4*>(cent + size_t(j) * D + c8 * 8);
    const int col = (j % 32) * CPL + j / 32;
    const __half* hv = reinterpret_cast<const __half*>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) mu_s[(c8 * 8 + i) * MP + col] = hv[i];
  }
  __syncthreads();
  for (int j = tid; j < MP; j += kThreads) {
    float acc = 0.0f, aabs = 0.0f;
    if (j < M) {
      const __half* col = mu_s + (j % 32) * CPL + j / 32;     // centroid j in the staged table
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        const float m = __half2float(col[c * MP]);
        const float wm = __fmul_rn(w_s[c], m);
        acc = __fmaf_rn(wm, m, acc);
        aabs = __fmaf_rn(fabsf(wm), fabsf(m), aabs);
      }
    }
    nrm_s[j] = acc;
    atomicMax(&na_bits, __float_as_uint(aabs));
  }
  __syncthreads();
  const float na = __uint_as_float(na_bits);

  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    // key k of this warp is row tile*KT + k*kWarps + warp, so that a short
    // append spreads over all warps
    const int rem = rows_total - tile * KT - warp;
    const int nk = rem > 0 ? min(KPT, (rem + kWarps - 1) / kWarps) : 0;
    if (nk <= 0) continue;                       // warp-uniform
    auto row_of = [&](int k) { return tile * KT + k * kWarps + warp; };

    // ---- w*k for this warp's keys, transposed to [D][KPT]; lane l handles
    // key l % KPT only (32 is a multiple of KPT) and sums its share of
    // Ka = sum_c |w_c| k_c^2 for the ranking bound
    float ka = 0.0f;
    for (int idx = lane; idx < KPT * (D / 8); idx += 32) {
      const int k = idx % KPT, c8 = idx / KPT;
      float f[8];
      if (k < nk) {
        const uint4 v = *reinterpret_cast<const uint4*>(key_ptr(a.K, row_of(k)) + c8 * 8);
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
      for (int i = 0; i < 8; ++i) {
        const float wk = __fmul_rn(w_s[c8 * 8 + i], f[i]);
        wk_w[(c8 * 8 + i) * KPT + k] = wk;
        ka = __fmaf_rn(fabsf(wk), fabsf(f[i]), ka);
      }
    }
#pragma unroll
    for (int o = 16; o >= KPT; o >>= 1) ka += __shfl_xor_sync(0xffffffffu, ka, o);
    if (lane < KPT) best_w[lane] = ~0ull;
    __syncwarp();

    // ---- ranking scores: KPT keys x CPL centres per lane
    uint32_t ord[KPT][CPL];
    {
      float acc[KPT][CPL];
#pragma unroll
      for (int k = 0; k < KPT; ++k)
#pragma unroll
        for (int j = 0; j < CPL; ++j) acc[k][j] = 0.0f;
      const __half* mu_base = mu_s + lane * CPL;
#pragma unroll 2
      for (int c = 0; c < D; ++c) {
        float wk[KPT];
        if constexpr (KPT % 4 == 0) {
#pragma unroll
          for (int k = 0; k < KPT; k += 4) {
            const float4 v = *reinterpret_cast<const float4*>(wk_w + c * KPT + k);
            wk[k] = v.x; wk[k + 1] = v.y; wk[k + 2] = v.z; wk[k + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int k = 0; k < KPT; ++k) wk[k] = wk_w[c * KPT + k];
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
        // the same fmaf per (key, centre), two at a time (fma.rn.f32x2 rounds
        // each lane as fmaf): pairs of centres when CPL >= KPT, else of keys
        if constexpr (CPL >= 2 && CPL >= KPT) {
#pragma unroll
          for (int k = 0; k < KPT; ++k) {
            const f32x2 w2 = pk2(wk[k], wk[k]);
#pragma unroll
            for (int j = 0; j < CPL; j += 2) {
              const float2 r = up2(ffma2(w2, pk2(m[j], m[j + 1]), pk2(acc[k][j], acc[k][j + 1])));
              acc[k][j] = r.x;
              acc[k][j + 1] = r.y;
            }
          }
        } else if constexpr (KPT >= 2) {
#pragma unroll
          for (int j = 0; j < CPL; ++j) {
            const f32x2 m2 = pk2(m[j], m[j]);
#pragma unroll
            for (int k = 0; k < KPT; k += 2) {
              const float2 r = up2(ffma2(pk2(wk[k], wk[k + 1]), m2, pk2(acc[k][j], acc[k + 1][j])));
              acc[k][j] = r.x;
              acc[k + 1][j] = r.y;
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < KPT; ++k)
#pragma unroll
            for (int j = 0; j < CPL; ++j) acc[k][j] = __fmaf_rn(wk[k], m[j], acc[k][j]);
        }
      }
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int cj = j * 32 + lane;            // centroid id of this lane's column j
        const float nrm = nrm_s[cj];
#pragma unroll
        for (int k = 0; k < KPT; ++k)
          ord[k][j] = (cj < M) ? float_order(__fadd_rn(__fmaf_rn(-2.0f, acc[k][j], nrm), 0.0f)) : 0xFFFFFFFFu;
      }
    }

    // ---- top-C per key: C rounds of a warp-wide min of (score order, id);
    // then the check that no other centre's fast score lies within the
    // ranking bound of the C-th. A key that fails it (rare) has its centres
    // under the threshold listed (ids, 32 per key, in this warp's w*k buffer,
    // free once the ranking products are done) and is decided by the exact
    // distances after this loop, which keeps the unrolled loop small.
    int* lists = reinterpret_cast<int*>(wk_w);               // [KPT][32]
    uint32_t exact_keys = 0, long_lists = 0;                 // bit k: key k needs the exact pass / has > 32
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      if (k >= nk) break;
      uint32_t taken = 0, last = 0;
      for (int i = 0; i < C; ++i) {
        uint32_t best = 0xFFFFFFFFu;
        int bj = 0;
#pragma unroll
        for (int j = 0; j < CPL; ++j)
          if (ord[k][j] < best) { best = ord[k][j]; bj = j; }   // lowest id among equal scores
        const uint32_t wmin = __reduce_min_sync(0xffffffffu, best);
        const uint32_t myid = (best == wmin) ? uint32_t(bj * 32 + lane) : 0xFFFFFFFFu;
        const uint32_t wid = __reduce_min_sync(0xffffffffu, myid);
        if (uint32_t(bj * 32 + lane) == wid) {
#pragma unroll
          for (int j = 0; j < CPL; ++j)
            if (j == bj) ord[k][j] = 0xFFFFFFFFu;                // taken
          taken |= 1u << bj;
        }
        if (lane == 0) cand_w[k * C + i] = uint16_t(wid);
        last = wmin;
      }
      const float thr = rank_threshold(order_float(last), __shfl_sync(0xffffffffu, ka, k), na, D);
      const uint32_t thr_o = float_order(thr);
      bool near = false;
#pragma unroll
      for (int j = 0; j < CPL; ++j) near |= ord[k][j] <= thr_o;
      if (__any_sync(0xffffffffu, near)) {
        lists[k * 32 + lane] = -1;                           // no centre
        __syncwarp();
        int n = 0;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          const bool in = ((taken >> j) & 1u) || ord[k][j] <= thr_o;
          const uint32_t m = __ballot_sync(0xffffffffu, in);
          const int at = n + __popc(m & ((1u << lane) - 1u));
          if (in && at < 32) lists[k * 32 + at] = j * 32 + lane;
          n += __popc(m);
        }
        exact_keys |= 1u << k;
        if (n > 32) long_lists |= 1u << k;
      }
    }
    __syncwarp();
    // ---- the keys whose candidate set the bound left open: fp32 D_j by the
    // definition, one listed centre per lane, and the C smallest (D_j, j);
    // with more than 32 centres under the threshold (degenerate tables), C
    // rounds over every centre instead
    for (int k = 0; k < nk; ++k) {
      if (!((exact_keys >> k) & 1u)) continue;                // warp-uniform
      // the key row (bf16) staged after the lists, so the serial chains
      // read it from shared memory: D/2 words fit since D * KPT >= 32 * KPT + D/2
      uint16_t* krow = reinterpret_cast<uint16_t*>(lists + 32 * KPT);
      if (lane < D / 8)
        reinterpret_cast<uint4*>(krow)[lane] = reinterpret_cast<const uint4*>(key_ptr(a.K, row_of(k)))[lane];
      __syncwarp();
      if (!((long_lists >> k) & 1u)) {
        const int id = lists[k * 32 + lane];                  // -1: no centre in this slot
        uint32_t o = 0xFFFFFFFFu;
        if (id >= 0)
          o = float_order(__fadd_rn(exact_distance<D, MP>(krow, mu_s + (id % 32) * CPL + id / 32, w_s), 0.0f));
        for (int i = 0; i < C; ++i) {
          const uint32_t wmin = __reduce_min_sync(0xffffffffu, o);
          const uint32_t wid = __reduce_min_sync(0xffffffffu, o == wmin ? uint32_t(id) : 0xFFFFFFFFu);
          if (uint32_t(id) == wid) o = 0xFFFFFFFFu;
          if (lane == 0) cand_w[k * C + i] = uint16_t(wid);
        }
      } else {
        uint64_t prev = 0;                                    // (order, id) of the last one taken
        for (int i = 0; i < C; ++i) {
          uint64_t best = ~0ull;
          for (int j = lane; j < M; j += 32) {
            const uint64_t key = (uint64_t(float_order(__fadd_rn(
                                      exact_distance<D, MP>(krow, mu_s + (j % 32) * CPL + j / 32, w_s), 0.0f)))
                                  << 32) | uint32_t(j);
            if ((i == 0 || key > prev) && key < best) best = key;
          }
          const uint32_t hi = __reduce_min_sync(0xffffffffu, uint32_t(best >> 32));
          const uint32_t lo = __reduce_min_sync(0xffffffffu, uint32_t(best >> 32) == hi ? uint32_t(best) : 0xFFFFFFFFu);
          prev = (uint64_t(hi) << 32) | lo;
          if (lane == 0) cand_w[k * C + i] = uint16_t(lo);
        }
      }
      __syncwarp();                                           // krow is rewritten for the next key
    }

    if constexpr (KPT == 1) {
      // One key per warp: the remaining phases run across the lanes (lane =
      // channel within a group, or (candidate, group)), with the same
      // arithmetic per decision as the general path below.
      const int row = row_of(0);
      const uint16_t* krow = key_ptr(a.K, row);
      const uint16_t* vrow = key_ptr(a.V, row);
      float kx[NS], vx[NS];                            // channel k * 32 + lane of sub-group k
#pragma unroll
      for (int k = 0; k < NS; ++k) {
        kx[k] = __uint_as_float(uint32_t(krow[k * kGroup + lane]) << 16);
        vx[k] = a.assign ? 0.0f : __uint_as_float(uint32_t(vrow[k * kGroup + lane]) << 16);
      }
      // ---- perturbation estimate: lane (candidate i, group g) takes the
      // group's scale; E_i = fmaf chain over ascending g of (W_g s_g) s_g;
      // least (E, centre id)
      int jc = cand_w[0];
      if (C > 1) {
        uint32_t best_e = 0xFFFFFFFFu, best_j = 0xFFFFFFFFu;
        for (int i0 = 0; i0 < C; i0 += 32 / NG) {
          const int i = i0 + lane / NG, g = lane % NG;
          float sg = 0.0f;
          int j = 0;
          if (i < C) {
            j = cand_w[i];
            const uint4* mseg = reinterpret_cast<const uint4*>(cent + size_t(j) * D + g * GS);   // global, L2
            const uint16_t* kseg = krow + g * GS;
            float mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
            for (int c = 0; c < GS; c += 8) {
              const uint4 kv = *reinterpret_cast<const uint4*>(kseg + c);
              const uint4 mv = __ldg(mseg + c / 8);
              const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
              const uint32_t mu4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float2 m = __half22float2(*reinterpret_cast<const __half2*>(&mu4[q]));
                const float x0 = __fsub_rn(__uint_as_float(ku[q] << 16), m.x);
                const float x1 = __fsub_rn(__uint_as_float(ku[q] & 0xffff0000u), m.y);
                mn = fmin3(mn, x0, x1);
                mx = fmax3(mx, x0, x1);
              }
            }
            sg = group_params(mn, mx).s;
          }
          float E = 0.0f;
#pragma unroll
          for (int gg = 0; gg < NG; ++gg) {
            const float sgg = __shfl_sync(0xffffffffu, sg, (lane / NG) * NG + gg);
            E = __fmaf_rn(__fmul_rn(a.Wg[size_t(h) * NG + gg], sgg), sgg, E);
          }
          const bool mine = (g == 0) && (i < C);
          const uint32_t eo = mine ? float_order(E) : 0xFFFFFFFFu;
          const uint32_t emin = __reduce_min_sync(0xffffffffu, eo);
          const uint32_t jmin = __reduce_min_sync(0xffffffffu, (mine && eo == emin) ? uint32_t(j) : 0xFFFFFFFFu);
          if (emin < best_e || (emin == best_e && jmin < best_j)) { best_e = emin; best_j = jmin; }
        }
        jc = int(best_j);
      }
      if (a.assign) {
        if (lane == 0) a.assign[size_t(row) * a.H + h] = jc;
      } else {
      // ---- K residual and V codecs, lane = channel of each 32-channel
      // sub-group; a group's range spans its SPG sub-groups and the lanes
      const __half* crow = cent + size_t(jc) * D;      // lanes read consecutive channels
      const size_t slot = slot_of(row);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          float x[SPG];
#pragma unroll
          for (int u = 0; u < SPG; ++u) {
            const int k = g * SPG + u, c = k * kGroup + lane;
            x[u] = (which == 0) ? __fsub_rn(kx[k], __half2float(crow[c])) : vx[k];
          }
          float mn = x[0], mx = x[0];
#pragma unroll
          for (int u = 1; u < SPG; ++u) {
            mn = fminf(mn, x[u]);
            mx = fmaxf(mx, x[u]);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          }
          const GroupParams gp = group_params(mn, mx);
          const float inv_s = __frcp_rn(gp.s);
#pragma unroll
          for (int u = 0; u < SPG; ++u) {
            const int k = g * SPG + u, c = k * kGroup + lane;
            const uint32_t q = group_code_recip(x[u], gp, inv_s);
            const uint32_t bits = q << (2 * (lane & 15));
            const uint32_t w0 = __reduce_or_sync(0xffffffffu, lane < 16 ? bits : 0u);
            const uint32_t w1 = __reduce_or_sync(0xffffffffu, lane >= 16 ? bits : 0u);
            if (lane == 0) {
              uint32_t* code = (which == 0 ? a.k_code : a.v_code) + slot * (D / 16) + k * 2;
              *reinterpret_cast<uint2*>(code) = make_uint2(w0, w1);
            }
            if (which == 0) e_w[c] = __fsub_rn(x[u], group_dequant(q, gp));
          }
          if (lane == 0) {
            (which == 0 ? a.k_sz : a.v_sz)[slot * NG + g] = uint32_t(gp.s_bits) | (uint32_t(gp.z_bits) << 16);
            if (which == 0 && g == 0) {
              if (M <= 256) static_cast<uint8_t*>(a.cidx)[slot] = uint8_t(jc);
              else static_cast<uint16_t*>(a.cidx)[slot] = uint16_t(jc);
            }
          }
        }
      }
      __syncwarp();
      // ---- PSAC coefficients a_i = sum_c P_ci e_c: lane partial sums over
      // channels lane, lane + 32, ..., then a warp tree (fp32; the fp16 result
      // is within one ulp of the ascending-c chain)
      for (int i0 = 0; i0 < a.r; i0 += 8) {
        float acc[8];
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) acc[ii] = 0.0f;
#pragma unroll
        for (int kc = 0; kc < D / 32; ++kc) {
          const int c = lane + 32 * kc;
          const float e = e_w[c];
          const float* Pr = P_s + c * a.r + i0;
#pragma unroll
          for (int ii = 0; ii < 8; ++ii)
            if (i0 + ii < a.r) acc[ii] = __fmaf_rn(Pr[ii], e, acc[ii]);
        }
        float mine = 0.0f;
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) {
          float v = acc[ii];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == ii) mine = v;
        }
        if (lane < 8 && i0 + lane < a.r) {
          if (r8) psa_w[i0 + lane] = mine;
          else a.psac[slot * a.r + i0 + lane] = f16_rn(mine);
        }
      }
      if (r8) {
        __syncwarp();
        if (lane == 0) psac_int8(psa_w, a.r, reinterpret_cast<int8_t*>(a.psac) + slot * a.r, a.psac_scale + slot);
      }
      }
    } else {
    // ---- perturbation estimate per (key, candidate); least (E, centre id)
    // per key
    if (C > 1) {
      for (int task = lane; task < nk * C; task += 32) {
        const int k = task / C, i = task - k * C;
        const int j = cand_w[k * C + i];
        // the candidate's row of the fp16 centre table in global memory (the
        // head's table stays in L2): 16-byte reads instead of 2-byte columns
        // of the transposed shared copy, whose lanes would collide on banks
        const uint4* mrow = reinterpret_cast<const uint4*>(cent + size_t(j) * D);
        const uint16_t* krow = key_ptr(a.K, row_of(k));
        float E = 0.0f;
#pragma unroll 1
        for (int g = 0; g < NG; ++g) {
          float mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
          for (int c = g * GS; c < (g + 1) * GS; c += 8) {
            const uint4 kv = *reinterpret_cast<const uint4*>(krow + c);
            const uint4 mv = __ldg(mrow + c / 8);
            const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
            const uint32_t mu4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 m = __half22float2(*reinterpret_cast<const __half2*>(&mu4[q]));
              const float x0 = __fsub_rn(__uint_as_float(ku[q] << 16), m.x);
              const float x1 = __fsub_rn(__uint_as_float(ku[q] & 0xffff0000u), m.y);
              mn = fmin3(mn, x0, x1);
              mx = fmax3(mx, x0, x1);
            }
          }
          const GroupParams p = group_params(mn, mx);
          E = __fmaf_rn(__fmul_rn(a.Wg[size_t(h) * NG + g], p.s), p.s, E);
        }
        atomicMin(&best_w[k], (static_cast<unsigned long long>(float_order(E)) << 32) | unsigned(j));
      }
      __syncwarp();
    }

    if (a.assign) {
      for (int k = lane; k < nk; k += 32) {
        a.assign[size_t(row_of(k)) * a.H + h] = (C > 1) ? int(best_w[k] & 0xffffffffu) : cand_w[k * C];
      }
    } else {
    // ---- K residual and V codecs per (key, group); a group larger than 32
    // channels takes its range over all its sub-groups first, then codes
    // them one sub-group at a time (residuals recomputed)
    for (int task = lane; task < nk * NG * 2; task += 32) {
      const int which = task / (nk * NG);   // 0: keys, 1: values
      const int kg = task - which * nk * NG;
      const int k = kg / NG, g = kg - k * NG;
      const int row = row_of(k);
      const size_t slot = slot_of(row);
      int j = 0;
      if (which == 0) j = (C > 1) ? int(best_w[k] & 0xffffffffu) : cand_w[k * C];
      const uint4* mrow = reinterpret_cast<const uint4*>(cent + size_t(j) * D);   // as in the estimate
      // the 32 residuals (keys) or values (which = 1) of channels c0 .. c0 + 31
      auto load32 = [&](int c0, float (&x)[kGroup]) {
        if (which == 0) {
          const uint16_t* krow = key_ptr(a.K, row) + c0;
#pragma unroll
          for (int c = 0; c < kGroup; c += 8) {
            const uint4 kv = *reinterpret_cast<const uint4*>(krow + c);
            const uint4 mv = __ldg(mrow + (c0 + c) / 8);
            const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
            const uint32_t mu4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 m = __half22float2(*reinterpret_cast<const __half2*>(&mu4[q]));
              x[c + 2 * q] = __fsub_rn(__uint_as_float(ku[q] << 16), m.x);
              x[c + 2 * q + 1] = __fsub_rn(__uint_as_float(ku[q] & 0xffff0000u), m.y);
            }
          }
        } else {
          const uint16_t* vrow = key_ptr(a.V, row) + c0;
#pragma unroll
          for (int c = 0; c < kGroup; c += 8) {
            const uint4 vv = *reinterpret_cast<const uint4*>(vrow + c);
            const uint32_t vu[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              x[c + 2 * q] = __uint_as_float(vu[q] << 16);
              x[c + 2 * q + 1] = __uint_as_float(vu[q] & 0xffff0000u);
            }
          }
        }
      };
      float x[kGroup];
      load32(g * GS, x);
      float mn = x[0], mx = x[0];
#pragma unroll
      for (int c = 1; c + 1 < kGroup; c += 2) { mn = fmin3(mn, x[c], x[c + 1]); mx = fmax3(mx, x[c], x[c + 1]); }
      mn = fminf(mn, x[kGroup - 1]);
      mx = fmaxf(mx, x[kGroup - 1]);
#pragma unroll 1
      for (int u = 1; u < SPG; ++u) {
        float y[kGroup];
        load32(g * GS + u * kGroup, y);
#pragma unroll
        for (int c = 0; c + 1 < kGroup; c += 2) { mn = fmin3(mn, y[c], y[c + 1]); mx = fmax3(mx, y[c], y[c + 1]); }
      }
      const GroupParams p = group_params(mn, mx);
      const float inv_s = __frcp_rn(p.s);
#pragma unroll 1
      for (int u = 0; u < SPG; ++u) {
        if (u > 0) load32(g * GS + u * kGroup, x);
        const int c0 = g * GS + u * kGroup;
        uint32_t w0 = 0, w1 = 0;
#pragma unroll
        for (int c = 0; c < kGroup; ++c) {
          const uint32_t q = group_code_recip(x[c], p, inv_s);
          if (c < 16) w0 |= q << (2 * c); else w1 |= q << (2 * (c - 16));
          if (which == 0) e_w[k * D + c0 + c] = __fsub_rn(x[c], group_dequant(q, p));
        }
        uint32_t* code = (which == 0 ? a.k_code : a.v_code) + slot * (D / 16) + c0 / 16;
        *reinterpret_cast<uint2*>(code) = make_uint2(w0, w1);
      }
      (which == 0 ? a.k_sz : a.v_sz)[slot * NG + g] = uint32_t(p.s_bits) | (uint32_t(p.z_bits) << 16);
      if (which == 0 && g == 0) {
        if (M <= 256) static_cast<uint8_t*>(a.cidx)[slot] = uint8_t(j);
        else static_cast<uint16_t*>(a.cidx)[slot] = uint16_t(j);
      }
    }
    __syncwarp();

    // ---- PSAC coefficients a_i = sum_c P_ci e_c (ascending c)
    for (int task = lane; task < nk * a.r; task += 32) {
      const int k = task / a.r, i = task - k * a.r;
      const float* Pcol = P_s + i;
      const float* e = e_w + k * D;
      float acc = 0.0f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = __fmaf_rn(Pcol[c * a.r], e[c], acc);
      if (r8) psa_w[k * a.r + i] = acc;
      else a.psac[slot_of(row_of(k)) * a.r + i] = f16_rn(acc);
    }
    if (r8) {
      __syncwarp();
      for (int k = lane; k < nk; k += 32) {
        const size_t slot = slot_of(row_of(k));
        psac_int8(psa_w + k * a.r, a.r, reinterpret_cast<int8_t*>(a.psac) + slot * a.r, a.psac_scale + slot);
      }
    }
    }
    }
    __syncwarp();    // e_w / wk_w and cand_w are reused by this warp's next tile
  }
}

template <int D, int CPL, int KPT, int GS>
cudaError_t launch_cfg(const QuantizeArgs& a, cudaStream_t s) {
  using Cfg = QCfg<D, CPL, KPT>;
  const size_t smem = Cfg::smem(a.C, a.r, a.psac_fmt == 1 ? a.r : 0);
  auto kern = quantize_kernel<D, CPL, KPT, GS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  // the SM's shared-memory split as large as the attention kernels': an SM
  // changes its split only when idle, so with a smaller one the attention
  // CTAs launched beside this kernel (as its programmatic dependents) could
  // not start on its SMs until it exits
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows = a.B * a.n_new;
  const int ntiles = (rows + Cfg::KT - 1) / Cfg::KT;
  int per_head = (sms * per_sm) / a.H;          // persistent CTAs per head: one wave in total
  per_head = per_head < 1 ? 1 : (per_head > ntiles ? ntiles : per_head);
  dim3 grid(per_head, a.H);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D, int GS>
cudaError_t launch_d(const QuantizeArgs& a, cudaStream_t s) {
  const int mp = (a.M + 31) / 32;
  if (a.B * a.n_new <= 8 * kWarps) {            // short appends: one key per warp and tile
    if (mp <= 1) return launch_cfg<D, 1, 1, GS>(a, s);
    if (mp <= 2) return launch_cfg<D, 2, 1, GS>(a, s);
    if (mp <= 4) return launch_cfg<D, 4, 1, GS>(a, s);
    if (mp <= 8) return launch_cfg<D, 8, 1, GS>(a, s);
    return launch_cfg<D, 16, 1, GS>(a, s);
  }
  if (mp <= 1) return launch_cfg<D, 1, 16, GS>(a, s);
  if (mp <= 2) return launch_cfg<D, 2, 16, GS>(a, s);
  if (mp <= 4) return launch_cfg<D, 4, 16, GS>(a, s);
  if (mp <= 8) return launch_cfg<D, 8, 8, GS>(a, s);
  return launch_cfg<D, 16, 4, GS>(a, s);
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t s) {
  if (a.B * a.n_new == 0) return cudaSuccess;
  if (a.d == 64) {
    switch (a.group) {
      case 32: return launch_d<64, 32>(a, s);
      case 64: return launch_d<64, 64>(a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (a.group) {
    case 32: return launch_d<128, 32>(a, s);
    case 64: return launch_d<128, 64>(a, s);
    case 128: return launch_d<128, 128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kv2
