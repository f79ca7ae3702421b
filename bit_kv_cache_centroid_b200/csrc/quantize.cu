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
// Structure: one wave of persistent CTAs, each taking an equal run of the
// head-major list of key tiles (8*KPT keys of one head) and staging a head's
// centroid table (fp16 rows [M][d], the 16-byte chunks of row j permuted by
// chunk ^ (j % 8) so that eight rows read at one logical chunk hit eight
// different bank groups) and norms when its run enters that head. Within a
// tile every warp runs its own KPT keys through the whole pipeline with warp
// synchronization only: w*k staging, the ranking products, top-C (lane l
// owns centres l, l+32, ...; each lane's scores become packed keys, the order
// with the centre id in its low bits, sorted per key; C rounds of one
// warp-wide integer minimum), the perturbation estimates, the K-residual
// codec and the PSAC coefficients. Warps with one key also code the values;
// the values of multi-key appends are coded by value_codec_kernel.
//
// Ranking in two steps. The M*d products (the dominant cost) run in the
// expanded form f_j = nrm_j - 2 dot_j, nrm_j = sum_c (w_c mu_jc) mu_jc,
// dot_j = sum_c (w_c k_c) mu_jc, which equals D_j - sum_c w_c k_c^2 in exact
// arithmetic. With Ka = sum_c |w_c| k_c^2 and Na = max_j sum_c |w_c| mu_jc^2,
// standard error bounds of fp32 fma chains give |f_j - (D_j - K)| <=
// g (Na + 2 sqrt(Ka Na)) (Cauchy-Schwarz bounds S = sum_c |w_c k_c mu_jc| by
// sqrt(Ka Na)) and |fp32 D_j - D_j| <= g (sqrt(Ka) + sqrt(Na))^2,
// g = gamma_{d+3} = (d+3) 2^-24 / (1 - (d+3) 2^-24). So every centre of the
// exact C smallest has f_j <= c + 2b, where c is the C-th smallest f and
// b = g (Ka + 2 Na + 4 sqrt(Ka Na)) + 2 e_dot (e_dot: the dot products' own
// error beyond an fp32 chain, below). The packed keys bound each true score
// from both sides, so any C centres S taken by them work: when no centre
// outside S lies under max_S f + 2b, S is the exact set (nearly always).
// Otherwise, with several keys per warp and 1 < C < 15, the key is listed:
// S and the centres under that threshold, a taken centre i marked sure when
// f_i < min_{j not in S} f_j - 2b (then D_i is below every D_j outside S).
// The perturbation E of every listed centre is estimated; the least (E, id)
// among the sure ones is the choice when it beats every doubtful one,
// whichever doubtful centres are in the exact set; otherwise (and with one
// key per warp, C = 1, C >= 15 or a longer list) the listed centres get their
// fp32 D_j by the definition and the C smallest (D_j, j) decide the set. The
// bounds are computed with g doubled and upward rounding, so they only ever
// err towards the exact path.
//
// Warps with several keys (KPT > 1) take the dot products on the tensor cores
// (mma.sync m16n8k16, fp16 operands, fp32 accumulation): A = 16 centres x 16
// channels of the exact fp16 table, B = the key's x_c = fp32(w_c k_c) times a
// power of two 2^e (max |x_c| 2^e in [2^14, 2^15)) split into hi = fp16(x 2^e)
// and lo = fp16(x 2^e - hi), both accumulated into the same fp32 sums, which
// are scaled back by 2^-e exactly. The split leaves |x 2^e - hi - lo| <=
// 2^-22 |x 2^e| + 2^-25 per channel; the products are exact in fp32; for the
// accumulation the bound takes kappa = 2^-12 of sum |hi mu| + |lo mu| over
// the whole chain of 2d/16 MMAs. That kappa is an assumption about the
// hardware, not a documented guarantee: a model of tensor-core addition that
// aligns each k16 block's products to the largest and truncates ("Numerical
// behavior of NVIDIA tensor cores", Fasi, Higham, Mikaitis and Pranesh, PeerJ
// Computer Science, 2021) bounds a chain of 16 such blocks by about 2^-13.8 S,
// and the largest error measured on this path's hardware (2^-19.1 of S,
// tests/test_gpu_tc_accumulation.py) is far below both.
// So e_dot = (2^-12 + 2^-18) sqrt(Ka Na) + 2^-24 2^-e sum_c |mu_jc|. A warp
// with one key (short appends) runs the products as fp32 FMAs (e_dot = 0).
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
  // w*k: fp32 [D] (KPT = 1) or the fp16 hi and lo halves [2][KPT][D] of the
  // scaled products (KPT > 1); then the lists and key rows of the decisions;
  // last the K residual errors e, [KPT] rows of ES = D + D/32 floats (one
  // spare word per 32 channels, so that the lanes coding different (key,
  // group) pairs hit different banks)
  static constexpr int ES = D + D / 32;
  static constexpr size_t warp_wk_bytes = size_t(ES) * KPT * 4;
  // tensor-core ranking: m16 tiles of centres, n8 tiles of keys, tiles kept
  // in registers at a time (64 accumulators), and the per-slice transpose
  // buffer [32 centres][TBS] (a row stride that keeps the lanes' 16-byte
  // reads on distinct bank groups), placed over the w*k halves when one pass
  // covers every centre
  static constexpr int MT = MP / 16, NT = (KPT + 7) / 8;
  static constexpr int MTP = (MT * NT > 16) ? 16 / NT : MT;
  static constexpr int PASSES = MT / MTP;
  static constexpr int TBS = KPT == 4 ? 4 : KPT + 4;
  static constexpr size_t tb_extra = (KPT > 1 && PASSES > 1) ? size_t(32) * TBS * 4 : 0;
  // per warp: w*k / e, best (E, centre id) per key, candidates, and (int8 PSAC
  // format only, r8 = r) the fp32 coefficients [KPT][r8] before quantization
  __host__ __device__ static size_t cand_end(int C) {
    return (warp_wk_bytes + tb_extra + size_t(KPT) * 8 + size_t(KPT) * C * 2 + 15) & ~size_t(15);
  }
  __host__ __device__ static size_t warp_bytes(int C, int r8) { return (cand_end(C) + size_t(KPT) * r8 * 4 + 15) & ~size_t(15); }
  __host__ __device__ static size_t head_bytes(int r) { return mu_bytes + size_t(MP) * 4 + size_t(D) * 4 + size_t(D) * r * 4; }
  static size_t smem(int C, int r, int r8) { return head_bytes(r) + size_t(kWarps) * warp_bytes(C, r8); }
  static_assert(KPT == 1 || (32 * TBS * 4 <= warp_wk_bytes || PASSES > 1), "transpose buffer fits");
  static_assert(MT % MTP == 0 && MTP % 2 == 0, "whole 32-centre slices per pass");
};

// element (j, c) of the staged centre table: row j, 16-byte chunk c/8 stored
// at position (c/8) ^ (j%8)
template <int D>
__device__ __forceinline__ int mu_index(int j, int c8) { return j * D + ((c8 ^ (j & 7)) << 3); }

// Half-width b of the fast scores' uncertainty, |f_j - (D_j - K)| <= b with
// the fp32 distance's own error folded in (derived in the file comment, with
// gamma_{d+3} doubled and every operation rounded up). A centre of the exact
// C smallest has f_j <= c + 2b (c: the C-th smallest fast score).
__device__ __forceinline__ float rank_bound(float ka, float na, int d) {
  const float g = float(2 * (d + 8)) * 0x1p-24f;
  const float cross = __fmul_ru(4.0f, __fsqrt_ru(__fmul_ru(ka, na)));
  return __fmul_ru(g, __fadd_ru(__fadd_ru(ka, __fmul_ru(2.0f, na)), cross));
}

// The same half-width with the tensor-core products' term 2 e_dot added
// (tc_abs = 2^-24 2^-e sum_c |mu_jc| for the key's scale exponent e).
__device__ __forceinline__ float rank_bound_tc(float ka, float na, float tc_abs, int d) {
  const float root = __fsqrt_ru(__fmul_ru(ka, na));
  return __fadd_ru(rank_bound(ka, na, d), __fmul_ru(2.0f, __fadd_ru(__fmul_ru(0x1p-12f + 0x1p-18f, root), tc_abs)));
}

// E_j = sum_g W_g s_g^2 of the key in row kr of `rows` and centre j (fp32,
// ascending g; s_g the group scale of the residual k - mu_j), both rows read
// from the staged shared-memory copies
template <int D, int GS>
__device__ __forceinline__ float perturbation(const uint16_t* rows, int kr, const __half* mu_s, int j,
                                             const float* Wg) {
  float E = 0.0f;
#pragma unroll 1
  for (int g = 0; g < D / GS; ++g) {
    float mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
    for (int c = g * GS; c < (g + 1) * GS; c += 8) {
      const uint4 kv = *reinterpret_cast<const uint4*>(rows + mu_index<D>(kr, c / 8));
      const uint4 mv = *reinterpret_cast<const uint4*>(mu_s + mu_index<D>(j, c / 8));
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
    E = __fmaf_rn(__fmul_rn(Wg[g], p.s), p.s, E);
  }
  return E;
}

// ascending bitonic sorting network over N (a power of two) registers
template <int N>
__device__ __forceinline__ void sort_asc(uint32_t (&v)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1)
#pragma unroll
    for (int stride = size / 2; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const uint32_t lo = min(v[i], v[j]), hi = max(v[i], v[j]);
          const bool up = (i & size) == 0;
          v[i] = up ? lo : hi;
          v[j] = up ? hi : lo;
        }
      }
}

// perturbation() of two (key row, centre) pairs with their chains interleaved
template <int D, int GS>
__device__ __forceinline__ void perturbation2(const uint16_t* rows, const int (&kr)[2], const int (&j)[2],
                                              const __half* mu_s, const float* Wg, float (&E)[2]) {
  E[0] = E[1] = 0.0f;
#pragma unroll 1
  for (int g = 0; g < D / GS; ++g) {
    float mn[2] = {FLT_MAX, FLT_MAX}, mx[2] = {-FLT_MAX, -FLT_MAX};
#pragma unroll
    for (int c = g * GS; c < (g + 1) * GS; c += 8) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint4 kv = *reinterpret_cast<const uint4*>(rows + mu_index<D>(kr[u], c / 8));
        const uint4 mv = *reinterpret_cast<const uint4*>(mu_s + mu_index<D>(j[u], c / 8));
        const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
        const uint32_t mu4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 m = __half22float2(*reinterpret_cast<const __half2*>(&mu4[q]));
          const float2 xx = up2(fsub2(pk2(__uint_as_float(ku[q] << 16), __uint_as_float(ku[q] & 0xffff0000u)),
                                      pk2(m.x, m.y)));
          mn[u] = fmin3(mn[u], xx.x, xx.y);
          mx[u] = fmax3(mx[u], xx.x, xx.y);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const GroupParams p = group_params(mn[u], mx[u]);
      E[u] = __fmaf_rn(__fmul_rn(Wg[g], p.s), p.s, E[u]);
    }
  }
}

// Codes of the 32 values x of one sub-group with the group's (s, z): the
// quotient (x - z) * inv_s rounded to the nearest integer and clamped to
// 0..3, two channels per packed instruction (each lane rounded as its scalar
// form); bit c of `redo` flags a quotient within 2^-18 of a half-integer
// (|q - rint(q)| > 1/2 - 2^-18), whose code the correctly rounded division
// must decide. With E, also the residual errors x - (code * s + z). A group
// of scale 0 holds x = z only (z is the rounded-down minimum and s the
// rounded-up range / 3): its codes are 0 and its errors x - z whatever the
// quotient gave.
template <bool E>
__device__ __forceinline__ void code32(const float (&x)[kGroup], const GroupParams& gp, float inv_s,
                                       uint32_t& w0, uint32_t& w1, uint32_t& redo, float (&ev)[kGroup]) {
  const f32x2 z2 = pk2(gp.z, gp.z), is2 = pk2(inv_s, inv_s), s2 = pk2(gp.s, gp.s);
  w0 = w1 = redo = 0;
#pragma unroll
  for (int c = 0; c < kGroup; c += 2) {
    const float2 qa = up2(fmul2(fsub2(pk2(x[c], x[c + 1]), z2), is2));
    const float r0 = rintf(qa.x), r1 = rintf(qa.y);
    redo |= (uint32_t(fabsf(__fsub_rn(qa.x, r0)) > 0.5f - 0x1p-18f) << c) |
            (uint32_t(fabsf(__fsub_rn(qa.y, r1)) > 0.5f - 0x1p-18f) << (c + 1));
    const float c0 = fminf(fmaxf(r0, 0.0f), 3.0f), c1 = fminf(fmaxf(r1, 0.0f), 3.0f);
    const uint32_t q = uint32_t(c0) | (uint32_t(c1) << 2);
    if (c < 16) w0 |= q << (2 * c); else w1 |= q << (2 * (c - 16));
    if constexpr (E) {
      const float2 e = up2(fsub2(pk2(x[c], x[c + 1]), ffma2(pk2(c0, c1), s2, z2)));
      ev[c] = e.x;
      ev[c + 1] = e.y;
    }
  }
  if (gp.s == 0.0f) w0 = w1 = redo = 0;
}

// warp-wide minimum of 64-bit keys (every lane gets it)
__device__ __forceinline__ unsigned long long warp_min64(unsigned long long v) {
  const uint32_t hi = __reduce_min_sync(0xffffffffu, uint32_t(v >> 32));
  const uint32_t lo = __reduce_min_sync(0xffffffffu, uint32_t(v >> 32) == hi ? uint32_t(v) : 0xFFFFFFFFu);
  return (static_cast<unsigned long long>(hi) << 32) | lo;
}

constexpr int kListLen = 15;   // listed centres per key in the decision by perturbations (slot 15: count and limit)

// D_j = sum_c w_c (k_c - mu_jc)^2 by the definition's fp32 order; the key:
// row kr of `rows` (bf16, chunks permuted like the centre table), mu_s: the
// staged table.
template <int D>
__device__ __forceinline__ float exact_distance(const uint16_t* rows, int kr, const __half* mu_s, int j,
                                               const float* w_s) {
  float acc = 0.0f;
#pragma unroll 2
  for (int c8 = 0; c8 < D / 8; ++c8) {
    const uint4 kv = *reinterpret_cast<const uint4*>(rows + mu_index<D>(kr, c8));
    const uint4 mv = *reinterpret_cast<const uint4*>(mu_s + mu_index<D>(j, c8));
    const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
    const uint32_t mu4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = c8 * 8 + q;
      const float kc = __uint_as_float((q & 1) ? (ku[q / 2] & 0xffff0000u) : (ku[q / 2] << 16));
      const float m = __half2float(__ushort_as_half(uint16_t((q & 1) ? (mu4[q / 2] >> 16) : (mu4[q / 2] & 0xffffu))));
      const float t = __fsub_rn(kc, m);
      acc = __fmaf_rn(__fmul_rn(w_s[c], t), t, acc);
    }
  }
  return acc;
}

// d += A B, m16n8k16, fp16 operands, fp32 accumulators
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// four 8x8 fp16 tiles; lane i gives the address of row i % 8 of tile i / 8
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* row) {
  const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(row));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(sa));
}
// scale exponent e of a key's products: max |x| 2^e in [2^14, 2^15) for
// normal max |x|, limited to [-126, 126] so that 2^e, 2^-e and 2^(1-e) are
// normal floats (0 for a zero or subnormal maximum)
__device__ __forceinline__ int tc_exponent(float maxabs) {
  const int E = int((__float_as_uint(maxabs) >> 23) & 0xffu) - 127;
  const int e = (E > -127) ? 14 - E : 0;
  return max(-126, min(126, e));
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// GS: channels per (scale, zero) group (32, 64 or 128); a group is SPG
// sub-groups of 32 channels (one code-word pair each)
template <int D, int CPL, int KPT, int GS>
__global__ void __launch_bounds__(kThreads, CPL >= 16 ? 1 : 2) quantize_kernel(QuantizeArgs a) {
  using Cfg = QCfg<D, CPL, KPT>;
  constexpr int MP = Cfg::MP, KT = Cfg::KT;
  constexpr int NG = D / GS, NS = D / kGroup, SPG = GS / kGroup;
  static_assert(GS % kGroup == 0 && D % GS == 0, "groups of whole 32-channel sub-groups");
  static_assert(D * KPT >= 32 * KPT + D / 2, "the w*k buffer holds the exact pass's lists and one key row");
  extern __shared__ __align__(16) unsigned char smem[];
  __half* mu_s = reinterpret_cast<__half*>(smem);                            // [MP][D], chunks permuted
  float* nrm_s = reinterpret_cast<float*>(smem + Cfg::mu_bytes);              // [MP]
  float* w_s = nrm_s + MP;                                                    // [D]
  float* P_s = w_s + D;                                                       // [D][r]
  __shared__ uint32_t na_bits;     // Na = max_j sum_c |w_c| mu_jc^2 (non-negative: ordered as its bits)
  __shared__ uint32_t mabs_bits;   // max_j sum_c |mu_jc|
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r8 = (a.psac_fmt == 1) ? a.r : 0;
  unsigned char* wbase = smem + Cfg::head_bytes(a.r) + size_t(warp) * Cfg::warp_bytes(a.C, r8);
  float* wk_w = reinterpret_cast<float*>(wbase);                              // w*k (see QCfg)
  float* e_w = wk_w;                                                          // [KPT][ES] after the decisions
  unsigned long long* best_w = reinterpret_cast<unsigned long long*>(wbase + Cfg::warp_wk_bytes + Cfg::tb_extra);  // [KPT]
  uint16_t* cand_w = reinterpret_cast<uint16_t*>(best_w + KPT);              // [KPT][C]
  float* psa_w = reinterpret_cast<float*>(wbase + Cfg::cand_end(a.C));         // [KPT][r8]

  // a decode launched as this kernel's programmatic dependent may start now;
  // it waits for this grid before reading the slots written here
  asm volatile("griddepcontrol.launch_dependents;");
  // work: the tiles of every head in one list (head-major); CTA b takes the
  // b-th of gridDim.x equal runs, so every resident CTA has the same number
  // of tiles, and stages a head's tables when its run enters that head
  const int rows_total = a.B * a.n_new;
  const int ntiles = (rows_total + KT - 1) / KT;       // per head
  const long long nwork = static_cast<long long>(ntiles) * a.H;
  const long long lo = nwork * blockIdx.x / gridDim.x, hi = nwork * (blockIdx.x + 1) / gridDim.x;
  const int M = a.M, C = a.C;
  int h = -1;
  const __half* cent = nullptr;
  float na = 0.0f, mabs = 0.0f;

  auto key_ptr = [&](const uint16_t* base, int row) {
    const int b = row / a.n_new, t = row - b * a.n_new;
    return base + ((size_t(b) * a.n_new + t) * a.H + h) * D;
  };
  auto slot_of = [&](int row) {
    const int b = row / a.n_new, t = row - b * a.n_new;
    return cache_slot(a.table, a.page, a.H, a.cap, b, h, a.pos + t);
  };

  for (long long wi = lo; wi < hi; ++wi) {
    const int tile = int(wi % ntiles);
    if (int(wi / ntiles) != h) {
      // ---- once per head in the run: centroid table (fp16 rows, chunks
      // permuted; zero rows past M), w, the PSAC basis, norms
      h = int(wi / ntiles);
      cent = reinterpret_cast<const __half*>(a.cent) + size_t(h) * M * D;
      __syncthreads();                                // the previous head's tables are no longer read
      if (tid == 0) na_bits = mabs_bits = 0;
      for (int i = tid; i < D; i += kThreads) w_s[i] = a.w[size_t(h) * D + i];
      for (int i = tid; i < D * a.r; i += kThreads) P_s[i] = a.P[size_t(h) * D * a.r + i];
      for (int idx = tid; idx < MP * (D / 8); idx += kThreads) {
        const int j = idx / (D / 8), c8 = idx % (D / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (j < M) v = *reinterpret_cast<const uint4*>(cent + size_t(j) * D + c8 * 8);
        *reinterpret_cast<uint4*>(mu_s + mu_index<D>(j, c8)) = v;
      }
      __syncthreads();
      for (int j = tid; j < MP; j += kThreads) {
        float acc = 0.0f, aabs = 0.0f, asum = 0.0f;
        if (j < M) {
#pragma unroll 2
          for (int c8 = 0; c8 < D / 8; ++c8) {
            const uint4 mv = *reinterpret_cast<const uint4*>(mu_s + mu_index<D>(j, c8));
            const __half* hv = reinterpret_cast<const __half*>(&mv);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float m = __half2float(hv[q]);
              const float wm = __fmul_rn(w_s[c8 * 8 + q], m);
              acc = __fmaf_rn(wm, m, acc);
              aabs = __fmaf_rn(fabsf(wm), fabsf(m), aabs);
              asum = __fadd_ru(asum, fabsf(m));
            }
          }
        }
        nrm_s[j] = acc;
        atomicMax(&na_bits, __float_as_uint(aabs));
        atomicMax(&mabs_bits, __float_as_uint(asum));
      }
      __syncthreads();
      na = __uint_as_float(na_bits);
      mabs = __uint_as_float(mabs_bits);
    }

    // key k of this warp is row tile*KT + k*kWarps + warp, so that a short
    // append spreads over all warps
    const int rem = rows_total - tile * KT - warp;
    const int nk = rem > 0 ? min(KPT, (rem + kWarps - 1) / kWarps) : 0;
    if (nk <= 0) continue;                       // warp-uniform
    auto row_of = [&](int k) { return tile * KT + k * kWarps + warp; };

    // ---- w*k for this warp's keys; lane l handles key l % KPT only (32 is a
    // multiple of KPT) and sums its share of Ka = sum_c |w_c| k_c^2 for the
    // ranking bound. KPT = 1: fp32 [D]. KPT > 1: the products' maximum sets
    // the key's scale 2^e, then the fp16 hi / lo halves of x 2^e go to rows of
    // [KPT][D] (chunks permuted like the centre table).
    float ka = 0.0f;
    uint32_t ord[KPT][CPL];
    float two_b_l;                                   // 2b of key lane % KPT (rounded up)
    if constexpr (KPT == 1) {
      for (int c8 = lane; c8 < D / 8; c8 += 32) {
        const uint4 v = *reinterpret_cast<const uint4*>(key_ptr(a.K, row_of(0)) + c8 * 8);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float f = __uint_as_float((i & 1) ? (u[i / 2] & 0xffff0000u) : (u[i / 2] << 16));
          const float wk = __fmul_rn(w_s[c8 * 8 + i], f);
          wk_w[c8 * 8 + i] = wk;
          ka = __fmaf_rn(fabsf(wk), fabsf(f), ka);
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) ka += __shfl_xor_sync(0xffffffffu, ka, o);
      two_b_l = __fmul_ru(2.0f, rank_bound(ka, na, D));
      if (lane == 0) best_w[0] = ~0ull;
      __syncwarp();
      // ranking scores: lane l, centres l + 32 j, fp32 FMAs over ascending c
      float acc[CPL];
#pragma unroll
      for (int j = 0; j < CPL; ++j) acc[j] = 0.0f;
#pragma unroll 2
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const float4 w0 = *reinterpret_cast<const float4*>(wk_w + c8 * 8);
        const float4 w1 = *reinterpret_cast<const float4*>(wk_w + c8 * 8 + 4);
        const float wk[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          const uint4 mv = *reinterpret_cast<const uint4*>(mu_s + mu_index<D>(j * 32 + lane, c8));
          const __half2* h2 = reinterpret_cast<const __half2*>(&mv);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 m = __half22float2(h2[i]);
            acc[j] = __fmaf_rn(wk[2 * i], m.x, acc[j]);
            acc[j] = __fmaf_rn(wk[2 * i + 1], m.y, acc[j]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int cj = j * 32 + lane;
        ord[0][j] = (cj < M) ? float_order(__fadd_rn(__fmaf_rn(-2.0f, acc[j], nrm_s[cj]), 0.0f)) : 0xFFFFFFFFu;
      }
    } else {
      using Cfg2 = QCfg<D, CPL, KPT>;
      constexpr int NT = Cfg2::NT, MTP = Cfg2::MTP, TBS = Cfg2::TBS;
      constexpr int NI = KPT * (D / 8) / 32;        // 8-channel chunks per lane
      __half* hi_w = reinterpret_cast<__half*>(wk_w);   // [KPT][D]
      __half* lo_w = hi_w + KPT * D;                    // [KPT][D]
      const int kk = lane % KPT;
      float x[NI][8];
      float mx = 0.0f;
#pragma unroll
      for (int it = 0; it < NI; ++it) {
        const int c8 = lane / KPT + it * (32 / KPT);
        float f[8];
        if (kk < nk) {
          const uint4 v = *reinterpret_cast<const uint4*>(key_ptr(a.K, row_of(kk)) + c8 * 8);
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
          x[it][i] = __fmul_rn(w_s[c8 * 8 + i], f[i]);
          ka = __fmaf_rn(fabsf(x[it][i]), fabsf(f[i]), ka);
          mx = fmaxf(mx, fabsf(x[it][i]));
        }
      }
#pragma unroll
      for (int o = 16; o >= KPT; o >>= 1) {
        ka += __shfl_xor_sync(0xffffffffu, ka, o);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      const int e = tc_exponent(mx);
      const float sigma = pow2f(e);
#pragma unroll
      for (int it = 0; it < NI; ++it) {
        const int c8 = lane / KPT + it * (32 / KPT);
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float y0 = __fmul_rn(x[it][2 * i], sigma), y1 = __fmul_rn(x[it][2 * i + 1], sigma);
          const __half h0 = __float2half_rn(y0), h1 = __float2half_rn(y1);
          const __half l0 = __float2half_rn(__fsub_rn(y0, __half2float(h0)));
          const __half l1 = __float2half_rn(__fsub_rn(y1, __half2float(h1)));
          hw[i] = uint32_t(__half_as_ushort(h0)) | (uint32_t(__half_as_ushort(h1)) << 16);
          lw[i] = uint32_t(__half_as_ushort(l0)) | (uint32_t(__half_as_ushort(l1)) << 16);
        }
        *reinterpret_cast<uint4*>(hi_w + mu_index<D>(kk, c8)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(lo_w + mu_index<D>(kk, c8)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      // per key (held by lane k): -2^(1-e) scales the MMA sums back into f_j,
      // tc_abs is the split's absolute term of the bound
      const float back = -pow2f(1 - e);
      const float tc_abs = __fmul_ru(__fmul_ru(mabs, 0x1p-24f), pow2f(-e));
      two_b_l = __fmul_ru(2.0f, rank_bound_tc(ka, na, tc_abs, D));
      if (lane < KPT) best_w[lane] = ~0ull;
      __syncwarp();

      // ranking scores on the tensor cores: D[centre][key] in m16n8 tiles,
      // then each 32-centre slice through the transpose buffer into ord
      const int g = lane >> 2, t = lane & 3;
      float bk[NT][2];                                  // back of the keys in this lane's D columns
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2) bk[nt][s2] = __shfl_sync(0xffffffffu, back, (nt * 8 + 2 * t + s2) % KPT);
      uint32_t* tb = (Cfg2::PASSES > 1) ? reinterpret_cast<uint32_t*>(wbase + Cfg2::warp_wk_bytes)
                                        : reinterpret_cast<uint32_t*>(wk_w);     // [32][TBS]
#pragma unroll
      for (int pass = 0; pass < Cfg2::PASSES; ++pass) {
        float acc[MTP][NT][4];
#pragma unroll
        for (int mt = 0; mt < MTP; ++mt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;
#pragma unroll 1
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t b[NT][4];                            // hi b0, hi b1, lo b0, lo b1
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int key = (nt * 8 + (lane & 7)) % KPT, m = lane >> 3;
            ldsm_x4(b[nt], ((m >> 1) ? lo_w : hi_w) + mu_index<D>(key, 2 * ks + (m & 1)));
          }
#pragma unroll
          for (int mt = 0; mt < MTP; ++mt) {
            const int row = (pass * MTP + mt) * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            uint32_t af[4];
            ldsm_x4(af, mu_s + mu_index<D>(row, 2 * ks + (lane >> 4)));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_f16(acc[mt][nt], af, b[nt][0], b[nt][1]);
              mma_f16(acc[mt][nt], af, b[nt][2], b[nt][3]);
            }
          }
        }
        __syncwarp();                                   // the halves are read (tb may lie over them)
#pragma unroll
        for (int sl = 0; sl < MTP / 2; ++sl) {
          const int q = pass * (MTP / 2) + sl;          // ord column: centres 32 q + lane
#pragma unroll
          for (int mh = 0; mh < 2; ++mh)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int key = nt * 8 + 2 * t + (i & 1), cl = mh * 16 + g + 8 * (i >> 1), cj = q * 32 + cl;
                if (key < KPT)
                  tb[cl * TBS + key] = (cj < M) ? float_order(__fmaf_rn(bk[nt][i & 1], acc[2 * sl + mh][nt][i], nrm_s[cj]))
                                                : 0xFFFFFFFFu;
              }
          __syncwarp();
#pragma unroll
          for (int k = 0; k < KPT; k += 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(tb + lane * TBS + k);
            ord[k][q] = v.x; ord[k + 1][q] = v.y; ord[k + 2][q] = v.z; ord[k + 3][q] = v.w;
          }
          __syncwarp();
        }
      }
      // the key rows for the decisions (after the lists), now that the
      // transpose buffer is free
      uint16_t* rows = reinterpret_cast<uint16_t*>(reinterpret_cast<unsigned char*>(wk_w) + KPT * 128);
      for (int idx = lane; idx < KPT * (D / 8); idx += 32) {
        const int k = idx / (D / 8), c8 = idx % (D / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (k < nk) v = *reinterpret_cast<const uint4*>(key_ptr(a.K, row_of(k)) + c8 * 8);
        *reinterpret_cast<uint4*>(rows + mu_index<D>(k, c8)) = v;
      }
    }

    // ---- top-C per key: C rounds of a warp-wide min over the lanes' sorted
    // lists of packed scores; then the check that no other centre's fast
    // score lies within the ranking bound of the C-th. A key that fails it
    // has its centres under the threshold listed in this warp's w*k buffer
    // (free once the ranking products are done) and is decided after the
    // perturbations. With several keys per warp and 1 < C < 15 the list
    // holds (score, id) of the C taken and of the others under the
    // threshold, and slot 15 the entry count and the limit below which a
    // taken centre is surely in the exact set (f_i < f_(C+1) - 2b: every
    // centre outside the taken set has D_j > D_i); the choice is then made on
    // perturbations and needs exact distances only when a centre in doubt
    // could win it. Otherwise (or with more listed centres than fit) the
    // list holds ids, 32 per key, and the exact distances decide the
    // candidate set.
    int* lists = reinterpret_cast<int*>(wk_w);               // [KPT][32] ids
    unsigned long long* lists64 = reinterpret_cast<unsigned long long*>(wk_w);   // [KPT][16] (score, id)
    // after the lists: the key rows (bf16 [KPT][D], chunks permuted like the
    // centre table; KPT * 128 + 2 * KPT * D bytes fit in 4 * KPT * D for
    // D >= 64), stored by the ranking above and read by the perturbations,
    // the codec and the exact distances; one key per warp stages its row
    // there only when its exact pass needs it
    uint16_t* rows_w = reinterpret_cast<uint16_t*>(reinterpret_cast<unsigned char*>(wk_w) + KPT * 128);
    const bool list_mode = KPT > 1 && C > 1 && C < kListLen;
    // a lane's scores as packed keys: the order with its low bits replaced by
    // the centre id j * 32 + lane (so every key is unique and carries its
    // centre), sorted ascending per key
    constexpr uint32_t JM = CPL * 32 - 1;
    uint32_t exact_keys = 0, long_lists = 0, listed = 0;     // bit k: key k's route
    uint32_t last[KPT];                                      // packed key of the C-th taken
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      last[k] = 0;
#pragma unroll
      for (int j = 0; j < CPL; ++j) ord[k][j] = (ord[k][j] & ~JM) | uint32_t(j * 32 + lane);
      sort_asc<CPL>(ord[k]);
    }
    // C rounds, the keys interleaved and without branches (so that the
    // reductions of different keys overlap): the least head over the lanes
    // is taken and its lane's list moves up
    for (int i = 0; i < C; ++i) {
#pragma unroll
      for (int k = 0; k < KPT; ++k) {
        const uint32_t head = ord[k][0];
        const uint32_t wmin = __reduce_min_sync(0xffffffffu, head);
        const bool up = head == wmin;
#pragma unroll
        for (int j = 0; j + 1 < CPL; ++j) ord[k][j] = up ? ord[k][j + 1] : ord[k][j];
        ord[k][CPL - 1] = up ? 0xFFFFFFFFu : ord[k][CPL - 1];
        const uint32_t id = wmin & JM;
        last[k] = wmin;
        const bool w0 = lane == 0 && k < nk;
        if (w0) cand_w[k * C + i] = uint16_t(id);
        if (w0 && list_mode) lists64[k * 16 + i] = (static_cast<unsigned long long>(wmin | JM) << 32) | id;
      }
    }
    __syncwarp();
    // The taken set S is C centres whose packed keys are least; a centre j
    // outside it with f_j > max_S f + 2b cannot be in the exact set, and one
    // in S with f_i < min_{j not in S} f_j - 2b surely is. The packed keys
    // bound the true orders from below (key & ~JM) and above (key | JM).
    uint32_t near_keys = 0;                                  // bit k: a centre outside S under the threshold
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      if (k >= nk) break;
      const uint32_t thr_o =
          float_order(__fadd_ru(order_float(last[k] | JM), __shfl_sync(0xffffffffu, two_b_l, k)));
      if (__any_sync(0xffffffffu, ord[k][0] <= thr_o)) near_keys |= 1u << k;   // the lists are sorted: heads decide
    }
    // the near keys one at a time (rare), from a copy of the key's lists, so
    // that this code is not repeated per key
#pragma unroll 1
    for (int k = 0; k < nk; ++k) {
      if (!((near_keys >> k) & 1u)) continue;                 // warp-uniform
      uint32_t cur[CPL], lastk = 0;
#pragma unroll
      for (int kk = 0; kk < KPT; ++kk) {
        const bool sel = kk == k;
        lastk = sel ? last[kk] : lastk;
#pragma unroll
        for (int j = 0; j < CPL; ++j) cur[j] = sel ? ord[kk][j] : (kk == 0 ? 0u : cur[j]);
      }
      const float two_b = __shfl_sync(0xffffffffu, two_b_l, k);
      const uint32_t thr_o = float_order(__fadd_ru(order_float(lastk | JM), two_b));
      if (list_mode) {
        const uint32_t nxt = __reduce_min_sync(0xffffffffu, cur[0]);
        int n = C;
#pragma unroll
        for (int q = 0; q < CPL; ++q) {
          const uint32_t v = cur[q];
          const bool in = v <= thr_o;
          const uint32_t m = __ballot_sync(0xffffffffu, in);
          const int at = n + __popc(m & ((1u << lane) - 1u));
          if (in && at < kListLen)
            lists64[k * 16 + at] = (static_cast<unsigned long long>(v | JM) << 32) | (v & JM);
          n += __popc(m);
        }
        if (n <= kListLen) {
          if (lane >= n && lane < kListLen) lists64[k * 16 + lane] = ~0ull;
          if (lane == 0)       // slot 15: the entry count and the limit
            lists64[k * 16 + kListLen] = (static_cast<unsigned long long>(n) << 32) |
                                         float_order(__fsub_rd(order_float(nxt & ~JM), two_b));
          listed |= 1u << k;
          continue;
        }
        __syncwarp();                                        // the id list below takes these slots
      }
      // ids: the C taken, then the others under the threshold
      const int taken_id = lane < C ? int(cand_w[k * C + lane]) : -1;
      __syncwarp();
      lists[k * 32 + lane] = taken_id;
      int n = C;
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        const uint32_t v = cur[q];
        const bool in = v <= thr_o;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        const int at = n + __popc(m & ((1u << lane) - 1u));
        if (in && at < 32) lists[k * 32 + at] = int(v & JM);
        n += __popc(m);
      }
      exact_keys |= 1u << k;
      if (n > 32) long_lists |= 1u << k;
    }
    __syncwarp();
    // ---- the keys whose candidate set the bound left open: fp32 D_j by the
    // definition, one listed centre per lane, and the C smallest (D_j, j);
    // with more than 32 centres under the threshold (degenerate tables), C
    // rounds over every centre instead
    for (int k = 0; k < nk; ++k) {
      if (!((exact_keys >> k) & 1u)) continue;                // warp-uniform
      // the key row (bf16) in shared memory, so the serial chains read it
      // from there: staged after the lists (one key per warp; D/2 words fit
      // since D * KPT >= 32 * KPT + D/2), or row k of the staged rows
      const int kr = (KPT == 1) ? 0 : k;
      if constexpr (KPT == 1) {
        if (lane < D / 8)
          reinterpret_cast<uint4*>(rows_w)[lane] = reinterpret_cast<const uint4*>(key_ptr(a.K, row_of(k)))[lane];
        __syncwarp();
      }
      if (!((long_lists >> k) & 1u)) {
        const int id = lists[k * 32 + lane];                  // -1: no centre in this slot
        uint32_t o = 0xFFFFFFFFu;
        if (id >= 0)
          o = float_order(__fadd_rn(exact_distance<D>(rows_w, kr, mu_s, id, w_s), 0.0f));
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
                                      exact_distance<D>(rows_w, kr, mu_s, j, w_s), 0.0f)))
                                  << 32) | uint32_t(j);
            if ((i == 0 || key > prev) && key < best) best = key;
          }
          const uint32_t hi = __reduce_min_sync(0xffffffffu, uint32_t(best >> 32));
          const uint32_t lo = __reduce_min_sync(0xffffffffu, uint32_t(best >> 32) == hi ? uint32_t(best) : 0xFFFFFFFFu);
          prev = (uint64_t(hi) << 32) | lo;
          if (lane == 0) cand_w[k * C + i] = uint16_t(lo);
        }
      }
      __syncwarp();                                           // the staged row is rewritten for the next key
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
    // ---- perturbation estimates: one task per (key, centre), the C
    // candidates of an ordinary key or the listed centres of a listed one,
    // spread over the lanes. Ordinary keys keep the least (E, centre id);
    // listed ones keep every entry's (E, sure flag, id) for the decision below.
    if (C > 1) {
      int off[KPT + 1];
      off[0] = 0;
#pragma unroll
      for (int k = 0; k < KPT; ++k)                     // tasks per key: C, or a listed key's entries
        off[k + 1] = off[k] + (k >= nk ? 0 : ((listed >> k) & 1u) ? int(lists64[k * 16 + kListLen] >> 32) : C);
      const float* Wg_h = a.Wg + size_t(h) * NG;
      // two tasks per lane at a time (t and t + 32), their chains independent;
      // the trip count is the same for every lane (the loop holds a
      // __syncwarp), lanes past the last task compute a copy and store nothing
      for (int t0 = 0; t0 < off[KPT]; t0 += 64) {
        int kt[2], et[2], jt[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int t = min(t0 + lane + 32 * u, off[KPT] - 1);
          int k = 0, base = 0;
#pragma unroll
          for (int kk = 1; kk < KPT; ++kk)
            if (t >= off[kk]) { k = kk; base = off[kk]; }
          kt[u] = k;
          et[u] = t - base;
          jt[u] = ((listed >> k) & 1u) ? int(uint32_t(lists64[k * 16 + et[u]]) & 0xffffu) : int(cand_w[k * C + et[u]]);
        }
        float E[2];
        perturbation2<D, GS>(rows_w, kt, jt, mu_s, Wg_h, E);
        __syncwarp();                                   // list entries are read before any is rewritten
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (t0 + lane + 32 * u >= off[KPT]) break;
          const int k = kt[u], e = et[u], j = jt[u];
          if ((listed >> k) & 1u) {
            const unsigned long long ent = lists64[k * 16 + e];
            const bool sure = uint32_t(ent >> 32) < uint32_t(lists64[k * 16 + kListLen]);
            lists64[k * 16 + e] = (static_cast<unsigned long long>(float_order(E[u])) << 32) | (sure ? 0x80000000u : 0u) | uint32_t(j);
          } else {
            atomicMin(&best_w[k], (static_cast<unsigned long long>(float_order(E[u])) << 32) | unsigned(j));
          }
        }
      }
      __syncwarp();
    }
    // ---- listed keys: the exact candidate set holds every centre sure to be
    // in it and C minus that many of the ones in doubt, so when the least
    // (E, id) among the sure ones is below every one in doubt it is the
    // choice whichever of those are in; otherwise (rare) the exact distances
    // of the listed centres decide the set, and the choice is the least
    // (E, id) in it.
    for (int k = 0; k < nk; ++k) {
      if (!((listed >> k) & 1u)) continue;                    // warp-uniform
      const unsigned long long ent = lane < kListLen ? lists64[k * 16 + lane] : ~0ull;
      const bool valid = ent != ~0ull;
      const bool sure = valid && ((ent >> 31) & 1u);
      const int id = int(uint32_t(ent) & 0xffffu);
      const unsigned long long ek = valid ? ((ent & 0xFFFFFFFF00000000ull) | uint32_t(id)) : ~0ull;
      const unsigned long long bs = warp_min64(sure ? ek : ~0ull);
      const unsigned long long bd = warp_min64(valid && !sure ? ek : ~0ull);
      unsigned long long choice = bs;
      if (bs == ~0ull || bd < bs) {
        unsigned long long dk = ~0ull;
        if (valid)
          dk = (static_cast<unsigned long long>(float_order(__fadd_rn(exact_distance<D>(rows_w, k, mu_s, id, w_s), 0.0f)))
                << 32) | uint32_t(id);
        bool in_set = false;
        for (int i = 0; i < C; ++i) {
          const unsigned long long m = warp_min64(dk);
          if (valid && dk == m) { in_set = true; dk = ~0ull; }
        }
        choice = warp_min64(in_set ? ek : ~0ull);
      }
      if (lane == 0) best_w[k] = choice;
    }
    __syncwarp();

    if (a.assign) {
      for (int k = lane; k < nk; k += 32) {
        a.assign[size_t(row_of(k)) * a.H + h] = (C > 1) ? int(best_w[k] & 0xffffffffu) : cand_w[k * C];
      }
    } else {
    // ---- K residual codec, one task per (key, 32-channel sub-group): the
    // residual k - mu_j of the chosen centre from the staged rows; a group of
    // GS channels spans SPG consecutive lanes, which share its range by
    // shuffles. The residual errors e go over the staged rows, so every
    // lane has read its rows before any writes. (Values are coded by their
    // own kernel, launched before this one.)
    {
      constexpr int MAXT = (KPT * NS + 31) / 32;
      float ev[MAXT][kGroup];
#pragma unroll
      for (int t = 0; t < MAXT; ++t) {
        const int task = lane + 32 * t;
        const bool live = task < nk * NS;
        const int k = live ? task / NS : 0, sg = task % NS;
        const int j = (C > 1) ? int(best_w[k] & 0xffffffffu) : cand_w[k * C];
        float x[kGroup];
#pragma unroll
        for (int c8 = 0; c8 < kGroup / 8; ++c8) {
          const uint4 kv = *reinterpret_cast<const uint4*>(rows_w + mu_index<D>(k, sg * 4 + c8));
          const uint4 mv = *reinterpret_cast<const uint4*>(mu_s + mu_index<D>(j, sg * 4 + c8));
          const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
          const uint32_t mu4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 m = __half22float2(*reinterpret_cast<const __half2*>(&mu4[q]));
            const float2 xx = up2(fsub2(pk2(__uint_as_float(ku[q] << 16), __uint_as_float(ku[q] & 0xffff0000u)),
                                        pk2(m.x, m.y)));
            x[c8 * 8 + 2 * q] = xx.x;
            x[c8 * 8 + 2 * q + 1] = xx.y;
          }
        }
        float mn = x[0], mx = x[0];
#pragma unroll
        for (int c = 1; c + 1 < kGroup; c += 2) { mn = fmin3(mn, x[c], x[c + 1]); mx = fmax3(mx, x[c], x[c + 1]); }
        mn = fminf(mn, x[kGroup - 1]);
        mx = fmaxf(mx, x[kGroup - 1]);
#pragma unroll
        for (int o = 1; o < SPG; o <<= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const GroupParams gp = group_params(mn, mx);
        const float inv_s = __frcp_rn(gp.s);
        uint32_t w0, w1, redo;
        code32<true>(x, gp, inv_s, w0, w1, redo, ev[t]);
        // the rare channels whose code the correctly rounded division decides
#pragma unroll 1
        for (; redo; redo &= redo - 1) {
          const int c = __ffs(redo) - 1, ch = sg * kGroup + c;
          const float xc = __fsub_rn(
              __uint_as_float(uint32_t(rows_w[mu_index<D>(k, ch / 8) + ch % 8]) << 16),
              __half2float(mu_s[mu_index<D>(j, ch / 8) + ch % 8]));
          const uint32_t q = group_code(xc, gp);
          if (c < 16) w0 = (w0 & ~(3u << (2 * c))) | (q << (2 * c));
          else w1 = (w1 & ~(3u << (2 * (c - 16)))) | (q << (2 * (c - 16)));
          const float e = __fsub_rn(xc, group_dequant(q, gp));
#pragma unroll
          for (int cc = 0; cc < kGroup; ++cc) ev[t][cc] = cc == c ? e : ev[t][cc];
        }
        if (live) {
          const size_t slot = slot_of(row_of(k));
          *reinterpret_cast<uint2*>(a.k_code + slot * (D / 16) + sg * 2) = make_uint2(w0, w1);
          if (sg % SPG == 0) a.k_sz[slot * NG + sg / SPG] = uint32_t(gp.s_bits) | (uint32_t(gp.z_bits) << 16);
          if (sg == 0) {
            if (M <= 256) static_cast<uint8_t*>(a.cidx)[slot] = uint8_t(j);
            else static_cast<uint16_t*>(a.cidx)[slot] = uint16_t(j);
          }
        }
      }
      __syncwarp();                                     // every lane's rows are read
#pragma unroll
      for (int t = 0; t < MAXT; ++t) {
        const int task = lane + 32 * t;
        if (task < nk * NS) {
          const int k = task / NS, sg = task % NS;
#pragma unroll
          for (int c = 0; c < kGroup; ++c) e_w[k * Cfg::ES + sg * (kGroup + 1) + c] = ev[t][c];
        }
      }
    }
    __syncwarp();

    // ---- PSAC coefficients a_i = sum_c P_ci e_c (ascending c)
    for (int task = lane; task < nk * a.r; task += 32) {
      const int k = task / a.r, i = task - k * a.r;
      const float* Pcol = P_s + i;
      const float* e = e_w + k * Cfg::ES;
      float acc = 0.0f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = __fmaf_rn(Pcol[c * a.r], e[c + (c >> 5)], acc);
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

// Value codec of the appends whose keys the multi-key warps take: one thread
// per 32-channel sub-group of one (row, head); the SPG threads of a group are
// consecutive lanes and share its range by shuffles (every thread takes part,
// those past the end with their stores off). Same arithmetic as the one-key
// path: group_params, then group_code_recip per channel. Launched as the key
// kernel's programmatic dependent (its blocks take the SMs the key kernel's
// CTAs leave); before it ends it waits for the key grid, so that whatever
// the stream runs next finds both kernels' writes.
template <int D, int GS>
__global__ void __launch_bounds__(256) value_codec_kernel(QuantizeArgs a) {
  constexpr int NS = D / kGroup, SPG = GS / kGroup, NG = D / GS;
  const long long total = static_cast<long long>(a.B) * a.n_new * a.H * NS;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool live = t < total;
  const long long tt = live ? t : 0;
  const int sg = int(tt % NS);
  const long long rh = tt / NS;
  const int h = int(rh % a.H);
  const long long row = rh / a.H;
  const int b = int(row / a.n_new), tok = int(row % a.n_new);
  const uint16_t* vrow = a.V + ((size_t(b) * a.n_new + tok) * a.H + h) * D + sg * kGroup;
  float x[kGroup];
#pragma unroll
  for (int c8 = 0; c8 < kGroup / 8; ++c8) {
    const uint4 vv = *reinterpret_cast<const uint4*>(vrow + c8 * 8);
    const uint32_t vu[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      x[c8 * 8 + 2 * q] = __uint_as_float(vu[q] << 16);
      x[c8 * 8 + 2 * q + 1] = __uint_as_float(vu[q] & 0xffff0000u);
    }
  }
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int c = 1; c + 1 < kGroup; c += 2) { mn = fmin3(mn, x[c], x[c + 1]); mx = fmax3(mx, x[c], x[c + 1]); }
  mn = fminf(mn, x[kGroup - 1]);
  mx = fmaxf(mx, x[kGroup - 1]);
#pragma unroll
  for (int o = 1; o < SPG; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const GroupParams gp = group_params(mn, mx);
  const float inv_s = __frcp_rn(gp.s);
  uint32_t w0, w1, redo;
  float unused[kGroup];
  code32<false>(x, gp, inv_s, w0, w1, redo, unused);
  // the rare channels whose code the correctly rounded division decides
#pragma unroll 1
  for (; redo; redo &= redo - 1) {
    const int c = __ffs(redo) - 1;
    const uint32_t q = group_code(__uint_as_float(uint32_t(vrow[c]) << 16), gp);
    if (c < 16) w0 = (w0 & ~(3u << (2 * c))) | (q << (2 * c));
    else w1 = (w1 & ~(3u << (2 * (c - 16)))) | (q << (2 * (c - 16)));
  }
  if (live) {
    const size_t slot = cache_slot(a.table, a.page, a.H, a.cap, b, h, a.pos + tok);
    *reinterpret_cast<uint2*>(a.v_code + slot * (D / 16) + sg * 2) = make_uint2(w0, w1);
    if (sg % SPG == 0) a.v_sz[slot * NG + sg / SPG] = uint32_t(gp.s_bits) | (uint32_t(gp.z_bits) << 16);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  const long long nwork = static_cast<long long>((rows + Cfg::KT - 1) / Cfg::KT) * a.H;
  const long long resident = static_cast<long long>(sms) * per_sm;   // one wave of persistent CTAs
  kern<<<unsigned(nwork < resident ? nwork : resident), kThreads, smem, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || KPT == 1 || a.assign) return e;
  // the values of a multi-key append: the key kernel's programmatic dependent
  const long long threads = static_cast<long long>(a.B) * a.n_new * a.H * (D / kGroup);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned((threads + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, value_codec_kernel<D, GS>, a);
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
