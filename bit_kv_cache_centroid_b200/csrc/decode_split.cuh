// decode_split.cuh — the split-K decode kernel over the packed 2-bit cache
// and its launch helpers, templated on the head dim, the query heads per KV
// head, the centroid id width and the PSAC format. Included by decode.cu.
//
// Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
// World Models", "1. QSAC" (a key is its centre plus an INT2 residual with a
// per-group fp16 scale and zero) and "2. PSAC" (the Key error's components on
// the top Query directions, added back to the score). Reading the 2-bit cache
// inside attention follows the principle stated on the OmniKVQuant page
// ("OmniKVQuant: KV Cache Quantization for Omni-LLMs", abstract); the design
// here is our own.
//
//   logit_t = q.mu[idx_t] + sum_g (s_g * sum_{c in g} q_c code_c + z_g * sum_{c in g} q_c)
//             + (q P) . a_t                      (all scaled by sm_scale * log2 e)
//   out     = sum_t softmax_t * (code_t s_t + z_t)
//
// Two kernels:
//   decode_split  grid (splits, B*H_kv), 4 warps. Prologue: the query-side
//                 tables of the G query heads sharing the KV head (q in log2
//                 units, q.mu_j for every centre, u = qP, per-group sums of q),
//                 built while the first tile is in flight. Then 128-token tiles
//                 of every packed stream arrive by 1-D bulk copies (three
//                 stages, one barrier each) and each tile takes three phases:
//                   q.k   the sums  sum_{c in g} q_c code_c  as 8-bit integer
//                         MMAs (mma.sync m16n8k32, A = codes as u8, B = q as
//                         two signed 8-bit digits, exact int32), scaled by the
//                         token's s_g; the zero-point and PSAC terms as fp16
//                         k-steps (A = the token's z_g and a_i, B = hi/lo
//                         halves of the query's group sums and qP);
//                   owner one thread per token adds the centre term, runs the
//                         online softmax and writes p_t s_t,g;
//                   p.v   sum_t (p_t s_t,g) code_t,c on the tensor cores
//                         (mma.sync m16n8k16): A = codes (channels x tokens),
//                         B = p s as fp16 hi = fp16(x), lo = fp16(x - hi)
//                         (about 22 significant bits) in separate columns of
//                         the n8 tile, so G <= 4 heads fill one tile and 8
//                         heads two; the two column sums are added in fp32.
//   decode_combine (decode.cu) log-sum-exp merge of the splits.
//
// Codes become operands with few integer/half instructions and no
// conversions. q.k: (word >> 2 tig) & 0x03030303 puts four codes in the bytes
// of an 8-bit operand (tig = lane % 4). p.v: a byte permute puts the byte
// holding channel c of two tokens into the two halves, and for a code at bits
// 2i..2i+1 (i <= 3) of a half, (half & (3 << 2i)) | 0x6400 is the fp16 number
// 1024 + code * 4^i; one fp16 fma with 4^-i and -1024 * 4^-i gives the code
// exactly.
#pragma once

#include <cfloat>

#include "common.cuh"
#include "internal.h"
#include "mbarrier.cuh"

namespace kv2 {
namespace dsplit {

constexpr int kTile = 128;        // tokens per tile
constexpr int kThreads = 128;     // one thread per token in the owner phase
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 3;        // tiles in shared memory (two copies ahead of the one in use)
constexpr float kLog2e = 1.4426950408889634f;

struct SplitParams {
  const uint32_t* k_code;
  const uint32_t* v_code;
  const uint32_t* k_sz;
  const uint32_t* v_sz;
  const void* cidx;
  const uint16_t* psac;
  const uint16_t* Q;      // bf16 [B][H_q][D]
  const uint16_t* cent;   // fp16 [H_kv][M][D]
  const float* P;         // [H_kv][D][r]
  float scale;            // sm_scale * log2(e)
  float* part;            // [B*H_kv][splits][G][D + 2]
  int* err;               // sticky error word: 1 after a wait ran out of its budget
  unsigned long long budget;   // SM clock cycles a wait may take
  int force_timeout;      // wait on copies that are never issued (tests)
  int wait_from;          // first slot the preceding (primary) kernel writes
  int H_kv, H_q, M, r, cap, len, splits, tiles_per_split;
  int psac_fmt;                 // 0: fp16 coefficients; 1: int8 codes + fp16 scale per token
  const uint16_t* psac_scale;
  const int32_t* table;         // paged cache: block table [B][cap / page] (null: contiguous)
  int page;
};

// d = a * b + c on two fp16 lanes
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// two codes (at the bits of `mask` in each half of x) -> two exact fp16 codes:
// (half & mask) | 0x6400 is the fp16 number 1024 + code * 4^i, and one fp16
// fma with 4^-i and -1024 * 4^-i leaves the code. (Reading the masked bits as
// fp16 subnormals, code * 4^i * 2^-24, would save the fma, but mma.sync then
// measured about 9x the error of this form against the oracle.)
__device__ __forceinline__ uint32_t unpack_codes(uint32_t x, uint32_t mask, uint32_t scale, uint32_t offset) {
  return hfma2((x & mask) | 0x64006400u, scale, offset);
}
// d += A B, m16n8k16, fp16 operands, fp32 accumulators
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// order-preserving map of floats (no NaN) to signed integers, and back
__device__ __forceinline__ int f2ord(float x) {
  const int i = __float_as_int(x);
  return i ^ ((i >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float ord2f(int k) { return __int_as_float(k ^ ((k >> 31) & 0x7fffffff)); }
// d = A B, m16n8k32, A unsigned 8-bit, B signed 8-bit, exact int32 sums
__device__ __forceinline__ void mma16832_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}
// four transposed 8x8 fp16 tiles; lane i gives the address of row i % 8 of tile i / 8
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* row) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(row));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(s));
}
// x = hi + lo with hi = fp16(x), lo = fp16(x - hi)
__device__ __forceinline__ uint16_t f16_hi(float x) { return __half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ uint16_t f16_lo(float x) {
  return __half_as_ushort(__float2half_rn(x - __half2float(__float2half_rn(x))));
}
__device__ __forceinline__ uint32_t pack_h2(uint16_t lo_half, uint16_t hi_half) {
  return uint32_t(lo_half) | (uint32_t(hi_half) << 16);
}

// G consecutive floats from shared memory with the widest aligned loads
template <int G>
__device__ __forceinline__ void load_vec(const float* src, float (&v)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int i = 0; i < G; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(src + i);
      v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
    }
  } else if constexpr (G == 2) {
    const float2 x = *reinterpret_cast<const float2*>(src);
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = src[0];
  }
}

// Column n of an n8 operand tile holds, for G <= 4, the hi half of head n
// (n < G) or the lo half of head n - G (G <= n < 2G), other columns zero; for
// G = 8, tile 0 holds the hi halves and tile 1 the lo halves of heads 0..7.
template <int G>
struct Cols {
  static constexpr int NT = (G == 8) ? 2 : 1;
  __device__ static int head(int n) { return (G == 8) ? n : (n < G ? n : n - G); }
  __device__ static bool used(int n) { return (G == 8) || n < 2 * G; }
  __device__ static bool is_lo(int nt, int n) { return (G == 8) ? nt == 1 : n >= G; }
};

// Adds the hi and lo column sums of a fragment (c0..c3 = rows r, r, r+8, r+8
// and columns 2 tig, 2 tig + 1 of each n8 tile) and calls f(row_sel, head,
// value) once per (row, head) on the lane that holds the sum. Every lane of
// the warp must call it (it shuffles).
template <int G, int NT, typename F>
__device__ __forceinline__ void combine_hi_lo(const float (&c)[NT][4], int tig, F&& f) {
  if constexpr (G == 8) {
#pragma unroll
    for (int i = 0; i < 4; ++i) f(i >> 1, 2 * tig + (i & 1), c[0][i] + c[NT - 1][i]);
  } else if constexpr (G == 4) {
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = c[0][i] + __shfl_xor_sync(0xffffffffu, c[0][i], 2);
    if (tig < 2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) f(i >> 1, 2 * tig + (i & 1), v[i]);
    }
  } else if constexpr (G == 2) {
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = c[0][i] + __shfl_xor_sync(0xffffffffu, c[0][i], 1);
    if (tig == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) f(i >> 1, i & 1, v[i]);
    }
  } else {
    if (tig == 0) {
      f(0, 0, c[0][0] + c[0][1]);
      f(1, 0, c[0][2] + c[0][3]);
    }
  }
}

// Shared memory of the split kernel:
//   stages  kStages x raw tile copies (codes, scale/zero words, ids, PSAC),
//           filled by bulk copies that complete on one barrier per stage
//           (reused at the end for the final reduction)
//   lg      [kTile][LS] fp32   q.k sums per token and head
//   wt      [NG][kTile][NCOL] fp16   p s_v per group, token and column
//   tables  q.mu [G][M], u [G][r], group sums [G][NG], reduction slots,
//           B fragments of the zero-point / PSAC k-steps [XK][NT][32 lanes]
// lg and wt also hold the prologue's scratch (q and rows of P).
// GS: channels per (scale, zero) group, 32, 64 or 128 (NG = D / GS groups).
template <int D, int G, bool U16, int GS>
struct DCfg {
  static_assert(GS % 32 == 0 && D % GS == 0, "groups of whole 32-channel sub-groups");
  static constexpr int NG = D / GS;            // scale/zero words per token
  static constexpr int NGP = (NG + 1) & ~1;    // zero-point columns of the aux k-steps (even)
  static constexpr int NS = D / 32;            // 32-channel sub-groups = 8-bit q.k k-steps
  static constexpr int SPG = GS / 32;          // sub-groups per group
  static constexpr int WPG = GS / 16;          // code words per group
  static constexpr int NW = D / 16;            // code words per token
  static constexpr int NT = Cols<G>::NT;
  static constexpr int NCOL = 8 * NT;
  static constexpr int MTK = kTile / 16 / kWarps;   // token m-tiles per warp in q.k
  static constexpr int MTV = NW / kWarps;           // channel m-tiles (words) per warp in p.v
  static_assert(MTV >= 1 && MTV <= 2 && MTV <= WPG, "one channel group per warp in p.v");
  static constexpr int IDXB = U16 ? 2 : 1;
  static constexpr int LS = G < 4 ? 4 : G;
  // per-stage byte offsets (all multiples of 16)
  static constexpr int kc_off = 0;
  static constexpr int vc_off = kc_off + kTile * NW * 4;
  static constexpr int ks_off = vc_off + kTile * NW * 4;
  static constexpr int vs_off = ks_off + kTile * NG * 4;
  static constexpr int ix_off = vs_off + kTile * NG * 4;
  static constexpr int ps_off = ix_off + kTile * IDXB;
  static constexpr int lg_bytes = kTile * LS * 4;
  static constexpr int wt_bytes = NG * kTile * NCOL * 2;
  static constexpr int scratch_floats = (lg_bytes + wt_bytes) / 4;
  static constexpr int red_bytes = (G * D + kWarps * G * NG) * 4;    // final reduction
  __host__ __device__ static int stage_bytes(int r) { return (ps_off + kTile * r * 2 + 15) & ~15; }
  __host__ __device__ static int stages_bytes(int r) {
    const int st = kStages * stage_bytes(r);
    return st > red_bytes ? st : red_bytes;
  }
  // k-steps of the zero-point and PSAC terms (columns z_0..z_NG-1, a zero
  // column when NG is odd, then a_0..a_r-1)
  __host__ __device__ static int xk(int r) { return (NGP + r + 15) / 16; }
  __host__ __device__ static int small_floats(int M, int r) {
    return (G * M + G * r + G * NG + kWarps * G + 2 * kWarps + 3) & ~3;
  }
  // one full-barrier per stage, after the other tables
  __host__ __device__ static int bar_off(int M, int r) {
    return lg_bytes + wt_bytes + small_floats(M, r) * 4 + xk(r) * NT * 32 * 8;
  }
  __host__ __device__ static int tables_bytes(int M, int r) { return bar_off(M, r) + kStages * 8 + 8; }
};

// Q8: the PSAC coefficients are int8 codes with a per-token fp16 scale
// (cache format 1), else fp16 (format 0). GS: channels per scale/zero group.
template <int D, int G, bool U16, bool Q8, int GS>
__global__ void __launch_bounds__(kThreads) decode_split(SplitParams p) {
  using Cfg = DCfg<D, G, U16, GS>;
  using CL = Cols<G>;
  constexpr int NG = Cfg::NG, NW = Cfg::NW, NT = Cfg::NT, NCOL = Cfg::NCOL;
  constexpr int NGP = Cfg::NGP, NS = Cfg::NS, SPG = Cfg::SPG, WPG = Cfg::WPG;
  constexpr int MTK = Cfg::MTK, MTV = Cfg::MTV, LS = Cfg::LS;
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = p.r, M = p.M;
  const int stage = Cfg::stage_bytes(r);
  unsigned char* tables = smem + Cfg::stages_bytes(r);
  float* lg_s = reinterpret_cast<float*>(tables);                                  // [kTile][LS]
  uint16_t* wt_s = reinterpret_cast<uint16_t*>(tables + Cfg::lg_bytes);            // [NG][kTile][NCOL]
  float* mus = reinterpret_cast<float*>(tables + Cfg::lg_bytes + Cfg::wt_bytes);   // [G][M]
  float* us = mus + G * M;                                                         // [G][r]
  float* sgs = us + G * r;                                                         // [G][NG]
  float* red = sgs + G * NG;                                                       // [kWarps][G], [2][kWarps]
  uint2* baux = reinterpret_cast<uint2*>(mus + Cfg::small_floats(M, r));           // [XK][NT][32]
  const int XK = Cfg::xk(r);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H_kv, h = bh % p.H_kv;
  const size_t base_slot = size_t(bh) * p.cap;
  const int t_begin = split * p.tiles_per_split * kTile;
  const int t_end = min(p.len, t_begin + p.tiles_per_split * kTile);
  const int ntiles = (t_end > t_begin) ? (t_end - t_begin + kTile - 1) / kTile : 0;

  // tile copies: thread 0 issues one bulk copy per stream into the tile's
  // stage; they complete on the stage's barrier
  const uint32_t bar0 = smem_u32(tables + Cfg::bar_off(M, r));
  int issued = 0;                                        // tiles issued (thread 0)
  bool dep_done = false;                                 // primary grid waited for (thread 0)
  auto issue = [&](int tile) {
    if (tile >= ntiles || p.force_timeout) return;
    const int st = tile % kStages;
    const uint32_t dst = smem_u32(smem + st * stage);
    const uint32_t bar = bar0 + 8 * st;
    const int t0 = t_begin + tile * kTile;
    const int n16 = (min(kTile, t_end - t0) + 15) & ~15;   // within capacity (cap % 16 == 0)
    if (!dep_done && t0 + n16 > p.wait_from) {
      // the tile reaches slots the primary kernel writes: wait for its grid
      // to complete (and its writes to be visible) before copying
      asm volatile("griddepcontrol.wait;" ::: "memory");
      dep_done = true;
    }
    // (a multiple of 16; a tile never leaves its page)
    const size_t s0 = p.table ? cache_slot(p.table, p.page, p.H_kv, p.cap, b, h, t0) : base_slot + t0;
    const int ps_bytes = Q8 ? (r ? r + 2 : 0) : 2 * r;   // per token
    mbar_arrive_expect_tx(bar, uint32_t(n16) * uint32_t(2 * NW * 4 + 2 * NG * 4 + Cfg::IDXB + ps_bytes));
    bulk_g2s(dst + Cfg::kc_off, p.k_code + s0 * NW, n16 * NW * 4, bar);
    bulk_g2s(dst + Cfg::vc_off, p.v_code + s0 * NW, n16 * NW * 4, bar);
    bulk_g2s(dst + Cfg::ks_off, p.k_sz + s0 * NG, n16 * NG * 4, bar);
    bulk_g2s(dst + Cfg::vs_off, p.v_sz + s0 * NG, n16 * NG * 4, bar);
    bulk_g2s(dst + Cfg::ix_off, static_cast<const unsigned char*>(p.cidx) + s0 * Cfg::IDXB, n16 * Cfg::IDXB, bar);
    if (Q8 && r) {
      // int8 codes [kTile][r], then the fp16 scales [kTile], in the PSAC region
      bulk_g2s(dst + Cfg::ps_off, reinterpret_cast<const int8_t*>(p.psac) + s0 * r, n16 * r, bar);
      bulk_g2s(dst + Cfg::ps_off + kTile * r, p.psac_scale + s0, n16 * 2, bar);
    } else if (r) {
      bulk_g2s(dst + Cfg::ps_off, p.psac + s0 * r, n16 * r * 2, bar);
    }
    issued = tile + 1;
  };
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(bar0 + 8 * i, 1);
    mbar_init_fence();
    for (int i = 0; i < kStages - 1; ++i) issue(i);
  }

  // ---- query-side tables of the G query heads sharing this KV head, built
  // while the first tile is in flight (lg and wt are not used before it):
  // q in log2 units, q . mu_j for every centre, u = q P, per-group sums of q
  float* qs = lg_s;                                      // [G][D]
  float* pst = lg_s + G * D;                             // a chunk of rows of P, [rows][r]
  for (int i = tid; i < G * D; i += kThreads)
    qs[i] = bf16_to_f32(p.Q[size_t(b * p.H_q + h * G) * D + i]) * p.scale;
  for (int i = tid; i < G * r; i += kThreads) us[i] = 0.0f;
  __syncthreads();
  {
    const __half* cent_h = reinterpret_cast<const __half*>(p.cent) + size_t(h) * M * D;
    for (int j = tid; j < M; j += kThreads) {
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = 0.0f;
      const uint4* row = reinterpret_cast<const uint4*>(cent_h + size_t(j) * D);
#pragma unroll 4
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 v = __ldg(row + c8);
        const __half2* h2 = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 m = __half22float2(h2[k]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            acc[g] = fmaf(qs[g * D + c8 * 8 + 2 * k], m.x, acc[g]);
            acc[g] = fmaf(qs[g * D + c8 * 8 + 2 * k + 1], m.y, acc[g]);
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) mus[g * M + j] = acc[g];
    }
    for (int i = tid; i < G * NG; i += kThreads) {
      const float* q = qs + (i / NG) * D + (i % NG) * GS;
      float acc = 0.0f;
      for (int c = 0; c < GS; ++c) acc += q[c];
      sgs[i] = acc;
    }
    if (r) {
      const float* Ph = p.P + size_t(h) * D * r;
      const int rows = min(D, (Cfg::scratch_floats - G * D) / r);   // >= 1 since r <= D
      for (int c0 = 0; c0 < D; c0 += rows) {
        const int nr = min(rows, D - c0);
        for (int i = tid; i < nr * r; i += kThreads) pst[i] = Ph[size_t(c0) * r + i];
        __syncthreads();
        for (int i = tid; i < G * r; i += kThreads) {
          const float* q = qs + (i / r) * D + c0;
          const float* pc = pst + i % r;
          float acc = us[i];
          for (int c = 0; c < nr; ++c) acc = fmaf(q[c], pc[c * r], acc);
          us[i] = acc;
        }
        __syncthreads();
      }
    }
  }
  __syncthreads();           // sgs and us are complete
  // scales for the tensor cores: max |q| 2^eq below 2^15 and
  // max(|sigma|, |u|) 2^ea below 2^14
  float qmax = 0.0f, amax = 0.0f;
  for (int i = tid; i < G * D; i += kThreads) qmax = fmaxf(qmax, fabsf(qs[i]));
  for (int i = tid; i < G * NG; i += kThreads) amax = fmaxf(amax, fabsf(sgs[i]));
  for (int i = tid; i < G * r; i += kThreads) amax = fmaxf(amax, fabsf(us[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  }
  if (lane == 0) {
    red[kWarps * G + warp] = qmax;
    red[kWarps * G + kWarps + warp] = amax;
  }
  __syncthreads();
  const float* rq = red + kWarps * G;
  qmax = fmaxf(fmaxf(rq[0], rq[1]), fmaxf(rq[2], rq[3]));
  amax = fmaxf(fmaxf(rq[4], rq[5]), fmaxf(rq[6], rq[7]));
  int qexp = 0, aexp = 0;
  frexpf(qmax, &qexp);
  frexpf(amax, &aexp);
  const int eq = (qmax > 0.0f) ? 15 - qexp : 0;
  const int ea = (amax > 0.0f) ? 14 - aexp : 0;
  // q enters q.k as the integer rint(q qmul), |.| <= 127 * 256 (two signed
  // 8-bit digits); qinv = 1 / qmul rounded to fp32
  const float qmul = ldexpf(127.0f / 128.0f, eq), qinv = 1.0f / qmul;
  const float amul = ldexpf(1.0f, ea), ainv = ldexpf(1.0f, -ea);
  // B fragments of the zero-point / PSAC k-steps: aux column c is sigma_c
  // (c < NG), zero (c = NG when NG is odd), u_(c-NGP) (c - NGP < r), zero
  // beyond
  for (int i = tid; i < XK * NT * 32; i += kThreads) {
    const int x = i / (NT * 32), nt = (i / 32) % NT, l = i % 32;
    const int n = l >> 2, tg = l & 3;
    const int hq = 4 * nt + n / 2;                        // q.k column convention
    const bool used = hq < G, lo = (n & 1) != 0;
    const int hd = min(hq, G - 1);
    uint16_t hv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 16 * x + 2 * tg + (e & 1) + 8 * (e >> 1);
      float v = 0.0f;
      if (c < NG) v = sgs[hd * NG + c];
      else if (c >= NGP && c - NGP < r) v = us[hd * r + c - NGP];
      v *= amul;
      hv[e] = used ? (lo ? f16_lo(v) : f16_hi(v)) : uint16_t(0);
    }
    baux[i] = make_uint2(pack_h2(hv[0], hv[1]), pack_h2(hv[2], hv[3]));
  }

  // B operand of q.k (8-bit, one k-step of 32 per 32-channel sub-group):
  // column n of n8 tile nt is head 4 nt + n / 2, digit n % 2 of q 2^eq
  // rounded to an integer q_int = d0 + 256 d1 (d0 in [-128, 127], |q_int| <=
  // 127 * 256); row 4 tig + i (i < 4) of the sub-group's k-step is channel
  // tig + 4 i of its first code word, row 16 + 4 tig + i channel tig + 4 i of
  // its second
  uint32_t bq8[NT][NS][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hd = 4 * nt + gid / 2, dg = gid & 1;
#pragma unroll
    for (int g = 0; g < NS; ++g) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          int qd = 0;
          if (hd < G) {
            const int c = 32 * g + 16 * hf + tig + 4 * i;
            const int qi = __float2int_rn(qs[hd * D + c] * qmul);
            const int d1 = (qi + 128) >> 8;
            qd = dg ? d1 : qi - 256 * d1;
          }
          word |= (uint32_t(qd) & 0xffu) << (8 * i);
        }
        bq8[nt][g][hf] = word;
      }
    }
  }
  // p.v code unpacking constants: this lane's channels sit at bits
  // 2 cv..2 cv + 1 of a byte (fp16 4^-cv and -1024 * 4^-cv in both halves)
  const int cv = gid & 3;
  const uint32_t mv = (3u << (2 * cv)) | (3u << (16 + 2 * cv));
  const uint32_t scv = 0x3C003C00u - 0x08000800u * uint32_t(cv);
  const uint32_t ofv = 0xE400E400u - 0x08000800u * uint32_t(cv);
  const uint32_t selv0 = uint32_t(gid >> 2) | (uint32_t(4 + (gid >> 2)) << 8);       // channel gid
  const uint32_t selv1 = uint32_t(2 + (gid >> 2)) | (uint32_t(6 + (gid >> 2)) << 8);  // channel gid + 8
  // heads of this lane's two accumulator columns in p.v
  const int hc0 = min(CL::head(2 * tig), G - 1), hc1 = min(CL::head(2 * tig + 1), G - 1);

  // per-thread running sums over the tokens it owns, heads in pairs (2j, 2j+1)
  constexpr int GP = (G + 1) / 2;
  float m_run[G], m_thr[G];   // running maximum and the bound m_run + 8 that forces a refresh
  f32x2 lsum2[GP], pz2[GP][NG];
  float oacc[MTV][NT][4];     // p.v sums scaled by 2^ev_acc
  int ev_acc = 0;
  uint32_t s_thr = 0;         // fp16 bits of 2^(6 - ev_acc): |s_v| at or above it forces a refresh
  float vmul = 1.0f;          // 2^ev_acc
#pragma unroll
  for (int g = 0; g < G; ++g) m_run[g] = m_thr[g] = -FLT_MAX;
#pragma unroll
  for (int j = 0; j < GP; ++j) {
    lsum2[j] = 0ull;
#pragma unroll
    for (int k = 0; k < NG; ++k) pz2[j][k] = 0ull;
  }
#pragma unroll
  for (int mt = 0; mt < MTV; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) oacc[mt][nt][i] = 0.0f;

  bool aborted = false;
  int tile = 0;
  // Iteration `tile` runs the q.k of tile `tile` and the p.v of tile
  // `tile - 1` (independent work in one barrier interval), then the owner
  // phase of tile `tile`; one more iteration finishes the last p.v.
  for (; tile <= ntiles; ++tile) {
    const bool have = tile < ntiles;
    const int st = tile % kStages;
    const bool ok = !have || mbar_wait(bar0 + 8 * st, (tile / kStages) & 1, p.budget);
    // (the barrier also orders the owner phase of tile - 1 before its p.v)
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    const unsigned char* cur = smem + st * stage;
    const unsigned char* prv = smem + ((tile + kStages - 1) % kStages) * stage;
    const int n = have ? min(kTile, t_end - (t_begin + tile * kTile)) : 0;

    if (have) {
      // ---- q.k on the tensor cores: warp w takes tokens 16 MTK w .. 16 MTK (w + 1) - 1
      {
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(cur + Cfg::kc_off);
        const uint32_t* ksz = reinterpret_cast<const uint32_t*>(cur + Cfg::ks_off);
#pragma unroll
        for (int mt = 0; mt < MTK; ++mt) {
          const int t0 = (warp * MTK + mt) * 16 + gid, t1 = t0 + 8;
          uint32_t w0[NW], w1[NW];
#pragma unroll
          for (int i = 0; i < NW; i += 4) {
            const uint4 x0 = *reinterpret_cast<const uint4*>(kw + t0 * NW + i);
            const uint4 x1 = *reinterpret_cast<const uint4*>(kw + t1 * NW + i);
            w0[i] = x0.x; w0[i + 1] = x0.y; w0[i + 2] = x0.z; w0[i + 3] = x0.w;
            w1[i] = x1.x; w1[i + 1] = x1.y; w1[i + 2] = x1.z; w1[i + 3] = x1.w;
          }
          // the two tokens' scale/zero words (all groups)
          uint32_t sz0[NG], sz1[NG];
          if constexpr (NG % 4 == 0) {
#pragma unroll
            for (int g = 0; g < NG; g += 4) {
              const uint4 y0 = *reinterpret_cast<const uint4*>(ksz + t0 * NG + g);
              const uint4 y1 = *reinterpret_cast<const uint4*>(ksz + t1 * NG + g);
              sz0[g] = y0.x; sz0[g + 1] = y0.y; sz0[g + 2] = y0.z; sz0[g + 3] = y0.w;
              sz1[g] = y1.x; sz1[g + 1] = y1.y; sz1[g + 2] = y1.z; sz1[g + 3] = y1.w;
            }
          } else {
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              sz0[g] = ksz[t0 * NG + g];
              sz1[g] = ksz[t1 * NG + g];
            }
          }
          // sum_{c in g} code_c q_int,c per group: one 8-bit k-step per
          // 32-channel sub-group (exact int32, |.| < 2^22 each and < 2^24 over
          // the at most 4 sub-groups of a group, so its conversion is exact),
          // scaled by the token's s_g (and once at the end by 1 / qmul); this
          // lane's column pair is head 4 nt + tig (both digits)
          const uint32_t m8 = 0x03030303u;
          float L[NT][2];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) L[nt][0] = L[nt][1] = 0.0f;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const float s0 = __half2float(__ushort_as_half(uint16_t(sz0[g] & 0xffff)));
            const float s1 = __half2float(__ushort_as_half(uint16_t(sz1[g] & 0xffff)));
            int S[NT][2];
#pragma unroll
            for (int u = 0; u < SPG; ++u) {
              const int k = g * SPG + u;
              const uint32_t a[4] = {(w0[2 * k] >> (2 * tig)) & m8, (w1[2 * k] >> (2 * tig)) & m8,
                                     (w0[2 * k + 1] >> (2 * tig)) & m8, (w1[2 * k + 1] >> (2 * tig)) & m8};
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                int C[4];
                mma16832_u8s8(C, a, bq8[nt][k][0], bq8[nt][k][1]);
                S[nt][0] = (u ? S[nt][0] : 0) + C[0] + 256 * C[1];
                S[nt][1] = (u ? S[nt][1] : 0) + C[2] + 256 * C[3];
              }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              L[nt][0] = fmaf(s0, __int2float_rn(S[nt][0]), L[nt][0]);
              L[nt][1] = fmaf(s1, __int2float_rn(S[nt][1]), L[nt][1]);
            }
          }
          // zero-point and PSAC terms, sum_g z_g sigma_g + sum_i a_i u_i, as XK
          // more k-steps over the columns (z_0 .. z_NG-1, [0], a_0 .. a_r-1) of
          // the token's scale/zero words and PSAC coefficients (exact fp16
          // values)
          {
            const uint32_t* kz0 = ksz + t0 * NG;
            const uint32_t* kz1 = ksz + t1 * NG;
            const uint32_t* ps0 = reinterpret_cast<const uint32_t*>(cur + Cfg::ps_off) + t0 * (r / 2);
            const uint32_t* ps1 = reinterpret_cast<const uint32_t*>(cur + Cfg::ps_off) + t1 * (r / 2);
            constexpr bool q8 = Q8;
            float sc0 = 0.0f, sc1 = 0.0f;              // int8 format: the tokens' scales
            if (q8 && r) {
              const uint16_t* scl = reinterpret_cast<const uint16_t*>(cur + Cfg::ps_off + kTile * r);
              sc0 = __half2float(__ushort_as_half(scl[t0]));
              sc1 = __half2float(__ushort_as_half(scl[t1]));
            }
            // (c is even: columns c, c + 1)
            auto aux_pair = [&](const uint32_t* kz, const uint32_t* ps, int t, float sc, int c) -> uint32_t {
              if (c < NGP) {
                if constexpr (NG % 2 == 0) return __byte_perm(kz[c], kz[c + 1], 0x7632);   // z_c, z_c+1
                else return (c + 1 < NG) ? __byte_perm(kz[c], kz[c + 1], 0x7632) : (kz[c] >> 16);   // z_c, 0
              }
              if (c - NGP >= r) return 0u;
              if (!q8) return ps[(c - NGP) >> 1];                           // an fp16 pair
              // int8 pair: fp16(code * scale) of coefficients c - NGP, c - NGP + 1
              const uint16_t two = reinterpret_cast<const uint16_t*>(cur + Cfg::ps_off)[(t * r + c - NGP) >> 1];
              const float a0 = float(int8_t(two & 0xff)) * sc, a1 = float(int8_t(two >> 8)) * sc;
              const __half2 hv = __floats2half2_rn(a0, a1);
              return *reinterpret_cast<const uint32_t*>(&hv);
            };
            float Ca[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) Ca[nt][i] = 0.0f;
            for (int x = 0; x < XK; ++x) {
              const int c = 16 * x + 2 * tig;
              const uint32_t a[4] = {aux_pair(kz0, ps0, t0, sc0, c), aux_pair(kz1, ps1, t1, sc1, c),
                                     aux_pair(kz0, ps0, t0, sc0, c + 8), aux_pair(kz1, ps1, t1, sc1, c + 8)};
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const uint2 bb = baux[(x * NT + nt) * 32 + lane];
                mma16816(Ca[nt], a, bb.x, bb.y);
              }
            }
            // (columns 2 tig, 2 tig + 1: hi and lo part of head 4 nt + tig)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const int hd = 4 * nt + tig;
              if (hd < G) {
                lg_s[t0 * LS + hd] = fmaf(L[nt][0], qinv, (Ca[nt][0] + Ca[nt][1]) * ainv);
                lg_s[t1 * LS + hd] = fmaf(L[nt][1], qinv, (Ca[nt][2] + Ca[nt][3]) * ainv);
              }
            }
          }
        }
      }
    }
    if (tile > 0) {
      // ---- p.v on the tensor cores: warp w takes code words (16-channel
      // m-tiles) MTV w .. MTV (w + 1) - 1, all in channel group MTV w / WPG. The
      // tile's sums start from zero and join the running sums in fp32 (the
      // tensor cores' accumulation truncates, and carried over a whole split
      // its bias would show through the cancellation of code and zero terms).
      {
        float tacc[MTV][NT][4];
#pragma unroll
        for (int mt = 0; mt < MTV; ++mt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) tacc[mt][nt][i] = 0.0f;
        const uint32_t* vw = reinterpret_cast<const uint32_t*>(prv + Cfg::vc_off);
        const int wi0 = warp * MTV;
        const uint16_t* wt_g = wt_s + size_t(wi0 / WPG) * kTile * NCOL;
#pragma unroll
        for (int ks2 = 0; ks2 < kTile / 32; ++ks2) {
          uint32_t bw[NT][4];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) ldmatrix_x4_trans(bw[nt], wt_g + (32 * ks2 + lane) * NCOL + 8 * nt);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const int ta = 32 * ks2 + 16 * kk + 2 * tig;
            uint32_t wa0[MTV], wb0[MTV], wa1[MTV], wb1[MTV];
            if constexpr (MTV == 2) {
              const uint2 x0 = *reinterpret_cast<const uint2*>(vw + ta * NW + wi0);
              const uint2 x1 = *reinterpret_cast<const uint2*>(vw + (ta + 1) * NW + wi0);
              const uint2 x2 = *reinterpret_cast<const uint2*>(vw + (ta + 8) * NW + wi0);
              const uint2 x3 = *reinterpret_cast<const uint2*>(vw + (ta + 9) * NW + wi0);
              wa0[0] = x0.x; wa0[1] = x0.y; wb0[0] = x1.x; wb0[1] = x1.y;
              wa1[0] = x2.x; wa1[1] = x2.y; wb1[0] = x3.x; wb1[1] = x3.y;
            } else {
              wa0[0] = vw[ta * NW + wi0];
              wb0[0] = vw[(ta + 1) * NW + wi0];
              wa1[0] = vw[(ta + 8) * NW + wi0];
              wb1[0] = vw[(ta + 9) * NW + wi0];
            }
#pragma unroll
            for (int mt = 0; mt < MTV; ++mt) {
              const uint32_t a[4] = {unpack_codes(__byte_perm(wa0[mt], wb0[mt], selv0), mv, scv, ofv),
                                     unpack_codes(__byte_perm(wa0[mt], wb0[mt], selv1), mv, scv, ofv),
                                     unpack_codes(__byte_perm(wa1[mt], wb1[mt], selv0), mv, scv, ofv),
                                     unpack_codes(__byte_perm(wa1[mt], wb1[mt], selv1), mv, scv, ofv)};
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) mma16816(tacc[mt][nt], a, bw[nt][2 * kk], bw[nt][2 * kk + 1]);
            }
          }
        }
#pragma unroll
        for (int mt = 0; mt < MTV; ++mt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) oacc[mt][nt][i] += tacc[mt][nt][i];
      }
    }
    if (!have) break;
    __syncthreads();   // lg complete; the p.v of tile - 1 is done with its stage and wt
    if (tid == 0) issue(tile + kStages - 1);   // into the stage of tile - 1

    // ---- owner phase (thread = token): the centre term, online softmax
    const int t = tid;
    float lg[G];
    {
      load_vec<G>(lg_s + t * LS, lg);
      int idx;
      if constexpr (U16) idx = reinterpret_cast<const uint16_t*>(cur + Cfg::ix_off)[t];
      else idx = cur[Cfg::ix_off + t];
      idx = min(idx, M - 1);
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g] = (t < n) ? lg[g] + mus[g * M + idx] : -FLT_MAX;
    }
    uint32_t vszr[NG];
    uint32_t smaxb = 0;                              // largest |s_v| of the token, fp16 bits
    {
      const uint32_t* vsz = reinterpret_cast<const uint32_t*>(cur + Cfg::vs_off) + t * NG;
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        vszr[k] = (t < n) ? vsz[k] : 0u;
        smaxb = max(smaxb, vszr[k] & 0x7fffu);
      }
    }
    // Probabilities are taken against the running maximum, which may trail
    // the true one (p <= 2^8), and p s_v enters p.v scaled by 2^ev_acc with
    // |s_v| 2^ev_acc < 2^6, so p s_v 2^ev_acc < 2^14 keeps its fp16 halves
    // normal. The first tile, and a tile that breaks either bound, refresh
    // both from the block-wide tile maxima and rescale the running sums; the
    // exponents stay consistent because the partial sums and the running
    // maximum always move together.
    bool need = (tile == 0) || smaxb >= s_thr;
#pragma unroll
    for (int g = 0; g < G; ++g) need |= lg[g] > m_thr[g];
    if (__syncthreads_or(need)) {
      // (warp maxima by integer reductions of order-preserving keys)
      int* redi = reinterpret_cast<int*>(red);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int m = __reduce_max_sync(0xffffffffu, f2ord(lg[g]));
        if (lane == 0) redi[warp * G + g] = m;
      }
      {
        const int m = __reduce_max_sync(0xffffffffu, int(min(smaxb, 0x7bffu)));   // finite fp16
        if (lane == 0) redi[kWarps * G + warp] = m;
      }
      __syncthreads();
      int ev = ev_acc;
      {
        const int sb = max(max(redi[kWarps * G], redi[kWarps * G + 1]), max(redi[kWarps * G + 2], redi[kWarps * G + 3]));
        const float st = __half2float(__ushort_as_half(uint16_t(sb)));
        int se = 0;
        frexpf(st, &se);                             // st < 2^se
        if (st > 0.0f) ev = 6 - se;
      }
      float alpha[G];
      bool rescale = false;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float tmax = ord2f(max(max(redi[g], redi[G + g]), max(redi[2 * G + g], redi[3 * G + g])));
        const float m_new = fmaxf(m_run[g], tmax);
        alpha[g] = ex2(m_run[g] - m_new);
        rescale |= (m_new != m_run[g]);
        m_run[g] = m_new;
        m_thr[g] = m_new + 8.0f;
      }
      if (rescale || ev != ev_acc) {                 // uniform across the CTA
        const float f = ldexpf(1.0f, ev - ev_acc);
        float ac0 = f, ac1 = f;
#pragma unroll
        for (int j = 0; j < GP; ++j) {
          const f32x2 a2 = pk2(alpha[2 * j], alpha[min(2 * j + 1, G - 1)]);
          lsum2[j] = fmul2(lsum2[j], a2);
#pragma unroll
          for (int k = 0; k < NG; ++k) pz2[j][k] = fmul2(pz2[j][k], a2);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (g == hc0) ac0 = alpha[g] * f;
          if (g == hc1) ac1 = alpha[g] * f;
        }
        ev_acc = ev;
        vmul = ldexpf(1.0f, ev);
        const int e = 6 - ev;                        // s_thr = fp16 bits of 2^e
        s_thr = (e > 15) ? 0x8000u : (e >= -14) ? uint32_t(e + 15) << 10 : (e >= -24) ? 1u << (e + 24) : 0u;
#pragma unroll
        for (int mt = 0; mt < MTV; ++mt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            oacc[mt][nt][0] *= ac0; oacc[mt][nt][1] *= ac1;
            oacc[mt][nt][2] *= ac0; oacc[mt][nt][3] *= ac1;
          }
      }
    }
    // ---- probabilities; p s_v as (hi, lo) fp16 columns per group; sum p z_v
    {
      f32x2 pr2[GP];
#pragma unroll
      for (int j = 0; j < GP; ++j) {
        const float p0 = ex2(lg[2 * j] - m_run[2 * j]);                      // 0 for t >= n
        const int g1 = min(2 * j + 1, G - 1);
        const float p1 = (2 * j + 1 < G) ? ex2(lg[g1] - m_run[g1]) : 0.0f;
        pr2[j] = pk2(p0, p1);
        lsum2[j] = fadd2(lsum2[j], pr2[j]);
      }
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        const uint32_t sz = vszr[k];                 // 0 for t >= n
        const float sv = __half2float(__ushort_as_half(uint16_t(sz & 0xffff))) * vmul;
        const float zv = __half2float(__ushort_as_half(uint16_t(sz >> 16)));
        const f32x2 sv2 = pk2(sv, sv), zv2 = pk2(zv, zv);
        // columns as described for Cols: hi halves of the G heads, then lo halves
        uint32_t hw[NCOL / 2];
#pragma unroll
        for (int i = 0; i < NCOL / 2; ++i) hw[i] = 0u;
#pragma unroll
        for (int j = 0; j < GP; ++j) {
          pz2[j][k] = ffma2(pr2[j], zv2, pz2[j][k]);
          const float2 w = up2(fmul2(pr2[j], sv2));
          const __half2 hi = __floats2half2_rn(w.x, w.y);
          const float2 hf = __half22float2(hi);
          const float2 d = up2(fsub2(pk2(w.x, w.y), pk2(hf.x, hf.y)));
          const __half2 lo = __floats2half2_rn(d.x, d.y);
          const uint32_t hb = *reinterpret_cast<const uint32_t*>(&hi), lb = *reinterpret_cast<const uint32_t*>(&lo);
          if constexpr (G == 1) {
            hw[0] = (hb & 0xffffu) | (lb << 16);
          } else {
            hw[j] = hb;
            hw[(G >= 4 ? G / 2 : 1) + j] = lb;
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(wt_s + (size_t(k) * kTile + t) * NCOL);
#pragma unroll
        for (int q4 = 0; q4 < NT; ++q4) dst[q4] = make_uint4(hw[4 * q4], hw[4 * q4 + 1], hw[4 * q4 + 2], hw[4 * q4 + 3]);
      }
    }
    // no barrier here: the next iteration's first barrier orders the writes
    // of wt before the p.v that reads them
  }
  // the merge kernel (this grid's programmatic dependent) may be scheduled
  // now; it waits for this grid's completion before reading the partials
  asm volatile("griddepcontrol.launch_dependents;");
  if (aborted) {
    // a tile's copies did not arrive within the budget: report it, let the
    // copies still in flight land (bounded), and poison this split's output
    if (tid == 0) {
      atomicExch(p.err, 1);
      for (int j = tile; j < issued; ++j) mbar_wait(bar0 + 8 * (j % kStages), (j / kStages) & 1, p.budget);
    }
    float* dst = p.part + (size_t(bh) * p.splits + split) * G * (D + 2);
    for (int i = tid; i < G * (D + 2); i += kThreads) {
      const int c = i % (D + 2);
      dst[i] = (c == D + 1) ? 1.0f : (c == D ? 0.0f : __int_as_float(0x7fc00000));
    }
    return;
  }
  __syncthreads();

  // ---- reduce: p.v sums (one lane per channel and head); p z_v and p sums
  // over the owner threads (warp shuffles, then the 4 warps' partials)
  float* ofin = reinterpret_cast<float*>(smem);            // [G][D]
  float* zred = ofin + G * D;                               // [kWarps][G][NG]
  const float vinv = ldexpf(1.0f, -ev_acc);
#pragma unroll
  for (int mt = 0; mt < MTV; ++mt) {
    const int c0 = (warp * MTV + mt) * 16 + gid;
    combine_hi_lo<G, NT>(oacc[mt], tig, [&](int rs, int g, float v) { ofin[g * D + c0 + 8 * rs] = v * vinv; });
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      const float2 zz = up2(pz2[g / 2][k]);
      float z = (g & 1) ? zz.y : zz.x;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      if (lane == 0) zred[(warp * G + g) * NG + k] = z;
    }
    const float2 ll = up2(lsum2[g / 2]);
    float l = (g & 1) ? ll.y : ll.x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) red[warp * G + g] = l;
  }
  __syncthreads();
  float* dst = p.part + (size_t(bh) * p.splits + split) * G * (D + 2);
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, k = (i % D) / GS;
    float z = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) z += zred[(w * G + g) * NG + k];
    dst[g * (D + 2) + i % D] = ofin[i] + z;
  }
  if (tid < G) {
    float mr = m_run[0];
#pragma unroll
    for (int g = 1; g < G; ++g) if (tid == g) mr = m_run[g];
    dst[tid * (D + 2) + D] = mr;
    dst[tid * (D + 2) + D + 1] = red[tid] + red[G + tid] + red[2 * G + tid] + red[3 * G + tid];
  }
}

template <int D, int G, bool U16, int GS>
size_t split_smem(int M, int r) {
  using Cfg = DCfg<D, G, U16, GS>;
  return size_t(Cfg::stages_bytes(r)) + size_t(Cfg::tables_bytes(M, r));
}

template <int D, int G, bool U16, int GS>
cudaError_t launch_split(const SplitParams& sp, int B, cudaStream_t s) {
  const size_t smem = split_smem<D, G, U16, GS>(sp.M, sp.r);
  auto kern = sp.psac_fmt == 1 ? decode_split<D, G, U16, true, GS> : decode_split<D, G, U16, false, GS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(sp.splits, B * sp.H_kv);
  if (sp.wait_from == INT32_MAX) {
    kern<<<grid, kThreads, smem, s>>>(sp);
    return cudaGetLastError();
  }
  // programmatic dependent of the kernel before it on the stream
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, sp);
}

// the split kernel for G = H_q / H_kv query heads per KV head
template <int D, bool U16, int GS>
cudaError_t launch_g(int G, const SplitParams& sp, int B, cudaStream_t s) {
  switch (G) {
    case 1: return launch_split<D, 1, U16, GS>(sp, B, s);
    case 2: return launch_split<D, 2, U16, GS>(sp, B, s);
    case 4: return launch_split<D, 4, U16, GS>(sp, B, s);
    case 8: return launch_split<D, 8, U16, GS>(sp, B, s);
    default: return cudaErrorInvalidValue;
  }
}

// resident split CTAs per SM for this shape (occupancy query; 4 if unknown)
template <int D, int G, bool U16, int GS>
int ctas_per_sm_t(int M, int r) {
  const size_t smem = split_smem<D, G, U16, GS>(M, r);
  auto kern = decode_split<D, G, U16, false, GS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 4;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, smem) != cudaSuccess || n <= 0) return 4;
  return n;
}
template <int D, bool U16, int GS>
int ctas_per_sm_g(int G, int M, int r) {
  switch (G) {
    case 1: return ctas_per_sm_t<D, 1, U16, GS>(M, r);
    case 2: return ctas_per_sm_t<D, 2, U16, GS>(M, r);
    case 4: return ctas_per_sm_t<D, 4, U16, GS>(M, r);
    default: return ctas_per_sm_t<D, 8, U16, GS>(M, r);
  }
}

// Groups of 64 and 128 channels are instantiated in decode_groups.cu.
#define KV2_DSPLIT_GROUP_INSTANCES(X)                                   \
  X(64, false, 64) X(64, true, 64) X(128, false, 64) X(128, true, 64)   \
  X(128, false, 128) X(128, true, 128)
#define KV2_DSPLIT_EXTERN(D, U16, GS)                                                              \
  extern template cudaError_t launch_g<D, U16, GS>(int, const SplitParams&, int, cudaStream_t); \
  extern template int ctas_per_sm_g<D, U16, GS>(int, int, int);
KV2_DSPLIT_GROUP_INSTANCES(KV2_DSPLIT_EXTERN)

}  // namespace dsplit
}  // namespace kv2
