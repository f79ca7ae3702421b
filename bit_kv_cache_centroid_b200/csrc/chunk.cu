// chunk.cu — chunk attention for video world models on the 5th-generation
// tensor cores (tcgen05, accumulators in TMEM).
//
// Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
// World Models": a chunk of new latent frames attends to the whole quantized
// history (keys = centre + INT2 residual, "1. QSAC") with the principal-subspace
// compensation of "2. PSAC" added to every score, plus its own keys/values,
// block-causal by latent frame. Thousands of queries per call make Q K^T and
// P V dense contractions, so they run on tcgen05.mma:
//
//   S  = Q . Khat^T           fp16 x fp16, Khat = fp16(code s + fp16(z + mu[idx]))
//                             (Q scaled per row by a power of two, undone in
//                             the softmax)
//      + U . A^T              fp16 x fp16, U = fp16(q P), A = the stored fp16
//                             PSAC coefficients (K = 16 extra contraction columns)
//   O += P . Vhat             fp16 x fp16, Vhat = fp16(code s + z), P = fp16
//
// One CTA (17 warps) serves two 128-query tiles of one (batch, query head);
// every dequantized key/value tile feeds both. Warp roles:
//   warps 0-3, 4-7  softmax of query tile 0 / 1 (thread = query row = TMEM lane):
//                   S from TMEM, online softmax, P written back into the S
//                   columns as fp16 pairs, O rescaled in TMEM when a row max grows;
//   warps 8-15      producer (two threads per key row, 64 channels each):
//                   packed key/value tiles -> 128-byte-swizzled fp16 Khat /
//                   Vhat and PSAC tiles in a 2-stage ring (fp16x2 arithmetic);
//   warp 16         issues the MMAs (one thread) and owns the TMEM allocation.
// TMEM (512 columns): S0, S1, O0, O1. The PV MMA reads P straight from TMEM.
// mbarriers: kv_full/kv_empty (ring), s_full, p_full, o_done (per query tile).
// A commit covers every earlier MMA of the issuing thread, so "S of tile j
// done" also means "P.V of tile j-1 done": the softmax may then overwrite P
// and rescale O.
//
// Every wait is bounded by an SM-clock budget; on expiry the waiting thread
// raises a CTA-wide abort flag that ends every other wait, the kernel records
// 1 in the workspace's first word, waits (bounded) for its MMAs in flight,
// frees its TMEM and returns.
#include <cfloat>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "mbarrier.cuh"
#include "umma.cuh"

namespace kv2 {
namespace {

constexpr int kRows = 128;        // queries per query tile (= TMEM lanes)
constexpr int kKeys = 128;        // keys per tile
constexpr int kD = 128;
constexpr int kThreads = 544;     // 17 warps
// floats per partial output row of a key-range piece: kD sums, the running
// maximum, the running sum, padded so every row starts on 16 bytes
constexpr int kPartRow = kD + 4;
constexpr int kProdWarp0 = 8, kProdThreads = 256, kMmaWarp = 16;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_Q0 = 0;           // Q tile 0 [2 k-chunks][128 rows][128 B], SW128, K-major
constexpr uint32_t OFF_Q1 = 32768;       // Q tile 1
constexpr uint32_t OFF_U0 = 65536;       // U = fp16(qP) tile 0 [16 row groups][2][8 rows][16 B]
constexpr uint32_t OFF_U1 = 69632;       // U tile 1
constexpr uint32_t OFF_STAGE = 73728;    // 2 stages of STAGE_BYTES
constexpr uint32_t ST_K = 0;             // Khat [2 k-chunks][128 keys][128 B], SW128, K-major
constexpr uint32_t ST_V = 32768;         // Vhat [2 n-blocks][128 keys][128 B], SW128, MN-major
constexpr uint32_t ST_A = 65536;         // A    [16 key groups][2][8 keys][16 B]
constexpr uint32_t STAGE_BYTES = 69632;
constexpr uint32_t OFF_BAR = OFF_STAGE + 2 * STAGE_BYTES;   // 212992
constexpr uint32_t SMEM_USED = OFF_BAR + 128;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;
// barrier slots (8 bytes each) from OFF_BAR
constexpr uint32_t B_KV_FULL = 0, B_KV_EMPTY = 16, B_S_FULL = 32, B_P_FULL = 48, B_O_DONE = 64, B_FINAL = 80,
                   B_NEVER = 88, B_TMEM_SLOT = 96, B_ABORT = 100;

constexpr uint32_t kTmemCols = 512;

// ---------------------------------------------------------------------------
// PTX wrappers (sm_100a)
// ---------------------------------------------------------------------------

constexpr uint32_t IDESC_QK = make_idesc(0, 0, 0, kKeys, kRows);
constexpr uint32_t IDESC_UA = make_idesc(0, 0, 0, kKeys, kRows);
constexpr uint32_t IDESC_PV = make_idesc(0, 0, 1, kD, kRows);

// byte offset of 16-byte chunk `c` (0, 1) of row `row` in a no-swizzle
// [row/8][2][8][16 B] operand tile (K = 16 columns of 16-bit values)
__device__ __forceinline__ uint32_t nosw_off(int row, int c) {
  return uint32_t((row >> 3) * 256 + c * 128 + (row & 7) * 16);
}

// two fp32 -> packed bf16x2 / f16x2 (one paired conversion, round to nearest even)
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  const __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}


// d = a * b + c on two fp16 lanes; d = a + b
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The codes of channels 2i, 2i+1 of an 8-channel chunk sit at bits 4i and
// 4i+2 of its 16-bit code field. With the field in both halves of x (and x
// shifted right by 8 for i >= 2), (x & mask) | 0x6400 puts the fp16 numbers
// 1024 + code * 16^i' in the low half and 1024 + 4 code * 16^i' in the high
// half (i' = i mod 2, bits within the fp16 mantissa); one fp16 fma with the
// exact constants below leaves the two codes (exact small integers).
__device__ __forceinline__ uint32_t code_pair_f16(uint32_t x, uint32_t x8, int i) {
  const uint32_t src = (i < 2) ? x : x8;
  const int ip = i & 1;
  const uint32_t mask = (3u << (4 * ip)) | (3u << (16 + 4 * ip + 2));
  const uint32_t scale = ip ? 0x24002C00u : 0x34003C00u;    // {1/16, 1/64} : {1, 1/4}
  const uint32_t offset = ip ? 0xCC00D400u : 0xDC00E400u;   // {-64, -16} : {-1024, -256}
  return hfma2((src & mask) | 0x64006400u, scale, offset);
}
// the 16-bit code field `lc & 1` of word w in both halves of a word
__device__ __forceinline__ uint32_t field_both(uint32_t w, int lc) {
  return __byte_perm(w, 0u, (lc & 1) ? 0x3232u : 0x1010u);
}

struct ChunkParams {
  const uint32_t* k_code;
  const uint32_t* v_code;
  const uint32_t* k_sz;
  const uint32_t* v_sz;
  const void* cidx;
  const uint16_t* psac;
  const uint16_t* cent;
  const float* P;
  const uint16_t* Q;
  const uint16_t* Ks;
  const uint16_t* Vs;
  void* out;
  int* err;
  int B, H_kv, H_q, M, r, cap, len, Nq, F, out_dtype;
  float scale_log2;
  unsigned long long budget;
  int force_timeout;
  // work decomposition: QP query-tile pairs per (batch, head); the first
  // n_full units run whole, each later unit as `pieces` ranges of key tiles
  // whose partial results (part) are merged by chunk_merge
  int QP, n_full, pieces;
  float* part;            // [split units][pieces][2][kRows][kPartRow]
  int psac_fmt;           // 0: fp16 coefficients; 1: int8 codes + fp16 scale per token
  const uint16_t* psac_scale;
  const int32_t* table;   // paged cache: block table [B][cap / page] (null: contiguous)
  int page;
};

// ---------------------------------------------------------------------------
// operand producers (thread = one row)
// ---------------------------------------------------------------------------

// Packed fields of half a cached token row (channels 64*half .. 64*half+63),
// loaded one tile ahead of their use.
struct RawHalf {
  uint4 kw, vw;       // 4 code words each
  uint2 ksz, vsz;     // the (fp16 scale | fp16 zero << 16) words of channels
                      // 64*half .. +31 and 64*half+32 .. +63
  int idx;            // centroid id
};

// GS: channels per (scale, zero) group (32, 64 or 128): a row holds 128 / GS
// scale/zero words, and both 32-channel quarters of a half share one word
// when GS > 32
template <int GS>
__device__ __forceinline__ void load_raw_half(const ChunkParams& p, size_t slot, int half, RawHalf& r) {
  r.kw = *reinterpret_cast<const uint4*>(p.k_code + slot * 8 + half * 4);
  r.vw = *reinterpret_cast<const uint4*>(p.v_code + slot * 8 + half * 4);
  if constexpr (GS == 32) {
    r.ksz = *reinterpret_cast<const uint2*>(p.k_sz + slot * 4 + half * 2);
    r.vsz = *reinterpret_cast<const uint2*>(p.v_sz + slot * 4 + half * 2);
  } else {
    constexpr int NG = kD / GS;
    const uint32_t k = p.k_sz[slot * NG + (half * 64) / GS], v = p.v_sz[slot * NG + (half * 64) / GS];
    r.ksz = make_uint2(k, k);
    r.vsz = make_uint2(v, v);
  }
  r.idx = (p.M <= 256) ? int(static_cast<const uint8_t*>(p.cidx)[slot])
                       : int(static_cast<const uint16_t*>(p.cidx)[slot]);
}

// the PSAC row of a cached token (fp16, zero-padded to 16 coefficients);
// loaded with the centroid half-row, not with the prefetched fields
__device__ __forceinline__ void load_psac(const ChunkParams& p, size_t slot, uint4& a0, uint4& a1) {
  a0 = make_uint4(0, 0, 0, 0);
  a1 = make_uint4(0, 0, 0, 0);
  if (p.psac_fmt == 1) {
    // int8 codes (r = 8 or 16) and the token's scale: fp16(code * scale)
    if (p.r == 0) return;
    const float sc = __half2float(__ushort_as_half(p.psac_scale[slot]));
    const int8_t* q8 = reinterpret_cast<const int8_t*>(p.psac) + slot * p.r;
    uint32_t w[4];
    const uint2 lo = *reinterpret_cast<const uint2*>(q8);
    w[0] = lo.x; w[1] = lo.y;
    if (p.r >= 16) {
      const uint2 hi = *reinterpret_cast<const uint2*>(q8 + 8);
      w[2] = hi.x; w[3] = hi.y;
    } else {
      w[2] = w[3] = 0u;
    }
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t two = (w[i >> 1] >> (16 * (i & 1))) & 0xffffu;
      h[i] = pack_f16(float(int8_t(two & 0xff)) * sc, float(int8_t(two >> 8)) * sc);
    }
    a0 = make_uint4(h[0], h[1], h[2], h[3]);
    a1 = make_uint4(h[4], h[5], h[6], h[7]);
    return;
  }
  if (p.r >= 8) a0 = *reinterpret_cast<const uint4*>(p.psac + slot * p.r);
  if (p.r >= 16) a1 = *reinterpret_cast<const uint4*>(p.psac + slot * p.r + 8);
}

// half a Khat row and half a Vhat row (both fp16) from the packed fields and
// the centroid half-row m4; half 0 also writes the PSAC row. In fp16
// arithmetic: Khat = fma(code, s, z + mu), Vhat = fma(code, s, z), codes exact.
__device__ void dequant_cache_half(const RawHalf& r, const uint4 (&m4)[8], const uint4& a0, const uint4& a1, int row,
                                   int half, uint8_t* stage) {
  const uint32_t kw[4] = {r.kw.x, r.kw.y, r.kw.z, r.kw.w};
  const uint32_t vw[4] = {r.vw.x, r.vw.y, r.vw.z, r.vw.w};
  const uint32_t ksz[2] = {r.ksz.x, r.ksz.y};
  const uint32_t vsz[2] = {r.vsz.x, r.vsz.y};
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const uint32_t ks2 = __byte_perm(ksz[g], 0u, 0x1010u), kz2 = __byte_perm(ksz[g], 0u, 0x3232u);
    const uint32_t vs2 = __byte_perm(vsz[g], 0u, 0x1010u), vz2 = __byte_perm(vsz[g], 0u, 0x3232u);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {                // 8 channels per chunk
      const int c16 = half * 8 + g * 4 + cc;         // chunk index within the row
      const int lc = g * 4 + cc;                      // chunk index within this half
      const uint32_t mu[4] = {m4[lc].x, m4[lc].y, m4[lc].z, m4[lc].w};
      const uint32_t kx = field_both(kw[lc >> 1], lc), vx = field_both(vw[lc >> 1], lc);
      const uint32_t kx8 = kx >> 8, vx8 = vx >> 8;
      uint32_t kb[4], vb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kb[i] = hfma2(code_pair_f16(kx, kx8, i), ks2, hadd2(kz2, mu[i]));
        vb[i] = hfma2(code_pair_f16(vx, vx8, i), vs2, vz2);
      }
      *reinterpret_cast<uint4*>(stage + ST_K + sw128_off(row, c16)) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
      *reinterpret_cast<uint4*>(stage + ST_V + sw128_off(row, c16)) = make_uint4(vb[0], vb[1], vb[2], vb[3]);
    }
  }
  if (half == 0) {
    *reinterpret_cast<uint4*>(stage + ST_A + nosw_off(row, 0)) = a0;
    *reinterpret_cast<uint4*>(stage + ST_A + nosw_off(row, 1)) = a1;
  }
}

// eight bf16 values -> eight fp16 values (round to nearest even)
__device__ __forceinline__ uint4 bf16x8_to_f16(const uint4& v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = pack_f16(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// chunk token -> half a Khat row and half a Vhat row (bf16 -> fp16)
__device__ void copy_self_half(const uint16_t* krow, const uint16_t* vrow, int row, int half, uint8_t* stage) {
  const uint4* k4 = reinterpret_cast<const uint4*>(krow) + half * 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(vrow) + half * 8;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int c16 = half * 8 + c;
    *reinterpret_cast<uint4*>(stage + ST_K + sw128_off(row, c16)) = bf16x8_to_f16(__ldg(k4 + c));
    *reinterpret_cast<uint4*>(stage + ST_V + sw128_off(row, c16)) = bf16x8_to_f16(__ldg(v4 + c));
  }
}

__device__ __forceinline__ void zero_half(uint8_t* tile, int row, int half) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(tile + sw128_off(row, half * 8 + c)) = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------------------
template <int GS>
__global__ void __launch_bounds__(kThreads, 1) chunk_attn_kernel(ChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar = sb + OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + B_TMEM_SLOT);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_BAR + B_ABORT);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // work item: a whole unit (pair of query tiles of one (batch, head)), or,
  // for the units of the last wave, one of p.pieces ranges of its key tiles
  int unit = blockIdx.x, piece = -1;
  if (unit >= p.n_full) {
    const int e = unit - p.n_full;
    unit = p.n_full + e / p.pieces;
    piece = e % p.pieces;
  }
  const int qt = unit % p.QP, hq = (unit / p.QP) % p.H_q, b = unit / (p.QP * p.H_q);
  const int G = p.H_q / p.H_kv, h = hq / G;
  const int q0 = qt * 2 * kRows;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + B_KV_FULL + 8 * i, kProdThreads);   // one arrival per producer thread
      mbar_init(bar + B_KV_EMPTY + 8 * i, 1);         // MMA commit
      mbar_init(bar + B_S_FULL + 8 * i, 1);           // MMA commit
      mbar_init(bar + B_P_FULL + 8 * i, kRows);       // one arrival per softmax thread
      mbar_init(bar + B_O_DONE + 8 * i, 1);           // MMA commit
    }
    mbar_init(bar + B_FINAL, 1);
    mbar_init(bar + B_NEVER, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    *abort = 0;
  }
  if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), kTmemCols);

  // ---- Q tiles (fp16, SW128 K-major) and U = fp16(q P) (no swizzle, K = 16),
  // each row scaled by 2^qexp with max(|q|, |u|) 2^qexp below 2^15: fp16 range
  // whatever the bf16 input (the bf16 -> fp16 conversion of q exact); the
  // softmax thread of the row undoes the factor in its score scale
  int qexp = 0;
  if (warp < 8) {
    const int x = warp >> 2, row = tid - x * kRows;
    const int qi = q0 + x * kRows + row;
    const bool q_ok = qi < p.Nq;
    uint8_t* qtile = smem + (x ? OFF_Q1 : OFF_Q0);
    const uint4* src = reinterpret_cast<const uint4*>(p.Q + ((size_t(b) * p.Nq + min(qi, p.Nq - 1)) * p.H_q + hq) * kD);
    uint32_t amax = 0;                                // largest |q| of the row, as bf16 bits in both halves
    float u[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) u[j] = 0.0f;
    const float* Ph = p.P + size_t(h) * kD * p.r;
#pragma unroll 1
    for (int c16 = 0; c16 < 16; ++c16) {
      const uint4 v = q_ok ? __ldg(src + c16) : make_uint4(0, 0, 0, 0);
      amax = __vmaxu2(amax, __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                                     __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu)));
      if (p.r > 0) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float qc = (i & 1) ? __uint_as_float(w[i >> 1] & 0xffff0000u) : __uint_as_float(w[i >> 1] << 16);
          const float* Prow = Ph + size_t(c16 * 8 + i) * p.r;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < p.r) u[j] = fmaf(qc, __ldg(Prow + j), u[j]);
        }
      }
    }
    float rmax = __uint_as_float(max(amax & 0xffffu, amax >> 16) << 16);
#pragma unroll
    for (int j = 0; j < 16; ++j) rmax = fmaxf(rmax, fabsf(u[j]));
    if (rmax > 0.0f && rmax < 1e30f) {
      int e = 0;
      frexpf(rmax, &e);                               // rmax < 2^e
      qexp = min(max(15 - e, -64), 64);
    }
    const float qmul = ldexpf(1.0f, qexp);
#pragma unroll 1
    for (int c16 = 0; c16 < 16; ++c16) {
      const uint4 v = q_ok ? __ldg(src + c16) : make_uint4(0, 0, 0, 0);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t hq4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        hq4[i] = pack_f16(__uint_as_float(w[i] << 16) * qmul, __uint_as_float(w[i] & 0xffff0000u) * qmul);
      *reinterpret_cast<uint4*>(qtile + sw128_off(row, c16)) = make_uint4(hq4[0], hq4[1], hq4[2], hq4[3]);
    }
    uint32_t uw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) uw[j] = pack_f16(u[2 * j] * qmul, u[2 * j + 1] * qmul);
    uint8_t* utile = smem + (x ? OFF_U1 : OFF_U0);
    *reinterpret_cast<uint4*>(utile + nosw_off(row, 0)) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
    *reinterpret_cast<uint4*>(utile + nosw_off(row, 1)) = make_uint4(uw[4], uw[5], uw[6], uw[7]);
  }
  fence_proxy_async();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const int n_cache = (p.len + kKeys - 1) / kKeys;
  const int last_q = min(q0 + 2 * kRows, p.Nq) - 1;
  const int self_len = min(p.Nq, (last_q / p.F + 1) * p.F);
  const int n_self = (self_len + kKeys - 1) / kKeys;
  const int n_tiles = n_cache + n_self;
  const int jA = piece < 0 ? 0 : piece * n_tiles / p.pieces;          // key tiles [jA, jB)
  const int jB = piece < 0 ? n_tiles : (piece + 1) * n_tiles / p.pieces;
  const int nloc = jB - jA;

  if (warp == kMmaWarp) {
    // ================= MMA issue (one thread) =================
    // Shared-memory descriptors are built once: an operand's address field
    // is its address / 16 (14 bits, no carry for any address of the CTA's
    // shared memory), so a k-step's descriptor is the base plus its offset
    // / 16 (one 64-bit add instead of the full encoding per MMA).
    const uint64_t dQ0 = make_sdesc(sb + OFF_Q0, 16, 1024, kLayoutSW128);
    const uint64_t dQ1 = make_sdesc(sb + OFF_Q1, 16, 1024, kLayoutSW128);
    const uint64_t dU0 = make_sdesc(sb + OFF_U0, 128, 256, kLayoutNone);
    const uint64_t dU1 = make_sdesc(sb + OFF_U1, 128, 256, kLayoutNone);
    const uint64_t dK0 = make_sdesc(sb + OFF_STAGE + ST_K, 16, 1024, kLayoutSW128);
    const uint64_t dA0 = make_sdesc(sb + OFF_STAGE + ST_A, 128, 256, kLayoutNone);
    const uint64_t dV0 = make_sdesc(sb + OFF_STAGE + ST_V, 16384, 1024, kLayoutSW128);
    const uint64_t dStage = uint64_t(STAGE_BYTES >> 4);     // the second stage's offset
    for (int jj = 0; jj < nloc; ++jj) {
      const int j = jA + jj;
      const int s = jj & 1;
      const uint32_t use = uint32_t(jj >> 1);
      const bool cache = j < n_cache;
      if (p.force_timeout && jj == 0 && !mbar_wait_or_abort(bar + B_NEVER, 0, p.budget, abort)) break;
      if (!mbar_wait_or_abort(bar + B_KV_FULL + 8 * s, use & 1, p.budget, abort)) break;
      fence_after_sync();
      bool ok = true;
      for (int x = 0; x < 2 && ok; ++x) {
        if (jj > 0 && !mbar_wait_or_abort(bar + B_O_DONE + 8 * x, (jj - 1) & 1, p.budget, abort)) { ok = false; break; }
        fence_after_sync();
        if (lane == 0) {
          const uint32_t tS = tmem + x * kKeys;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t off = uint64_t(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_f16(tS, (x ? dQ1 : dQ0) + off, dK0 + s * dStage + off, IDESC_QK, kk > 0);
          }
          if (cache && p.r > 0) mma_f16(tS, x ? dU1 : dU0, dA0 + s * dStage, IDESC_UA, 1);
          mma_commit(bar + B_S_FULL + 8 * x);
        }
        __syncwarp();
      }
      if (!ok) break;
      for (int x = 0; x < 2 && ok; ++x) {
        if (!mbar_wait_or_abort(bar + B_P_FULL + 8 * x, jj & 1, p.budget, abort)) { ok = false; break; }
        fence_after_sync();
        if (lane == 0) {
          const uint32_t tP = tmem + x * kKeys, tO = tmem + 2 * kKeys + x * kD;
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            mma_f16_tmem_a(tO, tP + kk * 8, dV0 + s * dStage + uint64_t(kk * 2048 >> 4), IDESC_PV, (jj > 0 || kk > 0));
          mma_commit(bar + B_O_DONE + 8 * x);
          if (x == 1) mma_commit(bar + B_KV_EMPTY + 8 * s);   // stage free once every MMA on it is done
        }
        __syncwarp();
      }
      if (!ok) break;
    }
  } else if (warp >= kProdWarp0) {
    // ================= producer: packed tiles -> operand tiles =================
    // The packed fields of cached tile j+1 are loaded while tile j is
    // dequantized; the centroid half-row is fetched as soon as its id is known.
    // lanes 8q..8q+7 of a producer warp take 8 consecutive rows and one half:
    // their 16-byte stores then fall on 8 distinct swizzled bank groups
    const int pt = tid - kProdWarp0 * 32;
    const int row = (pt >> 5) * 16 + (pt & 7) + 8 * ((pt >> 4) & 1), half = (pt >> 3) & 1;
    auto slot_of = [&](int t) { return cache_slot(p.table, p.page, p.H_kv, p.cap, b, h, t); };
    const uint4* cent4 = reinterpret_cast<const uint4*>(p.cent) + size_t(h) * p.M * (kD / 8) + half * 8;
    RawHalf raw;
    bool raw_ok = nloc > 0 && jA < n_cache && row < min(kKeys, p.len - jA * kKeys);
    if (raw_ok) load_raw_half<GS>(p, slot_of(jA * kKeys + row), half, raw);
    for (int jj = 0; jj < nloc; ++jj) {
      const int j = jA + jj;
      const int s = jj & 1;
      const uint32_t use = uint32_t(jj >> 1);
      const bool cache = j < n_cache;
      const int k0 = cache ? j * kKeys : (j - n_cache) * kKeys;
      const int kvalid = cache ? min(kKeys, p.len - k0) : min(kKeys, self_len - k0);
      uint4 m4[8], a0, a1;
      if (cache && raw_ok) {
        const uint4* mu = cent4 + size_t(min(raw.idx, p.M - 1)) * (kD / 8);
#pragma unroll
        for (int c = 0; c < 8; ++c) m4[c] = __ldg(mu + c);
        if (half == 0) load_psac(p, slot_of(j * kKeys + row), a0, a1);
      }
      RawHalf next;
      const int jn = j + 1;
      const bool next_ok = jn < jB && jn < n_cache && row < min(kKeys, p.len - jn * kKeys);
      if (next_ok) load_raw_half<GS>(p, slot_of(jn * kKeys + row), half, next);
      if (use >= 1 && !mbar_wait_or_abort(bar + B_KV_EMPTY + 8 * s, (use - 1) & 1, p.budget, abort)) break;
      uint8_t* stage = smem + OFF_STAGE + s * STAGE_BYTES;
      if (row < kvalid) {
        if (cache) {
          dequant_cache_half(raw, m4, a0, a1, row, half, stage);
        } else {
          const size_t srow = (size_t(b) * p.Nq + k0 + row) * p.H_kv + h;
          copy_self_half(p.Ks + srow * kD, p.Vs + srow * kD, row, half, stage);
        }
      } else {
        zero_half(stage + ST_K, row, half);
        zero_half(stage + ST_V, row, half);
        if (half == 0) {
          *reinterpret_cast<uint4*>(stage + ST_A + nosw_off(row, 0)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(stage + ST_A + nosw_off(row, 1)) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async();
      mbar_arrive(bar + B_KV_FULL + 8 * s);
      raw = next;
      raw_ok = next_ok;
    }
  } else {
    // ================= softmax of query tile x =================
    const int x = warp >> 2, row = tid - x * kRows;
    const int qi = q0 + x * kRows + row;
    const bool q_ok = qi < p.Nq;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + x * kKeys + lane_base, tO = tmem + 2 * kKeys + x * kD + lane_base;
    const int my_self_lim = min(self_len, (min(qi, p.Nq - 1) / p.F + 1) * p.F);
    const float sc_row = p.scale_log2 * ldexpf(1.0f, -qexp);   // the row's Q carries 2^qexp
    float m_run = -INFINITY, l_run = 0.0f;
    bool done = true;
    for (int jj = 0; jj < nloc; ++jj) {
      const int j = jA + jj;
      if (!mbar_wait_or_abort(bar + B_S_FULL + 8 * x, jj & 1, p.budget, abort)) { done = false; break; }
      fence_after_sync();
      const bool cache = j < n_cache;
      const int k0 = cache ? j * kKeys : (j - n_cache) * kKeys;
      const int lim = cache ? min(kKeys, p.len - k0) : (my_self_lim - k0);
      const bool full = __all_sync(0xffffffffu, lim >= kKeys);   // no masked key in the warp's rows
      // row max and row sum with 8 independent partial accumulators (short
      // dependency chains on the critical S -> softmax -> P.V path)
      float mpart[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mpart[i] = -INFINITY;
#pragma unroll 1
      for (int c0 = 0; c0 < kKeys; c0 += 64) {      // 64 columns per wait
        uint32_t ra[32], rb[32];
        tmem_ld32_issue(tS + c0, ra);
        tmem_ld32_issue(tS + c0 + 32, rb);
        tmem_wait_ld(ra);
        tmem_anchor(rb);
        if (full) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            mpart[(i >> 1) & 7] = fmax3(mpart[(i >> 1) & 7], __uint_as_float(ra[i]), __uint_as_float(ra[i + 1]));
            mpart[(i >> 1) & 7] = fmax3(mpart[(i >> 1) & 7], __uint_as_float(rb[i]), __uint_as_float(rb[i + 1]));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (c0 + i < lim) mpart[i & 7] = fmaxf(mpart[i & 7], __uint_as_float(ra[i]));
            if (c0 + 32 + i < lim) mpart[i & 7] = fmaxf(mpart[i & 7], __uint_as_float(rb[i]));
          }
        }
      }
      const float mt = fmaxf(fmaxf(fmaxf(mpart[0], mpart[1]), fmaxf(mpart[2], mpart[3])),
                             fmaxf(fmaxf(mpart[4], mpart[5]), fmaxf(mpart[6], mpart[7])));
      const float m_new = fmaxf(m_run, mt * sc_row);
      const float alpha = (m_new == -INFINITY) ? 1.0f : ex2(m_run - m_new);
      f32x2 spart[4];                                   // 8 partial sums as 4 pairs
#pragma unroll
      for (int i = 0; i < 4; ++i) spart[i] = 0ull;
      const f32x2 sc2 = pk2(sc_row, sc_row), nm2 = pk2(-m_new, -m_new);
#pragma unroll 1
      for (int c0 = 0; c0 < kKeys; c0 += 32) {
        float v[32];
        tmem_ld32(tS + c0, v);
        uint32_t pw[16];
        if (full) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 x = up2(ffma2(pk2(v[i], v[i + 1]), sc2, nm2));
            const float p0 = ex2(x.x), p1 = ex2(x.y);
            spart[(i >> 1) & 3] = fadd2(spart[(i >> 1) & 3], pk2(p0, p1));
            pw[i / 2] = pack_f16(p0, p1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 x = up2(ffma2(pk2(v[i], v[i + 1]), sc2, nm2));
            const float p0 = (c0 + i < lim) ? ex2(x.x) : 0.0f;
            const float p1 = (c0 + i + 1 < lim) ? ex2(x.y) : 0.0f;
            spart[(i >> 1) & 3] = fadd2(spart[(i >> 1) & 3], pk2(p0, p1));
            pw[i / 2] = pack_f16(p0, p1);
          }
        }
        tmem_st16(tS + c0 / 2, pw);       // P over S columns already read (no wait: later loads read other columns)
      }
      tmem_wait_st();
      const float2 s01 = up2(fadd2(spart[0], spart[1])), s23 = up2(fadd2(spart[2], spart[3]));
      const float lsum = (s01.x + s23.x) + (s01.y + s23.y);
      l_run = l_run * alpha + lsum;
      m_run = m_new;
      if (__any_sync(0xffffffffu, jj > 0 && alpha != 1.0f)) {   // warp-wide TMEM access
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
          float v[32];
          tmem_ld32(tO + c0, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(tO + c0, v);
        }
        tmem_wait_st();
      }
      fence_before_sync();
      mbar_arrive(bar + B_P_FULL + 8 * x);
    }
    if (piece >= 0) {
      // a piece: unnormalised output rows, running maximum and sum for the merge
      float* part = p.part + ((size_t(unit - p.n_full) * p.pieces + piece) * 2 + x) * kRows * kPartRow +
                    size_t(row) * kPartRow;
      const bool have = done && nloc > 0 &&
                        mbar_wait_or_abort(bar + B_O_DONE + 8 * x, (nloc - 1) & 1, p.budget, abort);
      if (have) {
        fence_after_sync();
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
          float v[32];
          tmem_ld32(tO + c0, v);          // every lane: warp-wide TMEM load
          float4* dst = reinterpret_cast<float4*>(part + c0);
#pragma unroll
          for (int i = 0; i < 32; i += 4) dst[i / 4] = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
        part[kD] = m_run;
        part[kD + 1] = l_run;
      } else if (nloc == 0 && done) {
        for (int c = 0; c < kD; ++c) part[c] = 0.0f;
        part[kD] = -INFINITY;
        part[kD + 1] = 0.0f;
      } else {                             // the pipeline gave up: poison the merged rows
        for (int c = 0; c < kD; ++c) part[c] = __int_as_float(0x7fc00000);
        part[kD] = 0.0f;
        part[kD + 1] = 1.0f;
      }
    } else if (done && mbar_wait_or_abort(bar + B_O_DONE + 8 * x, (n_tiles - 1) & 1, p.budget, abort)) {
      fence_after_sync();
      const float inv = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
      const size_t obase = ((size_t(b) * p.Nq + min(qi, p.Nq - 1)) * p.H_q + hq) * kD;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float v[32];
        tmem_ld32(tO + c0, v);            // every lane: warp-wide TMEM load
        if (!q_ok) continue;
        if (p.out_dtype == KV2_OUT_F32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + c0);
#pragma unroll
          for (int i = 0; i < 32; i += 4) dst[i / 4] = make_float4(v[i] * inv, v[i + 1] * inv, v[i + 2] * inv, v[i + 3] * inv);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + obase + c0);
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            dst[i / 8] = make_uint4(pack_bf16(v[i] * inv, v[i + 1] * inv), pack_bf16(v[i + 2] * inv, v[i + 3] * inv),
                                    pack_bf16(v[i + 4] * inv, v[i + 5] * inv), pack_bf16(v[i + 6] * inv, v[i + 7] * inv));
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    if (*abort) {
      if (lane == 0) {
        atomicExch(p.err, 1);
        mma_commit(bar + B_FINAL);                       // wait (bounded) for MMAs in flight
      }
      __syncwarp();
      mbar_wait(bar + B_FINAL, 0, 1ull << 32);
    }
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merges the pieces of each split unit: log-sum-exp of the partial rows
// (one block per query row of the unit, one thread per channel).
__global__ void chunk_merge(const float* __restrict__ part, int n_full, int pieces, int QP, int H_q, int Nq,
                            void* out, int out_dtype) {
  const int su = blockIdx.x / (2 * kRows), r2 = blockIdx.x % (2 * kRows);
  const int unit = n_full + su;
  const int qt = unit % QP, hq = (unit / QP) % H_q, b = unit / (QP * H_q);
  const int qi = qt * 2 * kRows + r2;
  if (qi >= Nq) return;
  const int c = threadIdx.x;
  const size_t stride = size_t(2) * kRows * kPartRow;      // between pieces
  const float* base = part + (size_t(su) * pieces * 2 + r2 / kRows) * kRows * kPartRow + size_t(r2 % kRows) * kPartRow;
  float m = -INFINITY;
  for (int pc = 0; pc < pieces; ++pc) {
    const float* pr = base + pc * stride;
    if (pr[kD + 1] > 0.0f) m = fmaxf(m, pr[kD]);
  }
  float o = 0.0f, l = 0.0f;
  for (int pc = 0; pc < pieces; ++pc) {
    const float* pr = base + pc * stride;
    const float lp = pr[kD + 1];
    if (!(lp > 0.0f)) continue;
    const float f = exp2f(pr[kD] - m);
    o = fmaf(f, pr[c], o);
    l = fmaf(f, lp, l);
  }
  const float v = (l > 0.0f) ? o / l : 0.0f;
  const size_t oi = ((size_t(b) * Nq + qi) * H_q + hq) * kD + c;
  if (out_dtype == KV2_OUT_F32) static_cast<float*>(out)[oi] = v;
  else static_cast<__nv_bfloat16*>(out)[oi] = __float2bfloat16_rn(v);
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Units beyond the last whole wave are split into ranges of key tiles so the
// last wave fills the GPU: split = units mod SMs, pieces = SMs / split (at
// most max_pieces); no split when that leaves fewer than 2 pieces.
struct ChunkPlan {
  int QP, n_units, split, pieces;
};
ChunkPlan plan_chunk(int B, int H_q, int Nq, int max_pieces) {
  ChunkPlan pl{};
  pl.QP = (Nq + 2 * kRows - 1) / (2 * kRows);
  pl.n_units = pl.QP * H_q * B;
  const int sms = sm_count();
  pl.split = 0;
  pl.pieces = 1;
  const int rem = pl.n_units % sms;
  if (pl.n_units > sms && rem > 0) {
    const int k = min(sms / rem, max_pieces);
    if (k >= 2) {
      pl.split = rem;
      pl.pieces = k;
    }
  }
  return pl;
}

constexpr size_t kChunkWsHeader = 256;

}  // namespace

size_t chunk_workspace_bytes(const kv2_cache& c, int H_q, int Nq) {
  const ChunkPlan pl = plan_chunk(c.B, H_q, Nq, 1 << 20);
  return kChunkWsHeader + size_t(pl.split) * pl.pieces * 2 * kRows * kPartRow * 4;
}

cudaError_t launch_chunk(const ChunkArgs& a, cudaStream_t s) {
  const kv2_cache& c = *a.c;
  ChunkParams p{};
  p.k_code = c.k_code; p.v_code = c.v_code; p.k_sz = c.k_sz; p.v_sz = c.v_sz;
  p.cidx = c.cidx; p.psac = c.psac; p.cent = c.centroids; p.P = c.P;
  p.psac_fmt = c.psac_fmt; p.psac_scale = c.psac_scale;
  p.table = c.block_table; p.page = c.page_tokens;
  p.Q = a.Q; p.Ks = a.Kself; p.Vs = a.Vself; p.out = a.out;
  p.err = static_cast<int*>(a.ws);
  p.B = c.B; p.H_kv = c.H_kv; p.H_q = a.H_q; p.M = c.M; p.r = c.r; p.cap = c.capacity;
  p.len = a.len; p.Nq = a.Nq; p.F = a.frame_tokens; p.out_dtype = a.out_dtype;
  p.scale_log2 = a.sm_scale * 1.4426950408889634f;
  p.budget = env_wait_budget();
  p.force_timeout = env_force_timeout();
  if (p.force_timeout) p.budget = 1u << 20;
  // every unit has at least n_cache + 1 key tiles: pieces never come out empty
  const int n_cache = (a.len + kKeys - 1) / kKeys;
  const ChunkPlan pl = plan_chunk(c.B, a.H_q, a.Nq, n_cache + 1);
  p.QP = pl.QP;
  p.n_full = pl.n_units - pl.split;
  p.pieces = pl.pieces;
  p.part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + kChunkWsHeader);
  cudaError_t e = cudaMemsetAsync(a.ws, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  const int group = cache_group(c);
  auto kern = group == 128 ? chunk_attn_kernel<128> : group == 64 ? chunk_attn_kernel<64> : chunk_attn_kernel<32>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_ALLOC));
  if (e != cudaSuccess) return e;
  const int items = p.n_full + pl.split * pl.pieces;
  if (items == 0) return cudaSuccess;
  kern<<<items, kThreads, SMEM_ALLOC, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || pl.split == 0) return e;
  chunk_merge<<<pl.split * 2 * kRows, kD, 0, s>>>(p.part, p.n_full, pl.pieces, pl.QP, a.H_q, a.Nq, a.out,
                                                   a.out_dtype);
  return cudaGetLastError();
}

}  // namespace kv2
