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
//   S  = Q . Khat^T           bf16 x bf16, Khat = bf16(fmaf(code, s, z) + mu[idx])
//      + U . A^T              fp16 x fp16, U = fp16(q P), A = the stored fp16
//                             PSAC coefficients (K = 16 extra contraction columns)
//   O  = P . Vhat             fp16 x fp16, Vhat = fp16(fmaf(code, s, z)), P = fp16
//
// Packed key/value tiles are dequantized into shared memory in the canonical
// 128-byte-swizzled layouts the MMA descriptors describe; no dense cache is
// kept anywhere. One CTA handles 128 queries of one (batch, query head); TMEM
// holds S (128 columns) and the tile's P.V (128 columns); the softmax keeps
// the running max / sum / output in registers (thread = query row = TMEM lane).
//
// Every mbarrier wait is bounded by a clock-cycle budget; a wait that runs out
// records 1 in the first word of the workspace and the CTA waits (bounded) for
// its MMAs in flight, frees its TMEM and returns.
#include <cfloat>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"

namespace kv2 {
namespace {

constexpr int kRows = 128;       // queries per CTA (= TMEM lanes)
constexpr int kKeys = 128;       // keys per tile
constexpr int kD = 128;
constexpr int kThreads = 128;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_Q = 0;            // Q    [2 k-chunks][128 rows][128 B], SW128, K-major
constexpr uint32_t OFF_K = 32768;        // Khat [2 k-chunks][128 keys][128 B], SW128, K-major
constexpr uint32_t OFF_V = 65536;        // Vhat [2 n-blocks][128 keys][128 B], SW128, MN-major
constexpr uint32_t OFF_P = 98304;        // P    [2 k-chunks][128 rows][128 B], SW128, K-major
constexpr uint32_t OFF_U = 131072;       // U    [16 row groups][2 k-chunks][8 rows][16 B]
constexpr uint32_t OFF_A = 135168;       // A    [16 key groups][2 k-chunks][8 keys][16 B]
constexpr uint32_t OFF_BAR = 139264;     // mbarriers + TMEM address
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;

constexpr uint32_t kTmemCols = 256;

// ---------------------------------------------------------------------------
// PTX wrappers (sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// UMMA shared-memory matrix descriptor: start, leading / stride byte offsets,
// version 1 (Blackwell), layout (0 = no swizzle, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(layout & 7u) << 61);
}
constexpr uint32_t kLayoutNone = 0, kLayoutSW128 = 2;

// kind::f16 instruction descriptor: fp32 accumulate, A/B formats (0 f16, 1 bf16),
// B major (0 K, 1 MN), N, M.
constexpr uint32_t make_idesc(uint32_t a_fmt, uint32_t b_fmt, uint32_t b_mn_major, uint32_t N, uint32_t M) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | (b_mn_major << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}
constexpr uint32_t IDESC_QK = make_idesc(1, 1, 0, kKeys, kRows);
constexpr uint32_t IDESC_UA = make_idesc(0, 0, 0, kKeys, kRows);
constexpr uint32_t IDESC_PV = make_idesc(0, 0, 1, kD, kRows);

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t phase) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred P1;\n\tmbarrier.test_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}\n"
      : "=r"(done)
      : "r"(bar), "r"(phase)
      : "memory");
  return done != 0;
}
// Bounded wait: spins until the phase completes or `budget` SM clock cycles pass.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, unsigned long long budget) {
  const unsigned long long t0 = clock64();
  while (!mbar_test(bar, phase)) {
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// byte offset of 16-byte chunk `c16` (0..15) of row `row` in a [2][128][128 B]
// 128-byte-swizzled operand tile (K-major: chunks along K; MN-major: along N)
__device__ __forceinline__ uint32_t sw128_off(int row, int c16) {
  return uint32_t((c16 >> 3) * 16384 + row * 128 + (((c16 & 7) ^ (row & 7)) << 4));
}
// byte offset of 16-byte chunk `c` (0, 1) of row `row` in a no-swizzle
// [row/8][2][8][16 B] operand tile (K = 16 columns of 16-bit values)
__device__ __forceinline__ uint32_t nosw_off(int row, int c) {
  return uint32_t((row >> 3) * 256 + c * 128 + (row & 7) * 16);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(a))) |
         (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(b))) << 16);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  return uint32_t(__half_as_ushort(__float2half_rn(a))) | (uint32_t(__half_as_ushort(__float2half_rn(b))) << 16);
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
};

// ---------------------------------------------------------------------------
// operand producers (thread = one row)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void zero_rows(uint8_t* tile, int row) {
#pragma unroll
  for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(tile + sw128_off(row, c)) = make_uint4(0, 0, 0, 0);
}

// cached token -> Khat (bf16) row, PSAC row, Vhat (fp16) row
__device__ void dequant_cache_row(const ChunkParams& p, size_t slot, int h, int row, uint8_t* smem) {
  const uint4* kw4 = reinterpret_cast<const uint4*>(p.k_code + slot * 8);
  const uint4* vw4 = reinterpret_cast<const uint4*>(p.v_code + slot * 8);
  const uint4 k0 = kw4[0], k1 = kw4[1], v0 = vw4[0], v1 = vw4[1];
  const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
  const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  const uint4 ks = *reinterpret_cast<const uint4*>(p.k_sz + slot * 4);
  const uint4 vs = *reinterpret_cast<const uint4*>(p.v_sz + slot * 4);
  const uint32_t ksz[4] = {ks.x, ks.y, ks.z, ks.w};
  const uint32_t vsz[4] = {vs.x, vs.y, vs.z, vs.w};
  const int idx = (p.M <= 256) ? int(static_cast<const uint8_t*>(p.cidx)[slot])
                               : int(static_cast<const uint16_t*>(p.cidx)[slot]);
  const uint4* mu = reinterpret_cast<const uint4*>(p.cent + (size_t(h) * p.M + min(idx, p.M - 1)) * kD);
#pragma unroll
  for (int c16 = 0; c16 < 16; ++c16) {              // 8 channels per chunk
    const int g = c16 >> 2;
    const float ksc = __half2float(__ushort_as_half(uint16_t(ksz[g] & 0xffff)));
    const float kz = __half2float(__ushort_as_half(uint16_t(ksz[g] >> 16)));
    const float vsc = __half2float(__ushort_as_half(uint16_t(vsz[g] & 0xffff)));
    const float vz = __half2float(__ushort_as_half(uint16_t(vsz[g] >> 16)));
    const uint4 m4 = __ldg(mu + c16);
    const __half2* mh = reinterpret_cast<const __half2*>(&m4);
    const uint32_t kword = kw[c16 >> 1] >> ((c16 & 1) * 16);
    const uint32_t vword = vw[c16 >> 1] >> ((c16 & 1) * 16);
    uint32_t kb[4], vb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 m = __half22float2(mh[i]);
      const float c0 = float((kword >> (4 * i)) & 3u), c1 = float((kword >> (4 * i + 2)) & 3u);
      const float k0f = __fadd_rn(__fmaf_rn(c0, ksc, kz), m.x);
      const float k1f = __fadd_rn(__fmaf_rn(c1, ksc, kz), m.y);
      kb[i] = pack_bf16(k0f, k1f);
      const float d0 = float((vword >> (4 * i)) & 3u), d1 = float((vword >> (4 * i + 2)) & 3u);
      vb[i] = pack_f16(__fmaf_rn(d0, vsc, vz), __fmaf_rn(d1, vsc, vz));
    }
    *reinterpret_cast<uint4*>(smem + OFF_K + sw128_off(row, c16)) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
    *reinterpret_cast<uint4*>(smem + OFF_V + sw128_off(row, c16)) = make_uint4(vb[0], vb[1], vb[2], vb[3]);
  }
  // PSAC coefficients: r (0, 8 or 16) fp16 values, zero-padded to 16
  uint4 a0 = make_uint4(0, 0, 0, 0), a1 = make_uint4(0, 0, 0, 0);
  if (p.r >= 8) a0 = *reinterpret_cast<const uint4*>(p.psac + slot * p.r);
  if (p.r >= 16) a1 = *reinterpret_cast<const uint4*>(p.psac + slot * p.r + 8);
  *reinterpret_cast<uint4*>(smem + OFF_A + nosw_off(row, 0)) = a0;
  *reinterpret_cast<uint4*>(smem + OFF_A + nosw_off(row, 1)) = a1;
}

// chunk token -> Khat row (bf16 copy), Vhat row (bf16 -> fp16)
__device__ void copy_self_row(const ChunkParams& p, const uint16_t* krow, const uint16_t* vrow, int row,
                              uint8_t* smem) {
  const uint4* k4 = reinterpret_cast<const uint4*>(krow);
  const uint4* v4 = reinterpret_cast<const uint4*>(vrow);
#pragma unroll
  for (int c16 = 0; c16 < 16; ++c16) {
    *reinterpret_cast<uint4*>(smem + OFF_K + sw128_off(row, c16)) = __ldg(k4 + c16);
    const uint4 v = __ldg(v4 + c16);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = pack_f16(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
    *reinterpret_cast<uint4*>(smem + OFF_V + sw128_off(row, c16)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) chunk_attn_kernel(ChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_s = sb + OFF_BAR, bar_o = sb + OFF_BAR + 8, bar_never = sb + OFF_BAR + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 32);
  volatile int* s_fail = reinterpret_cast<volatile int*>(smem + OFF_BAR + 40);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qt = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int G = p.H_q / p.H_kv, h = hq / G;
  const int q0 = qt * kRows;
  const int qi = q0 + tid;                  // this thread's query (row, TMEM lane)
  const bool q_ok = qi < p.Nq;

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_never, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    *s_fail = 0;
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);

  // ---- Q tile (bf16, SW128 K-major) and U = fp16(q P) (no swizzle, K = 16)
  {
    float u[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) u[j] = 0.0f;
    const uint4* src = reinterpret_cast<const uint4*>(p.Q + ((size_t(b) * p.Nq + min(qi, p.Nq - 1)) * p.H_q + hq) * kD);
    const float* Ph = p.P + size_t(h) * kD * p.r;
#pragma unroll 1
    for (int c16 = 0; c16 < 16; ++c16) {
      const uint4 v = q_ok ? __ldg(src + c16) : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(smem + OFF_Q + sw128_off(tid, c16)) = v;
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
    uint32_t uw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) uw[j] = pack_f16(u[2 * j], u[2 * j + 1]);
    *reinterpret_cast<uint4*>(smem + OFF_U + nosw_off(tid, 0)) = make_uint4(uw[0], uw[1], uw[2], uw[3]);
    *reinterpret_cast<uint4*>(smem + OFF_U + nosw_off(tid, 1)) = make_uint4(uw[4], uw[5], uw[6], uw[7]);
  }
  fence_proxy_async();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + kKeys;
  const uint32_t lane_base = uint32_t(warp * 32) << 16;

  const int n_cache = (p.len + kKeys - 1) / kKeys;
  const int last_q = min(q0 + kRows, p.Nq) - 1;
  const int self_len = min(p.Nq, (last_q / p.F + 1) * p.F);
  const int n_self = (self_len + kKeys - 1) / kKeys;
  const int my_self_lim = min(self_len, (min(qi, p.Nq - 1) / p.F + 1) * p.F);

  float m_run = -INFINITY, l_run = 0.0f;
  uint32_t phase = 0;
  bool failed = false;
  int pending = 0;     // MMA group committed and not yet waited for: 1 = S, 2 = O
  const int n_tiles = n_cache + n_self;

  for (int j = 0; j < n_tiles; ++j) {
    const bool cache = j < n_cache;
    const int k0 = cache ? j * kKeys : (j - n_cache) * kKeys;
    const int kvalid = cache ? min(kKeys, p.len - k0) : min(kKeys, self_len - k0);
    // ---- produce Khat, A, Vhat rows (the previous tile's MMAs have completed)
    const int key = k0 + tid;
    if (tid < kvalid) {
      if (cache) {
        dequant_cache_row(p, (size_t(b) * p.H_kv + h) * p.cap + key, h, tid, smem);
      } else {
        const size_t srow = (size_t(b) * p.Nq + key) * p.H_kv + h;
        copy_self_row(p, p.Ks + srow * kD, p.Vs + srow * kD, tid, smem);
      }
    } else {
      zero_rows(smem + OFF_K, tid);
      zero_rows(smem + OFF_V, tid);
      *reinterpret_cast<uint4*>(smem + OFF_A + nosw_off(tid, 0)) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(smem + OFF_A + nosw_off(tid, 1)) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // ---- S = Q Khat^T (+ U A^T)
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tS, make_sdesc(sb + OFF_Q + off, 16, 1024, kLayoutSW128),
                make_sdesc(sb + OFF_K + off, 16, 1024, kLayoutSW128), IDESC_QK, kk > 0);
      }
      if (cache && p.r > 0)
        mma_f16(tS, make_sdesc(sb + OFF_U, 128, 256, kLayoutNone), make_sdesc(sb + OFF_A, 128, 256, kLayoutNone),
                IDESC_UA, 1);
      mma_commit(bar_s);
    }
    pending = 1;
    if (p.force_timeout && !mbar_wait(bar_never, 0, p.budget)) *s_fail = 1;
    if (!*s_fail && !mbar_wait(bar_s, phase, p.budget)) *s_fail = 1;
    __syncthreads();
    if (*s_fail) { failed = true; break; }
    pending = 0;
    fence_after_sync();

    // ---- softmax of this row over the tile; P (fp16) to shared memory
    const int lim = cache ? kvalid : (my_self_lim - k0);
    float mt = -INFINITY;
#pragma unroll
    for (int c0 = 0; c0 < kKeys; c0 += 32) {
      float v[32];
      tmem_ld32(tS + lane_base + c0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c0 + i < lim) mt = fmaxf(mt, v[i]);
    }
    const float m_new = fmaxf(m_run, mt * p.scale_log2);
    const float alpha = (m_new == -INFINITY) ? 1.0f : exp2f(m_run - m_new);
    float lsum = 0.0f;
#pragma unroll
    for (int c0 = 0; c0 < kKeys; c0 += 32) {
      float v[32];
      tmem_ld32(tS + lane_base + c0, v);
      uint32_t pw[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float p0 = (c0 + i < lim) ? exp2f(fmaf(v[i], p.scale_log2, -m_new)) : 0.0f;
        const float p1 = (c0 + i + 1 < lim) ? exp2f(fmaf(v[i + 1], p.scale_log2, -m_new)) : 0.0f;
        lsum += p0 + p1;
        pw[i / 2] = pack_f16(p0, p1);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(smem + OFF_P + sw128_off(tid, c0 / 8 + q)) =
            make_uint4(pw[4 * q], pw[4 * q + 1], pw[4 * q + 2], pw[4 * q + 3]);
    }
    l_run = l_run * alpha + lsum;
    m_run = m_new;
    // ---- rescale the running output in TMEM when a row's max grew. The TMEM
    // load/store are .sync.aligned warp instructions: the whole warp executes
    // them when any of its rows needs it (alpha is 1 for the others).
    if (__any_sync(0xffffffffu, j > 0 && alpha != 1.0f)) {
#pragma unroll
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float v[32];
        tmem_ld32(tO + lane_base + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= alpha;
        tmem_st32(tO + lane_base + c0, v);
      }
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // ---- O += P Vhat
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; ++kk) {
        mma_f16(tO, make_sdesc(sb + OFF_P + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSW128),
                make_sdesc(sb + OFF_V + kk * 2048, 16384, 1024, kLayoutSW128), IDESC_PV, (j > 0 || kk > 0));
      }
      mma_commit(bar_o);
    }
    pending = 2;
    if (!mbar_wait(bar_o, phase, p.budget)) *s_fail = 1;
    __syncthreads();
    if (*s_fail) { failed = true; break; }
    pending = 0;
    fence_after_sync();
    phase ^= 1u;
  }

  if (failed) {
    if (tid == 0) atomicExch(p.err, 1);
    // wait (bounded) for the MMA group still in flight before freeing TMEM
    if (pending == 1) mbar_wait(bar_s, phase, 1ull << 32);
    if (pending == 2) mbar_wait(bar_o, phase, 1ull << 32);
  } else {
    // every lane runs the (warp-wide) TMEM loads; only valid rows store
    const float inv = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
    const size_t obase = ((size_t(b) * p.Nq + min(qi, p.Nq - 1)) * p.H_q + hq) * kD;
#pragma unroll
    for (int c0 = 0; c0 < kD; c0 += 32) {
      float v[32];
      if (n_tiles > 0) {
        tmem_ld32(tO + lane_base + c0, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.0f;
      }
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
  fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

unsigned long long env_budget() {
  const char* e = std::getenv("KV2_WAIT_BUDGET_CYCLES");
  return e ? std::strtoull(e, nullptr, 10) : (1ull << 31);   // ~1 s at 2 GHz
}

}  // namespace

size_t chunk_workspace_bytes(const kv2_cache&, int, int) { return 256; }

cudaError_t launch_chunk(const ChunkArgs& a, cudaStream_t s) {
  const kv2_cache& c = *a.c;
  ChunkParams p{};
  p.k_code = c.k_code; p.v_code = c.v_code; p.k_sz = c.k_sz; p.v_sz = c.v_sz;
  p.cidx = c.cidx; p.psac = c.psac; p.cent = c.centroids; p.P = c.P;
  p.Q = a.Q; p.Ks = a.Kself; p.Vs = a.Vself; p.out = a.out;
  p.err = static_cast<int*>(a.ws);
  p.B = c.B; p.H_kv = c.H_kv; p.H_q = a.H_q; p.M = c.M; p.r = c.r; p.cap = c.capacity;
  p.len = a.len; p.Nq = a.Nq; p.F = a.frame_tokens; p.out_dtype = a.out_dtype;
  p.scale_log2 = a.sm_scale * 1.4426950408889634f;
  p.budget = env_budget();
  const char* ft = std::getenv("KV2_FORCE_WAIT_TIMEOUT");
  p.force_timeout = (ft && ft[0] == '1') ? 1 : 0;
  if (p.force_timeout) p.budget = 1u << 20;
  cudaError_t e = cudaMemsetAsync(a.ws, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(chunk_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_ALLOC));
  if (e != cudaSuccess) return e;
  dim3 grid((a.Nq + kRows - 1) / kRows, a.H_q, c.B);
  chunk_attn_kernel<<<grid, kThreads, SMEM_ALLOC, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kv2
