// decode.cu — attention of one query token per sequence over the packed
// 2-bit cache, dequantizing in registers (no dense fp16 cache is built).
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
// Three kernels:
//   decode_prep   per query head: q' (q scaled, with a per-channel power-of-4
//                 factor matching the code extraction), q.mu_j for every centre,
//                 u = qP, per-group sums of q;
//   decode_split  grid (splits, B*H_kv): streams 128-token tiles of every packed
//                 stream with cp.async (double-buffered), one thread per token for
//                 the logits of the G query heads sharing the KV head (so each
//                 byte is read once per KV head), online softmax, values
//                 accumulated as sum_t (p_t s_t) code_t + sum_t p_t z_t;
//   decode_combine log-sum-exp merge of the splits.
// Codes become floats without integer->float conversions: for channel i of a
// 32-bit code word, (word & (3 << 2i)) | 0x4B000000 is the float 2^23 + code*4^i;
// subtracting 2^23 leaves code*4^i exactly, and q carries the factor 4^-i.
#include <cfloat>

#include "common.cuh"
#include "internal.h"

namespace kv2 {
namespace {

constexpr int kTile = 128;        // tokens per tile
constexpr int kThreads = 128;     // one thread per token in the logit phase
constexpr float kLog2e = 1.4426950408889634f;

// power-of-4 exponent carried by channel i (0..15) of a code word
__host__ __device__ constexpr int code_exp(int i) { return i <= 10 ? i : i - 6; }

__device__ __forceinline__ float code_val(uint32_t word, int i) {
  // code * 4^code_exp(i), exact
  const uint32_t src = (i <= 10) ? word : (word >> 12);
  const int sh = 2 * code_exp(i);
  return __uint_as_float((src & (3u << sh)) | 0x4B000000u) - 8388608.0f;
}

struct PrepLayout {
  int D, M, r, NG, stride;
  __host__ __device__ PrepLayout(int d, int m, int rr) : D(d), M(m), r(rr), NG(d / 32) {
    stride = (D + M + r + NG + 3) & ~3;
  }
  __host__ __device__ int q_off() const { return 0; }
  __host__ __device__ int mu_off() const { return D; }
  __host__ __device__ int u_off() const { return D + M; }
  __host__ __device__ int sig_off() const { return D + M + r; }
};

// ---------------------------------------------------------------------------
__global__ void decode_prep(const uint16_t* __restrict__ Q, const uint16_t* __restrict__ cent,
                            const float* __restrict__ P, int H_q, int H_kv, int D, int M, int r,
                            float scale, float* __restrict__ prep) {
  const int bq = blockIdx.x;                 // b * H_q + hq
  const int hq = bq % H_q;
  const int h = hq / (H_q / H_kv);
  const PrepLayout L(D, M, r);
  float* out = prep + size_t(bq) * L.stride;
  __shared__ float q_s[128];
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const float q = bf16_to_f32(Q[size_t(bq) * D + c]) * scale;
    q_s[c] = q;
    out[L.q_off() + c] = ldexpf(q, -2 * code_exp(c % 16));
  }
  __syncthreads();
  const __half* ch = reinterpret_cast<const __half*>(cent) + size_t(h) * M * D;
  for (int j = threadIdx.x; j < M; j += blockDim.x) {
    float acc = 0.0f;
    const __half2* row = reinterpret_cast<const __half2*>(ch + size_t(j) * D);
    for (int c = 0; c < D / 2; ++c) {
      const float2 m = __half22float2(row[c]);
      acc = fmaf(q_s[2 * c], m.x, acc);
      acc = fmaf(q_s[2 * c + 1], m.y, acc);
    }
    out[L.mu_off() + j] = acc;
  }
  for (int i = threadIdx.x; i < r; i += blockDim.x) {
    float acc = 0.0f;
    for (int c = 0; c < D; ++c) acc = fmaf(q_s[c], P[(size_t(h) * D + c) * r + i], acc);
    out[L.u_off() + i] = acc;
  }
  for (int g = threadIdx.x; g < D / 32; g += blockDim.x) {
    float acc = 0.0f;
    for (int c = 0; c < 32; ++c) acc += q_s[g * 32 + c];
    out[L.sig_off() + g] = acc;
  }
}

// ---------------------------------------------------------------------------
struct SplitParams {
  const uint32_t* k_code;
  const uint32_t* v_code;
  const uint32_t* k_sz;
  const uint32_t* v_sz;
  const void* cidx;
  const uint16_t* psac;
  const float* prep;
  float* part;        // [B*H_kv][splits][G][D + 2]
  int H_kv, H_q, M, r, cap, len, splits, tiles_per_split;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

template <int D, int G, bool U16>
struct DCfg {
  static constexpr int NG = D / 32;
  static constexpr int NW = D / 16;            // code words per token
  static constexpr int CH = (G >= 8) ? 8 : 16; // channels per thread in the value phase
  static constexpr int CB = D / CH;            // channel blocks
  static constexpr int TS = kThreads / CB;     // token slices
  static constexpr int IDXB = U16 ? 2 : 1;
  // per-stage byte offsets (all multiples of 16)
  static constexpr int kc_off = 0;
  static constexpr int vc_off = kc_off + kTile * NW * 4;
  static constexpr int ks_off = vc_off + kTile * NW * 4;
  static constexpr int vs_off = ks_off + kTile * NG * 4;
  static constexpr int ix_off = vs_off + kTile * NG * 4;
  static constexpr int ps_off = ix_off + kTile * IDXB;
  static constexpr int red_bytes = TS * G * D * 4;   // final value reduction
  __host__ __device__ static int stage_bytes(int r) { return ps_off + kTile * r * 2; }
  __host__ __device__ static int tables_off(int r) {
    const int two = 2 * stage_bytes(r);
    return two > red_bytes ? two : red_bytes;
  }
};

template <int D, int G, bool U16>
__global__ void __launch_bounds__(kThreads) decode_split(SplitParams p) {
  using Cfg = DCfg<D, G, U16>;
  constexpr int NG = Cfg::NG, NW = Cfg::NW, CH = Cfg::CH, CB = Cfg::CB, TS = Cfg::TS;
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = p.r, M = p.M;
  const int stage = Cfg::stage_bytes(r);
  unsigned char* st[2] = {smem, smem + stage};
  float* qs = reinterpret_cast<float*>(smem + Cfg::tables_off(r));   // [D][G]  q'
  float* mus = qs + D * G;                                  // [G][M]
  float* us = mus + G * M;                                  // [G][r]
  float* sgs = us + G * r;                                  // [G][NG]
  float* ps = sgs + G * NG;                                 // [G][kTile] probabilities
  float* red = ps + G * kTile;                              // [4 warps][G] reductions
  float* mrun = red + 4 * G;                                // [G] running max
  float* alpha_s = mrun + G;                                // [G]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H_kv, h = bh % p.H_kv;
  const PrepLayout L(D, M, r);
  const size_t base_slot = size_t(bh) * p.cap;
  const int t_begin = split * p.tiles_per_split * kTile;
  const int t_end = min(p.len, t_begin + p.tiles_per_split * kTile);
  const int ntiles = (t_end > t_begin) ? (t_end - t_begin + kTile - 1) / kTile : 0;

  // query-side tables of the G query heads
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, c = i % D;
    qs[c * G + g] = p.prep[size_t(b * p.H_q + h * G + g) * L.stride + L.q_off() + c];
  }
  for (int i = tid; i < G * M; i += kThreads) {
    const int g = i / M, j = i % M;
    mus[i] = p.prep[size_t(b * p.H_q + h * G + g) * L.stride + L.mu_off() + j];
  }
  for (int i = tid; i < G * r; i += kThreads) {
    const int g = i / r, k = i % r;
    us[i] = p.prep[size_t(b * p.H_q + h * G + g) * L.stride + L.u_off() + k];
  }
  for (int i = tid; i < G * NG; i += kThreads) {
    const int g = i / NG, k = i % NG;
    sgs[i] = p.prep[size_t(b * p.H_q + h * G + g) * L.stride + L.sig_off() + k];
  }
  if (tid < G) mrun[tid] = -FLT_MAX;

  auto issue = [&](int tile, unsigned char* dst) {
    const int t0 = t_begin + tile * kTile;
    const int n = min(kTile, t_end - t0);
    const int n16 = (n + 15) & ~15;                      // within capacity (cap % 16 == 0)
    const size_t s0 = base_slot + t0;
    auto copy = [&](int off, const void* src, int bytes_per_tok) {
      const int chunks = n16 * bytes_per_tok / 16;
      const char* g = static_cast<const char*>(src) + s0 * bytes_per_tok;
      for (int i = tid; i < chunks; i += kThreads) cp_async16(dst + off + i * 16, g + i * 16);
    };
    copy(Cfg::kc_off, p.k_code, NW * 4);
    copy(Cfg::vc_off, p.v_code, NW * 4);
    copy(Cfg::ks_off, p.k_sz, NG * 4);
    copy(Cfg::vs_off, p.v_sz, NG * 4);
    copy(Cfg::ix_off, p.cidx, Cfg::IDXB);
    if (r) copy(Cfg::ps_off, p.psac, r * 2);
  };

  // value accumulators: CH channels x G heads, scaled by 4^code_exp per channel
  const int cb = tid % CB, ts = tid / CB;
  float acc[G][CH];
  float pz[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    pz[g] = 0.0f;
#pragma unroll
    for (int c = 0; c < CH; ++c) acc[g][c] = 0.0f;
  }
  float lsum[G];
#pragma unroll
  for (int g = 0; g < G; ++g) lsum[g] = 0.0f;

  if (ntiles > 0) issue(0, st[0]);
  cp_async_commit();
  __syncthreads();

  for (int tile = 0; tile < ntiles; ++tile) {
    unsigned char* cur = st[tile & 1];
    if (tile + 1 < ntiles) issue(tile + 1, st[(tile + 1) & 1]);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const int t0 = t_begin + tile * kTile;
    const int n = min(kTile, t_end - t0);

    // ---- logits: thread = token, all G heads
    float lg[G];
    {
      const int t = tid;
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(cur + Cfg::kc_off) + t * NW;
      const uint32_t* ksz = reinterpret_cast<const uint32_t*>(cur + Cfg::ks_off) + t * NG;
      float dot[G][NG];
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int k = 0; k < NG; ++k) dot[g][k] = 0.0f;
#pragma unroll
      for (int w4 = 0; w4 < NW; w4 += 4) {
        const uint4 wv = *reinterpret_cast<const uint4*>(kw + w4);
        const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) {
          const int w = w4 + ww, grp = w / 2;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float f = code_val(words[ww], i);
            const float* qc = qs + (w * 16 + i) * G;
            if constexpr (G == 4) {
              const float4 q4 = *reinterpret_cast<const float4*>(qc);
              dot[0][grp] = fmaf(q4.x, f, dot[0][grp]);
              dot[1][grp] = fmaf(q4.y, f, dot[1][grp]);
              dot[2][grp] = fmaf(q4.z, f, dot[2][grp]);
              dot[3][grp] = fmaf(q4.w, f, dot[3][grp]);
            } else {
#pragma unroll
              for (int g = 0; g < G; ++g) dot[g][grp] = fmaf(qc[g], f, dot[g][grp]);
            }
          }
        }
      }
      int idx;
      if constexpr (U16) idx = reinterpret_cast<const uint16_t*>(cur + Cfg::ix_off)[t];
      else idx = (cur + Cfg::ix_off)[t];
      idx = min(idx, M - 1);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float l = mus[g * M + idx];
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          const uint32_t sz = ksz[k];
          const float s = __half2float(__ushort_as_half(uint16_t(sz & 0xffff)));
          const float z = __half2float(__ushort_as_half(uint16_t(sz >> 16)));
          l = fmaf(s, dot[g][k], l);
          l = fmaf(z, sgs[g * NG + k], l);
        }
        lg[g] = l;
      }
      if (r) {
        const __half2* a2 = reinterpret_cast<const __half2*>(cur + Cfg::ps_off) + t * (r / 2);
        for (int k = 0; k < r / 2; ++k) {
          const float2 a = __half22float2(a2[k]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            lg[g] = fmaf(us[g * r + 2 * k], a.x, lg[g]);
            lg[g] = fmaf(us[g * r + 2 * k + 1], a.y, lg[g]);
          }
        }
      }
      if (t >= n) {
#pragma unroll
        for (int g = 0; g < G; ++g) lg[g] = -FLT_MAX;
      }
    }
    // ---- tile max per head, new running max, probabilities
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float m = lg[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[warp * G + g] = m;
    }
    __syncthreads();
    if (tid < G) {
      const float m_old = mrun[tid];
      const float m_new = fmaxf(m_old, fmaxf(fmaxf(red[tid], red[G + tid]), fmaxf(red[2 * G + tid], red[3 * G + tid])));
      alpha_s[tid] = exp2f(m_old - m_new);
      mrun[tid] = m_new;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float pr = (tid < n) ? exp2f(lg[g] - mrun[g]) : 0.0f;
      ps[g * kTile + tid] = pr;
      const float al = alpha_s[g];
      lsum[g] = lsum[g] * al + pr;        // per-thread partial sums, rescaled alike
#pragma unroll
      for (int c = 0; c < CH; ++c) acc[g][c] *= al;
      pz[g] *= al;
    }
    __syncthreads();

    // ---- values: thread = (channel block, token slice)
    {
      const uint32_t* vw = reinterpret_cast<const uint32_t*>(cur + Cfg::vc_off);
      const uint32_t* vsz = reinterpret_cast<const uint32_t*>(cur + Cfg::vs_off);
      const int c0 = cb * CH;
      const int word = c0 / 16, sub = c0 % 16, grp = c0 / 32;
      for (int t = ts; t < n; t += TS) {
        const uint32_t wv = vw[t * NW + word];
        const uint32_t sz = vsz[t * NG + grp];
        const float s = __half2float(__ushort_as_half(uint16_t(sz & 0xffff)));
        const float z = __half2float(__ushort_as_half(uint16_t(sz >> 16)));
        float pw[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pr = ps[g * kTile + t];
          pw[g] = pr * s;
          pz[g] = fmaf(pr, z, pz[g]);
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const float f = code_val(wv, sub + c);
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g][c] = fmaf(pw[g], f, acc[g][c]);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- reduce: probabilities' sum over threads, value partials over token slices
  float* rbuf = reinterpret_cast<float*>(smem);      // reuse the stage buffers
  __syncthreads();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float l = lsum[g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) red[warp * G + g] = l;
  }
  // value partials: [TS][G][D], then the zero term per group (only channel block's group)
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = cb * CH + c;
      rbuf[(ts * G + g) * D + ch] = ldexpf(acc[g][c], -2 * code_exp(ch % 16)) + pz[g];
    }
  __syncthreads();
  float* dst = p.part + (size_t(bh) * p.splits + split) * G * (D + 2);
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, ch = i % D;
    float o = 0.0f;
    for (int k = 0; k < TS; ++k) o += rbuf[(k * G + g) * D + ch];
    dst[g * (D + 2) + ch] = o;
  }
  if (tid < G) {
    dst[tid * (D + 2) + D] = mrun[tid];
    dst[tid * (D + 2) + D + 1] = red[tid] + red[G + tid] + red[2 * G + tid] + red[3 * G + tid];
  }
}

// ---------------------------------------------------------------------------
__global__ void decode_combine(const float* __restrict__ part, int H_q, int H_kv, int D,
                               int splits, void* out, int out_dtype) {
  const int bq = blockIdx.x;
  const int b = bq / H_q, hq = bq % H_q;
  const int G = H_q / H_kv, h = hq / G, g = hq % G;
  const float* base = part + (size_t(b * H_kv + h) * splits) * G * (D + 2) + g * (D + 2);
  const size_t sstride = size_t(G) * (D + 2);
  float m = -FLT_MAX;
  for (int s = 0; s < splits; ++s) {
    const float l = base[s * sstride + D + 1];
    if (l > 0.0f) m = fmaxf(m, base[s * sstride + D]);
  }
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float o = 0.0f, l = 0.0f;
    for (int s = 0; s < splits; ++s) {
      const float ls = base[s * sstride + D + 1];
      if (!(ls > 0.0f)) continue;
      const float f = exp2f(base[s * sstride + D] - m);
      o = fmaf(f, base[s * sstride + c], o);
      l = fmaf(f, ls, l);
    }
    const float v = (l > 0.0f) ? o / l : 0.0f;
    if (out_dtype == KV2_OUT_F32) static_cast<float*>(out)[size_t(bq) * D + c] = v;
    else static_cast<__nv_bfloat16*>(out)[size_t(bq) * D + c] = __float2bfloat16_rn(v);
  }
}

template <int D, int G, bool U16>
cudaError_t launch_split(const SplitParams& sp, int B, cudaStream_t s) {
  using Cfg = DCfg<D, G, U16>;
  const int stage = Cfg::stage_bytes(sp.r);
  const size_t tables = (size_t(D) * G + size_t(G) * sp.M + size_t(G) * sp.r + G * Cfg::NG +
                         size_t(G) * kTile + 4 * G + 2 * G) * 4;
  (void)stage;
  const size_t smem = size_t(Cfg::tables_off(sp.r)) + tables;
  auto kern = decode_split<D, G, U16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(sp.splits, B * sp.H_kv);
  kern<<<grid, kThreads, smem, s>>>(sp);
  return cudaGetLastError();
}

template <int D, bool U16>
cudaError_t launch_g(int G, const SplitParams& sp, int B, cudaStream_t s) {
  switch (G) {
    case 1: return launch_split<D, 1, U16>(sp, B, s);
    case 2: return launch_split<D, 2, U16>(sp, B, s);
    case 4: return launch_split<D, 4, U16>(sp, B, s);
    case 8: return launch_split<D, 8, U16>(sp, B, s);
    default: return cudaErrorInvalidValue;
  }
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

void plan_splits(const kv2_cache& c, int len, int* splits, int* tiles_per_split) {
  const int tiles = (len + kTile - 1) / kTile;
  const int pairs = c.B * c.H_kv;
  int want = (sm_count() * 4 + pairs - 1) / pairs;
  want = want < 1 ? 1 : want;
  int tps = (tiles + want - 1) / want;
  tps = tps < 1 ? 1 : tps;
  *tiles_per_split = tps;
  *splits = tiles > 0 ? (tiles + tps - 1) / tps : 1;
}

}  // namespace

size_t decode_workspace_bytes(const kv2_cache& c, int H_q, int len) {
  int splits, tps;
  plan_splits(c, len, &splits, &tps);
  const PrepLayout L(c.d, c.M, c.r);
  const size_t prep = size_t(c.B) * H_q * L.stride * 4;
  const size_t part = size_t(c.B) * c.H_kv * splits * (H_q / c.H_kv) * (c.d + 2) * 4;
  return ((prep + 255) & ~size_t(255)) + part;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const kv2_cache& c = *a.c;
  int splits, tps;
  plan_splits(c, a.len, &splits, &tps);
  const PrepLayout L(c.d, c.M, c.r);
  float* prep = static_cast<float*>(a.ws);
  const size_t prep_bytes = (size_t(c.B) * a.H_q * L.stride * 4 + 255) & ~size_t(255);
  float* part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + prep_bytes);
  decode_prep<<<c.B * a.H_q, 128, 0, s>>>(a.Q, c.centroids, c.P, a.H_q, c.H_kv, c.d, c.M, c.r,
                                          a.sm_scale * kLog2e, prep);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  SplitParams sp{c.k_code, c.v_code, c.k_sz, c.v_sz, c.cidx, c.psac, prep, part,
                 c.H_kv, a.H_q, c.M, c.r, c.capacity, a.len, splits, tps};
  const int G = a.H_q / c.H_kv;
  if (c.d == 64) e = (c.M > 256) ? launch_g<64, true>(G, sp, c.B, s) : launch_g<64, false>(G, sp, c.B, s);
  else e = (c.M > 256) ? launch_g<128, true>(G, sp, c.B, s) : launch_g<128, false>(G, sp, c.B, s);
  if (e != cudaSuccess) return e;
  decode_combine<<<c.B * a.H_q, 128, 0, s>>>(part, a.H_q, c.H_kv, c.d, splits, a.out, a.out_dtype);
  return cudaGetLastError();
}

}  // namespace kv2
