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
// subtracting 2^23 leaves code*4^i exactly, and q carries the factor 4^-i
// (channels 10..15 use the word shifted right by 12, so the exponent stays
// below 10). Two channels are extracted at once into an fp32 pair with 64-bit
// logic on a duplicated word, then consumed by packed f32x2 arithmetic.
#include <cfloat>

#include "common.cuh"
#include "internal.h"

namespace kv2 {
namespace {

constexpr int kTile = 128;        // tokens per tile
constexpr int kThreads = 128;     // one thread per token in the logit phase
constexpr float kLog2e = 1.4426950408889634f;

// power-of-4 exponent carried by channel i (0..15) of a code word: channels
// 0..9 are read in place, channels 10..15 from the word shifted right by 12
__host__ __device__ constexpr int code_exp(int i) { return i < 10 ? i : i - 6; }

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

// Packed fp32 pairs (Blackwell f32x2 arithmetic): one instruction, two lanes.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pack2u(uint32_t lo, uint32_t hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2(f32x2 v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ f32x2 ffma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 fsub2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 fmul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// {w, w} and {w >> 12, w >> 12}: the two 64-bit sources of a code word's pairs
struct WordPair {
  f32x2 lo, hi;
};
__device__ __forceinline__ WordPair word_pair(uint32_t w) {
  const uint32_t wh = w >> 12;
  return WordPair{pack2u(w, w), pack2u(wh, wh)};
}
// codes of channels (2k, 2k+1) of a code word as {code*4^e(2k), code*4^e(2k+1)}
__device__ __forceinline__ f32x2 code_pair(const WordPair& wp, int k) {
  const int c0 = 2 * k, c1 = 2 * k + 1;
  const f32x2 src = (c0 < 10) ? wp.lo : wp.hi;            // pairs never straddle channel 10
  const unsigned long long mask =
      (static_cast<unsigned long long>(3u << (2 * code_exp(c1))) << 32) | (3u << (2 * code_exp(c0)));
  f32x2 bits;
  asm("{\n\t.reg .b64 t;\n\tand.b64 t, %1, %2;\n\tor.b64 %0, t, 0x4B0000004B000000;\n\t}\n"
      : "=l"(bits) : "l"(src), "l"(mask));
  return fsub2(bits, 0x4B0000004B000000ull);
}

constexpr int kStages = 3;

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
  // tables after the stages
  static constexpr int qs_bytes = D * G * 4;                  // q' as [D/2][G] pairs
  static constexpr int pw_bytes = kTile * NG * G * 4;          // p s_v per (token, group, head)
  static constexpr int red_bytes = (TS * G * D + kThreads * G * NG) * 4;   // final reduction
  __host__ __device__ static int stage_bytes(int r) { return (ps_off + kTile * r * 2 + 15) & ~15; }
  __host__ __device__ static int stages_bytes(int r) {
    const int st = kStages * stage_bytes(r);
    return st > red_bytes ? st : red_bytes;
  }
  __host__ __device__ static int tables_bytes(int M, int r) {
    return qs_bytes + pw_bytes + (G * M + G * r + G * NG + 4 * G + 4) * 4;
  }
};

template <int D, int G, bool U16>
__global__ void __launch_bounds__(kThreads) decode_split(SplitParams p) {
  using Cfg = DCfg<D, G, U16>;
  constexpr int NG = Cfg::NG, NW = Cfg::NW, CH = Cfg::CH, CB = Cfg::CB, TS = Cfg::TS;
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = p.r, M = p.M;
  const int stage = Cfg::stage_bytes(r);
  unsigned char* tables = smem + Cfg::stages_bytes(r);
  f32x2* qs2 = reinterpret_cast<f32x2*>(tables);                              // [D/2][G]
  float* pw_s = reinterpret_cast<float*>(tables + Cfg::qs_bytes);               // [kTile][NG][G]
  float* mus = pw_s + kTile * NG * G;                                           // [G][M]
  float* us = mus + G * M;                                                      // [G][r]
  float* sgs = us + G * r;                                                      // [G][NG]
  float* red = sgs + G * NG;                                                    // [4 warps][G]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H_kv, h = bh % p.H_kv;
  const PrepLayout L(D, M, r);
  const size_t base_slot = size_t(bh) * p.cap;
  const int t_begin = split * p.tiles_per_split * kTile;
  const int t_end = min(p.len, t_begin + p.tiles_per_split * kTile);
  const int ntiles = (t_end > t_begin) ? (t_end - t_begin + kTile - 1) / kTile : 0;

  auto issue = [&](int tile) {
    if (tile < ntiles) {
      unsigned char* dst = smem + (tile % kStages) * stage;
      const int t0 = t_begin + tile * kTile;
      const int n16 = (min(kTile, t_end - t0) + 15) & ~15;   // within capacity (cap % 16 == 0)
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
    }
    cp_async_commit();
  };
  issue(0);
  issue(1);

  // query-side tables of the G query heads sharing this KV head
  const float* prep_h = p.prep + size_t(b * p.H_q + h * G) * L.stride;
  for (int i = tid; i < G * (D / 2); i += kThreads) {
    const int g = i % G, c2 = i / G;
    const float* q = prep_h + size_t(g) * L.stride + L.q_off();
    qs2[c2 * G + g] = pack2(q[2 * c2], q[2 * c2 + 1]);
  }
  for (int i = tid; i < G * M; i += kThreads) mus[i] = prep_h[size_t(i / M) * L.stride + L.mu_off() + i % M];
  for (int i = tid; i < G * r; i += kThreads) us[i] = prep_h[size_t(i / r) * L.stride + L.u_off() + i % r];
  for (int i = tid; i < G * NG; i += kThreads) sgs[i] = prep_h[size_t(i / NG) * L.stride + L.sig_off() + i % NG];

  // per-thread state; the running max is identical in every thread
  float m_run[G], lsum[G], pz[G][NG];
  f32x2 oacc[G][CH / 2];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -FLT_MAX;
    lsum[g] = 0.0f;
#pragma unroll
    for (int k = 0; k < NG; ++k) pz[g][k] = 0.0f;
#pragma unroll
    for (int c = 0; c < CH / 2; ++c) oacc[g][c] = 0ull;
  }
  const int cb = tid % CB, ts = tid / CB;
  const int vword = (cb * CH) / 16, vsub = ((cb * CH) % 16) / 2, vgrp = (cb * CH) / 32;

  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<1>();
    __syncthreads();          // tile data ready; every thread is done with tile - 1
    issue(tile + 2);          // into the stage tile - 1 used
    const unsigned char* cur = smem + (tile % kStages) * stage;
    const int n = min(kTile, t_end - (t_begin + tile * kTile));
    const int t = tid;                                 // logit phase: thread = token

    // ---- logits of the G query heads
    float lg[G];
    {
      int idx;
      if constexpr (U16) idx = reinterpret_cast<const uint16_t*>(cur + Cfg::ix_off)[t];
      else idx = cur[Cfg::ix_off + t];
      idx = min(idx, M - 1);
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g] = mus[g * M + idx];
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(cur + Cfg::kc_off) + t * NW;
      const uint32_t* ksz = reinterpret_cast<const uint32_t*>(cur + Cfg::ks_off) + t * NG;
#pragma unroll
      for (int grp = 0; grp < NG; grp += 2) {          // two groups' chains interleaved
        const uint4 wv = *reinterpret_cast<const uint4*>(kw + 2 * grp);
        const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
        f32x2 dacc[2][G];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int g = 0; g < G; ++g) dacc[u][g] = 0ull;
#pragma unroll
        for (int ww = 0; ww < 2; ++ww) {
          const WordPair wp0 = word_pair(words[ww]), wp1 = word_pair(words[2 + ww]);
          const f32x2* q0 = qs2 + (grp * 2 + ww) * 8 * G;
          const f32x2* q1 = qs2 + (grp * 2 + 2 + ww) * 8 * G;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const f32x2 c0 = code_pair(wp0, k), c1 = code_pair(wp1, k);
#pragma unroll
            for (int g = 0; g < G; ++g) {
              dacc[0][g] = ffma2(q0[k * G + g], c0, dacc[0][g]);
              dacc[1][g] = ffma2(q1[k * G + g], c1, dacc[1][g]);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint32_t sz = ksz[grp + u];
          const float s = __half2float(__ushort_as_half(uint16_t(sz & 0xffff)));
          const float z = __half2float(__ushort_as_half(uint16_t(sz >> 16)));
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float2 d2 = unpack2(dacc[u][g]);
            lg[g] = fmaf(s, d2.x + d2.y, fmaf(z, sgs[g * NG + grp + u], lg[g]));
          }
        }
      }
      if (r) {
        const __half2* a2 = reinterpret_cast<const __half2*>(cur + Cfg::ps_off) + t * (r / 2);
        for (int k = 0; k < r / 2; ++k) {
          const float2 a = __half22float2(a2[k]);
#pragma unroll
          for (int g = 0; g < G; ++g) lg[g] = fmaf(us[g * r + 2 * k], a.x, fmaf(us[g * r + 2 * k + 1], a.y, lg[g]));
        }
      }
      if (t >= n) {
#pragma unroll
        for (int g = 0; g < G; ++g) lg[g] = -FLT_MAX;
      }
    }
    // ---- tile max per head (block-wide), new running max
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float m = lg[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[warp * G + g] = m;
    }
    __syncthreads();
    float alpha[G];
    bool rescale = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float tmax = fmaxf(fmaxf(red[g], red[G + g]), fmaxf(red[2 * G + g], red[3 * G + g]));
      const float m_new = fmaxf(m_run[g], tmax);
      alpha[g] = exp2f(m_run[g] - m_new);
      rescale |= (m_new != m_run[g]);
      m_run[g] = m_new;
    }
    if (rescale) {                                   // uniform across the CTA
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const f32x2 a2 = pack2(alpha[g], alpha[g]);
        lsum[g] *= alpha[g];
#pragma unroll
        for (int k = 0; k < NG; ++k) pz[g][k] *= alpha[g];
#pragma unroll
        for (int c = 0; c < CH / 2; ++c) oacc[g][c] = fmul2(oacc[g][c], a2);
      }
    }
    // ---- probabilities; p s_v per (group, head) for the value phase; sum p z_v
    {
      const uint32_t* vsz = reinterpret_cast<const uint32_t*>(cur + Cfg::vs_off) + t * NG;
      float pr[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        pr[g] = (t < n) ? exp2f(lg[g] - m_run[g]) : 0.0f;
        lsum[g] += pr[g];
      }
#pragma unroll
      for (int grp = 0; grp < NG; ++grp) {
        const uint32_t sz = vsz[grp];
        const float s = (t < n) ? __half2float(__ushort_as_half(uint16_t(sz & 0xffff))) : 0.0f;
        const float z = (t < n) ? __half2float(__ushort_as_half(uint16_t(sz >> 16))) : 0.0f;
        float* dst = pw_s + (t * NG + grp) * G;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          dst[g] = pr[g] * s;
          pz[g][grp] = fmaf(pr[g], z, pz[g][grp]);
        }
      }
    }
    __syncthreads();

    // ---- values: thread = (channel block, token slice)
    {
      const uint32_t* vw = reinterpret_cast<const uint32_t*>(cur + Cfg::vc_off);
      for (int tt = ts; tt < n; tt += TS) {
        const WordPair wp = word_pair(vw[tt * NW + vword]);
        const float* pws = pw_s + (tt * NG + vgrp) * G;
        f32x2 pw[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pw[g] = pack2(pws[g], pws[g]);
#pragma unroll
        for (int k = 0; k < CH / 2; ++k) {
          const f32x2 cpair = code_pair(wp, vsub + k);
#pragma unroll
          for (int g = 0; g < G; ++g) oacc[g][k] = ffma2(pw[g], cpair, oacc[g][k]);
        }
      }
    }
    // no barrier here: the next tile's first barrier orders these reads before
    // the copy into this stage and before the next writes of pw_s
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- reduce: value partials over token slices, p z_v and p sums over threads
  float* rbuf = reinterpret_cast<float*>(smem);            // [TS][G][D], then [kThreads][G][NG]
  float* zbuf = rbuf + TS * G * D;
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int k = 0; k < CH / 2; ++k) {
      const float2 v = unpack2(oacc[g][k]);
      const int c = cb * CH + 2 * k;
      rbuf[(ts * G + g) * D + c] = ldexpf(v.x, -2 * code_exp(c % 16));
      rbuf[(ts * G + g) * D + c + 1] = ldexpf(v.y, -2 * code_exp((c + 1) % 16));
    }
#pragma unroll
    for (int k = 0; k < NG; ++k) zbuf[(tid * G + g) * NG + k] = pz[g][k];
    float l = lsum[g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) red[warp * G + g] = l;
  }
  __syncthreads();
  float* dst = p.part + (size_t(bh) * p.splits + split) * G * (D + 2);
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, c = i % D;
    float o = 0.0f;
    for (int k = 0; k < TS; ++k) o += rbuf[(k * G + g) * D + c];
    float z = 0.0f;
    for (int k = 0; k < kThreads; ++k) z += zbuf[(k * G + g) * NG + c / 32];
    dst[g * (D + 2) + c] = o + z;
  }
  if (tid < G) {
    dst[tid * (D + 2) + D] = m_run[tid];
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
size_t split_smem(int M, int r) {
  using Cfg = DCfg<D, G, U16>;
  return size_t(Cfg::stages_bytes(r)) + size_t(Cfg::tables_bytes(M, r));
}

template <int D, int G, bool U16>
cudaError_t launch_split(const SplitParams& sp, int B, cudaStream_t s) {
  const size_t smem = split_smem<D, G, U16>(sp.M, sp.r);
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

// resident split CTAs per SM for this shape (occupancy query; 4 if unknown)
template <int D, int G, bool U16>
int ctas_per_sm_t(int M, int r) {
  const size_t smem = split_smem<D, G, U16>(M, r);
  auto kern = decode_split<D, G, U16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 4;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, smem) != cudaSuccess || n <= 0) return 4;
  return n;
}
template <int D, bool U16>
int ctas_per_sm_g(int G, int M, int r) {
  switch (G) {
    case 1: return ctas_per_sm_t<D, 1, U16>(M, r);
    case 2: return ctas_per_sm_t<D, 2, U16>(M, r);
    case 4: return ctas_per_sm_t<D, 4, U16>(M, r);
    default: return ctas_per_sm_t<D, 8, U16>(M, r);
  }
}
int ctas_per_sm(const kv2_cache& c, int G) {
  if (c.d == 64) return c.M > 256 ? ctas_per_sm_g<64, true>(G, c.M, c.r) : ctas_per_sm_g<64, false>(G, c.M, c.r);
  return c.M > 256 ? ctas_per_sm_g<128, true>(G, c.M, c.r) : ctas_per_sm_g<128, false>(G, c.M, c.r);
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

// Splits along the sequence: as many CTAs as fit in one wave (resident CTAs
// per SM x SMs), each covering a whole number of 128-token tiles.
void plan_splits(const kv2_cache& c, int H_q, int len, int* splits, int* tiles_per_split) {
  const int tiles = (len + kTile - 1) / kTile;
  const int pairs = c.B * c.H_kv;
  const int slots = sm_count() * ctas_per_sm(c, H_q / c.H_kv);
  int want = slots / pairs;
  want = want < 1 ? 1 : want;
  int tps = (tiles + want - 1) / want;
  tps = tps < 1 ? 1 : tps;
  *tiles_per_split = tps;
  *splits = tiles > 0 ? (tiles + tps - 1) / tps : 1;
}

}  // namespace

size_t decode_workspace_bytes(const kv2_cache& c, int H_q, int len) {
  int splits, tps;
  plan_splits(c, H_q, len, &splits, &tps);
  const PrepLayout L(c.d, c.M, c.r);
  const size_t prep = size_t(c.B) * H_q * L.stride * 4;
  const size_t part = size_t(c.B) * c.H_kv * splits * (H_q / c.H_kv) * (c.d + 2) * 4;
  return ((prep + 255) & ~size_t(255)) + part;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const kv2_cache& c = *a.c;
  int splits, tps;
  plan_splits(c, a.H_q, a.len, &splits, &tps);
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
