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
//   decode_split  grid (splits, B*H_kv): first the query-side tables of the G
//                 query heads sharing the KV head (q scaled, with a per-channel
//                 power-of-4 factor matching the code extraction; q.mu_j for
//                 every centre; u = qP; per-group sums of q), built while the
//                 first tile is in flight; then it streams 128-token tiles of
//                 every packed stream with cp.async (double-buffered), one
//                 thread per token for the logits of the G query heads (so
//                 each byte is read once per KV head), online softmax, values
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

// ---------------------------------------------------------------------------
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

constexpr int kStages = 2;

// G consecutive floats to / from shared memory with the widest aligned accesses
template <int G>
__device__ __forceinline__ void store_vec(float* dst, const float (&v)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int i = 0; i < G; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  } else if constexpr (G == 2) {
    *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
  } else {
    dst[0] = v[0];
  }
}
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

// Thread mapping of the split kernel (128 threads, 128-token tiles):
//   cb = tid % 16: 8-channel block (half of code word cb/2, group cb/4)
//   ts = tid / 16: token slice, tokens ts, ts+8, ... of the tile
// In both phases a thread works on its 8 channels of 16 tokens, so the query
// values of its channels stay in registers. Per-token partial logits go
// through shared memory to the token's owner thread (tid = token).
template <int D, int G, bool U16>
struct DCfg {
  static constexpr int NG = D / 32;
  static constexpr int NW = D / 16;            // code words per token
  static constexpr int CB = D / 8;             // 8-channel blocks
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
  // per-token rows padded by 4 floats so that 8 consecutive tokens start in
  // distinct 16-byte bank groups (conflict-free 16-byte accesses)
  static constexpr int PS = CB * G + 4;                        // partial logits [token][cb][G]
  static constexpr int PWS = NG * G + 4;                       // p s_v [token][group][G]
  static constexpr int part_bytes = kTile * PS * 4;
  static constexpr int pw_bytes = kTile * PWS * 4;
  static constexpr int red_bytes = (TS * G * D + kThreads * G * NG) * 4;  // final reduction
  __host__ __device__ static int stage_bytes(int r) { return (ps_off + kTile * r * 2 + 15) & ~15; }
  __host__ __device__ static int stages_bytes(int r) {
    const int st = kStages * stage_bytes(r);
    return st > red_bytes ? st : red_bytes;
  }
  __host__ __device__ static int tables_bytes(int M, int r) {
    return part_bytes + pw_bytes + (G * M + G * r + G * NG + 4 * G + 4) * 4;
  }
};

template <int D, int G, bool U16>
__global__ void __launch_bounds__(kThreads) decode_split(SplitParams p) {
  using Cfg = DCfg<D, G, U16>;
  constexpr int NG = Cfg::NG, NW = Cfg::NW, CB = Cfg::CB, TS = Cfg::TS;
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = p.r, M = p.M;
  const int stage = Cfg::stage_bytes(r);
  unsigned char* tables = smem + Cfg::stages_bytes(r);
  float* part_s = reinterpret_cast<float*>(tables);                             // [kTile][CB][G]
  float* pw_s = reinterpret_cast<float*>(tables + Cfg::part_bytes);            // [kTile][NG][G]
  float* mus = reinterpret_cast<float*>(tables + Cfg::part_bytes + Cfg::pw_bytes);  // [G][M]
  float* us = mus + G * M;                                                      // [G][r]
  float* sgs = us + G * r;                                                      // [G][NG]
  float* red = sgs + G * NG;                                                    // [4 warps][G]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H_kv, h = bh % p.H_kv;
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

  // ---- query-side tables of the G query heads sharing this KV head, built
  // while the first tile is in flight (part_s is not used before that tile):
  // q in log2 units, q . mu_j for every centre, u = q P, per-group sums of q
  float* qs = part_s;                                    // [G][D]
  float* pst = part_s + G * D;                           // a chunk of rows of P, [rows][r]
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
      const float* q = qs + (i / NG) * D + (i % NG) * 32;
      float acc = 0.0f;
      for (int c = 0; c < 32; ++c) acc += q[c];
      sgs[i] = acc;
    }
    if (r) {
      const float* Ph = p.P + size_t(h) * D * r;
      const int rows = min(D, (Cfg::part_bytes / 4 - G * D) / r);   // >= 1 since r <= D
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

  const int cb = tid % CB, ts = tid / CB;
  const int word = cb >> 1, sub = (cb & 1) * 4, grp = cb >> 2;   // channel pairs sub..sub+3 of the word
  // this thread's query values: 8 channels x G heads as channel pairs, each
  // channel carrying the factor 4^-e that matches its code extraction
  f32x2 q2[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float* q = qs + g * D + cb * 8;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c0 = cb * 8 + 2 * k;
      q2[g][k] = pack2(ldexpf(q[2 * k], -2 * code_exp(c0 % 16)), ldexpf(q[2 * k + 1], -2 * code_exp((c0 + 1) % 16)));
    }
  }

  float m_run[G], lsum[G], pz[G][NG];
  f32x2 oacc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -FLT_MAX;
    lsum[g] = 0.0f;
#pragma unroll
    for (int k = 0; k < NG; ++k) pz[g][k] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) oacc[g][c] = 0ull;
  }

  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<0>();
    __syncthreads();          // tile data ready; every thread is done with tile - 1
    issue(tile + 1);          // into the stage tile - 1 used
    const unsigned char* cur = smem + (tile % kStages) * stage;
    const int n = min(kTile, t_end - (t_begin + tile * kTile));

    // ---- K: partial dot products of this thread's 8 channels, scaled by s_grp
    {
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(cur + Cfg::kc_off);
      const uint32_t* ksz = reinterpret_cast<const uint32_t*>(cur + Cfg::ks_off);
#pragma unroll 4
      for (int k = 0; k < kTile / TS; ++k) {
        const int t = ts + k * TS;
        const WordPair wp = word_pair(kw[t * NW + word]);
        f32x2 dacc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) dacc[g] = 0ull;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const f32x2 cpair = code_pair(wp, sub + c);
#pragma unroll
          for (int g = 0; g < G; ++g) dacc[g] = ffma2(q2[g][c], cpair, dacc[g]);
        }
        const float s = __half2float(__ushort_as_half(uint16_t(ksz[t * NG + grp] & 0xffff)));
        float pd[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float2 d2 = unpack2(dacc[g]);
          pd[g] = s * (d2.x + d2.y);
        }
        store_vec<G>(part_s + t * Cfg::PS + cb * G, pd);
      }
    }
    __syncthreads();

    // ---- logits (thread = token): partials + centre + zero terms + PSAC
    const int t = tid;
    float lg[G];
    {
      int idx;
      if constexpr (U16) idx = reinterpret_cast<const uint16_t*>(cur + Cfg::ix_off)[t];
      else idx = cur[Cfg::ix_off + t];
      idx = min(idx, M - 1);
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g] = mus[g * M + idx];
      const float* src = part_s + t * Cfg::PS;
#pragma unroll
      for (int c = 0; c < CB; ++c) {
        float pd[G];
        load_vec<G>(src + c * G, pd);
#pragma unroll
        for (int g = 0; g < G; ++g) lg[g] += pd[g];
      }
      const uint32_t* ksz = reinterpret_cast<const uint32_t*>(cur + Cfg::ks_off) + t * NG;
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        const float z = __half2float(__ushort_as_half(uint16_t(ksz[k] >> 16)));
#pragma unroll
        for (int g = 0; g < G; ++g) lg[g] = fmaf(z, sgs[g * NG + k], lg[g]);
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
        for (int c = 0; c < 4; ++c) oacc[g][c] = fmul2(oacc[g][c], a2);
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
      for (int k = 0; k < NG; ++k) {
        const uint32_t sz = vsz[k];
        const float sv = (t < n) ? __half2float(__ushort_as_half(uint16_t(sz & 0xffff))) : 0.0f;
        const float zv = (t < n) ? __half2float(__ushort_as_half(uint16_t(sz >> 16))) : 0.0f;
        float pw[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          pw[g] = pr[g] * sv;
          pz[g][k] = fmaf(pr[g], zv, pz[g][k]);
        }
        store_vec<G>(pw_s + t * Cfg::PWS + k * G, pw);
      }
    }
    __syncthreads();

    // ---- values: this thread's 8 channels over its 16 tokens
    {
      const uint32_t* vw = reinterpret_cast<const uint32_t*>(cur + Cfg::vc_off);
#pragma unroll 4
      for (int k = 0; k < kTile / TS; ++k) {
        const int tt = ts + k * TS;
        const WordPair wp = word_pair(vw[tt * NW + word]);
        float pv[G];
        load_vec<G>(pw_s + tt * Cfg::PWS + grp * G, pv);
        f32x2 pw[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pw[g] = pack2(pv[g], pv[g]);   // {p s_v, p s_v}
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const f32x2 cpair = code_pair(wp, sub + c);
#pragma unroll
          for (int g = 0; g < G; ++g) oacc[g][c] = ffma2(pw[g], cpair, oacc[g][c]);
        }
      }
    }
    // no barrier here: the next tile's first barrier orders these reads before
    // the copy into this stage and the next writes of part_s / pw_s
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- reduce: value partials over token slices, p z_v and p sums over threads
  float* rbuf = reinterpret_cast<float*>(smem);            // [TS][G][D], then [kThreads][G][NG]
  float* zbuf = rbuf + TS * G * D;
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 v = unpack2(oacc[g][c]);
      const int ch = cb * 8 + 2 * c;
      rbuf[(ts * G + g) * D + ch] = ldexpf(v.x, -2 * code_exp(ch % 16));
      rbuf[(ts * G + g) * D + ch + 1] = ldexpf(v.y, -2 * code_exp((ch + 1) % 16));
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
    float mr = m_run[0];
#pragma unroll
    for (int g = 1; g < G; ++g) if (tid == g) mr = m_run[g];
    dst[tid * (D + 2) + D] = mr;
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
  return size_t(c.B) * c.H_kv * splits * (H_q / c.H_kv) * (c.d + 2) * 4;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const kv2_cache& c = *a.c;
  int splits, tps;
  plan_splits(c, a.H_q, a.len, &splits, &tps);
  float* part = static_cast<float*>(a.ws);
  SplitParams sp{c.k_code, c.v_code, c.k_sz, c.v_sz, c.cidx, c.psac,
                 static_cast<const uint16_t*>(a.Q), static_cast<const uint16_t*>(c.centroids), c.P,
                 a.sm_scale * kLog2e, part, c.H_kv, a.H_q, c.M, c.r, c.capacity, a.len, splits, tps};
  const int G = a.H_q / c.H_kv;
  cudaError_t e;
  if (c.d == 64) e = (c.M > 256) ? launch_g<64, true>(G, sp, c.B, s) : launch_g<64, false>(G, sp, c.B, s);
  else e = (c.M > 256) ? launch_g<128, true>(G, sp, c.B, s) : launch_g<128, false>(G, sp, c.B, s);
  if (e != cudaSuccess) return e;
  decode_combine<<<c.B * a.H_q, 128, 0, s>>>(part, a.H_q, c.H_kv, c.d, splits, a.out, a.out_dtype);
  return cudaGetLastError();
}

}  // namespace kv2
