// Device helpers shared by the libkv2 kernels.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace kv2 {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float f16_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// fp32 -> fp16 bit patterns with an explicit rounding direction.
__device__ __forceinline__ uint16_t f16_rd(float x) { return __half_as_ushort(__float2half_rd(x)); }
__device__ __forceinline__ uint16_t f16_ru(float x) { return __half_as_ushort(__float2half_ru(x)); }
__device__ __forceinline__ uint16_t f16_rn(float x) { return __half_as_ushort(__float2half_rn(x)); }

// Order-preserving map of an fp32 value to uint32 (for packed argmin keys).
__device__ __forceinline__ uint32_t float_order(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of float_order.
__device__ __forceinline__ float order_float(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// INT2 group codec, shared by the quantizer's decision and encoding stages.
// zero = round-down of the minimum, scale = round-up of (max - zero)/3.
struct GroupParams {
  uint16_t s_bits, z_bits;
  float s, z;
};

__device__ __forceinline__ GroupParams group_params(float mn, float mx) {
  GroupParams p;
  p.z_bits = f16_rd(mn);
  p.z = f16_to_f32(p.z_bits);
  float q = __fdiv_rn(__fsub_rn(mx, p.z), 3.0f);
  p.s_bits = f16_ru(q);
  p.s = f16_to_f32(p.s_bits);
  return p;
}

__device__ __forceinline__ uint32_t group_code(float x, const GroupParams& p) {
  if (p.s == 0.0f) return 0u;
  float c = rintf(__fdiv_rn(__fsub_rn(x, p.z), p.s));
  c = fminf(fmaxf(c, 0.0f), 3.0f);
  return static_cast<uint32_t>(c);
}

// The same code as group_code, with the quotient taken as (x - z) * inv_s
// (inv_s = 1/s correctly rounded): that product is within 2.5 ulp of the
// correctly rounded quotient, so their rint agrees unless the product lies
// within 2^-18 of a half-integer (the quotient is below 4, where 3 ulp is
// under 2^-20); those rare cases take the correctly rounded division.
__device__ __forceinline__ uint32_t group_code_recip(float x, const GroupParams& p, float inv_s) {
  if (p.s == 0.0f) return 0u;
  const float d = __fsub_rn(x, p.z);
  const float qa = __fmul_rn(d, inv_s);
  float c = rintf(qa);
  if (fabsf(__fsub_rn(__fsub_rn(qa, floorf(qa)), 0.5f)) < 0x1p-18f) c = rintf(__fdiv_rn(d, p.s));
  c = fminf(fmaxf(c, 0.0f), 3.0f);
  return static_cast<uint32_t>(c);
}

// min / max of three floats in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed fp32 pairs (Blackwell f32x2 arithmetic: one instruction, two lanes,
// each rounded as its scalar counterpart)
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 up2(f32x2 v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ f32x2 ffma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 fadd2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
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
// 2^x by the hardware approximation (ex2.approx.ftz: relative error about
// 2^-22; 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Slot of token t of (sequence b, KV head h): contiguous streams
// [B][H_kv][cap], or a pool of pages [pages][H_kv][page] addressed through the
// block table [B][cap / page] (a page holds `page` consecutive tokens of one
// sequence; page is a multiple of 128, so a 128-token tile never leaves it)
__device__ __forceinline__ size_t cache_slot(const int32_t* table, int page, int H_kv, int cap, int b, int h,
                                             int t) {
  if (!table) return (size_t(b) * H_kv + h) * cap + t;
  const int pg = table[size_t(b) * (cap / page) + t / page];
  return (size_t(pg) * H_kv + h) * page + (t % page);
}

// INT8 PSAC coefficients of one token: scale = fp16 round-up of the fp32
// quotient max|a| / 127, code = clamp(round-half-even(a / scale), -127, 127)
// (0 when the scale is 0); the coefficient read back is code * scale
__device__ __forceinline__ void psac_int8(const float* a, int r, int8_t* q, uint16_t* scale_bits) {
  float amax = 0.0f;
  for (int i = 0; i < r; ++i) amax = fmaxf(amax, fabsf(a[i]));
  const uint16_t sb = f16_ru(__fdiv_rn(amax, 127.0f));
  const float s = f16_to_f32(sb);
  for (int i = 0; i < r; ++i) {
    const float v = (s > 0.0f) ? rintf(__fdiv_rn(a[i], s)) : 0.0f;
    q[i] = static_cast<int8_t>(fminf(fmaxf(v, -127.0f), 127.0f));
  }
  *scale_bits = sb;
}

__device__ __forceinline__ float group_dequant(uint32_t code, const GroupParams& p) {
  return __fmaf_rn(static_cast<float>(code), p.s, p.z);
}

}  // namespace kv2
