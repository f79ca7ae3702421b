// decode.cu — attention of one query token per sequence over the packed
// 2-bit cache: the host side of kv2_attention_decode (split planning,
// launches) and the log-sum-exp merge of the splits. The split kernel is in
// decode_split.cuh.
#include <cfloat>

#include "decode_split.cuh"

namespace kv2 {
namespace {

using namespace dsplit;

// ---------------------------------------------------------------------------
__global__ void decode_combine(const float* __restrict__ part, int H_q, int H_kv, int D,
                               int splits, void* out, int out_dtype) {
  // launched as the split kernel's programmatic dependent: its partials are
  // complete and visible after this wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int bq = blockIdx.x;
  const int b = bq / H_q, hq = bq % H_q;
  const int G = H_q / H_kv, h = hq / G, g = hq % G;
  const float* base = part + (size_t(b * H_kv + h) * splits) * G * (D + 2) + g * (D + 2);
  const size_t sstride = size_t(G) * (D + 2);
  const int c = threadIdx.x, lane = c & 31;          // one thread per channel (blockDim = D)
  // lane s of every warp reads split s (32 at a time): the overall maximum
  float m = -FLT_MAX;
  for (int s0 = 0; s0 < splits; s0 += 32) {
    const int sp = s0 + lane;
    if (sp < splits && base[sp * sstride + D + 1] > 0.0f) m = fmaxf(m, base[sp * sstride + D]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // weights 2^(m_s - m) per split (0 for an empty split), shared by shuffles;
  // the channel sums' loads are independent of one another
  float o = 0.0f, l = 0.0f;
  for (int s0 = 0; s0 < splits; s0 += 32) {
    const int sp = s0 + lane;
    float f = 0.0f;
    if (sp < splits) {
      const float ls = base[sp * sstride + D + 1];
      if (ls > 0.0f) {
        f = exp2f(base[sp * sstride + D] - m);
        l = fmaf(f, ls, l);
      }
    }
    const int ns = min(32, splits - s0);
    const float* col = base + size_t(s0) * sstride + c;
#pragma unroll 8
    for (int j = 0; j < ns; ++j) o = fmaf(__shfl_sync(0xffffffffu, f, j), col[j * sstride], o);
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) l += __shfl_xor_sync(0xffffffffu, l, k);
  const float v = (l > 0.0f) ? o / l : 0.0f;
  if (out_dtype == KV2_OUT_F32) static_cast<float*>(out)[size_t(bq) * D + c] = v;
  else static_cast<__nv_bfloat16*>(out)[size_t(bq) * D + c] = __float2bfloat16_rn(v);
}

template <int GS>
int ctas_per_sm_gs(const kv2_cache& c, int G) {
  if constexpr (GS <= 64) {
    if (c.d == 64)
      return c.M > 256 ? ctas_per_sm_g<64, true, GS>(G, c.M, c.r) : ctas_per_sm_g<64, false, GS>(G, c.M, c.r);
  }
  return c.M > 256 ? ctas_per_sm_g<128, true, GS>(G, c.M, c.r) : ctas_per_sm_g<128, false, GS>(G, c.M, c.r);
}
int ctas_per_sm(const kv2_cache& c, int G) {
  switch (cache_group(c)) {
    case 64: return ctas_per_sm_gs<64>(c, G);
    case 128: return ctas_per_sm_gs<128>(c, G);
    default: return ctas_per_sm_gs<32>(c, G);
  }
}

// the split kernel for the cache's head dim and centroid id width
template <int GS>
cudaError_t launch_gs(const kv2_cache& c, int G, const SplitParams& sp, cudaStream_t s) {
  if constexpr (GS <= 64) {
    if (c.d == 64) return c.M > 256 ? launch_g<64, true, GS>(G, sp, c.B, s) : launch_g<64, false, GS>(G, sp, c.B, s);
  }
  if (c.d != 128) return cudaErrorInvalidValue;
  return c.M > 256 ? launch_g<128, true, GS>(G, sp, c.B, s) : launch_g<128, false, GS>(G, sp, c.B, s);
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

// workspace: a 256-byte header (word 0: the sticky error word), then the
// split partials
constexpr size_t kWsHeader = 256;

size_t decode_workspace_bytes(const kv2_cache& c, int H_q, int len) {
  int splits, tps;
  plan_splits(c, H_q, len, &splits, &tps);
  return kWsHeader + size_t(c.B) * c.H_kv * splits * (H_q / c.H_kv) * (c.d + 2) * 4;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const kv2_cache& c = *a.c;
  int splits, tps;
  plan_splits(c, a.H_q, a.len, &splits, &tps);
  float* part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + kWsHeader);
  const int force = env_force_timeout();
  SplitParams sp{c.k_code, c.v_code, c.k_sz, c.v_sz, c.cidx, c.psac,
                 static_cast<const uint16_t*>(a.Q), static_cast<const uint16_t*>(c.centroids), c.P,
                 a.sm_scale * kLog2e, part, static_cast<int*>(a.ws),
                 force ? (1ull << 20) : env_wait_budget(), force, a.wait_from,
                 c.H_kv, a.H_q, c.M, c.r, c.capacity, a.len, splits, tps, c.psac_fmt, c.psac_scale,
                 c.block_table, c.page_tokens};
  const int G = a.H_q / c.H_kv;
  cudaError_t e;
  switch (cache_group(c)) {
    case 32: e = launch_gs<32>(c, G, sp, s); break;
    case 64: e = launch_gs<64>(c, G, sp, s); break;
    case 128: e = launch_gs<128>(c, G, sp, s); break;
    default: e = cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  // the merge runs as the split kernel's programmatic dependent (its launch
  // overlaps the split kernel's last CTAs)
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(c.B * a.H_q);
  cfg.blockDim = dim3(c.d);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine, static_cast<const float*>(part), a.H_q, c.H_kv, c.d, splits,
                            a.out, a.out_dtype);
}

}  // namespace kv2
