// api.cu — extern "C" entry points of libkv2 (declared in include/kv2.h):
// argument validation, workspace sizing and kernel dispatch. The library never
// allocates device memory; every buffer is the caller's.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"

namespace {

thread_local char g_last_error[512] = "";

// An NVTX range named after the entry point, open for the call (profilers
// show the library's calls on the host timeline; no cost without a tool).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
};

kv2_status fail(kv2_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

kv2_status ok() {
  g_last_error[0] = '\0';
  return KV2_OK;
}

kv2_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(KV2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape and pointer checks common to every call that reads the cache.
// Channels per (scale, zero) group (0 selects 32): 32, 64 or 128, at most d.
kv2_status check_group(int d, int group) {
  const int g = group ? group : kv2::kGroup;
  if (g != 32 && g != 64 && g != 128) return fail(KV2_ERR_UNSUPPORTED, "group=%d (32, 64 or 128)", group);
  if (g > d) return fail(KV2_ERR_UNSUPPORTED, "group=%d larger than d=%d", g, d);
  return KV2_OK;
}

kv2_status check_cache(const kv2_cache* c, bool need_cache_streams, bool need_fit) {
  if (!c) return fail(KV2_ERR_INVALID_ARG, "cache descriptor is NULL");
  if (c->B <= 0 || c->H_kv <= 0 || c->capacity < 0 || c->M <= 0 || c->r < 0)
    return fail(KV2_ERR_INVALID_ARG, "cache sizes must be positive (B=%d H_kv=%d M=%d r=%d cap=%d)",
                c->B, c->H_kv, c->M, c->r, c->capacity);
  if (c->d != 64 && c->d != 128) return fail(KV2_ERR_UNSUPPORTED, "head dim d=%d (supported: 64, 128)", c->d);
  if (c->M > kv2::kMaxCentroids) return fail(KV2_ERR_UNSUPPORTED, "M=%d centroids (max 512)", c->M);
  if (c->r > c->d || (c->r & 1)) return fail(KV2_ERR_UNSUPPORTED, "PSAC rank r=%d (even, <= d)", c->r);
  if (kv2_status st = check_group(c->d, c->group); st != KV2_OK) return st;
  if (c->capacity % 16) return fail(KV2_ERR_UNSUPPORTED, "capacity %d is not a multiple of 16", c->capacity);
  if (c->psac_fmt != 0 && c->psac_fmt != 1) return fail(KV2_ERR_INVALID_ARG, "psac_fmt=%d (0: fp16, 1: int8)", c->psac_fmt);
  if (c->block_table && (c->page_tokens < 128 || c->page_tokens % 128 || c->capacity % c->page_tokens))
    return fail(KV2_ERR_UNSUPPORTED, "paged cache: page_tokens=%d (a multiple of 128 dividing capacity %d)",
                c->page_tokens, c->capacity);
  if (!c->centroids || !aligned16(c->centroids))
    return fail(KV2_ERR_INVALID_ARG, "centroids must be a non-NULL 16-byte aligned pointer");
  if (need_cache_streams) {
    const void* ptrs[] = {c->k_code, c->v_code, c->k_sz, c->v_sz, c->cidx};
    for (const void* p : ptrs)
      if (!p || !aligned16(p)) return fail(KV2_ERR_INVALID_ARG, "cache stream pointer NULL or not 16-byte aligned");
    if (c->r && (!c->psac || !aligned16(c->psac)))
      return fail(KV2_ERR_INVALID_ARG, "psac pointer NULL or not 16-byte aligned");
    if (c->psac_fmt == 1 && c->r && (!c->psac_scale || !aligned16(c->psac_scale)))
      return fail(KV2_ERR_INVALID_ARG, "psac_scale pointer NULL or not 16-byte aligned (int8 PSAC format)");
  }
  if (need_fit) {
    if (!c->w || !c->Wg || !aligned16(c->w) || !aligned16(c->Wg))
      return fail(KV2_ERR_INVALID_ARG, "w / Wg pointers NULL or not 16-byte aligned");
  }
  if (c->r && (!c->P || !aligned16(c->P))) return fail(KV2_ERR_INVALID_ARG, "P pointer NULL or not 16-byte aligned");
  return KV2_OK;
}

}  // namespace

namespace kv2 {
kv2_status set_last_error(kv2_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}
}  // namespace kv2

extern "C" {

const char* kv2_status_string(kv2_status s) {
  switch (s) {
    case KV2_OK: return "KV2_OK";
    case KV2_ERR_INVALID_ARG: return "KV2_ERR_INVALID_ARG";
    case KV2_ERR_UNSUPPORTED: return "KV2_ERR_UNSUPPORTED";
    case KV2_ERR_CAPACITY: return "KV2_ERR_CAPACITY";
    case KV2_ERR_CUDA: return "KV2_ERR_CUDA";
    case KV2_ERR_TIMEOUT: return "KV2_ERR_TIMEOUT";
    case KV2_ERR_WORKSPACE: return "KV2_ERR_WORKSPACE";
  }
  return "KV2_ERR_UNKNOWN";
}

const char* kv2_last_error(void) { return g_last_error; }

int kv2_version(void) { return 200; }

size_t kv2_fit_workspace_size(int H_kv, int d) {
  if (H_kv <= 0 || (d != 64 && d != 128)) return 0;
  return kv2::fit_workspace_bytes(H_kv, d);
}

kv2_status kv2_fit_psac_basis(const uint16_t* Qhist, int n, int H_q, int H_kv, int d, int r, int group,
                              float* P, float* w, float* Wg, float* energy, void* ws,
                              size_t ws_bytes, void* stream) {
  const CallRange range_("kv2_fit_psac_basis");
  if (n <= 0 || H_q <= 0 || H_kv <= 0 || r < 0) return fail(KV2_ERR_INVALID_ARG, "fit: sizes must be positive");
  if (H_q % H_kv) return fail(KV2_ERR_UNSUPPORTED, "fit: H_q=%d not a multiple of H_kv=%d", H_q, H_kv);
  if (d != 64 && d != 128) return fail(KV2_ERR_UNSUPPORTED, "fit: head dim d=%d (supported: 64, 128)", d);
  if (r > d) return fail(KV2_ERR_UNSUPPORTED, "fit: r=%d > d=%d", r, d);
  if (kv2_status st = check_group(d, group); st != KV2_OK) return st;
  if (!Qhist || !w || !Wg || !ws || (r && !P)) return fail(KV2_ERR_INVALID_ARG, "fit: NULL pointer");
  if (!aligned16(Qhist) || !aligned16(ws)) return fail(KV2_ERR_INVALID_ARG, "fit: misaligned pointer");
  if (ws_bytes < kv2::fit_workspace_bytes(H_kv, d))
    return fail(KV2_ERR_WORKSPACE, "fit: workspace %zu < %zu bytes", ws_bytes, kv2::fit_workspace_bytes(H_kv, d));
  kv2::FitArgs a{Qhist, n, H_q, H_kv, d, r, P, w, Wg, energy, ws, group ? group : kv2::kGroup};
  return cuda_status(kv2::launch_fit(a, static_cast<cudaStream_t>(stream)), "fit launch");
}

size_t kv2_top1_workspace_size(int B, int nq, int H_q, int len) {
  if (B <= 0 || nq <= 0 || H_q <= 0 || len < 0) return 0;
  return kv2::top1_workspace_bytes(B, nq, H_q, len);
}

kv2_status kv2_decode_top1(const kv2_cache* c, int len, const uint16_t* Q, int nq, int H_q, int32_t* top1,
                           void* ws, size_t ws_bytes, void* stream) {
  const CallRange range_("kv2_decode_top1");
  kv2_status st = check_cache(c, true, false);
  if (st != KV2_OK) return st;
  if (H_q <= 0 || H_q % c->H_kv) return fail(KV2_ERR_UNSUPPORTED, "top1: H_q=%d not a multiple of H_kv=%d", H_q, c->H_kv);
  if (len < 0 || len > c->capacity) return fail(KV2_ERR_CAPACITY, "top1: len=%d outside 0..capacity=%d", len, c->capacity);
  if (nq <= 0) return fail(KV2_ERR_INVALID_ARG, "top1: nq=%d", nq);
  if (!Q || !top1 || !ws || !aligned16(ws)) return fail(KV2_ERR_INVALID_ARG, "top1: NULL or misaligned pointer");
  const size_t need = kv2::top1_workspace_bytes(c->B, nq, H_q, len);
  if (ws_bytes < need) return fail(KV2_ERR_WORKSPACE, "top1: workspace %zu < %zu bytes", ws_bytes, need);
  kv2::Top1Args a{c, Q, nullptr, c->B, nq, H_q, c->H_kv, c->d, len, top1, ws};
  return cuda_status(kv2::launch_top1(a, static_cast<cudaStream_t>(stream)), "top1 launch");
}

kv2_status kv2_dense_top1(const uint16_t* K, int B, int len, int H_kv, int d, const uint16_t* Q, int nq, int H_q,
                          int32_t* top1, void* ws, size_t ws_bytes, void* stream) {
  const CallRange range_("kv2_dense_top1");
  if (B <= 0 || nq <= 0 || H_kv <= 0 || len < 0 || d <= 0 || d > 1024)
    return fail(KV2_ERR_INVALID_ARG, "dense_top1: B=%d H_kv=%d len=%d d=%d", B, H_kv, len, d);
  if (H_q <= 0 || H_q % H_kv) return fail(KV2_ERR_UNSUPPORTED, "dense_top1: H_q=%d not a multiple of H_kv=%d", H_q, H_kv);
  if ((len && !K) || !Q || !top1 || !ws || !aligned16(ws))
    return fail(KV2_ERR_INVALID_ARG, "dense_top1: NULL or misaligned pointer");
  const size_t need = kv2::top1_workspace_bytes(B, nq, H_q, len);
  if (ws_bytes < need) return fail(KV2_ERR_WORKSPACE, "dense_top1: workspace %zu < %zu bytes", ws_bytes, need);
  kv2::Top1Args a{nullptr, Q, K, B, nq, H_q, H_kv, d, len, top1, ws};
  return cuda_status(kv2::launch_top1(a, static_cast<cudaStream_t>(stream)), "dense_top1 launch");
}

size_t kv2_fit_centroids_workspace_size(int H_kv, int d, int M) {
  if (H_kv <= 0 || (d != 64 && d != 128) || M < 1 || M > 512) return 0;
  return kv2::fit_centroids_workspace_bytes(H_kv, d, M);
}

kv2_status kv2_fit_centroids(const uint16_t* X, int n, int H_kv, int d, int M, int candidates, int group,
                             const float* w, const float* Wg, int iters, uint16_t* centroids, int32_t* assign,
                             void* ws, size_t ws_bytes, void* stream) {
  const CallRange range_("kv2_fit_centroids");
  if (H_kv <= 0 || n < 0 || n > 65536) return fail(KV2_ERR_INVALID_ARG, "fit_centroids: H_kv=%d, n=%d", H_kv, n);
  if (d != 64 && d != 128) return fail(KV2_ERR_UNSUPPORTED, "fit_centroids: head dim d=%d (supported: 64, 128)", d);
  if (M < 1 || M > 512) return fail(KV2_ERR_UNSUPPORTED, "fit_centroids: M=%d outside 1..512", M);
  if (candidates < 1 || candidates > M)
    return fail(KV2_ERR_INVALID_ARG, "fit_centroids: candidates=%d outside 1..M=%d", candidates, M);
  if (iters < 0) return fail(KV2_ERR_INVALID_ARG, "fit_centroids: iters=%d < 0", iters);
  if (kv2_status st = check_group(d, group); st != KV2_OK) return st;
  if (iters == 0 || n == 0) return KV2_OK;
  if (!X || !w || !Wg || !centroids || !assign || !ws)
    return fail(KV2_ERR_INVALID_ARG, "fit_centroids: NULL pointer");
  if (!aligned16(X) || !aligned16(centroids) || !aligned16(ws))
    return fail(KV2_ERR_INVALID_ARG, "fit_centroids: misaligned pointer");
  const size_t need = kv2::fit_centroids_workspace_bytes(H_kv, d, M);
  if (ws_bytes < need) return fail(KV2_ERR_WORKSPACE, "fit_centroids: workspace %zu < %zu bytes", ws_bytes, need);
  kv2::FitCentroidsArgs a{X, n, H_kv, d, M, candidates, iters, w, Wg, centroids, assign, ws,
                          group ? group : kv2::kGroup};
  return cuda_status(kv2::launch_fit_centroids(a, static_cast<cudaStream_t>(stream)), "fit_centroids launch");
}

namespace {

// argument checks of a quantize/append call (the cache already checked)
kv2_status check_quantize(const kv2_cache* c, const uint16_t* K, const uint16_t* V, int n_new, int pos,
                          int candidates) {
  if (n_new < 0) return fail(KV2_ERR_INVALID_ARG, "quantize: n_new=%d < 0", n_new);
  if (pos < 0 || pos > c->capacity - n_new)
    return fail(KV2_ERR_CAPACITY, "quantize: slots [%d, %d) exceed capacity %d", pos, pos + n_new, c->capacity);
  if (candidates < 1 || candidates > c->M)
    return fail(KV2_ERR_INVALID_ARG, "quantize: candidates=%d outside 1..M=%d", candidates, c->M);
  if (n_new > 0 && (!K || !V || !aligned16(K) || !aligned16(V)))
    return fail(KV2_ERR_INVALID_ARG, "quantize: K / V NULL or not 16-byte aligned");
  return KV2_OK;
}

kv2::QuantizeArgs quantize_args(const kv2_cache* c, const uint16_t* K, const uint16_t* V, int n_new, int pos,
                                int candidates) {
  kv2::QuantizeArgs a{K, V, c->B, c->H_kv, c->d, c->M, c->r, c->capacity, n_new, pos, candidates,
                      c->centroids, c->P, c->w, c->Wg, c->k_code, c->v_code, c->k_sz, c->v_sz,
                      c->cidx, c->psac};
  a.psac_fmt = c->psac_fmt;
  a.psac_scale = c->psac_scale;
  a.table = c->block_table;
  a.page = c->page_tokens;
  a.group = kv2::cache_group(*c);
  return a;
}

// argument checks of a decode call (the cache already checked)
// Decode arguments other than the workspace.
kv2_status check_decode_args(const kv2_cache* c, int len, const uint16_t* Q, int H_q, void* out, int out_dtype) {
  if (H_q <= 0 || H_q % c->H_kv) return fail(KV2_ERR_UNSUPPORTED, "decode: H_q=%d not a multiple of H_kv=%d", H_q, c->H_kv);
  const int G = H_q / c->H_kv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(KV2_ERR_UNSUPPORTED, "decode: H_q/H_kv=%d (supported 1, 2, 4, 8)", G);
  if (len < 0 || len > c->capacity) return fail(KV2_ERR_CAPACITY, "decode: len=%d outside 0..capacity=%d", len, c->capacity);
  if (out_dtype != KV2_OUT_F32 && out_dtype != KV2_OUT_BF16) return fail(KV2_ERR_INVALID_ARG, "decode: out_dtype=%d", out_dtype);
  if (!Q || !out || !aligned16(Q) || !aligned16(out))
    return fail(KV2_ERR_INVALID_ARG, "decode: Q / out NULL or not 16-byte aligned");
  return KV2_OK;
}

kv2_status check_decode(const kv2_cache* c, int len, const uint16_t* Q, int H_q, void* out, int out_dtype,
                        void* ws, size_t ws_bytes) {
  if (kv2_status st = check_decode_args(c, len, Q, H_q, out, out_dtype); st != KV2_OK) return st;
  if (!ws || !aligned16(ws)) return fail(KV2_ERR_INVALID_ARG, "decode: ws NULL or not 16-byte aligned");
  const size_t need = kv2::decode_workspace_bytes(*c, H_q, len);
  if (ws_bytes < need) return fail(KV2_ERR_WORKSPACE, "decode: workspace %zu < %zu bytes", ws_bytes, need);
  return KV2_OK;
}

}  // namespace

}  // extern "C"

namespace kv2 {
kv2_status validate_decode(const kv2_cache* c, int len, const uint16_t* Q, int H_q, void* out, int out_dtype,
                           size_t* ws_need) {
  kv2_status st = check_cache(c, true, false);
  if (st == KV2_OK) st = check_decode_args(c, len, Q, H_q, out, out_dtype);
  if (st == KV2_OK) *ws_need = decode_workspace_bytes(*c, H_q, len);
  return st;
}
}  // namespace kv2

extern "C" {

kv2_status kv2_quantize_append(const kv2_cache* c, const uint16_t* K, const uint16_t* V, int n_new,
                               int pos, int candidates, void* stream) {
  const CallRange range_("kv2_quantize_append");
  kv2_status st = check_cache(c, true, true);
  if (st != KV2_OK) return st;
  st = check_quantize(c, K, V, n_new, pos, candidates);
  if (st != KV2_OK) return st;
  if (n_new == 0) return ok();
  return cuda_status(kv2::launch_quantize(quantize_args(c, K, V, n_new, pos, candidates),
                                          static_cast<cudaStream_t>(stream)), "quantize launch");
}

size_t kv2_decode_workspace_size(const kv2_cache* c, int H_q, int len) {
  if (!c || H_q <= 0 || c->H_kv <= 0 || H_q % c->H_kv || len < 0) return 0;
  if (check_cache(c, false, false) != KV2_OK) return 0;
  return kv2::decode_workspace_bytes(*c, H_q, len);
}

kv2_status kv2_attention_decode(const kv2_cache* c, int len, const uint16_t* Q, int H_q, float sm_scale,
                                void* out, int out_dtype, void* ws, size_t ws_bytes, void* stream) {
  const CallRange range_("kv2_attention_decode");
  kv2_status st = check_cache(c, true, false);
  if (st != KV2_OK) return st;
  st = check_decode(c, len, Q, H_q, out, out_dtype, ws, ws_bytes);
  if (st != KV2_OK) return st;
  kv2::DecodeArgs a{c, len, H_q, Q, sm_scale, out, out_dtype, ws, ws_bytes};
  return cuda_status(kv2::launch_decode(a, static_cast<cudaStream_t>(stream)), "decode launch");
}

kv2_status kv2_append_attention_decode(const kv2_cache* c, const uint16_t* K_new, const uint16_t* V_new,
                                       int n_new, int pos, int candidates, const uint16_t* Q, int H_q,
                                       float sm_scale, void* out, int out_dtype, void* ws, size_t ws_bytes,
                                       void* stream) {
  const CallRange range_("kv2_append_attention_decode");
  kv2_status st = check_cache(c, true, true);
  if (st != KV2_OK) return st;
  st = check_quantize(c, K_new, V_new, n_new, pos, candidates);
  if (st != KV2_OK) return st;
  const int len = pos + n_new;
  st = check_decode(c, len, Q, H_q, out, out_dtype, ws, ws_bytes);
  if (st != KV2_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  kv2::DecodeArgs a{c, len, H_q, Q, sm_scale, out, out_dtype, ws, ws_bytes};
  if (n_new > 0) {
    st = cuda_status(kv2::launch_quantize(quantize_args(c, K_new, V_new, n_new, pos, candidates), s),
                     "quantize launch");
    if (st != KV2_OK) return st;
    a.wait_from = pos;
  }
  return cuda_status(kv2::launch_decode(a, s), "decode launch");
}

size_t kv2_chunk_workspace_size(const kv2_cache* c, int H_q, int Nq) {
  if (!c || H_q <= 0 || c->H_kv <= 0 || H_q % c->H_kv || Nq < 0) return 0;
  if (check_cache(c, false, false) != KV2_OK) return 0;
  return kv2::chunk_workspace_bytes(*c, H_q, Nq);
}

kv2_status kv2_attention_chunk(const kv2_cache* c, int len, const uint16_t* Q, int H_q, int Nq,
                               const uint16_t* Kself, const uint16_t* Vself, int frame_tokens,
                               float sm_scale, void* out, int out_dtype, void* ws, size_t ws_bytes,
                               void* stream) {
  const CallRange range_("kv2_attention_chunk");
  kv2_status st = check_cache(c, true, false);
  if (st != KV2_OK) return st;
  if (c->d != 128) return fail(KV2_ERR_UNSUPPORTED, "chunk: head dim d=%d (supported: 128)", c->d);
  if (c->r != 0 && c->r != 8 && c->r != 16) return fail(KV2_ERR_UNSUPPORTED, "chunk: r=%d (supported 0, 8, 16)", c->r);
  if (H_q <= 0 || H_q % c->H_kv) return fail(KV2_ERR_UNSUPPORTED, "chunk: H_q=%d not a multiple of H_kv=%d", H_q, c->H_kv);
  if (Nq < 0 || frame_tokens <= 0) return fail(KV2_ERR_INVALID_ARG, "chunk: Nq=%d frame_tokens=%d", Nq, frame_tokens);
  if (len < 0 || len > c->capacity) return fail(KV2_ERR_CAPACITY, "chunk: len=%d outside 0..capacity=%d", len, c->capacity);
  if (out_dtype != KV2_OUT_F32 && out_dtype != KV2_OUT_BF16) return fail(KV2_ERR_INVALID_ARG, "chunk: out_dtype=%d", out_dtype);
  if (Nq == 0) return ok();
  if (!Q || !Kself || !Vself || !out || !ws)
    return fail(KV2_ERR_INVALID_ARG, "chunk: NULL pointer");
  if (!aligned16(Q) || !aligned16(Kself) || !aligned16(Vself) || !aligned16(out) || !aligned16(ws))
    return fail(KV2_ERR_INVALID_ARG, "chunk: pointer not 16-byte aligned");
  const size_t need = kv2::chunk_workspace_bytes(*c, H_q, Nq);
  if (ws_bytes < need) return fail(KV2_ERR_WORKSPACE, "chunk: workspace %zu < %zu bytes", ws_bytes, need);
  kv2::ChunkArgs a{c, len, H_q, Nq, frame_tokens, Q, Kself, Vself, sm_scale, out, out_dtype, ws, ws_bytes, nullptr};
  cudaError_t e = kv2::launch_chunk(a, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return fail(KV2_ERR_UNSUPPORTED, "chunk: kernel not available");
  return cuda_status(e, "chunk launch");
}

namespace {

// one stream of a paged cache: device base and bytes per token slot
struct PageStream {
  char* base;
  size_t per_token;
};

// the streams of a cache in the order of a page's host image; returns how many
int page_streams(const kv2_cache* c, PageStream (&s)[7]) {
  const size_t words = size_t(c->d / 16) * 4, groups = size_t(c->d / kv2::cache_group(*c)) * 4;
  int n = 0;
  s[n++] = {reinterpret_cast<char*>(c->k_code), words};
  s[n++] = {reinterpret_cast<char*>(c->v_code), words};
  s[n++] = {reinterpret_cast<char*>(c->k_sz), groups};
  s[n++] = {reinterpret_cast<char*>(c->v_sz), groups};
  s[n++] = {static_cast<char*>(c->cidx), size_t(c->M <= 256 ? 1 : 2)};
  if (c->r) s[n++] = {reinterpret_cast<char*>(c->psac), size_t(c->psac_fmt == 1 ? c->r : 2 * c->r)};
  if (c->r && c->psac_fmt == 1) s[n++] = {reinterpret_cast<char*>(c->psac_scale), 2};
  return n;
}

size_t page_image_bytes(const kv2_cache* c) {
  PageStream s[7];
  const int n = page_streams(c, s);
  size_t per_token = 0;
  for (int i = 0; i < n; ++i) per_token += s[i].per_token;
  return size_t(c->H_kv) * size_t(c->page_tokens) * per_token;
}

kv2_status check_page(const kv2_cache* c, int page, int num_pages, const void* host) {
  kv2_status st = check_cache(c, true, false);
  if (st != KV2_OK) return st;
  if (!c->block_table) return fail(KV2_ERR_INVALID_ARG, "page: the cache is not paged (block_table is NULL)");
  if (num_pages <= 0 || page < 0 || page >= num_pages)
    return fail(KV2_ERR_INVALID_ARG, "page: page %d outside 0..num_pages-1 (num_pages=%d)", page, num_pages);
  if (!host) return fail(KV2_ERR_INVALID_ARG, "page: host buffer is NULL");
  return KV2_OK;
}

// page `page` of every stream (slots page*H_kv*page_tokens .. +H_kv*page_tokens,
// contiguous in each stream) to or from the host image
kv2_status page_copy(const kv2_cache* c, int page, char* host, bool store, cudaStream_t stream) {
  PageStream s[7];
  const int n = page_streams(c, s);
  const size_t slots = size_t(c->H_kv) * size_t(c->page_tokens);
  for (int i = 0; i < n; ++i) {
    const size_t bytes = slots * s[i].per_token;
    char* dev = s[i].base + size_t(page) * bytes;
    const cudaError_t e = store ? cudaMemcpyAsync(host, dev, bytes, cudaMemcpyDeviceToHost, stream)
                                : cudaMemcpyAsync(dev, host, bytes, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_status(e, store ? "page_store copy" : "page_load copy");
    host += bytes;
  }
  return ok();
}

}  // namespace

size_t kv2_page_bytes(const kv2_cache* c) {
  if (!c || !c->block_table || check_cache(c, false, false) != KV2_OK) return 0;
  return page_image_bytes(c);
}

kv2_status kv2_page_store(const kv2_cache* c, int page, int num_pages, void* host, void* stream) {
  const CallRange range_("kv2_page_store");
  const kv2_status st = check_page(c, page, num_pages, host);
  if (st != KV2_OK) return st;
  return page_copy(c, page, static_cast<char*>(host), true, static_cast<cudaStream_t>(stream));
}

kv2_status kv2_page_load(const kv2_cache* c, int page, int num_pages, const void* host, void* stream) {
  const CallRange range_("kv2_page_load");
  const kv2_status st = check_page(c, page, num_pages, host);
  if (st != KV2_OK) return st;
  return page_copy(c, page, const_cast<char*>(static_cast<const char*>(host)), false,
                   static_cast<cudaStream_t>(stream));
}

}  // extern "C"
