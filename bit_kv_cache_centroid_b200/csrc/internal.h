// Internal declarations shared by the host entry points and the kernel files
// of libkv2. Nothing here is part of the C ABI (see include/kv2.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <climits>

#include <cuda_runtime.h>

#include "kv2.h"

namespace kv2 {

constexpr int kGroup = 32;          // channels of a sub-group: one code-word pair, one 8-bit q.k k-step
constexpr int kMaxCentroids = 512;  // centroid ids fit in u16 above 256

// Channels per (scale, zero) group of a cache descriptor (0 selects 32).
inline int cache_group(const kv2_cache& c) { return c.group ? c.group : kGroup; }

// Arguments of one quantize/append call (validated by the host entry point).
struct QuantizeArgs {
  const uint16_t* K;   // bf16 [B][n_new][H][d]
  const uint16_t* V;
  int B, H, d, M, r, cap, n_new, pos, C;
  const uint16_t* cent;  // fp16 [H][M][d]
  const float* P;        // [H][d][r]
  const float* w;        // [H][d]
  const float* Wg;       // [H][d/group]
  uint32_t* k_code;
  uint32_t* v_code;
  uint32_t* k_sz;
  uint32_t* v_sz;
  void* cidx;
  uint16_t* psac;
  // assignment only (centre fitting): when set, the chosen centre of row
  // (b * n_new + t) and head h goes to assign[row * H + h] and nothing is
  // packed (V, P and the cache streams are not read or written)
  int32_t* assign = nullptr;
  // PSAC storage: 0 = fp16 coefficients in psac; 1 = int8 codes in psac and
  // one fp16 scale per token in psac_scale
  int psac_fmt = 0;
  uint16_t* psac_scale = nullptr;
  // paged cache: block table [B][cap / page] (null: contiguous streams)
  const int32_t* table = nullptr;
  int page = 0;
  int group = kGroup;  // channels per (scale, zero) group: 32, 64 or 128
};
cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t s);

// QSAC-aware centre fitting (Lloyd iterations with the QSAC assignment).
struct FitCentroidsArgs {
  const uint16_t* X;   // bf16 [n][H][D] sample keys
  int n, H, D, M, C, iters;
  const float* w;      // [H][D]
  const float* Wg;     // [H][D/group]
  uint16_t* cent;      // fp16 [H][M][D], initial centres in, fitted centres out
  int32_t* assign;     // [n][H]: the last assignment
  void* ws;            // fit_centroids_workspace_bytes(H, D, M)
  int group = kGroup;  // channels per (scale, zero) group of the QSAC estimate
};
size_t fit_centroids_workspace_bytes(int H, int D, int M);

// Most-attended token per query (retrieval analysis): over the packed cache
// (c set, K null) or over dense bf16 keys K [B][len][H_kv][d] (c null).
struct Top1Args {
  const kv2_cache* c;
  const uint16_t* Q;   // bf16 [B][nq][H_q][d]
  const uint16_t* K;
  int B, nq, H_q, H_kv, d, len;
  int32_t* top1;       // [B][nq][H_q]
  void* ws;            // top1_workspace_bytes(B, nq, H_q, len)
};
size_t top1_workspace_bytes(int B, int nq, int H_q, int len);
cudaError_t launch_top1(const Top1Args& a, cudaStream_t s);
cudaError_t launch_fit_centroids(const FitCentroidsArgs& a, cudaStream_t s);

// Decode attention.
struct DecodeArgs {
  const kv2_cache* c;   // host copy of the descriptor
  int len, H_q;
  const uint16_t* Q;    // bf16 [B][H_q][d]
  float sm_scale;
  void* out;
  int out_dtype;
  void* ws;
  size_t ws_bytes;
  // Slots at or after wait_from are written by the kernel just before on the
  // stream; the decode then starts as its programmatic dependent and waits
  // for it only before copying a tile that reaches such a slot. INT32_MAX:
  // ordinary stream order.
  int wait_from = INT32_MAX;
};
size_t decode_workspace_bytes(const kv2_cache& c, int H_q, int len);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);

// PSAC basis fit.
struct FitArgs {
  const uint16_t* Qhist;  // bf16 [n][H_q][d]
  int n, H_q, H_kv, d, r;
  float* P;
  float* w;
  float* Wg;
  float* energy;
  void* ws;
  int group = kGroup;     // Wg sums w over groups of this many channels
};
size_t fit_workspace_bytes(int H_kv, int d);
cudaError_t launch_fit(const FitArgs& a, cudaStream_t s);

// Chunk attention (tcgen05).
struct ChunkArgs {
  const kv2_cache* c;
  int len, H_q, Nq, frame_tokens;
  const uint16_t* Q;      // bf16 [B][Nq][H_q][d]
  const uint16_t* Kself;  // bf16 [B][Nq][H_kv][d]
  const uint16_t* Vself;
  float sm_scale;
  void* out;
  int out_dtype;
  void* ws;
  size_t ws_bytes;
  int* err_flag;          // device word for bounded-wait timeouts (in ws)
};
size_t chunk_workspace_bytes(const kv2_cache& c, int H_q, int Nq);
cudaError_t launch_chunk(const ChunkArgs& a, cudaStream_t s);

// Records the detail returned by kv2_last_error() on this thread; returns st.
kv2_status set_last_error(kv2_status st, const char* fmt, ...);
// Every check kv2_attention_decode makes except those of the workspace; on
// success *ws_need is the workspace size the call needs.
kv2_status validate_decode(const kv2_cache* c, int len, const uint16_t* Q, int H_q, void* out, int out_dtype,
                           size_t* ws_need);

}  // namespace kv2
