/*
 * kv2.h — C ABI of libkv2: a training-free 2-bit KV cache with
 * sensitivity-aware centroids (QSAC) and principal-subspace compensation
 * (PSAC), and attention that reads the packed cache directly, for NVIDIA B200
 * (sm_100a).
 *
 * Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
 * World Models" (besthub.dev article), sections "1. Quantization
 * Sensitivity-Aware Clustering (QSAC)" and "2. Principal Subspace Attention
 * Compensation (PSAC)". The principle of unpacking a 2-bit cache inside the
 * attention kernel, so that no dense fp16 cache is ever built, is the one the
 * OmniKVQuant page ("OmniKVQuant: KV Cache Quantization for Omni-LLMs",
 * abstract) states for its decode kernel.
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    never allocates or frees device memory. Pointers must be 16-byte aligned.
 *  - 16-bit floats travel as uint16_t bit patterns: bf16 for keys, values and
 *    queries; fp16 for centroid tables, scales, zeros and PSAC coefficients.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Work is
 *    enqueued asynchronously; argument errors are returned synchronously
 *    before anything is enqueued; a failed launch returns KV2_ERR_CUDA.
 *  - Supported shapes: head dim d in {64, 128}; quantization groups of 32, 64
 *    or 128 channels, group <= d (the `group` field and argument below; 0
 *    selects 32); 1 <= M <= 512 centroids per KV head (ids stored as u8 when
 *    M <= 256, else u16); 0 <= r <= d PSAC rank (r a multiple of 8 for the
 *    chunk kernel, r <= 16 there); H_q a multiple of H_kv. Anything else
 *    returns KV2_ERR_UNSUPPORTED.
 *  - Input magnitudes: keys, values and centroid-relative residuals must stay
 *    within +-60000 (fp16 range of the stored zero and scale); larger inputs
 *    give unspecified codes. NaN inputs propagate to the affected outputs.
 *  - Dense tensors use the token-major layout [batch][token][head][d].
 */
#ifndef KV2_H
#define KV2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kv2_status {
  KV2_OK = 0,
  KV2_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, negative size      */
  KV2_ERR_UNSUPPORTED = 2,  /* shape outside the supported set (see above)   */
  KV2_ERR_CAPACITY = 3,     /* pos + n_new > capacity, or len > capacity     */
  KV2_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed          */
  KV2_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out            */
  KV2_ERR_WORKSPACE = 6     /* workspace smaller than the *_workspace_size() */
} kv2_status;

enum { KV2_OUT_F32 = 0, KV2_OUT_BF16 = 1 };

/*
 * Packed cache of one layer (caller-owned device memory). Per (batch b,
 * KV head h) every stream is contiguous along tokens, slot = (b*H_kv + h)*capacity + t:
 *   k_code, v_code : uint32 [B][H_kv][capacity][d/16]; channel c of a token is
 *                    in word c/16 at bits 2(c%16)..2(c%16)+1 (INT2 codes 0..3)
 *   k_sz, v_sz     : uint32 [B][H_kv][capacity][d/group]; per group of `group`
 *                    consecutive channels (group g = channels g*group ..
 *                    g*group + group - 1), low half = fp16 scale s, high half =
 *                    fp16 zero z; the dequantized value of code q is fmaf(q, s, z)
 *   cidx           : centroid id per token, uint8 (M <= 256) or uint16 [B][H_kv][capacity]
 *   psac           : PSAC coefficients a = P^T e, [B][H_kv][capacity][r]:
 *                    fp16 (psac_fmt 0), or int8 codes (psac_fmt 1) whose
 *                    coefficient is code * psac_scale[slot]
 *   psac_scale     : fp16 [B][H_kv][capacity], one scale per token (psac_fmt 1
 *                    only; NULL otherwise)
 * Paged cache (block_table set): every stream above is instead a pool of pages
 * [pages][H_kv][page_tokens][...]; token t of sequence b lives in page
 * block_table[b][t / page_tokens] at offset t % page_tokens. capacity is the
 * logical length per sequence (a multiple of page_tokens); the pool may hold
 * any number of pages, shared by the sequences through their tables.
 *   centroids      : fp16 [H_kv][M][d] (read-only; shared by the batch)
 *   P, w, Wg       : fp32 [H_kv][d][r] basis, [H_kv][d] channel sensitivities,
 *                    [H_kv][d/group] group sensitivities, as written by
 *                    kv2_fit_psac_basis with the same group (read-only)
 *   group          : channels per (scale, zero) group: 32 (0 also selects 32),
 *                    64 or 128. Larger groups store fewer scales and zeros (the
 *                    compression QuantWM's evaluation counts) at a coarser INT2
 *                    grid.
 * A key is reconstructed as centroid[cidx] + fmaf(code, s, z) (+ P a for the
 * logit correction), a value as fmaf(code, s, z).
 */
typedef struct kv2_cache {
  int32_t B, H_kv, d, M, r, capacity;
  uint32_t* k_code;
  uint32_t* v_code;
  uint32_t* k_sz;
  uint32_t* v_sz;
  void* cidx;
  uint16_t* psac;
  const uint16_t* centroids;
  const float* P;
  const float* w;
  const float* Wg;
  int32_t psac_fmt;      /* 0: fp16 coefficients; 1: int8 codes + fp16 scale per token */
  uint16_t* psac_scale;
  const int32_t* block_table;  /* paged cache: page ids [B][capacity / page_tokens]; NULL: contiguous */
  int32_t page_tokens;         /* tokens per page (a multiple of 128) when block_table is set */
  int32_t group;               /* channels per (scale, zero) group; 0 selects 32 */
} kv2_cache;

/* Human-readable name of a status. Never NULL. */
const char* kv2_status_string(kv2_status s);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char* kv2_last_error(void);

/* Library ABI version (major*100 + minor). 200: the group field of kv2_cache
 * and the group argument of kv2_fit_psac_basis / kv2_fit_centroids. */
int kv2_version(void);

/*
 * Workspace for kv2_fit_psac_basis, in bytes: 2*H_kv*d*d*8 (fp64 Gram
 * matrices and eigenvector accumulators). Returns 0 for unsupported shapes.
 */
size_t kv2_fit_workspace_size(int H_kv, int d);

/*
 * kv2_fit_psac_basis — Query statistics of article section "2. PSAC"
 * (historical Query energy concentrates in a few principal directions) and
 * the sensitivity weights of "1. QSAC".
 * Qhist  : bf16 [n][H_q][d] history (calibration) queries. For KV head h the
 *          statistics pool the n*G vectors of its query heads h*G..h*G+G-1
 *          (G = H_q/H_kv).
 * Outputs (fp32, device): S = (1/(n*G)) sum q q^T (uncentred second moment),
 *   w[h][c] = S_cc; Wg[h][g] = sum of w over group g's `group` channels
 *   (ascending channel order, fp32), Wg of [H_kv][d/group];
 *   P[h][c][i] = i-th eigenvector of S by decreasing eigenvalue (i < r), sign
 *   fixed so its largest-magnitude entry is positive; energy[h] (may be NULL)
 *   = share of trace(S) in the top r eigenvalues.
 * Method on the device: fp64 Gram accumulation, cyclic Jacobi in fp64.
 * group: channels per (scale, zero) group of the cache the statistics serve
 *   (32, or 0 for 32; 64 and 128 return KV2_ERR_UNSUPPORTED from this
 *   version).
 * ws: device workspace of kv2_fit_workspace_size(H_kv, d) bytes.
 */
kv2_status kv2_fit_psac_basis(const uint16_t* Qhist, int n, int H_q, int H_kv, int d,
                              int r, int group, float* P, float* w, float* Wg, float* energy,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * Workspace for kv2_fit_centroids, in bytes: (H_kv*M*d + H_kv*M)*8 (64-bit
 * integer sums and counts). Returns 0 for unsupported shapes.
 */
size_t kv2_fit_centroids_workspace_size(int H_kv, int d, int M);

/*
 * kv2_fit_centroids — Key centres for the QSAC assignment (article "1. QSAC":
 * the clustering picks INT2-friendly centres). The pages do not print the
 * loop; it is read as Lloyd iterations whose assignment step is the QSAC
 * decision of kv2_quantize_append (same ranking, candidates and choice,
 * bit for bit) and whose update step moves every centre to the mean of the
 * keys assigned to it; a centre that no key chooses keeps its value.
 * Mean: each bf16 key value as a whole number of 2^-24 units (truncated
 * toward zero), summed in 64-bit integers (exact, order-free), divided by
 * the count in fp64, times 2^-24, rounded to fp16 (nearest even).
 * X        : bf16 [n][H_kv][d] sample keys (read-only), n <= 65536,
 *            |k| < 2^23 (so the 64-bit sums cannot overflow).
 * w, Wg    : the sensitivities of kv2_fit_psac_basis (read-only), Wg for
 *            groups of `group` channels (32, or 0 for 32; 64 and 128 return
 *            KV2_ERR_UNSUPPORTED from this version).
 * centroids: fp16 [H_kv][M][d], initial centres in, fitted centres out.
 * assign   : int32 [n][H_kv] out: the assignment of the last iteration.
 * iters >= 0 iterations (0 leaves everything unchanged); candidates 1..M.
 * ws       : device workspace of kv2_fit_centroids_workspace_size bytes.
 * All pointers are device memory owned by the caller; asynchronous on stream.
 * Errors: KV2_ERR_INVALID_ARG (NULL / misaligned pointers, n out of range,
 * candidates outside 1..M, iters < 0), KV2_ERR_UNSUPPORTED (d not 64/128,
 * M outside 1..512), KV2_ERR_WORKSPACE.
 */
kv2_status kv2_fit_centroids(const uint16_t* X, int n, int H_kv, int d, int M, int candidates, int group,
                             const float* w, const float* Wg, int iters, uint16_t* centroids,
                             int32_t* assign, void* ws, size_t ws_bytes, void* stream);

/*
 * Workspace for kv2_decode_top1 / kv2_dense_top1, in bytes:
 * B*nq*H_q*ceil(len/4096)*8. Returns 0 for invalid sizes.
 */
size_t kv2_top1_workspace_size(int B, int nq, int H_q, int len);

/*
 * kv2_decode_top1 — the most-attended cached token of each query: the index
 * of the largest logit q . khat_t + (q P) . a_t over tokens [0, len) of the
 * packed cache (the logit decode uses, before scaling), computed in fp32 with
 * the channels in order; ties go to the lower index; -1 when len = 0. With
 * kv2_dense_top1 on the original keys it measures the retrieval shift that
 * Key quantization causes (article introduction and Table 1: which
 * temporal-spatial tokens a Query selects). Not on the attention hot path.
 * Q: bf16 [B][nq][H_q][d] (nq queries per sequence); top1: int32
 * [B][nq][H_q] (device, written); ws: kv2_top1_workspace_size(B, nq, H_q, len)
 * bytes.
 */
kv2_status kv2_decode_top1(const kv2_cache* cache, int len, const uint16_t* Q, int nq, int H_q, int32_t* top1,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * kv2_dense_top1 — the same over dense bf16 keys K [B][len][H_kv][d]:
 * the index of the largest q . k_t (fp32, channels in order, ties to the
 * lower index).
 */
kv2_status kv2_dense_top1(const uint16_t* K, int B, int len, int H_kv, int d, const uint16_t* Q, int nq, int H_q,
                          int32_t* top1, void* ws, size_t ws_bytes, void* stream);

/*
 * kv2_quantize_append — QSAC centroid assignment, INT2 residual/value
 * packing and PSAC coefficients for n_new new tokens of every (batch, KV
 * head), written to slots [pos, pos + n_new) (article "1. QSAC", "2. PSAC").
 * K, V   : bf16 [B][n_new][H_kv][d].
 * candidates (C, 1..M): the C centres of smallest Query-sensitivity-weighted
 *   distance D_j = sum_c w_c (k_c - mu_jc)^2 (fp32: t = k_c - mu_jc, then
 *   fmaf(w_c t, t, acc) over ascending c), ties to the lower id, are kept; of
 *   those, the one whose residual gives the least E_j = sum_g W_g s_g^2 (s_g
 *   the group's fp16 scale) is chosen, ties to the lower id. C = 1 with w = 1
 *   is the plain nearest-centre (QVG) assignment.
 * Codec per group of `group` channels (residual k - mu for keys, v for values): zero =
 *   fp16 round-down of the minimum, scale = fp16 round-up of (max - zero)/3,
 *   code = clamp(round-half-even((x - zero)/scale), 0, 3) (0 when scale = 0).
 * PSAC: a_i = sum_c P_ci (x_c - fmaf(code_c, s, z)), rounded to fp16
 *   (psac_fmt 0), or (psac_fmt 1) stored as int8 codes with one fp16 scale per
 *   token: scale = fp16 round-up of max_i |a_i| / 127, code_i =
 *   clamp(round-half-even(a_i / scale), -127, 127) (0 when the scale is 0).
 * All quantizer decisions are those fp32 definitions, bit for bit. The
 * kernel ranks by a faster expanded form with an error bound; with more than
 * 64 rows per head its dot products run on the tensor cores, and that bound
 * then assumes the tensor cores' fp32 accumulation errs by at most 2^-12 of
 * the summed product magnitudes (128x the largest error measured on B200).
 * When the bound leaves the candidate set open, the choice comes from the
 * perturbations of every centre that may be in the set if they decide it,
 * else from D_j itself. Tokens outside [pos, pos+n_new) are never read or
 * written; concurrent calls on overlapping slots race.
 * Errors: KV2_ERR_CAPACITY if pos < 0 or pos + n_new > capacity.
 */
kv2_status kv2_quantize_append(const kv2_cache* cache, const uint16_t* K, const uint16_t* V,
                               int n_new, int pos, int candidates, void* stream);

/*
 * Workspace for kv2_attention_decode, in bytes: a 256-byte header whose
 * first 32-bit word is the sticky error word (below), then the split-K
 * partials (per query head and split, d output sums, the running maximum and
 * the softmax denominator, fp32). Returns 0 for unsupported shapes.
 */
size_t kv2_decode_workspace_size(const kv2_cache* cache, int H_q, int len);

/*
 * kv2_attention_decode — one query token per sequence against the first
 * `len` cached tokens of every (batch, KV head), reading the packed cache
 * directly, as the OmniKVQuant page's abstract describes for its decode
 * kernel (the 2-bit cache unpacked inside attention, no dense cache built).
 * Logits follow "2. PSAC" of the QuantWM article (the Key error's projection
 * on the top Query directions compensates the score):
 * logit_t = sm_scale * (q.mu[cidx_t] + sum_g (s_g sum_{c in g} q_c code_c +
 * z_g sum_{c in g} q_c) + (qP).a_t); online softmax; values dequantized in
 * registers. Split-K over the sequence, then a log-sum-exp merge.
 * Arithmetic: the code sums sum_{c in g} q_c code_c run as 8-bit integer
 * tensor-core products (codes exact; q as a 16-bit fixed-point value, two
 * signed 8-bit digits, rounding at most 2^-16 of its largest component) with
 * exact int32 sums; the zero-point and PSAC terms and p.v use fp16 tensor-core
 * operands (stored fp16 values exact, the query's group sums, qP and p*s_v
 * as fp16 hi/lo pairs, about 22 significant bits); every sum is fp32;
 * exponentials use the hardware ex2.approx (relative error about 2^-22).
 * Q   : bf16 [B][H_q][d]; out: [B][H_q][d], fp32 (KV2_OUT_F32) or bf16
 *       (KV2_OUT_BF16, round to nearest even). len = 0 writes zeros.
 * ws  : device workspace of kv2_decode_workspace_size(cache, H_q, len) bytes,
 *       zeroed by the caller before its first use. Its first 32-bit word is
 *       a sticky error word: the kernel sets it to 1 when one of its waits
 *       for the cache tiles it copies into shared memory runs out of its
 *       budget (KV2_WAIT_BUDGET_CYCLES SM cycles, default 2^31); the outputs
 *       of the affected (batch, KV head) are then NaN. The library never
 *       clears it. Errors of the launch itself are returned as KV2_ERR_CUDA.
 */
kv2_status kv2_attention_decode(const kv2_cache* cache, int len, const uint16_t* Q, int H_q,
                                float sm_scale, void* out, int out_dtype,
                                void* ws, size_t ws_bytes, void* stream);

/*
 * kv2_attention_decode_noalloc — the same computation and arguments as
 * kv2_attention_decode, minus the workspace: the scratch lives in a fixed
 * 8 MiB array inside the library, so the caller allocates nothing. It serves
 * callers that may not allocate device memory themselves (a plugin inside a
 * framework that owns the allocator, a serving loop where cudaMalloc would
 * synchronize the device). The paper has no counterpart; it is a convenience
 * of this library.
 *  - Every argument is checked first, with the errors of kv2_attention_decode;
 *    shapes whose kv2_decode_workspace_size exceeds 8 MiB (8388608 bytes) are
 *    then rejected with KV2_ERR_WORKSPACE.
 *  - Every GPU that loads the library holds the 8 MiB array until exit.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it per device ordinal; make that first
 *    call before any stream capture. The address is that of the device's
 *    primary context: do not call from another driver context or after
 *    cudaDeviceReset in the same process.
 *  - All calls share the array and it keeps the last call's contents: calls
 *    that overlap on the GPU race on it and must be serialized by the caller.
 *  - The array's first 32-bit word is the decode error word of
 *    kv2_attention_decode: it starts at 0, a decode call sets it to 1 when a
 *    wait for its cache tiles runs out of budget (those outputs are NaN), and
 *    no decode call clears it. Read and clear it with kv2_decode_noalloc_error.
 *  - No cudaMalloc, cudaFree or other allocating call is made.
 */
kv2_status kv2_attention_decode_noalloc(const kv2_cache* cache, int len, const uint16_t* Q,
                                        int H_q, float sm_scale, void* out, int out_dtype,
                                        void* stream);

/*
 * kv2_decode_noalloc_error — the error word of kv2_attention_decode_noalloc's
 * fixed array on the current device, for callers that cannot hold a
 * workspace of their own to inspect. Allocates nothing. Enqueues a 4-byte
 * device-to-host copy on `stream` and waits for the stream (so it sees every
 * decode call enqueued there before it), stores the word in *flag (host
 * memory: 0 = no wait ran out, 1 = at least one did), and when `clear` is
 * non-zero and the word was set, zeroes it (on `stream`, waited for). The
 * paper has no counterpart.
 * Errors: KV2_ERR_INVALID_ARG (flag NULL), KV2_ERR_CUDA.
 */
kv2_status kv2_decode_noalloc_error(int* flag, int clear, void* stream);

/*
 * kv2_append_attention_decode — one decode step of a serving loop: appends
 * the n_new new tokens of every sequence at slots [pos, pos + n_new) exactly
 * as kv2_quantize_append does, then attends exactly as kv2_attention_decode
 * does over len = pos + n_new cached tokens ("QuantWM: Training-Free 2-bit KV
 * Cache Quantization for Stable Video World Models", "1. QSAC" and "2. PSAC":
 * new Keys are quantized as they enter the cache and attention reads the
 * packed cache). The results are those of the two calls in sequence, bit for
 * bit. The two kernels overlap: the attention kernel is launched as the
 * programmatic dependent of the append kernel and waits for it only before
 * copying a tile that reaches slot pos, so the append's latency hides behind
 * the attention over the older tokens. The pages have no counterpart; it is a
 * convenience of this library.
 * K_new, V_new: bf16 [B][n_new][H_kv][d] (device); n_new = 0 only attends.
 * Q, H_q, sm_scale, out, out_dtype, ws, ws_bytes: as kv2_attention_decode,
 *   with ws of kv2_decode_workspace_size(cache, H_q, pos + n_new) bytes.
 * Errors: those of both calls, checked before anything is launched.
 */
kv2_status kv2_append_attention_decode(const kv2_cache* cache, const uint16_t* K_new,
                                       const uint16_t* V_new, int n_new, int pos, int candidates,
                                       const uint16_t* Q, int H_q, float sm_scale, void* out,
                                       int out_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Workspace for kv2_attention_chunk, in bytes (fp16 q P per query). Returns 0
 * for unsupported shapes.
 */
size_t kv2_chunk_workspace_size(const kv2_cache* cache, int H_q, int Nq);

/*
 * kv2_attention_chunk — Nq queries per (batch, query head) of a video-world-
 * model chunk against the whole packed cache (first `len` tokens) plus the
 * chunk's own dense keys/values, block-causal by latent frame: query i sees
 * every cached token and the self tokens j with j/frame_tokens <= i/frame_tokens.
 * The score is the compensated one of "2. PSAC" in the QuantWM article,
 * q.(k^ + P a) = q.k^ + (qP).a, over the 2-bit cache unpacked inside the
 * kernel (the principle the OmniKVQuant page's abstract states); the chunk
 * shape (thousands of queries per step attending to the whole history) is
 * that of the article's video world models ("Experimental Validation").
 * Tensor cores (tcgen05, accumulators in TMEM): packed key tiles are
 * dequantized in shared memory to fp16(code*s + fp16(z + centroid)), value
 * tiles to fp16(code*s + z), the chunk's own keys and values are rounded
 * from bf16 to fp16, each query row is scaled by a power of two and
 * converted to fp16, the PSAC term (qP).a enters as fp16 extra contraction
 * columns, probabilities are fp16, accumulation fp32.
 * Q     : bf16 [B][Nq][H_q][d]; Kself, Vself: bf16 [B][Nq][H_kv][d];
 * out   : [B][Nq][H_q][d] fp32 or bf16. Requires d = 128.
 * ws    : device workspace of kv2_chunk_workspace_size(cache, H_q, Nq) bytes.
 */
kv2_status kv2_attention_chunk(const kv2_cache* cache, int len, const uint16_t* Q, int H_q,
                               int Nq, const uint16_t* Kself, const uint16_t* Vself,
                               int frame_tokens, float sm_scale, void* out, int out_dtype,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * Pages of a paged cache moved out of HBM and back (long-horizon memory:
 * a sequence's older chunks kept in host memory and brought back when the
 * caller wants them in the attention window again; which pages to move is
 * the caller's policy).
 *
 * A page holds page_tokens consecutive tokens of every KV head in each
 * stream: k_code, v_code, k_sz, v_sz, cidx, then psac (r > 0) and
 * psac_scale (int8 PSAC format, r > 0). Its image in host memory is those
 * streams' page slices back to back in that order, kv2_page_bytes(cache)
 * bytes: H_kv * page_tokens * (8*(d/16) + 8*(d/group) + id bytes + PSAC
 * bytes per token).
 *
 * kv2_page_store copies page `page` (0 <= page < num_pages, the pool's page
 * count) of the cache's device streams into `host`; kv2_page_load copies an
 * image from `host` into page `page`. To evict, store a page and drop it
 * from the block table; to retrieve, load the image into a free page and
 * point the table entry at it (the block table is the caller's device
 * memory). Both are cudaMemcpyAsync calls on `stream`, one per stream: with
 * page-locked host memory they are asynchronous, with pageable memory a
 * store returns after its copies. The page's device bytes are not otherwise
 * read or written.
 * Errors: KV2_ERR_INVALID_ARG (cache not paged, page outside 0..num_pages-1,
 * NULL host buffer), the cache checks of kv2_quantize_append, KV2_ERR_CUDA.
 * kv2_page_bytes returns 0 for a descriptor that is not a valid paged cache.
 */
size_t kv2_page_bytes(const kv2_cache* cache);
kv2_status kv2_page_store(const kv2_cache* cache, int page, int num_pages, void* host, void* stream);
kv2_status kv2_page_load(const kv2_cache* cache, int page, int num_pages, const void* host, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KV2_H */
