/*
 * kv2_oracle.c — plain, slow CPU oracle of the 2-bit KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file's library; the product path never does.
 * It shares no code, header or table with the CUDA library.
 *
 * Source of the method: "QuantWM: Training-Free 2-bit KV Cache Quantization for
 * Stable Video World Models" (besthub.dev article), sections
 *   "1. Quantization Sensitivity-Aware Clustering (QSAC)" and
 *   "2. Principal Subspace Attention Compensation (PSAC)".
 * The pages leave the exact formulas open; every reading taken here is the one
 * written out below and in the design notes (codec, ranking score, perturbation
 * estimate, coefficient precision, sign and order of eigenvectors).
 *
 * Precision: quantizer decisions (centroid choice, INT2 codes, fp16 scale and
 * zero) are taken in fp32 in the stated operation order, using fmaf only where
 * stated (compile with -ffp-contract=off). Eigen-decomposition and attention are
 * fp64. 16-bit float conversions are written from the IEEE 754 definition.
 *
 * Parity pins (tests/test_oracle_*.py): rounding functions vs numpy/torch casts
 * and directed-rounding brackets; codec invariants and per-element brute force;
 * QSAC vs brute-force argmin (candidates = M) and vs plain nearest centre
 * (candidates = 1, unit weights); PSAC r = d and r = 0 closed forms; Jacobi vs
 * numpy.linalg.eigh; attention vs a two-pass softmax and a centroid-only closed
 * form; group sizes 64 and 128 by per-group codec invariants, exact
 * reconstruction of group-constant residuals, the single-group QSAC choice as
 * the least residual range, and W over one whole-row group as the trace of
 * the Gram matrix; 4-element groups exhaustively over a value grid (nearest
 * level, exact ties to even) and QSAC by brute force; the chunk operands'
 * fp16 rounding (keys, values, q P) on hand-derived ties; the centre update's
 * truncation below one 2^-24 unit. Parity unpinned: whether the perturbation estimate is the authors' exact
 * heuristic (the pages print no worked example).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 / bfloat16                                             */
/* ------------------------------------------------------------------------ */

enum { RND_NEAREST_EVEN = 0, RND_DOWN = 1, RND_UP = 2 };

/* Round a finite or infinite double to a binary format with `man` fraction
 * bits, minimum normal exponent `emin` and largest finite value `maxf`, under
 * the given rounding mode. Returns the rounded value as a double (exact). */
static double round_to_format(double x, int man, int emin, double maxf, int mode)
{
    if (isnan(x)) return x;
    int neg = signbit(x) != 0;
    double a = fabs(x);
    if (isinf(a)) return x;
    if (a == 0.0) return x;
    int e2;
    frexp(a, &e2);                 /* a in [2^(e2-1), 2^e2) */
    int e = e2 - 1;                /* floor(log2 a) */
    if (e < emin) e = emin;        /* subnormal range shares the emin quantum */
    double quantum = ldexp(1.0, e - man);
    double n = a / quantum;        /* exact: division by a power of two */
    double k;
    if (mode == RND_NEAREST_EVEN) {
        double f = floor(n), rem = n - f;
        if (rem > 0.5) k = f + 1.0;
        else if (rem < 0.5) k = f;
        else k = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
    } else {
        /* magnitude toward zero for (down, positive) and (up, negative) */
        int toward_zero = (mode == RND_DOWN) ? !neg : neg;
        k = toward_zero ? floor(n) : ceil(n);
    }
    double r = k * quantum;
    if (r > maxf) {
        int toward_zero = (mode == RND_NEAREST_EVEN) ? 0 : ((mode == RND_DOWN) ? !neg : neg);
        r = toward_zero ? maxf : INFINITY;
    }
    return neg ? -r : r;
}

static const double F16_MAX = 65504.0;

static uint16_t f16_encode_exact(double r)
{
    /* r is already representable in binary16 (or +-inf / nan) */
    uint16_t sign = signbit(r) ? 0x8000u : 0u;
    double a = fabs(r);
    if (isnan(r)) return 0x7e00u;
    if (isinf(a)) return (uint16_t)(sign | 0x7c00u);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(a / ldexp(1.0, -24)));
    int e2;
    frexp(a, &e2);
    int e = e2 - 1;
    uint16_t mant = (uint16_t)(a / ldexp(1.0, e - 10) - 1024.0);
    return (uint16_t)(sign | ((uint16_t)(e + 15) << 10) | mant);
}

uint16_t or_f16_from_f32(float x, int mode)
{
    return f16_encode_exact(round_to_format((double)x, 10, -14, F16_MAX, mode));
}

float or_f32_from_f16(uint16_t h)
{
    int neg = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m | 0x400), e - 25);
    return (float)(neg ? -v : v);
}

float or_f32_from_bf16(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp16 nearest-even rounding of an exact (double) value: one rounding, as an
 * fp16 add or fused multiply-add performs it */
static double f16_round(double x)
{
    return (double)or_f32_from_f16(f16_encode_exact(round_to_format(x, 10, -14, F16_MAX, RND_NEAREST_EVEN)));
}

uint16_t or_bf16_from_f32(float x)
{
    if (isnan(x)) return 0x7fc0u;
    double bmax = ldexp(2.0 - ldexp(1.0, -7), 127);
    float r = (float)round_to_format((double)x, 7, -126, bmax, RND_NEAREST_EVEN);
    uint32_t u;
    memcpy(&u, &r, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* INT2 group codec                                                          */
/*   QuantWM article, "1. QSAC": the centre-relative residual is quantized to  */
/*   2 bits; the cache stores an fp16 scale and an fp16 zero per group of      */
/*   consecutive channels (asymmetric INT2). The pages fix no group size: the  */
/*   cache format takes 32 (default), 64 or 128, the larger ones trading       */
/*   accuracy for the compression the evaluation counts. Reading taken: zero = */
/*   the group minimum rounded down to fp16, scale = (max - zero)/3 rounded up */
/*   to fp16, so that [zero, zero + 3 scale] covers the group; codes round     */
/*   half to even.                                                             */
/* ------------------------------------------------------------------------ */

static void codec_params(const float* x, int n, uint16_t* s_bits, uint16_t* z_bits)
{
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    uint16_t zb = or_f16_from_f32(mn, RND_DOWN);
    float z = or_f32_from_f16(zb);
    float range = mx - z;              /* fp32, round to nearest */
    float q = range / 3.0f;            /* fp32 correctly rounded division */
    *z_bits = zb;
    *s_bits = or_f16_from_f32(q, RND_UP);
}

static uint32_t codec_code(float x, float s, float z)
{
    if (s == 0.0f) return 0u;
    float t = (x - z) / s;             /* fp32 subtraction, fp32 division */
    float c = rintf(t);                /* round half to even */
    if (c < 0.0f) c = 0.0f;
    if (c > 3.0f) c = 3.0f;
    return (uint32_t)c;
}

static float codec_dequant(uint32_t code, float s, float z)
{
    return fmaf((float)code, s, z);
}

/* exported for the tests: one group of n values */
void or_codec_group(const float* x, int n, uint16_t* s_bits, uint16_t* z_bits,
                    uint8_t* codes, float* deq)
{
    codec_params(x, n, s_bits, z_bits);
    float s = or_f32_from_f16(*s_bits), z = or_f32_from_f16(*z_bits);
    for (int i = 0; i < n; ++i) {
        codes[i] = (uint8_t)codec_code(x[i], s, z);
        if (deq) deq[i] = codec_dequant(codes[i], s, z);
    }
}

/* ------------------------------------------------------------------------ */
/* PSAC basis fit (article section "2. PSAC": historical Query energy          */
/* concentrates in a few principal directions; QSAC's sensitivity weights are  */
/* the per-channel Query energy).                                              */
/*   S = (1/N) sum q q^T over the N = n*G history queries of the KV head's     */
/*   query-head group (uncentred second moment), w_c = S_cc, W_g = sum of w_c   */
/*   over the group's channels (fp32, ascending c), P = top-r eigenvectors of S */
/*   (eigenvalues descending, each vector's largest-magnitude entry positive).  */
/* ------------------------------------------------------------------------ */

/* cyclic Jacobi eigen-decomposition of a symmetric n x n matrix A (destroyed);
 * eigenvalues on return in A's diagonal, eigenvectors in the columns of V */
static void jacobi_eigen(double* A, double* V, int n)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) V[i * n + j] = (i == j) ? 1.0 : 0.0;
    double total = 0.0;
    for (int i = 0; i < n * n; ++i) total += A[i] * A[i];
    for (int sweep = 0; sweep < 100; ++sweep) {
        double off = 0.0;
        for (int p = 0; p < n; ++p)
            for (int q = p + 1; q < n; ++q) off += 2.0 * A[p * n + q] * A[p * n + q];
        if (off <= 1e-28 * total || off == 0.0) break;
        for (int p = 0; p < n - 1; ++p) {
            for (int q = p + 1; q < n; ++q) {
                double apq = A[p * n + q];
                if (apq == 0.0) continue;
                double app = A[p * n + p], aqq = A[q * n + q];
                double theta = (aqq - app) / (2.0 * apq);
                double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
                double c = 1.0 / sqrt(t * t + 1.0), s = t * c;
                /* A <- J^T A J with J the rotation in the (p, q) plane */
                for (int k = 0; k < n; ++k) {
                    double akp = A[k * n + p], akq = A[k * n + q];
                    A[k * n + p] = c * akp - s * akq;
                    A[k * n + q] = s * akp + c * akq;
                }
                for (int k = 0; k < n; ++k) {
                    double apk = A[p * n + k], aqk = A[q * n + k];
                    A[p * n + k] = c * apk - s * aqk;
                    A[q * n + k] = s * apk + c * aqk;
                }
                for (int k = 0; k < n; ++k) {
                    double vkp = V[k * n + p], vkq = V[k * n + q];
                    V[k * n + p] = c * vkp - s * vkq;
                    V[k * n + q] = s * vkp + c * vkq;
                }
            }
        }
    }
}

int or_fit(const uint16_t* Qh, int n, int Hq, int Hkv, int d, int r,
           float* P, float* w, float* Wg, double* evals, double* energy, int group)
{
    if (Hkv <= 0 || Hq % Hkv || group <= 0 || d % group || r < 0 || r > d || n <= 0) return 1;
    int G = Hq / Hkv, ng = d / group;
    double* S = (double*)calloc((size_t)d * d, sizeof(double));
    double* Vec = (double*)malloc((size_t)d * d * sizeof(double));
    double* lam = (double*)malloc((size_t)d * sizeof(double));
    int* order = (int*)malloc((size_t)d * sizeof(int));
    double* q = (double*)malloc((size_t)d * sizeof(double));
    for (int h = 0; h < Hkv; ++h) {
        memset(S, 0, (size_t)d * d * sizeof(double));
        for (int t = 0; t < n; ++t)
            for (int g = 0; g < G; ++g) {
                const uint16_t* qr = Qh + ((size_t)t * Hq + (size_t)h * G + g) * d;
                for (int c = 0; c < d; ++c) q[c] = or_f32_from_bf16(qr[c]);
                for (int a = 0; a < d; ++a)
                    for (int b = 0; b < d; ++b) S[a * d + b] += q[a] * q[b];
            }
        double N = (double)n * G;
        for (int i = 0; i < d * d; ++i) S[i] /= N;
        for (int c = 0; c < d; ++c) w[(size_t)h * d + c] = (float)S[c * d + c];
        for (int g = 0; g < ng; ++g) {
            float acc = 0.0f;
            for (int c = g * group; c < (g + 1) * group; ++c) acc = acc + w[(size_t)h * d + c];
            Wg[(size_t)h * ng + g] = acc;
        }
        jacobi_eigen(S, Vec, d);
        for (int i = 0; i < d; ++i) { lam[i] = S[i * d + i]; order[i] = i; }
        /* eigenvalues descending; equal values keep the lower index first */
        for (int i = 1; i < d; ++i) {
            int o = order[i], j = i - 1;
            while (j >= 0 && lam[order[j]] < lam[o]) { order[j + 1] = order[j]; --j; }
            order[j + 1] = o;
        }
        double tot = 0.0, top = 0.0;
        for (int i = 0; i < d; ++i) tot += lam[i];
        for (int i = 0; i < r; ++i) top += lam[order[i]];
        if (energy) energy[h] = tot > 0.0 ? top / tot : 0.0;
        if (evals)
            for (int i = 0; i < d; ++i) evals[(size_t)h * d + i] = lam[order[i]];
        for (int i = 0; i < r; ++i) {
            int col = order[i];
            int arg = 0;
            for (int c = 1; c < d; ++c)
                if (fabs(Vec[c * d + col]) > fabs(Vec[arg * d + col])) arg = c;
            double sg = Vec[arg * d + col] < 0.0 ? -1.0 : 1.0;
            for (int c = 0; c < d; ++c)
                P[((size_t)h * d + c) * r + i] = (float)(sg * Vec[c * d + col]);
        }
    }
    free(S); free(Vec); free(lam); free(order); free(q);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* QSAC + INT2 packing + PSAC coefficients for appended tokens.               */
/*   Ranking (article "1. QSAC": candidates by a Query-sensitivity-weighted    */
/*   distance): the weighted squared distance itself,                          */
/*       D_j = sum_c w_c (k_c - mu_jc)^2,                                      */
/*   in fp32 as written: t = k_c - mu_jc (fp32 subtraction), then              */
/*   acc = fmaf(w_c * t, t, acc) over ascending c from 0 (the product w_c * t  */
/*   rounded to fp32 first). Candidates: the set of the C smallest (D_j, j),   */
/*   equal distances to the lower index.                                       */
/*   Choice (same section: estimated perturbation from the residual group's    */
/*   dynamic range and its sensitivity): E_j = sum_g (W_g s_g) s_g, an fp32     */
/*   fmaf chain over ascending g with s_g the group's fp16 scale; the least    */
/*   (E_j, j) over the candidate set wins, so the choice depends on the set    */
/*   alone, not on the order the ranking lists it in.                          */
/*   PSAC coefficients (article "2. PSAC"): a_i = sum_c P_ci e_c with          */
/*   e = residual - dequantized residual, an fp32 fmaf chain over ascending c, */
/*   stored as fp16 (round to nearest even).                                   */
/* Layouts: K, V bf16 [B][n_new][Hkv][d]; centroids fp16 [Hkv][M][d];          */
/* P [Hkv][d][r]; w [Hkv][d]; Wg [Hkv][d/group]; packed streams as in the      */
/* library: [B][Hkv][cap][...], (scale, zero) per group of `group` channels.  */
/* ------------------------------------------------------------------------ */

/* weighted squared distance of key k to centre m, fp32 in the order above */
static float qsac_distance(const float* k, const float* m, const float* wh, int d)
{
    float acc = 0.0f;
    for (int c = 0; c < d; ++c) {
        float t = k[c] - m[c];
        float wt = wh[c] * t;
        acc = fmaf(wt, t, acc);
    }
    return acc;
}

/* QSAC decision for one key k (fp32 [d]) of KV head h: returns the chosen
 * centre and leaves its residual k - mu_j in xbest. mu [M][d]; scratch:
 * score [M], cand [C], used [M], x [d]. Optional debug outputs (candidate ids
 * in rank order, their distances D_j, E per candidate) when non-NULL. */
static int qsac_choose(const float* k, const float* wh, const float* Wgh, const float* mu,
                       int M, int C, int d, int group, float* score, int* cand, char* used, float* x,
                       float* xbest, int32_t* cand_out, float* score_out, float* E_out)
{
    int ng = d / group;
    /* ranking */
    for (int j = 0; j < M; ++j) score[j] = qsac_distance(k, mu + (size_t)j * d, wh, d);
    memset(used, 0, (size_t)M);
    for (int i = 0; i < C; ++i) {
        int best = -1;
        for (int j = 0; j < M; ++j) {
            if (used[j]) continue;
            if (best < 0 || score[j] < score[best]) best = j;
        }
        used[best] = 1;
        cand[i] = best;
        if (cand_out) cand_out[i] = best;
        if (score_out) score_out[i] = score[best];
    }
    /* choice by estimated perturbation */
    int chosen = -1;
    float bestE = 0.0f;
    for (int i = 0; i < C; ++i) {
        int j = cand[i];
        const float* m = mu + (size_t)j * d;
        for (int c = 0; c < d; ++c) x[c] = k[c] - m[c];
        float E = 0.0f;
        for (int g = 0; g < ng; ++g) {
            uint16_t sb, zb;
            codec_params(x + g * group, group, &sb, &zb);
            float s = or_f32_from_f16(sb);
            float ws = Wgh[g] * s;
            E = fmaf(ws, s, E);
        }
        if (E_out) E_out[i] = E;
        if (chosen < 0 || E < bestE || (E == bestE && j < chosen)) {
            chosen = j;
            bestE = E;
            memcpy(xbest, x, (size_t)d * sizeof(float));
        }
    }
    return chosen;
}

/* the centres of KV head h as fp32 */
static void qsac_tables(const uint16_t* cent, int h, int M, int d, float* mu)
{
    for (size_t i = 0; i < (size_t)M * d; ++i) mu[i] = or_f32_from_f16(cent[(size_t)h * M * d + i]);
}

/* Slot of token t of (sequence b, KV head h): contiguous streams
 * [B][Hkv][cap], or a pool of pages [pages][Hkv][page] addressed through the
 * block table (a page holds `page` consecutive tokens of one sequence). */
static size_t slot_at(int Hkv, int cap, const int32_t* table, int page, int b, int h, int t)
{
    if (!table) return ((size_t)b * Hkv + h) * cap + (size_t)t;
    int32_t pg = table[(size_t)b * (cap / page) + t / page];
    return ((size_t)pg * Hkv + h) * page + (size_t)(t % page);
}

/* INT8 PSAC coefficients with one fp16 scale per token (the compensation
 * information stored compactly, article "2. PSAC" and the compression count
 * of the evaluation). Reading taken: symmetric, scale = fp16 round-up of the
 * fp32 quotient max|a| / 127, so every |a / scale| <= 127; code =
 * clamp(round-half-even(a / scale), -127, 127) (fp32 division), 0 when the
 * scale is 0; the coefficient read back is code * scale. */
static void psac_int8(const float* a, int r, float amax, int8_t* q, uint16_t* scale_bits)
{
    uint16_t sb = or_f16_from_f32(amax / 127.0f, RND_UP);
    float s = or_f32_from_f16(sb);
    *scale_bits = sb;
    for (int i = 0; i < r; ++i) {
        float v = (s > 0.0f) ? rintf(a[i] / s) : 0.0f;
        if (v > 127.0f) v = 127.0f;
        if (v < -127.0f) v = -127.0f;
        q[i] = (int8_t)v;
    }
}

static uint32_t pack_word(const uint32_t* codes16)
{
    uint32_t w = 0;
    for (int i = 0; i < 16; ++i) w |= (codes16[i] & 3u) << (2 * i);
    return w;
}

/* One row of d channels in groups of `group` consecutive channels: each
 * group's fp16 (scale, zero) into sz[g], then every channel's code under its
 * own group's parameters, 16 codes per word in channel order. */
static void quantize_row(const float* x, int d, int group, uint32_t* code_words, uint32_t* sz, float* deq)
{
    uint32_t codes[16];
    for (int g = 0; g < d / group; ++g) {
        uint16_t sb, zb;
        codec_params(x + g * group, group, &sb, &zb);
        sz[g] = (uint32_t)sb | ((uint32_t)zb << 16);
    }
    for (int wd = 0; wd < d / 16; ++wd) {
        for (int i = 0; i < 16; ++i) {
            int c = wd * 16 + i;
            uint32_t p = sz[c / group];
            float s = or_f32_from_f16((uint16_t)(p & 0xffff)), z = or_f32_from_f16((uint16_t)(p >> 16));
            codes[i] = codec_code(x[c], s, z);
            if (deq) deq[c] = codec_dequant(codes[i], s, z);
        }
        code_words[wd] = pack_word(codes);
    }
}

int or_quantize(int B, int Hkv, int d, int M, int r, int cap,
                const uint16_t* K, const uint16_t* V, int n_new, int pos, int C,
                const uint16_t* cent, const float* P, const float* w, const float* Wg,
                uint32_t* k_code, uint32_t* v_code, uint32_t* k_sz, uint32_t* v_sz,
                void* cidx, uint16_t* psac, int psac_fmt, uint16_t* psac_scale,
                const int32_t* table, int page,
                int32_t* cand_out, float* score_out, float* E_out, int group)
{
    if (group <= 0 || d % group || d % 16 || C < 1 || C > M || pos < 0 || pos + n_new > cap || (psac_fmt != 0 && psac_fmt != 1) ||
        (table && (page <= 0 || cap % page))) return 1;
    int ng = d / group, nw = d / 16;
    float* mu = (float*)malloc((size_t)M * d * sizeof(float));
    float* score = (float*)malloc((size_t)M * sizeof(float));
    int* cand = (int*)malloc((size_t)C * sizeof(int));
    float* k = (float*)malloc((size_t)d * sizeof(float));
    float* x = (float*)malloc((size_t)d * sizeof(float));
    float* deq = (float*)malloc((size_t)d * sizeof(float));
    float* xbest = (float*)malloc((size_t)d * sizeof(float));
    uint32_t* cw = (uint32_t*)malloc((size_t)nw * sizeof(uint32_t));
    uint32_t* szr = (uint32_t*)malloc((size_t)ng * sizeof(uint32_t));
    char* used = (char*)malloc((size_t)M);
    float* acoef = (float*)malloc(((size_t)r + 1) * sizeof(float));
    for (int h = 0; h < Hkv; ++h) {
        const float* wh = w + (size_t)h * d;
        qsac_tables(cent, h, M, d, mu);
        for (int b = 0; b < B; ++b) {
            for (int t = 0; t < n_new; ++t) {
                size_t in = (((size_t)b * n_new + t) * Hkv + h) * d;
                size_t slot = slot_at(Hkv, cap, table, page, b, h, pos + t);
                size_t dbg = (((size_t)b * n_new + t) * Hkv + h);
                for (int c = 0; c < d; ++c) k[c] = or_f32_from_bf16(K[in + c]);
                int chosen = qsac_choose(k, wh, Wg + (size_t)h * ng, mu, M, C, d, group, score, cand, used, x,
                                         xbest, cand_out ? cand_out + dbg * C : NULL,
                                         score_out ? score_out + dbg * C : NULL, E_out ? E_out + dbg * C : NULL);
                /* residual codes, scales, zeros */
                quantize_row(xbest, d, group, cw, szr, deq);
                memcpy(k_code + slot * nw, cw, (size_t)nw * 4);
                memcpy(k_sz + slot * ng, szr, (size_t)ng * 4);
                if (M <= 256) ((uint8_t*)cidx)[slot] = (uint8_t)chosen;
                else ((uint16_t*)cidx)[slot] = (uint16_t)chosen;
                /* PSAC coefficients of the key's quantization error */
                float amax = 0.0f;
                for (int i = 0; i < r; ++i) {
                    float a = 0.0f;
                    for (int c = 0; c < d; ++c) {
                        float e = xbest[c] - deq[c];
                        a = fmaf(P[((size_t)h * d + c) * r + i], e, a);
                    }
                    acoef[i] = a;
                    if (fabsf(a) > amax) amax = fabsf(a);
                    if (psac_fmt == 0) psac[slot * (size_t)r + i] = or_f16_from_f32(a, RND_NEAREST_EVEN);
                }
                if (psac_fmt == 1 && r > 0) psac_int8(acoef, r, amax, (int8_t*)psac + slot * (size_t)r,
                                                      psac_scale + slot);
                /* values: same codec, no centre */
                for (int c = 0; c < d; ++c) x[c] = or_f32_from_bf16(V[in + c]);
                quantize_row(x, d, group, cw, szr, NULL);
                memcpy(v_code + slot * nw, cw, (size_t)nw * 4);
                memcpy(v_sz + slot * ng, szr, (size_t)ng * 4);
            }
        }
    }
    free(mu); free(score); free(cand); free(k); free(x);
    free(deq); free(xbest); free(cw); free(szr); free(used); free(acoef);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* QSAC-aware centre fitting.                                                 */
/*   Article "1. QSAC" names the clustering (QSAC picks INT2-friendly Key     */
/*   centres) but not its loop. Reading taken: Lloyd iterations whose          */
/*   assignment step is the QSAC decision above (rank by the weighted          */
/*   distance, keep C candidates, choose the least estimated perturbation) and */
/*   whose update step moves every centre to the mean of the keys assigned to  */
/*   it; a centre with no key keeps its value. The mean: the keys' sum in      */
/*   64-bit fixed point (units of 2^-24, each bf16 value truncated toward 0    */
/*   to a whole number of units: exact for |k| >= 2^-17), divided by the count */
/*   in fp64 (one rounding), scaled by 2^-24 (exact), rounded to fp16 (nearest */
/*   even). Exact, order-free sums make the update independent of summation   */
/*   order. Valid while n * max|k| < 2^39.                                      */
/* X bf16 [n][Hkv][d]; cent fp16 [Hkv][M][d] (in: initial centres, out: the   */
/* fitted ones); assign [n][Hkv] (out, may be NULL): the last assignment.      */
/* ------------------------------------------------------------------------ */

int or_fit_centroids(int n, int Hkv, int d, int M, int C, const uint16_t* X, const float* w,
                     const float* Wg, int iters, uint16_t* cent, int32_t* assign, int group)
{
    if (group <= 0 || d % group || C < 1 || C > M || n < 0 || iters < 0) return 1;
    int ng = d / group;
    float* mu = (float*)malloc((size_t)M * d * sizeof(float));
    float* score = (float*)malloc((size_t)M * sizeof(float));
    int* cand = (int*)malloc((size_t)C * sizeof(int));
    float* k = (float*)malloc((size_t)d * sizeof(float));
    float* x = (float*)malloc((size_t)d * sizeof(float));
    float* xbest = (float*)malloc((size_t)d * sizeof(float));
    char* used = (char*)malloc((size_t)M);
    int* a = (int*)malloc(((size_t)n + 1) * sizeof(int));
    int64_t* sum = (int64_t*)malloc((size_t)M * d * sizeof(int64_t));
    int64_t* cnt = (int64_t*)malloc((size_t)M * sizeof(int64_t));
    for (int it = 0; it < iters; ++it) {
        for (int h = 0; h < Hkv; ++h) {
            const float* wh = w + (size_t)h * d;
            qsac_tables(cent, h, M, d, mu);
            /* assignment */
            for (int t = 0; t < n; ++t) {
                const uint16_t* xr = X + ((size_t)t * Hkv + h) * d;
                for (int c = 0; c < d; ++c) k[c] = or_f32_from_bf16(xr[c]);
                a[t] = qsac_choose(k, wh, Wg + (size_t)h * ng, mu, M, C, d, group, score, cand, used, x,
                                   xbest,
                                   NULL, NULL, NULL);
                if (assign) assign[(size_t)t * Hkv + h] = a[t];
            }
            /* update */
            memset(sum, 0, (size_t)M * d * sizeof(int64_t));
            memset(cnt, 0, (size_t)M * sizeof(int64_t));
            for (int t = 0; t < n; ++t) {
                const uint16_t* xr = X + ((size_t)t * Hkv + h) * d;
                cnt[a[t]] += 1;
                for (int c = 0; c < d; ++c)
                    sum[(size_t)a[t] * d + c] += (int64_t)ldexp((double)or_f32_from_bf16(xr[c]), 24);
            }
            for (int j = 0; j < M; ++j) {
                if (cnt[j] == 0) continue;
                for (int c = 0; c < d; ++c) {
                    double q = (double)sum[(size_t)j * d + c] / (double)cnt[j];
                    cent[((size_t)h * M + j) * d + c] =
                        f16_encode_exact(round_to_format(ldexp(q, -24), 10, -14, F16_MAX, RND_NEAREST_EVEN));
                }
            }
        }
    }
    free(mu); free(score); free(cand); free(k); free(x); free(xbest); free(used);
    free(a); free(sum); free(cnt);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention over the packed cache (fp64).                                    */
/*   logit_t = scale * (q . khat_t + (q P) . a_t), khat_t = mu_idx + deq_t:    */
/*   the PSAC term is the Key compensation of article "2. PSAC" applied to the */
/*   score, q.(khat + P a) = q.khat + (qP).a. Softmax in two passes.           */
/*   Decode: dequantized values are exact (mu + code s + z in fp64), matching   */
/*   a kernel that never rounds them. Chunk: the kernel's operand precision,   */
/*   fp16 arithmetic with one rounding per operation:                          */
/*   khat = fp16(code s + fp16(z + mu)), vhat = fp16(code s + z), u = qP as    */
/*   fp16, self keys and values rounded from bf16 to fp16.                     */
/* ------------------------------------------------------------------------ */

typedef struct {
    int B, Hkv, d, M, r, cap;
    const uint32_t *k_code, *v_code, *k_sz, *v_sz;
    const void* cidx;
    const uint16_t *psac, *cent;
    const float* P;
    int psac_fmt;                 /* 0: fp16 [r]; 1: int8 [r] + fp16 scale per token */
    const uint16_t* psac_scale;
    const int32_t* table;         /* paged: page ids [B][cap / page]; NULL: contiguous */
    int page;                     /* tokens per page (paged) */
    int group;                    /* channels per (scale, zero) group */
} or_cache;


/* PSAC coefficient i of a cached token, exact: the stored fp16 value, or
 * code * scale for the int8 format */
static double psac_value(const or_cache* c, size_t slot, int i)
{
    if (c->psac_fmt == 0) return (double)or_f32_from_f16(c->psac[slot * (size_t)c->r + i]);
    int8_t q = ((const int8_t*)c->psac)[slot * (size_t)c->r + i];
    return (double)q * (double)or_f32_from_f16(c->psac_scale[slot]);
}

static int cache_idx(const or_cache* c, size_t slot)
{
    return c->M <= 256 ? ((const uint8_t*)c->cidx)[slot] : ((const uint16_t*)c->cidx)[slot];
}

static uint32_t code_at(const uint32_t* words, int ch)
{
    return (words[ch / 16] >> (2 * (ch % 16))) & 3u;
}

/* exact dequantized key/value rows of one token (decode precision) */
static void dequant_exact(const or_cache* c, size_t slot, double* kh, double* vh)
{
    int d = c->d, ng = d / c->group;
    const uint32_t* kw = c->k_code + slot * (d / 16);
    const uint32_t* vw = c->v_code + slot * (d / 16);
    int j = cache_idx(c, slot);
    int h = (int)((slot / (size_t)(c->table ? c->page : c->cap)) % (size_t)c->Hkv);
    for (int g = 0; g < ng; ++g) {
        uint32_t ks = c->k_sz[slot * ng + g], vs = c->v_sz[slot * ng + g];
        double s = or_f32_from_f16((uint16_t)(ks & 0xffff)), z = or_f32_from_f16((uint16_t)(ks >> 16));
        double sv = or_f32_from_f16((uint16_t)(vs & 0xffff)), zv = or_f32_from_f16((uint16_t)(vs >> 16));
        for (int ch = g * c->group; ch < (g + 1) * c->group; ++ch) {
            double m = or_f32_from_f16(c->cent[((size_t)h * c->M + j) * d + ch]);
            kh[ch] = m + (double)code_at(kw, ch) * s + z;
            vh[ch] = (double)code_at(vw, ch) * sv + zv;
        }
    }
}

/* operand-precision dequantized rows (chunk kernel precision): fp16
 * arithmetic with one rounding per operation, Khat = fp16(code s + fp16(z + mu)),
 * Vhat = fp16(code s + z) */
static void dequant_operand(const or_cache* c, size_t slot, double* kh, double* vh)
{
    int d = c->d, ng = d / c->group;
    const uint32_t* kw = c->k_code + slot * (d / 16);
    const uint32_t* vw = c->v_code + slot * (d / 16);
    int j = cache_idx(c, slot);
    int h = (int)((slot / (size_t)(c->table ? c->page : c->cap)) % (size_t)c->Hkv);
    for (int g = 0; g < ng; ++g) {
        uint32_t ks = c->k_sz[slot * ng + g], vs = c->v_sz[slot * ng + g];
        double s = or_f32_from_f16((uint16_t)(ks & 0xffff)), z = or_f32_from_f16((uint16_t)(ks >> 16));
        double sv = or_f32_from_f16((uint16_t)(vs & 0xffff)), zv = or_f32_from_f16((uint16_t)(vs >> 16));
        for (int ch = g * c->group; ch < (g + 1) * c->group; ++ch) {
            double m = or_f32_from_f16(c->cent[((size_t)h * c->M + j) * d + ch]);
            kh[ch] = f16_round((double)code_at(kw, ch) * s + f16_round(z + m));
            vh[ch] = f16_round((double)code_at(vw, ch) * sv + zv);
        }
    }
}

/* softmax-weighted sum over n keys given logits and value rows */
static void softmax_combine(const double* logit, const double* vals, int n, int d, double* out)
{
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (n == 0) return;
    double m = logit[0];
    for (int i = 1; i < n; ++i) if (logit[i] > m) m = logit[i];
    double l = 0.0;
    for (int i = 0; i < n; ++i) l += exp(logit[i] - m);
    for (int i = 0; i < n; ++i) {
        double p = exp(logit[i] - m) / l;
        for (int c = 0; c < d; ++c) out[c] += p * vals[(size_t)i * d + c];
    }
}

int or_decode(int B, int Hkv, int d, int M, int r, int cap,
              const uint32_t* k_code, const uint32_t* v_code, const uint32_t* k_sz,
              const uint32_t* v_sz, const void* cidx, const uint16_t* psac,
              int psac_fmt, const uint16_t* psac_scale, const int32_t* table, int page,
              const uint16_t* cent, const float* P,
              int len, const uint16_t* Q, int Hq, double sm_scale, double* out, int group)
{
    if (Hq % Hkv || len < 0 || len > cap || group <= 0 || d % group) return 1;
    or_cache c = {B, Hkv, d, M, r, cap, k_code, v_code, k_sz, v_sz, cidx, psac, cent, P, psac_fmt, psac_scale,
                  table, page, group};
    int G = Hq / Hkv;
    double* logit = (double*)malloc(((size_t)len + 1) * sizeof(double));
    double* vals = (double*)malloc(((size_t)len + 1) * d * sizeof(double));
    double* kh = (double*)malloc((size_t)d * sizeof(double));
    double* q = (double*)malloc((size_t)d * sizeof(double));
    double* u = (double*)malloc(((size_t)r + 1) * sizeof(double));
    for (int b = 0; b < B; ++b)
        for (int hq = 0; hq < Hq; ++hq) {
            int h = hq / G;
            const uint16_t* qr = Q + ((size_t)b * Hq + hq) * d;
            for (int ch = 0; ch < d; ++ch) q[ch] = or_f32_from_bf16(qr[ch]);
            for (int i = 0; i < r; ++i) {
                u[i] = 0.0;
                for (int ch = 0; ch < d; ++ch) u[i] += q[ch] * (double)P[((size_t)h * d + ch) * r + i];
            }
            for (int t = 0; t < len; ++t) {
                size_t slot = slot_at(Hkv, cap, table, page, b, h, t);
                dequant_exact(&c, slot, kh, vals + (size_t)t * d);
                double acc = 0.0;
                for (int ch = 0; ch < d; ++ch) acc += q[ch] * kh[ch];
                for (int i = 0; i < r; ++i)
                    acc += u[i] * psac_value(&c, slot, i);
                logit[t] = acc * sm_scale;
            }
            softmax_combine(logit, vals, len, d, out + ((size_t)b * Hq + hq) * d);
        }
    free(logit); free(vals); free(kh); free(q); free(u);
    return 0;
}

/* Chunk attention for a list of query rows. Q bf16 [B][Nq][Hq][d]; Kself, Vself
 * bf16 [B][Nq][Hkv][d]; query i of frame i / frame_tokens sees every cached
 * token and the self tokens of frames <= its own. rows[k] = (b, i, hq) triples;
 * out [nrows][d]. */
int or_chunk(int B, int Hkv, int d, int M, int r, int cap,
             const uint32_t* k_code, const uint32_t* v_code, const uint32_t* k_sz,
             const uint32_t* v_sz, const void* cidx, const uint16_t* psac,
             int psac_fmt, const uint16_t* psac_scale, const int32_t* table, int page,
             const uint16_t* cent, const float* P, int len,
             const uint16_t* Q, int Hq, int Nq, const uint16_t* Kself, const uint16_t* Vself,
             int frame_tokens, double sm_scale, const int32_t* rows, int nrows, double* out, int group)
{
    if (Hq % Hkv || len < 0 || len > cap || frame_tokens <= 0 || group <= 0 || d % group) return 1;
    or_cache c = {B, Hkv, d, M, r, cap, k_code, v_code, k_sz, v_sz, cidx, psac, cent, P, psac_fmt, psac_scale,
                  table, page, group};
    int G = Hq / Hkv;
    size_t nmax = (size_t)len + (size_t)Nq + 1;
    double* logit = (double*)malloc(nmax * sizeof(double));
    double* vals = (double*)malloc(nmax * d * sizeof(double));
    double* kh = (double*)malloc((size_t)d * sizeof(double));
    double* q = (double*)malloc((size_t)d * sizeof(double));
    double* u = (double*)malloc(((size_t)r + 1) * sizeof(double));
    for (int k = 0; k < nrows; ++k) {
        int b = rows[3 * k], i = rows[3 * k + 1], hq = rows[3 * k + 2];
        int h = hq / G;
        const uint16_t* qr = Q + (((size_t)b * Nq + i) * Hq + hq) * d;
        for (int ch = 0; ch < d; ++ch) q[ch] = or_f32_from_bf16(qr[ch]);
        for (int a = 0; a < r; ++a) {
            double acc = 0.0;
            for (int ch = 0; ch < d; ++ch) acc += q[ch] * (double)P[((size_t)h * d + ch) * r + a];
            u[a] = or_f32_from_f16(or_f16_from_f32((float)acc, RND_NEAREST_EVEN));
        }
        size_t n = 0;
        for (int t = 0; t < len; ++t, ++n) {
            size_t slot = slot_at(Hkv, cap, table, page, b, h, t);
            dequant_operand(&c, slot, kh, vals + n * d);
            double acc = 0.0;
            for (int ch = 0; ch < d; ++ch) acc += q[ch] * kh[ch];
            for (int a = 0; a < r; ++a) acc += u[a] * f16_round(psac_value(&c, slot, a));
            logit[n] = acc * sm_scale;
        }
        int fi = i / frame_tokens;
        for (int j = 0; j < Nq && j / frame_tokens <= fi; ++j, ++n) {
            const uint16_t* kr = Kself + (((size_t)b * Nq + j) * Hkv + h) * d;
            const uint16_t* vr = Vself + (((size_t)b * Nq + j) * Hkv + h) * d;
            double acc = 0.0;
            for (int ch = 0; ch < d; ++ch) {
                acc += q[ch] * f16_round(or_f32_from_bf16(kr[ch]));
                vals[n * d + ch] = or_f32_from_f16(or_f16_from_f32(or_f32_from_bf16(vr[ch]), RND_NEAREST_EVEN));
            }
            logit[n] = acc * sm_scale;
        }
        softmax_combine(logit, vals, (int)n, d, out + (size_t)k * d);
    }
    free(logit); free(vals); free(kh); free(q); free(u);
    return 0;
}

/* Decode logits of one query against the packed cache (fp64), for tests of the
 * PSAC and centroid closed forms. q fp64 [d]; out [len]. */
int or_decode_logits(int Hkv, int d, int M, int r, int cap, int b, int h,
                     const uint32_t* k_code, const uint32_t* k_sz, const void* cidx,
                     const uint16_t* psac, int psac_fmt, const uint16_t* psac_scale,
                     const int32_t* table, int page,
                     const uint16_t* cent, const float* P, int len, const double* q, double* out, int group)
{
    if (group <= 0 || d % group) return 1;
    or_cache c = {b + 1, Hkv, d, M, r, cap, k_code, k_code, k_sz, k_sz, cidx, psac, cent, P, psac_fmt, psac_scale,
                  table, page, group};
    double* kh = (double*)malloc((size_t)d * sizeof(double));
    double* vh = (double*)malloc((size_t)d * sizeof(double));
    double* u = (double*)malloc(((size_t)r + 1) * sizeof(double));
    for (int i = 0; i < r; ++i) {
        u[i] = 0.0;
        for (int ch = 0; ch < d; ++ch) u[i] += q[ch] * (double)P[((size_t)h * d + ch) * r + i];
    }
    for (int t = 0; t < len; ++t) {
        size_t slot = slot_at(Hkv, cap, table, page, b, h, t);
        dequant_exact(&c, slot, kh, vh);
        double acc = 0.0;
        for (int ch = 0; ch < d; ++ch) acc += q[ch] * kh[ch];
        for (int i = 0; i < r; ++i) acc += u[i] * psac_value(&c, slot, i);
        out[t] = acc;
    }
    free(kh); free(vh); free(u);
    return 0;
}
