// fit.cu — Query statistics for QSAC and PSAC.
//
// Method: "QuantWM: Training-Free 2-bit KV Cache Quantization for Stable Video
// World Models", "2. Principal Subspace Attention Compensation (PSAC)":
// historical Query energy concentrates in a few principal directions; both
// components use statistics of already generated Queries. Here:
//   S_h  = (1/N) sum q q^T over the N = n*G history queries of KV head h's
//          query-head group (uncentred second moment, fp64);
//   w    = diag(S) (per-channel sensitivity, fp32), Wg = per-group sums of w
//          (groups of 32, 64 or 128 consecutive channels);
//   P    = top-r eigenvectors of S (descending eigenvalues, largest-magnitude
//          entry positive), energy = top-r share of trace(S).
// Kernels: fit_gram (fp64 32x32 output tiles), fit_jacobi (one CTA per head:
// parallel cyclic Jacobi with round-robin pairing, d/2 disjoint rotations per
// step; the matrix lives in shared memory in fp64, the eigenvector matrix is
// kept transposed in the workspace so every rotation is a row operation).
#include <cfloat>

#include "common.cuh"
#include "internal.h"

namespace kv2 {
namespace {

constexpr int kGramTile = 32;
constexpr int kGramChunk = 32;

__global__ void __launch_bounds__(256) fit_gram(const uint16_t* __restrict__ Qh, int n, int H_q,
                                                int H_kv, int D, double* __restrict__ S) {
  const int h = blockIdx.z;
  const int r0 = blockIdx.y * kGramTile, c0 = blockIdx.x * kGramTile;
  const int G = H_q / H_kv;
  const int N = n * G;
  __shared__ double a_s[kGramChunk][kGramTile + 1];
  __shared__ double b_s[kGramChunk][kGramTile + 1];
  const int tid = threadIdx.x;
  const int ty = tid / 8, tx = tid % 8;   // row ty, cols tx*4 .. +3
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int v0 = 0; v0 < N; v0 += kGramChunk) {
    for (int i = tid; i < kGramChunk * kGramTile; i += 256) {
      const int v = i / kGramTile, c = i % kGramTile;
      double x = 0.0, y = 0.0;
      if (v0 + v < N) {
        const int t = (v0 + v) / G, g = (v0 + v) % G;
        const uint16_t* q = Qh + (size_t(t) * H_q + size_t(h) * G + g) * D;
        x = bf16_to_f32(q[r0 + c]);
        y = bf16_to_f32(q[c0 + c]);
      }
      a_s[v][c] = x;
      b_s[v][c] = y;
    }
    __syncthreads();
#pragma unroll 4
    for (int v = 0; v < kGramChunk; ++v) {
      const double x = a_s[v][ty];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = fma(x, b_s[v][tx * 4 + k], acc[k]);
    }
    __syncthreads();
  }
  const double inv = 1.0 / double(N);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    S[(size_t(h) * D + r0 + ty) * D + c0 + tx * 4 + k] = acc[k] * inv;
}

__device__ __forceinline__ void pair_of(int round, int i, int D, int* p, int* q) {
  // round-robin tournament: D-1 rounds, D/2 disjoint pairs each
  const int m = D - 1;
  int a, b;
  if (i == 0) {
    a = round;
    b = m;
  } else {
    a = (round + i) % m;
    b = (round - i + m) % m;
  }
  *p = a < b ? a : b;
  *q = a < b ? b : a;
}

constexpr int kJacobiThreads = 512;

__global__ void __launch_bounds__(kJacobiThreads) fit_jacobi(const double* __restrict__ S_all,
                                                             double* __restrict__ Vt_all, int D, int r,
                                                             float* __restrict__ P, float* __restrict__ w,
                                                             float* __restrict__ Wg, float* __restrict__ energy,
                                                             int group) {
  constexpr int NT = kJacobiThreads;
  extern __shared__ __align__(16) unsigned char smem[];
  double* A = reinterpret_cast<double*>(smem);             // [D][D]
  double* cs = A + D * D;                                  // [D/2]
  double* sn = cs + D / 2;                                 // [D/2]
  double* red = sn + D / 2;                                // [NT]
  int* order = reinterpret_cast<int*>(red + NT);           // [D]
  int* pp = order + D;                                     // [D/2] this round's pairs
  int* qq = pp + D / 2;                                    // [D/2]
  const int h = blockIdx.x, tid = threadIdx.x;
  const double* S = S_all + size_t(h) * D * D;
  double* Vt = Vt_all + size_t(h) * D * D;
  for (int i = tid; i < D * D; i += NT) {
    A[i] = S[i];
    Vt[i] = (i / D == i % D) ? 1.0 : 0.0;
  }
  // sensitivity weights from the diagonal
  for (int c = tid; c < D; c += NT) w[size_t(h) * D + c] = float(S[size_t(c) * D + c]);
  __syncthreads();
  // group sensitivities: w summed over each group's channels in ascending order
  if (tid < D / group) {
    float acc = 0.0f;
    for (int c = tid * group; c < tid * group + group; ++c) acc = __fadd_rn(acc, w[size_t(h) * D + c]);
    Wg[size_t(h) * (D / group) + tid] = acc;
  }
  // total squared norm (convergence reference)
  double tot = 0.0;
  for (int i = tid; i < D * D; i += NT) tot += A[i] * A[i];
  red[tid] = tot;
  __syncthreads();
  for (int s = NT / 2; s > 0; s >>= 1) {
    if (tid < s) red[tid] += red[tid + s];
    __syncthreads();
  }
  const double total = red[0];
  __syncthreads();

  const int npairs = D / 2;
  for (int sweep = 0; sweep < 40; ++sweep) {
    double off = 0.0;
    for (int i = tid; i < D * D; i += NT) {
      const int a = i / D, b = i % D;
      if (a != b) off += A[i] * A[i];
    }
    red[tid] = off;
    __syncthreads();
    for (int s = NT / 2; s > 0; s >>= 1) {
      if (tid < s) red[tid] += red[tid + s];
      __syncthreads();
    }
    const double offn = red[0];
    __syncthreads();
    if (offn <= 1e-28 * total || offn == 0.0) break;
    for (int round = 0; round < D - 1; ++round) {
      if (tid < npairs) {
        int p, q;
        pair_of(round, tid, D, &p, &q);
        const double apq = A[p * D + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double theta = (A[q * D + q] - A[p * D + p]) / (2.0 * apq);
          const double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          s = t * c;
        }
        cs[tid] = c;
        sn[tid] = s;
        pp[tid] = p;
        qq[tid] = q;
      }
      __syncthreads();
      // rows p, q of A and of Vt (J^T applied from the left; Vt rows = V columns)
      for (int i = tid; i < npairs * D; i += NT) {
        const int pi = i / D, k = i - pi * D;
        const int p = pp[pi], q = qq[pi];
        const double c = cs[pi], s = sn[pi];
        const double apk = A[p * D + k], aqk = A[q * D + k];
        A[p * D + k] = c * apk - s * aqk;
        A[q * D + k] = s * apk + c * aqk;
        const double vpk = Vt[p * D + k], vqk = Vt[q * D + k];
        Vt[p * D + k] = c * vpk - s * vqk;
        Vt[q * D + k] = s * vpk + c * vqk;
      }
      __syncthreads();
      // columns p, q of A (J applied from the right)
      for (int i = tid; i < npairs * D; i += NT) {
        const int k = i / npairs, pi = i - k * npairs;
        const int p = pp[pi], q = qq[pi];
        const double c = cs[pi], s = sn[pi];
        const double akp = A[k * D + p], akq = A[k * D + q];
        A[k * D + p] = c * akp - s * akq;
        A[k * D + q] = s * akp + c * akq;
      }
      __syncthreads();
    }
  }
  // order eigenvalues descending (ties: lower index first)
  for (int i = tid; i < D; i += NT) {
    const double li = A[i * D + i];
    int rank = 0;
    for (int j = 0; j < D; ++j) {
      const double lj = A[j * D + j];
      rank += (lj > li) || (lj == li && j < i);
    }
    order[rank] = i;
  }
  __syncthreads();
  if (tid == 0 && energy) {
    double all = 0.0, top = 0.0;
    for (int i = 0; i < D; ++i) all += A[i * D + i];
    for (int i = 0; i < r; ++i) top += A[order[i] * D + order[i]];
    energy[h] = float(all > 0.0 ? top / all : 0.0);
  }
  for (int i = tid; i < r; i += NT) {
    const double* v = Vt + size_t(order[i]) * D;
    int arg = 0;
    for (int c = 1; c < D; ++c)
      if (fabs(v[c]) > fabs(v[arg])) arg = c;
    const double sg = v[arg] < 0.0 ? -1.0 : 1.0;
    for (int c = 0; c < D; ++c) P[(size_t(h) * D + c) * r + i] = float(sg * v[c]);
  }
}

}  // namespace

size_t fit_workspace_bytes(int H_kv, int d) { return size_t(2) * H_kv * d * d * sizeof(double); }

cudaError_t launch_fit(const FitArgs& a, cudaStream_t s) {
  const int D = a.d;
  double* S = static_cast<double*>(a.ws);
  double* Vt = S + size_t(a.H_kv) * D * D;
  dim3 g1(D / kGramTile, D / kGramTile, a.H_kv);
  fit_gram<<<g1, 256, 0, s>>>(a.Qhist, a.n, a.H_q, a.H_kv, D, S);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = size_t(D) * D * 8 + size_t(D) * 8 + kJacobiThreads * 8 + size_t(D) * 4 + size_t(D) * 4;
  e = cudaFuncSetAttribute(fit_jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  fit_jacobi<<<a.H_kv, kJacobiThreads, smem, s>>>(S, Vt, D, a.r, a.P, a.w, a.Wg, a.energy, a.group);
  return cudaGetLastError();
}

}  // namespace kv2
