// calibrate: the per-modality value bases U_m from calibration values, on the GPU
// (paperpeel.com section 2.3 "Modality-aware value rotation": one basis per
// modality, calibrated once per model; section 3.1; pchao.org 方法概览: an
// attention-contribution-weighted covariance matrix per modality and its
// eigendecomposition). Readings (the oracle's calibration module, c1-c4):
//   C_m = sum_{t of m, a_t > 0} a_t (v_t - mu_m)(v_t - mu_m)^T / sum a_t, mu_m the
//   a-weighted mean, in fp64; E_m = its eigenvectors, descending eigenvalues, each
//   column's entry of largest magnitude positive (the first on ties); U_m = E_m H
//   with H = 2^-3.5 H_128 (Sylvester); a modality without weight keeps U_m = H.
//   Tokens whose id is not 0, 1 or 2, or whose weight is not positive, are ignored.
//
// Four launches on the caller's stream, all in fp64 (the result is compared with an
// fp64 LAPACK eigensolver; a calibration runs once per model, so exactness wins
// over speed):
//   1. gram: CTA c sums, over its contiguous run of tokens and for each modality,
//      W = sum a, S = sum a v and the Gram matrix G = sum a v v^T; each of 256
//      threads owns an 8 x 8 tile of G (64 fp64 accumulators); the run's tokens are
//      staged in shared memory 64 at a time; partial sums go to the workspace (no
//      atomics: the result does not depend on scheduling);
//   2. reduce: C_m = G/W - (S/W)(S/W)^T from the partials, summed in run order;
//   3. jacobi: one CTA per modality holds C_m in shared memory (128 KB) and runs
//      cyclic parallel Jacobi sweeps (round-robin ordering: 64 disjoint rotations
//      per round, 127 rounds per sweep; Golub and Van Loan, Matrix Computations,
//      sections 8.5.2 "the symmetric Schur decomposition" and 8.5.3-8.5.5 on the
//      cyclic and parallel orderings), accumulating the eigenvectors in the
//      workspace, until the off-diagonal mass is below 1e-26 of the total (an
//      off-diagonal norm of 1e-13 of the matrix's; the sweeps converge
//      quadratically, so the last one is far below) or after 40 sweeps (the loop
//      is bounded; a singular covariance, fewer than 129 weighted tokens, keeps
//      rounding noise in its null space and stops there);
//   4. finish: rank the eigenvalues (descending, ties by index), apply the sign
//      rule, multiply by H with a fast Walsh-Hadamard transform of every row, store
//      U_m in fp32 and the sorted eigenvalues in fp64.
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace omnikv {
namespace {

constexpr int kGramThreads = 256;    // 16 x 16 tiles of 8 x 8
constexpr int kGramBatch = 64;       // tokens staged in shared memory at a time
constexpr int kMaxRuns = 148;        // token runs (CTAs) of the Gram launch
constexpr int kMinRunTokens = 64;
constexpr int kPartStride = 16520;   // fp64 per (run, modality): W, S[128], G[128][128], padding
constexpr int kJacThreads = 512;
constexpr int kMaxSweeps = 40;
constexpr int kMat = kHeadDim * kHeadDim;

int gram_runs(int T) { return max(1, min(kMaxRuns, (T + kMinRunTokens - 1) / kMinRunTokens)); }

struct CalWorkspace {  // offsets in doubles
  size_t part, cov, vec, eig, wsum, bytes;
  explicit CalWorkspace(int T) {
    const size_t runs = (size_t)gram_runs(T);
    part = 0;
    cov = part + runs * kMods * kPartStride;
    vec = cov + (size_t)kMods * kMat;
    eig = vec + (size_t)kMods * kMat;
    wsum = eig + (size_t)kMods * kHeadDim;
    bytes = (wsum + 8) * sizeof(double);
  }
};

__global__ void __launch_bounds__(kGramThreads) gram_kernel(const __half* __restrict__ v, const uint8_t* __restrict__ mod,
                                                           const float* __restrict__ a, int T, double* __restrict__ ws) {
  __shared__ float xs[kGramBatch][kHeadDim];  // the batch's values (exact from fp16)
  __shared__ double ws_a[kGramBatch];         // weights, 0 for tokens of another modality
  const int tid = threadIdx.x;
  const int runs = gridDim.x;
  const int per = (T + runs - 1) / runs;
  const int t0 = min(T, blockIdx.x * per), t1 = min(T, t0 + per);
  const int r0 = 8 * (tid >> 4), c0 = 8 * (tid & 15);
  for (int m = 0; m < kMods; ++m) {
    double acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
    double s_acc = 0.0, w_acc = 0.0;  // thread c < 128: S[c]; thread 0 also W
    for (int base = t0; base < t1; base += kGramBatch) {
      const int n = min(kGramBatch, t1 - base);
      for (int e = tid; e < kGramBatch * kHeadDim / 2; e += kGramThreads) {  // half2 pairs
        const int t = e / (kHeadDim / 2), c2 = e % (kHeadDim / 2);
        float2 f = make_float2(0.f, 0.f);
        if (t < n) f = __half22float2(reinterpret_cast<const __half2*>(v + (size_t)(base + t) * kHeadDim)[c2]);
        xs[t][2 * c2] = f.x;
        xs[t][2 * c2 + 1] = f.y;
      }
      if (tid < kGramBatch) {
        const int md = tid < n ? (int)mod[base + tid] : -1;
        const float w = tid < n ? a[base + tid] : 0.0f;
        ws_a[tid] = (md == m && w > 0.0f) ? (double)w : 0.0;
      }
      __syncthreads();
      for (int t = 0; t < n; ++t) {
        const double w = ws_a[t];
        if (w == 0.0) continue;  // the same decision in every thread
        double u[8], x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) u[i] = w * (double)xs[t][r0 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = (double)xs[t][c0 + j];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fma(u[i], x[j], acc[i][j]);
        if (tid < kHeadDim) s_acc = fma(w, (double)xs[t][tid], s_acc);
        if (tid == 0) w_acc += w;
      }
      __syncthreads();
    }
    double* part = ws + ((size_t)blockIdx.x * kMods + m) * kPartStride;
    if (tid == 0) part[0] = w_acc;
    if (tid < kHeadDim) part[1 + tid] = s_acc;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) part[1 + kHeadDim + (r0 + i) * kHeadDim + c0 + j] = acc[i][j];
  }
}

// Block (m, r), thread c: C_m[r][c] from the runs' partials, in run order.
__global__ void __launch_bounds__(kHeadDim) cov_reduce_kernel(double* __restrict__ ws, size_t cov_off,
                                                              size_t wsum_off, int runs) {
  const int m = blockIdx.x / kHeadDim, r = blockIdx.x % kHeadDim, c = threadIdx.x;
  double W = 0.0, Sr = 0.0, Sc = 0.0, G = 0.0;
  for (int k = 0; k < runs; ++k) {
    const double* part = ws + ((size_t)k * kMods + m) * kPartStride;
    W += part[0];
    Sr += part[1 + r];
    Sc += part[1 + c];
    G += part[1 + kHeadDim + r * kHeadDim + c];
  }
  double C = 0.0;
  if (W > 0.0) {
    const double mr = Sr / W, mc = Sc / W;
    C = G / W - mr * mc;
  }
  ws[cov_off + (size_t)m * kMat + r * kHeadDim + c] = C;
  if (r == 0 && c == 0) ws[wsum_off + m] = W;
}

// Round r of the round-robin ordering: pair i = (pos(i), pos(127 - i)) with pos(0)
// = 0 and pos(k) = 1 + (k - 1 + r) mod 127; every pair of indices meets once per sweep.
__device__ __forceinline__ int rr_pos(int k, int r) { return k == 0 ? 0 : 1 + (k - 1 + r) % (kHeadDim - 1); }

__global__ void __launch_bounds__(kJacThreads) jacobi_kernel(double* __restrict__ ws, size_t cov_off, size_t vec_off,
                                                            size_t eig_off, size_t wsum_off) {
  extern __shared__ double A[];  // [128][128]
  __shared__ double rc[kHeadDim / 2], rs[kHeadDim / 2];
  __shared__ int rp[kHeadDim / 2], rq[kHeadDim / 2];
  __shared__ double red[kJacThreads / 32][2];
  __shared__ int s_done;
  const int m = blockIdx.x, tid = threadIdx.x;
  double* V = ws + vec_off + (size_t)m * kMat;
  const double* C = ws + cov_off + (size_t)m * kMat;
  for (int e = tid; e < kMat; e += kJacThreads) {
    A[e] = C[e];
    V[e] = (e / kHeadDim == e % kHeadDim) ? 1.0 : 0.0;
  }
  if (tid == 0) s_done = ws[wsum_off + m] > 0.0 ? 0 : 1;  // no weight: the finish launch writes H
  __syncthreads();
  for (int sweep = 0; sweep < kMaxSweeps && !s_done; ++sweep) {
    for (int r = 0; r < kHeadDim - 1; ++r) {
      if (tid < kHeadDim / 2) {  // the rotation of pair tid (Golub and Van Loan, sym.schur2)
        const int p = rr_pos(tid, r), q = rr_pos(kHeadDim - 1 - tid, r);
        const double apq = A[p * kHeadDim + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (A[q * kHeadDim + q] - A[p * kHeadDim + p]) / (2.0 * apq);
          const double t = tau >= 0.0 ? 1.0 / (tau + sqrt(1.0 + tau * tau)) : -1.0 / (-tau + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        rc[tid] = c;
        rs[tid] = s;
        rp[tid] = p;
        rq[tid] = q;
      }
      __syncthreads();
      // rows p, q of A: (J^T A)
      for (int e = tid; e < (kHeadDim / 2) * kHeadDim; e += kJacThreads) {
        const int i = e / kHeadDim, k = e % kHeadDim;
        const double c = rc[i], s = rs[i];
        double* ap = &A[rp[i] * kHeadDim + k];
        double* aq = &A[rq[i] * kHeadDim + k];
        const double x = *ap, y = *aq;
        *ap = c * x - s * y;
        *aq = s * x + c * y;
      }
      __syncthreads();
      // columns p, q of A and of V: (A J), (V J)
      for (int e = tid; e < (kHeadDim / 2) * kHeadDim; e += kJacThreads) {
        const int i = e % (kHeadDim / 2), k = e / (kHeadDim / 2);
        const double c = rc[i], s = rs[i];
        const int p = rp[i], q = rq[i];
        double* ap = &A[k * kHeadDim + p];
        double* aq = &A[k * kHeadDim + q];
        const double x = *ap, y = *aq;
        *ap = c * x - s * y;
        *aq = s * x + c * y;
        double* vp = &V[k * kHeadDim + p];
        double* vq = &V[k * kHeadDim + q];
        const double vx = *vp, vy = *vq;
        *vp = c * vx - s * vy;
        *vq = s * vx + c * vy;
      }
      __syncthreads();
    }
    // converged when the off-diagonal mass is below 1e-26 of the total
    double off = 0.0, tot = 0.0;
    for (int e = tid; e < kMat; e += kJacThreads) {
      const double x = A[e] * A[e];
      tot += x;
      if (e / kHeadDim != e % kHeadDim) off += x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if ((tid & 31) == 0) {
      red[tid >> 5][0] = off;
      red[tid >> 5][1] = tot;
    }
    __syncthreads();
    if (tid == 0) {
      double o2 = 0.0, t2 = 0.0;
      for (int w = 0; w < kJacThreads / 32; ++w) {
        o2 += red[w][0];
        t2 += red[w][1];
      }
      s_done = (o2 <= 1e-26 * t2) ? 1 : 0;
    }
    __syncthreads();
  }
  if (tid < kHeadDim) ws[eig_off + (size_t)m * kHeadDim + tid] = A[tid * kHeadDim + tid];
}

// U_m = E_m H in fp32 and the eigenvalues in descending order.
__global__ void __launch_bounds__(kHeadDim) basis_finish_kernel(const double* __restrict__ ws, size_t vec_off,
                                                               size_t eig_off, size_t wsum_off,
                                                               float* __restrict__ bases,
                                                               double* __restrict__ eigenvalues) {
  extern __shared__ double E[];  // [128][128], rows i, sorted columns
  __shared__ double lam[kHeadDim];
  __shared__ int perm[kHeadDim];
  const int m = blockIdx.x, j = threadIdx.x;
  float* U = bases + (size_t)m * kMat;
  const double inv = 0.08838834764831845;  // 2^-3.5
  if (!(ws[wsum_off + m] > 0.0)) {  // no calibration weight: U_m = H
    for (int i = 0; i < kHeadDim; ++i) U[i * kHeadDim + j] = (float)((__popc(i & j) & 1) ? -inv : inv);
    if (eigenvalues) eigenvalues[(size_t)m * kHeadDim + j] = 0.0;
    return;
  }
  const double* V = ws + vec_off + (size_t)m * kMat;
  lam[j] = ws[eig_off + (size_t)m * kHeadDim + j];
  __syncthreads();
  int rank = 0;  // descending, ties by index
  for (int i = 0; i < kHeadDim; ++i) rank += (lam[i] > lam[j] || (lam[i] == lam[j] && i < j)) ? 1 : 0;
  perm[rank] = j;
  __syncthreads();
  // thread j: sorted column j = eigenvector perm[j], sign by its entry of largest magnitude
  const int src = perm[j];
  int imax = 0;
  double vmax = -1.0;
  for (int i = 0; i < kHeadDim; ++i) {
    const double x = fabs(V[i * kHeadDim + src]);
    if (x > vmax) {
      vmax = x;
      imax = i;
    }
  }
  const double sg = V[imax * kHeadDim + src] < 0.0 ? -1.0 : 1.0;
  for (int i = 0; i < kHeadDim; ++i) E[i * kHeadDim + j] = sg * V[i * kHeadDim + src];
  if (eigenvalues) eigenvalues[(size_t)m * kHeadDim + j] = lam[src];
  __syncthreads();
  // every row times H: butterflies h = 1 .. 64 on the rows, then the scale
  for (int h = 1; h < kHeadDim; h <<= 1) {
    for (int e = j; e < kHeadDim * kHeadDim / 2; e += kHeadDim) {
      const int i = e / (kHeadDim / 2), k = e % (kHeadDim / 2);
      const int lo = (k / h) * 2 * h + (k % h), hi = lo + h;
      const double x = E[i * kHeadDim + lo], y = E[i * kHeadDim + hi];
      E[i * kHeadDim + lo] = x + y;
      E[i * kHeadDim + hi] = x - y;
    }
    __syncthreads();
  }
  for (int i = 0; i < kHeadDim; ++i) U[i * kHeadDim + j] = (float)(E[i * kHeadDim + j] * inv);
}

}  // namespace

size_t calibrate_workspace_bytes(int num_tokens) { return num_tokens > 0 ? CalWorkspace(num_tokens).bytes : 0; }

cudaError_t launch_calibrate(const __half* values, const uint8_t* modality, const float* weights, int T,
                             void* workspace, float* bases, double* eigenvalues, cudaStream_t stream) {
  const CalWorkspace L(T);
  double* ws = static_cast<double*>(workspace);
  const int runs = gram_runs(T);
  gram_kernel<<<runs, kGramThreads, 0, stream>>>(values, modality, weights, T, ws + L.part);
  cov_reduce_kernel<<<kMods * kHeadDim, kHeadDim, 0, stream>>>(ws, L.cov, L.wsum, runs);
  const size_t smem = (size_t)kMat * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  jacobi_kernel<<<kMods, kJacThreads, smem, stream>>>(ws, L.cov, L.vec, L.eig, L.wsum);
  e = cudaFuncSetAttribute(basis_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  basis_finish_kernel<<<kMods, kHeadDim, smem, stream>>>(ws, L.vec, L.eig, L.wsum, bases, eigenvalues);
  return cudaGetLastError();
}

}  // namespace omnikv
