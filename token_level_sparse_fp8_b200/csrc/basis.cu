// Calibration, step 2: M = TopEig_r(G_Qbar / tr(G_Qbar) + G_K / tr(G_K))^T
// (JSSA summary, eq. (5); JSSA README, paper-to-code map "compute_basis" and section 2: one
// eigendecomposition per layer and KV head).
//
// One CTA per KV head runs a parallel cyclic Jacobi eigensolver in float64: the d x d matrix
// lives in shared memory at d = 128 (rows padded by one element) and in the workspace at
// d = 256 and 512 (the latent basis of multi-head latent attention; too large for shared
// memory, it stays in L2), the eigenvectors are
// accumulated as the rows of V^T in the workspace. Each sweep is d-1 rounds of the round-robin ("circle") pairing,
// so the d/2 rotations of a round touch disjoint index pairs and run in parallel: rotation
// parameters, then the row update (A <- J^T A, V^T <- J^T V^T), then the column update
// (A <- A J). Sweeps stop when the off-diagonal Frobenius norm is below 1e-14 of the total, or
// after kMaxSweeps. Then the eigenvalues are ranked (descending, lower index first on ties), the
// r leading eigenvectors become the rows of M, each signed so that its largest-magnitude entry
// is positive (lowest index on ties).
#include <math.h>

#include "common.cuh"

namespace jssa {

namespace basis_detail {

constexpr int kThreads = 512;
constexpr int kMaxSweeps = 30;

__device__ __forceinline__ void rr_pair(int round, int i, int d, int& p, int& q) {
  const int a = (i == 0) ? 0 : ((i - 1 + round) % (d - 1)) + 1;
  const int b = ((d - 2 - i + round) % (d - 1)) + 1;
  p = a < b ? a : b;
  q = a < b ? b : a;
}

__device__ double block_sum_d(double v, double* s_red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < kThreads / 32; ++w) t += s_red[w];
  return t;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    basis_kernel(const double* __restrict__ gram_q, const double* __restrict__ gram_k, int r,
                 float* __restrict__ basis, double* __restrict__ eigvals, double* __restrict__ ws) {
  constexpr int LD = D + 1;
  constexpr bool kGlobalA = D > 128;
  extern __shared__ __align__(16) double s_a[];  // [D][LD] (D = 128)
  __shared__ double s_c[D / 2], s_s[D / 2];
  __shared__ int s_p[D / 2], s_q[D / 2];
  __shared__ double s_red[kThreads / 32];
  __shared__ int s_rank[D];
  __shared__ double s_lam[D];

  const int tid = threadIdx.x;
  const int h = blockIdx.x;
  const double* gq = gram_q + (int64_t)h * D * D;
  const double* gk = gram_k + (int64_t)h * D * D;
  double* vt = ws + (int64_t)h * D * D;  // rows are eigenvectors
  double* sA = kGlobalA ? ws + (int64_t)gridDim.x * D * D + (int64_t)h * D * LD : s_a;

  double tq = 0.0, tk = 0.0;
  for (int i = tid; i < D; i += kThreads) {
    tq += gq[(int64_t)i * D + i];
    tk += gk[(int64_t)i * D + i];
  }
  tq = block_sum_d(tq, s_red);
  tk = block_sum_d(tk, s_red);
  const double iq = tq > 0.0 ? 1.0 / tq : 0.0;
  const double ik = tk > 0.0 ? 1.0 / tk : 0.0;
  for (int e = tid; e < D * D; e += kThreads) {
    const int i = e / D, j = e % D;
    const double aij = gq[(int64_t)i * D + j] * iq + gk[(int64_t)i * D + j] * ik;
    const double aji = gq[(int64_t)j * D + i] * iq + gk[(int64_t)j * D + i] * ik;
    sA[i * LD + j] = 0.5 * (aij + aji);
    vt[e] = (i == j) ? 1.0 : 0.0;
  }
  __syncthreads();

  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int e = tid; e < D * D; e += kThreads) {
      const int i = e / D, j = e % D;
      const double v = sA[i * LD + j];
      tot += v * v;
      if (i != j) off += v * v;
    }
    off = block_sum_d(off, s_red);
    tot = block_sum_d(tot, s_red);
    if (off <= 1e-28 * tot) break;

    for (int round = 0; round < D - 1; ++round) {
      if (tid < D / 2) {
        int p, q;
        rr_pair(round, tid, D, p, q);
        const double app = sA[p * LD + p], aqq = sA[q * LD + q], apq = sA[p * LD + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (aqq - app) / (2.0 * apq);
          double t;
          if (fabs(tau) > 1e150) t = 0.5 / tau;
          else t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        s_c[tid] = c;
        s_s[tid] = s;
        s_p[tid] = p;
        s_q[tid] = q;
      }
      __syncthreads();
      // rows: A <- J^T A and V^T <- J^T V^T
      for (int e = tid; e < (D / 2) * D; e += kThreads) {
        const int k = e / D, j = e % D;
        const int p = s_p[k], q = s_q[k];
        const double c = s_c[k], s = s_s[k];
        const double apj = sA[p * LD + j], aqj = sA[q * LD + j];
        sA[p * LD + j] = c * apj - s * aqj;
        sA[q * LD + j] = s * apj + c * aqj;
        const double vpj = vt[(int64_t)p * D + j], vqj = vt[(int64_t)q * D + j];
        vt[(int64_t)p * D + j] = c * vpj - s * vqj;
        vt[(int64_t)q * D + j] = s * vpj + c * vqj;
      }
      __syncthreads();
      // columns: A <- A J
      for (int e = tid; e < (D / 2) * D; e += kThreads) {
        const int k = e % (D / 2), i = e / (D / 2);
        const int p = s_p[k], q = s_q[k];
        const double c = s_c[k], s = s_s[k];
        const double aip = sA[i * LD + p], aiq = sA[i * LD + q];
        sA[i * LD + p] = c * aip - s * aiq;
        sA[i * LD + q] = s * aip + c * aiq;
      }
      __syncthreads();
    }
  }

  // rank eigenvalues: descending, lower index first on ties
  for (int i = tid; i < D; i += kThreads) s_lam[i] = sA[i * LD + i];
  __syncthreads();
  for (int i = tid; i < D; i += kThreads) {
    const double li = s_lam[i];
    int rank = 0;
    for (int j = 0; j < D; ++j) {
      const double lj = s_lam[j];
      rank += (lj > li) || (lj == li && j < i);
    }
    s_rank[i] = rank;
    if (eigvals) eigvals[(int64_t)h * D + rank] = li;
  }
  __syncthreads();
  // rows of M: one warp per eigenvector of rank < r
  const int warp = tid >> 5, lane = tid & 31;
  for (int i = warp; i < D; i += kThreads / 32) {
    const int rank = s_rank[i];
    if (rank >= r) continue;
    const double* v = vt + (int64_t)i * D;
    double best = -1.0;
    int bj = D;
    for (int j = lane; j < D; j += 32) {
      const double a = fabs(v[j]);
      if (a > best) { best = a; bj = j; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ob > best || (ob == best && oj < bj)) { best = ob; bj = oj; }
    }
    const double sgn = v[bj] < 0.0 ? -1.0 : 1.0;
    float* dst = basis + ((int64_t)h * r + rank) * D;
    for (int j = lane; j < D; j += 32) dst[j] = (float)(sgn * v[j]);
  }
}

}  // namespace basis_detail

cudaError_t launch_basis(const double* gram_q, const double* gram_k, int h_kv, int d, int r,
                         float* basis, double* eigvals, double* ws, cudaStream_t s) {
  if (h_kv <= 0) return cudaSuccess;
  if (d != 128 && d != 256 && d != 512) return cudaErrorInvalidValue;
  const size_t smem = d == 128 ? (size_t)d * (d + 1) * sizeof(double) : 0;
  auto kern = d == 128 ? basis_detail::basis_kernel<128>
                       : d == 256 ? basis_detail::basis_kernel<256> : basis_detail::basis_kernel<512>;
  cudaError_t e = configure_kernel((const void*)kern, (int)smem, false);
  if (e != cudaSuccess) return e;
  kern<<<h_kv, basis_detail::kThreads, smem, s>>>(gram_q, gram_k, r, basis, eigvals, ws);
  return cudaGetLastError();
}

}  // namespace jssa
