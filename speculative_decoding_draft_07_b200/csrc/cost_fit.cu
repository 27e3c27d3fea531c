// Non-negative least-squares fit of the verification cost
//   C_v(n; l) = a + b l + c n + e n^2,   a, b, c, e >= 0,
// to latency samples (n_i, l_i, t_i).
//
// "Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
// summary), "Method: CaDDTree": the verification cost is profiled offline as a
// convex function of the tree size that does not decrease as it grows (and
// grows with the context length); with this model that is the fit under
// a, b, c, e >= 0.
//
// One block. The threads accumulate the normal equations of X = [1, l, n, n^2]
// (G = X^T X, h = X^T t and t^T t) in fp64 over strided samples, reduced in a
// fixed order (lane tree, then warps in order). Thread s < 16 then solves the
// least squares restricted to the free set s (bit j: coefficient j free) on the
// unit-norm-scaled columns, by Gaussian elimination with partial pivoting on at
// most four unknowns, and keeps it when every coefficient is >= 0; a free set
// whose columns are linearly dependent is skipped. The optimum of the
// constrained problem is the least squares of its own free set, so thread 0
// takes the feasible set with the smallest residual and scales it back.
#include "common.cuh"
#include "internal.h"

namespace pct {
namespace {

constexpr int kFitThreads = 256;
constexpr int kFitSums = 15;   // 10 entries of G (upper triangle), 4 of h, t^T t

__global__ __launch_bounds__(kFitThreads) void cost_fit_kernel(long long m,
                                                               const float* __restrict__ n,
                                                               const float* __restrict__ ell,
                                                               const float* __restrict__ lat,
                                                               double* __restrict__ out,
                                                               int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  __shared__ double red[kFitThreads / 32][kFitSums];
  __shared__ double tot[kFitSums];
  __shared__ double res[16];
  __shared__ double sol[16][4];
  __shared__ int feasible[16];
  __shared__ int s_bad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();

  double acc[kFitSums];
#pragma unroll
  for (int q = 0; q < kFitSums; ++q) acc[q] = 0.0;
  int bad = 0;
  for (long long i = threadIdx.x; i < m; i += blockDim.x) {
    const double nv = (double)n[i], lv = (double)ell[i], tv = (double)lat[i];
    bad |= !(isfinite(nv) && isfinite(lv) && isfinite(tv));
    const double x[4] = {1.0, lv, nv, nv * nv};
    int q = 0;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = a; b < 4; ++b) acc[q++] += x[a] * x[b];
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[10 + a] += x[a] * tv;
    acc[14] += tv * tv;
  }
  if (bad) atomicOr(&s_bad, 1);
#pragma unroll
  for (int q = 0; q < kFitSums; ++q) {
    double v = acc[q];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][q] = v;
  }
  __syncthreads();
  if (threadIdx.x < kFitSums) {
    double v = 0.0;
    for (int w = 0; w < kFitThreads / 32; ++w) v += red[w][threadIdx.x];
    tot[threadIdx.x] = v;
  }
  __syncthreads();

  if (threadIdx.x < 16) {
    const int fs = threadIdx.x;
    double G[4][4], h[4], sc[4];
    int q = 0;
    for (int a = 0; a < 4; ++a)
      for (int b = a; b < 4; ++b) { G[a][b] = tot[q]; G[b][a] = tot[q]; ++q; }
    for (int a = 0; a < 4; ++a) {
      sc[a] = G[a][a] > 0.0 ? sqrt(G[a][a]) : 1.0;
      h[a] = tot[10 + a] / sc[a];
    }
    for (int a = 0; a < 4; ++a)
      for (int b = 0; b < 4; ++b) G[a][b] /= sc[a] * sc[b];
    // the system of the free set: A x = r on the free coefficients
    int idx[4], k = 0;
    for (int a = 0; a < 4; ++a)
      if (fs & (1 << a)) idx[k++] = a;
    double A[4][5];
    for (int i = 0; i < k; ++i) {
      for (int j = 0; j < k; ++j) A[i][j] = G[idx[i]][idx[j]];
      A[i][4] = h[idx[i]];
    }
    bool ok = true;
    for (int c = 0; c < k && ok; ++c) {
      int piv = c;
      for (int i = c + 1; i < k; ++i)
        if (fabs(A[i][c]) > fabs(A[piv][c])) piv = i;
      // unit diagonal before elimination: a pivot this small means dependent columns
      if (!(fabs(A[piv][c]) > 1e-12)) { ok = false; break; }
      if (piv != c)
        for (int j = 0; j < 5; ++j) { const double t = A[c][j]; A[c][j] = A[piv][j]; A[piv][j] = t; }
      for (int i = c + 1; i < k; ++i) {
        const double f = A[i][c] / A[c][c];
        for (int j = c; j < 5; ++j) A[i][j] -= f * A[c][j];
      }
    }
    double x[4] = {0.0, 0.0, 0.0, 0.0};
    if (ok) {
      for (int i = k - 1; i >= 0; --i) {
        double v = A[i][4];
        for (int j = i + 1; j < k; ++j) v -= A[i][j] * x[idx[j]];
        x[idx[i]] = v / A[i][i];
      }
      for (int i = 0; i < k; ++i) ok = ok && x[idx[i]] >= 0.0;
    }
    // residual sum of squares at the free set's least squares: t^T t - x . h
    double r = tot[14];
    for (int a = 0; a < 4; ++a) r -= x[a] * h[a];
    feasible[fs] = ok;
    res[fs] = r;
    for (int a = 0; a < 4; ++a) sol[fs][a] = x[a] / sc[a];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int best = 0;   // the empty free set (all zero) is always feasible
    for (int fs = 1; fs < 16; ++fs)
      if (feasible[fs] && res[fs] < res[best]) best = fs;
    for (int a = 0; a < 4; ++a) out[a] = sol[best][a];
    out[4] = sqrt(fmax(res[best], 0.0) / (double)m);
    if (s_bad) atomicOr(status, PCT_DEV_BAD_COST);
  }
}

}  // namespace

cudaError_t launch_cost_fit(long long m, const float* n, const float* ell, const float* lat,
                            double* out, int32_t* status, cudaStream_t s) {
  TraceScope t(s, "cadd_cost_fit");
  return launch_pdl(cost_fit_kernel, dim3(1), dim3(kFitThreads), 0, s, 1, m, n, ell, lat, out,
                    status);
}

}  // namespace pct
