// Batched parent scoring for fp32 Markov parameters (FP32 pipes).
//
// PCTree article (qiita), section on the chain draft's weakness and the tree
// built in its place: every frontier parent p is scored as
// z_d(p) = L_d + Markov(p) in one batched call. With the rank-r stand-in
// Markov(p) = E[p] . W and fp32 E, W the contraction is done with FMAs (the
// fp32 inputs keep their full precision; the bf16 variant runs on the tensor
// cores in pct_umma.cu). Block = one parent row x one V-slice; each thread
// walks a strided set of columns keeping an online log-sum-exp and a register
// top-k, and the block folds them into one partial for the slice.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace pct {
namespace {

constexpr int kSimtThreads = 128;

template <typename TL, int KMAX>
__global__ __launch_bounds__(kSimtThreads) void score_simt_kernel(ScoreArgs a, int cols_per_slice) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float eg[];                       // [r]
  __shared__ float rm[kSimtThreads / 32], rs[kSimtThreads / 32];
  __shared__ float bv[kSimtThreads / 32];
  __shared__ int bi[kSimtThreads / 32];
  const int row = blockIdx.x, sl = blockIdx.y;
  const int req = row / a.n_par;
  const int r = a.r;
  const float* Eg = static_cast<const float*>(a.Eg) + (size_t)row * a.r_pad;
  for (int j = threadIdx.x; j < r; j += blockDim.x) eg[j] = Eg[j];
  __syncthreads();
  const TL* Lr = static_cast<const TL*>(a.L) + (size_t)req * a.L_req_stride;
  const float* W = static_cast<const float*>(a.W);
  const int V = a.V, k = a.k;
  const int c0 = sl * cols_per_slice, c1 = min(V, c0 + cols_per_slice);

  float m = neg_inf(), s = 0.f;
  TopK<KMAX> tk;
  tk.init(k);
  for (int v = c0 + threadIdx.x; v < c1; v += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < r; ++j) acc = fmaf(eg[j], W[(size_t)j * V + v], acc);
    const float z = load_f(Lr + v) + acc;
    lse_combine(m, s, z, 1.f);
    if (tk.admits(z, v)) tk.insert(z, v);
  }
  tk.finish(k);
  // fold the block: log-sum-exp pairs, then k rounds of block-wide best head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_combine(m, s, m2, s2);
  }
  if (lane == 0) { rm[warp] = m; rs[warp] = s; }
  __syncthreads();
  const size_t ps = (size_t)row * a.S + sl;
  if (threadIdx.x == 0) {
    float M = neg_inf(), Ssum = 0.f;
    for (int w = 0; w < kSimtThreads / 32; ++w) lse_combine(M, Ssum, rm[w], rs[w]);
    a.part.ms[ps] = make_float2(M, Ssum);
  }
  for (int j = 0; j < k; ++j) {
    float v = tk.v[0];
    int i = tk.i[0];
    warp_best(v, i);
    if (lane == 0) { bv[warp] = v; bi[warp] = i; }
    __syncthreads();
    v = bv[0]; i = bi[0];
    for (int w = 1; w < kSimtThreads / 32; ++w)
      if (better(bv[w], bi[w], v, i)) { v = bv[w]; i = bi[w]; }
    if (tk.v[0] == v && tk.i[0] == i) tk.pop();
    if (threadIdx.x == 0) { a.part.val[ps * k + j] = v; a.part.idx[ps * k + j] = i; }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_score_simt(const ScoreArgs& a, cudaStream_t s) {
  const int rows = a.n_req * a.n_par;
  const int cps = (a.V + a.S - 1) / a.S;
  dim3 grid(rows, a.S);
  const size_t smem = (size_t)a.r * sizeof(float);
  TraceScope t(s, "pct_score_simt");
#define PCT_SIMT(TL, KM) \
  launch_pdl(score_simt_kernel<TL, KM>, grid, dim3(kSimtThreads), smem, s, 1, a, cps)
  if (a.logits_dtype == PCT_BF16) {
    if (a.k <= 4) return PCT_SIMT(__nv_bfloat16, 4);
    if (a.k <= 8) return PCT_SIMT(__nv_bfloat16, 8);
    return PCT_SIMT(__nv_bfloat16, 16);
  }
  if (a.k <= 4) return PCT_SIMT(float, 4);
  if (a.k <= 8) return PCT_SIMT(float, 8);
  return PCT_SIMT(float, 16);
#undef PCT_SIMT
}

}  // namespace pct
