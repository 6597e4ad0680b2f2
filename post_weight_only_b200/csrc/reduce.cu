// reduce.cu -- L(alpha) from the search kernel's per-(alpha, token half-tile,
// column) partial sums, and alpha* = argmin L.
// compassingai.com AWQ concept page, flow steps 4c-5 (L(alpha) = ||X S^-1 W'_hat
// - X W||^2, alpha* = argmin L); the smallest index wins exact ties.
//
// Every sum runs in a fixed order in fp64, so L and alpha* are reproducible
// run to run:  L_col[a][n] = sum_h partial[a][h][n] (h ascending), then per
// block a fixed binary tree over 256 columns, then the block totals in
// ascending order.
#include "internal.cuh"

namespace awq {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    loss_cols_kernel(const float* __restrict__ partial, int H, int64_t D_out, double* __restrict__ L_col,
                     double* __restrict__ blk, int nblk) {
  __shared__ double red[kThreads];
  const int a = blockIdx.y;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  double acc = 0.0;
  if (n < D_out) {
    const float* p = partial + static_cast<int64_t>(a) * H * D_out + n;
    for (int h = 0; h < H; ++h) acc += static_cast<double>(p[static_cast<int64_t>(h) * D_out]);
    if (L_col) L_col[static_cast<int64_t>(a) * D_out + n] = acc;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) blk[static_cast<int64_t>(a) * nblk + blockIdx.x] = red[0];
}

__global__ void loss_final_kernel(const double* __restrict__ blk, int A, int nblk, AlphaList alphas,
                                  double* __restrict__ L, float* __restrict__ alpha_star,
                                  int* __restrict__ alpha_idx) {
  __shared__ double Ls[kMaxAlpha];
  const int a = threadIdx.x;
  if (a < A) {
    double s = 0.0;
    for (int b = 0; b < nblk; ++b) s += blk[static_cast<int64_t>(a) * nblk + b];
    Ls[a] = s;
    if (L) L[a] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int best = 0;
    for (int i = 1; i < A; ++i)
      if (Ls[i] < Ls[best]) best = i;
    if (alpha_idx) *alpha_idx = best;
    if (alpha_star) *alpha_star = alphas.v[best];
  }
}

// Per-layer losses of a joint search: L_layer[l][a] = sum of L_col[a][n] over
// the layer's column range [off[l], off[l+1]), each thread a strided share in
// ascending order, then a fixed binary tree.
__global__ void __launch_bounds__(kThreads)
    segment_sums_kernel(const double* __restrict__ L_col, int64_t D, Segments seg, double* __restrict__ out) {
  __shared__ double red[kThreads];
  const int a = blockIdx.x, l = blockIdx.y;
  const int A = gridDim.x;
  double acc = 0.0;
  for (int64_t n = seg.off[l] + threadIdx.x; n < seg.off[l + 1]; n += kThreads)
    acc += L_col[static_cast<int64_t>(a) * D + n];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[static_cast<int64_t>(l) * A + a] = red[0];
}

}  // namespace

cudaError_t launch_segment_sums(const double* L_col, int A, int64_t D, const Segments& seg, int n_seg, double* out,
                                cudaStream_t st) {
  segment_sums_kernel<<<dim3(static_cast<unsigned>(A), static_cast<unsigned>(n_seg)), kThreads, 0, st>>>(L_col, D,
                                                                                                         seg, out);
  return cudaGetLastError();
}

int loss_reduce_blocks(int64_t D_out) { return static_cast<int>((D_out + kThreads - 1) / kThreads); }

cudaError_t launch_loss_reduce(const float* partial, int A, int H, int64_t D_out, double* L_col, double* blk,
                               int nblk, const AlphaList& alphas, double* L, float* alpha_star, int* alpha_idx,
                               cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(nblk), static_cast<unsigned>(A));
  loss_cols_kernel<<<grid, kThreads, 0, st>>>(partial, H, D_out, L_col, blk, nblk);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  loss_final_kernel<<<1, kMaxAlpha, 0, st>>>(blk, A, nblk, alphas, L, alpha_star, alpha_idx);
  return cudaGetLastError();
}

}  // namespace awq
