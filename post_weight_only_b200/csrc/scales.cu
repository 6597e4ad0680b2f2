// scales.cu -- the candidate scale table s_alpha[j] = a_j^alpha and its
// reciprocal 1/s_alpha[j] (fp32, IEEE division).
// compassingai.com AWQ concept page, flow step 3 (s_j(alpha) =
// activation_scale[j]^alpha, alpha in {0, 0.05, ..., 1}); mudrobot.github.io
// AWQ notes, "searching the optimal scale" (s = s_X^alpha).
//
// Reading for a dead channel (the pages are silent): a_j is floored at
// 1e-6 * max_j a_j (fp32 product) so that 1/s stays finite; when every a_j is
// 0 all scales are 1.  The power is taken in fp64 and rounded once to fp32,
// so alpha = 0 gives exactly 1 and alpha = 1 gives exactly a_j.
//
// Balanced scale (laojiahuo2003.github.io GPTQ/AWQ/SmoothQuant notes, section 4.4, the per-channel
// scale): with a weight statistic b_j = mean_n |W_jn|, s_j = a_j^alpha /
// b_j^(1-alpha); b is floored the same way, and the quotient of the two fp64
// powers is rounded once.
#include "internal.cuh"

namespace awq {
namespace {

constexpr int kThreads = 256;

__device__ float block_max(const float* __restrict__ v, int64_t D, float* red) {
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < D; j += kThreads) m = fmaxf(m, v[j]);
  red[threadIdx.x] = m;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  const float r = red[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads)
    scale_table_kernel(const float* __restrict__ a, const float* __restrict__ b, int64_t D, AlphaList alphas,
                       const float* __restrict__ alpha_dev, float* __restrict__ s_tab, float* __restrict__ r_tab) {
  __shared__ float red[kThreads];
  const float amax = block_max(a, D, red);
  const float bmax = b ? block_max(b, D, red) : 0.0f;
  const float floor_ = __fmul_rn(1e-6f, amax);
  const int ai = blockIdx.y;
  const float alpha = alpha_dev ? alpha_dev[0] : alphas.v[ai];
  const int64_t j = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (j >= D) return;
  float aj = 1.0f;
  if (amax != 0.0f) aj = a[j] > floor_ ? a[j] : floor_;
  double sv = pow(static_cast<double>(aj), static_cast<double>(alpha));
  if (b) {
    const float bfl = __fmul_rn(1e-6f, bmax);
    float bj = 1.0f;
    if (bmax != 0.0f) bj = b[j] > bfl ? b[j] : bfl;
    sv = sv / pow(static_cast<double>(bj), 1.0 - static_cast<double>(alpha));
  }
  const float s = static_cast<float>(sv);
  if (s_tab) s_tab[static_cast<int64_t>(ai) * D + j] = s;
  if (r_tab) r_tab[static_cast<int64_t>(ai) * D + j] = __fdiv_rn(1.0f, s);
}

// b_j = (sum_n |W_jn|) / D_out, one block per row j: per-thread fp64 sums
// over a strided slice of the row, then a fixed-order tree; rounded to fp32
// once.  Reads each row once, coalesced.
__global__ void __launch_bounds__(kThreads)
    weight_mean_kernel(const float* __restrict__ W, int64_t D_in, int64_t D_out, float* __restrict__ b) {
  __shared__ double red[kThreads];
  const float* row = W + static_cast<int64_t>(blockIdx.x) * D_out;
  double acc = 0.0;
  for (int64_t n = threadIdx.x; n < D_out; n += kThreads) acc += fabs(static_cast<double>(__ldcs(row + n)));
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) b[blockIdx.x] = static_cast<float>(red[0] / static_cast<double>(D_out));
}

}  // namespace

cudaError_t launch_scale_table(const float* a, const float* b, int64_t D, const AlphaList& alphas,
                               const float* alpha_dev, int A, float* s_tab, float* r_tab, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((D + kThreads - 1) / kThreads), static_cast<unsigned>(A));
  scale_table_kernel<<<grid, kThreads, 0, st>>>(a, b, D, alphas, alpha_dev, s_tab, r_tab);
  return cudaGetLastError();
}

cudaError_t launch_weight_mean(const float* W, int64_t D_in, int64_t D_out, float* b, cudaStream_t st) {
  weight_mean_kernel<<<static_cast<unsigned>(D_in), kThreads, 0, st>>>(W, D_in, D_out, b);
  return cudaGetLastError();
}

}  // namespace awq
