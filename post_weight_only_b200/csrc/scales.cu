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
#include "internal.cuh"

namespace awq {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    scale_table_kernel(const float* __restrict__ a, int64_t D, AlphaList alphas, const float* __restrict__ alpha_dev,
                       float* __restrict__ s_tab, float* __restrict__ r_tab) {
  __shared__ float red[kThreads];
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < D; j += kThreads) m = fmaxf(m, a[j]);
  red[threadIdx.x] = m;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  const float amax = red[0];
  const float floor_ = __fmul_rn(1e-6f, amax);
  const int ai = blockIdx.y;
  const float alpha = alpha_dev ? alpha_dev[0] : alphas.v[ai];
  const int64_t j = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  if (j >= D) return;
  float aj = 1.0f;
  if (amax != 0.0f) aj = a[j] > floor_ ? a[j] : floor_;
  const float s = static_cast<float>(pow(static_cast<double>(aj), static_cast<double>(alpha)));
  if (s_tab) s_tab[static_cast<int64_t>(ai) * D + j] = s;
  if (r_tab) r_tab[static_cast<int64_t>(ai) * D + j] = __fdiv_rn(1.0f, s);
}

}  // namespace

cudaError_t launch_scale_table(const float* a, int64_t D, const AlphaList& alphas, const float* alpha_dev, int A,
                               float* s_tab, float* r_tab, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((D + kThreads - 1) / kThreads), static_cast<unsigned>(A));
  scale_table_kernel<<<grid, kThreads, 0, st>>>(a, D, alphas, alpha_dev, s_tab, r_tab);
  return cudaGetLastError();
}

}  // namespace awq
