// act_stats.cu -- per-input-channel activation statistic
//   a_j = (1/N) sum_i |X_ij|   (or max_i |X_ij|)
// compassingai.com AWQ concept page, "statistical basis of salient channels"
// (activation_scale[j] = mean(|X_calib[:, j]|), or max); mudrobot.github.io
// AWQ notes, "searching the optimal scale" (s_X = average magnitude per
// channel).
//
// HBM-bound column reduction over a row-major bf16 matrix.  One cluster of 8
// CTAs owns a slab of 64 channels (128 bytes of every row); each warp reads
// four rows per instruction (8 lanes x 16 bytes per row) and keeps eight such
// loads in flight.  Every thread accumulates 8 channels in fp32 over its rows;
// the CTA folds its 32 row-lanes in a fixed order in shared memory, and CTA
// rank 0 folds the 8 CTA totals of the cluster through distributed shared
// memory, again in a fixed order.  No atomics and no scratch memory: the result
// is bit-for-bit reproducible for a given shape.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace awq {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kSlab = 64;                // channels per cluster
constexpr int kLanesPerRow = kSlab / 8;  // 16-byte chunks per row slab
constexpr int kRowLanesCta = kThreads / kLanesPerRow;
constexpr int kRowLanes = kCluster * kRowLanesCta;
constexpr int kUnroll = 8;

__device__ __forceinline__ void unpack8_abs(const uint4& v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = fabsf(__uint_as_float(w[i] << 16));
    x[2 * i + 1] = fabsf(__uint_as_float(w[i] & 0xFFFF0000u));
  }
}

template <bool kMax>
__device__ __forceinline__ void fold8(float (&acc)[8], const uint4& v) {
  float x[8];
  unpack8_abs(v, x);
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = kMax ? fmaxf(acc[e], x[e]) : acc[e] + x[e];
}

template <bool kMax>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads)
    act_stats_kernel(const uint16_t* __restrict__ X, int64_t N, int64_t D, float* __restrict__ a) {
  __shared__ float part[kRowLanesCta][kSlab + 1];
  __shared__ float cta_total[kSlab];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int chunk = threadIdx.x % kLanesPerRow;
  const int rl = threadIdx.x / kLanesPerRow;               // row-lane within the CTA
  const int64_t ch0 = static_cast<int64_t>(blockIdx.y) * kSlab + chunk * 8;
  const int row_lane = rank * kRowLanesCta + rl;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;

  if (ch0 < D) {
    const uint4* base = reinterpret_cast<const uint4*>(X + ch0);
    const int64_t stride = D / 8;   // uint4 per row
    int64_t r = row_lane;
    for (; r + (kUnroll - 1) * kRowLanes < N; r += kUnroll * kRowLanes) {
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) v[u] = __ldcs(base + (r + u * kRowLanes) * stride);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) fold8<kMax>(acc, v[u]);
    }
    for (; r < N; r += kRowLanes) fold8<kMax>(acc, __ldcs(base + r * stride));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rl][chunk * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < kSlab) {
    float t = part[0][threadIdx.x];
#pragma unroll
    for (int l = 1; l < kRowLanesCta; ++l) t = kMax ? fmaxf(t, part[l][threadIdx.x]) : t + part[l][threadIdx.x];
    cta_total[threadIdx.x] = t;
  }
  cluster.sync();
  if (rank == 0 && threadIdx.x < kSlab) {
    float t = 0.0f;
    for (int q = 0; q < kCluster; ++q) {
      const float* remote = cluster.map_shared_rank(cta_total, q);
      t = kMax ? fmaxf(t, remote[threadIdx.x]) : t + remote[threadIdx.x];
    }
    const int64_t j = static_cast<int64_t>(blockIdx.y) * kSlab + threadIdx.x;
    if (j < D) a[j] = kMax ? t : __fdiv_rn(t, static_cast<float>(N));
  }
  cluster.sync();   // keep every CTA's shared memory alive until rank 0 has read it
}

}  // namespace

cudaError_t launch_act_stats(const uint16_t* X, int64_t N, int64_t D, int stat, float* a, cudaStream_t st) {
  dim3 grid(kCluster, static_cast<unsigned>((D + kSlab - 1) / kSlab));
  if (stat == 1)
    act_stats_kernel<true><<<grid, kThreads, 0, st>>>(X, N, D, a);
  else
    act_stats_kernel<false><<<grid, kThreads, 0, st>>>(X, N, D, a);
  return cudaGetLastError();
}

}  // namespace awq
