// act_stats.cu -- per-input-channel activation statistic
//   a_j = (1/N) sum_i |X_ij|   (or max_i |X_ij|)
// compassingai.com AWQ concept page, "statistical basis of salient channels"
// (activation_scale[j] = mean(|X_calib[:, j]|), or max); mudrobot.github.io
// AWQ notes, "searching the optimal scale" (s_X = average magnitude per
// channel).
//
// HBM-bound column reduction over a row-major bf16 matrix, in one wave of CTA
// pairs (clusters of two, one CTA per SM).  The channels are cut into slabs
// whose width is a multiple of 64 channels, so that every row segment a CTA
// reads is whole 128-byte lines (segments that straddle lines cost a third
// more time on B200), as many slabs as there are pairs or fewer; the two CTAs
// of a pair split the slab's rows.  Inside a CTA a thread owns one 8-channel
// chunk and one row lane and streams its rows through private slots in shared
// memory with 16-byte asynchronous copies, sixteen rows in flight, so the data
// in flight costs no registers and needs no barrier (a thread reads back only
// its own copies).  The row lanes fold in two fixed-order steps in shared
// memory and the pair folds its two halves through distributed shared memory,
// again in a fixed order: no atomics, no scratch in global memory, and the
// result is bit-for-bit reproducible for a given shape.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace awq {
namespace {

constexpr int kThreads = 512;
constexpr int kCluster = 2;                              // CTAs per slab: the row split
constexpr int kSlabAlign = 64;                           // channels: one 128-byte line of bf16
constexpr int kMaxSlabChunks = 2048;                     // 8-channel chunks per slab at most
constexpr int kRowsPerStage = 4;
constexpr int kStages = 4;
constexpr int kDepth = kRowsPerStage * kStages;          // rows in flight per thread
constexpr int kRingBytes = kDepth * kThreads * 16;       // 128 KiB
constexpr int kSmemBytes = kRingBytes + kMaxSlabChunks * 8 * 4 /*channel totals*/;

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

// The inputs of one launch: input i is X [N][D] bf16 with output a [D], cut
// into slabs of slab_ch channels that are clusters first_slab[i] ..
// first_slab[i + 1] - 1 of the grid.
struct StatsInputs {
  const uint16_t* X[kMaxStatsInputs];
  float* a[kMaxStatsInputs];
  int64_t N[kMaxStatsInputs], D[kMaxStatsInputs], slab_ch[kMaxStatsInputs];
  int first_slab[kMaxStatsInputs + 1];
  int n;
};

// Cluster blockIdx.x / kCluster owns channels [slab * W, min(D, (slab + 1) * W))
// of the input whose slab range holds it.
template <bool kMax>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
    act_stats_kernel(const StatsInputs in) {
  const int slab_id = static_cast<int>(blockIdx.x / kCluster);
  int which = 0;
  while (which + 1 < in.n && slab_id >= in.first_slab[which + 1]) ++which;
  const uint16_t* __restrict__ X = in.X[which];
  float* __restrict__ a = in.a[which];
  const int64_t N = in.N[which], D = in.D[which], slab_ch = in.slab_ch[which];
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* ring = reinterpret_cast<uint4*>(smem);
  float* fold = reinterpret_cast<float*>(smem);                 // reuses the ring after the stream
  float* tot = reinterpret_cast<float*>(smem + kRingBytes);     // this CTA's channel totals
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int t = threadIdx.x;
  const int64_t c0 = static_cast<int64_t>(slab_id - in.first_slab[which]) * slab_ch;   // first channel of the slab
  const int64_t c1 = c0 + slab_ch < D ? c0 + slab_ch : D;
  const int nck = static_cast<int>((c1 - c0) / 8);              // chunks, >= 1
  const int RL = nck < kThreads ? kThreads / nck : 1;           // row lanes
  const int lanes = nck * RL;
  const int64_t r0 = N * rank / kCluster, r1 = N * (rank + 1) / kCluster;
  const int64_t stride = D / 8;                                 // uint4 per row

  const int rounds = (lanes + kThreads - 1) / kThreads;       // > 1 only with one row lane
  for (int j = 0; j < rounds; ++j) {
    const int L = t + j * kThreads;
    const bool active = L < lanes;
    const int ck = active ? L % nck : 0, rl = active ? L / nck : 0;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    if (active) {
      const int64_t first = r0 + rl;
      const int nr = first < r1 ? static_cast<int>((r1 - first + RL - 1) / RL) : 0;   // rows of this lane
      const int nst = (nr + kRowsPerStage - 1) / kRowsPerStage;
      // The next row to copy, advanced by a pointer step (no per-row products);
      // row i lands in ring slot i % kDepth, so stage g's slots are
      // (g % kStages) * kRowsPerStage + q with q a compile-time offset.
      const uint4* next = reinterpret_cast<const uint4*>(X) + c0 / 8 + ck + first * stride;
      const int64_t step = static_cast<int64_t>(RL) * stride;
      uint4* const mine = ring + t;
      // One pass covers the prologue, the steady state and the drain: pass g
      // issues stage g (if any) and folds stage g - (kStages - 1) (if any).
      for (int g = 0; g < nst + kStages - 1; ++g) {
        if (g < nst) {
          uint4* slots = mine + (g % kStages) * kRowsPerStage * kThreads;
          const int left = nr - g * kRowsPerStage;
#pragma unroll
          for (int q = 0; q < kRowsPerStage; ++q) {
            if (q < left) {
              cp_async16(slots + q * kThreads, next, 16u);
              next += step;
            }
          }
        }
        cp_async_commit();
        const int f = g - (kStages - 1);
        if (f >= 0) {
          cp_async_wait<kStages - 1>();    // this thread's rows of stage f have landed
          const uint4* slots = mine + (f % kStages) * kRowsPerStage * kThreads;
          const int left = nr - f * kRowsPerStage;
#pragma unroll
          for (int q = 0; q < kRowsPerStage; ++q)
            if (q < left) fold8<kMax>(acc, slots[q * kThreads]);
        }
      }
      cp_async_wait<0>();
    }
    if (RL == 1) {
      // one row lane: a lane's sums are the CTA's totals for its chunk
      if (active) {
        float4* d4 = reinterpret_cast<float4*>(tot + ck * 8);
        d4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        d4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    } else {
      // several row lanes (then a single round): fold them in order through
      // the ring, which every thread has finished streaming through
      __syncthreads();
      if (active) {
        float4* f4 = reinterpret_cast<float4*>(fold + (static_cast<int64_t>(rl) * nck + ck) * 8);
        f4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        f4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
      __syncthreads();
      // Step 1: P parts per channel, part p folding row lanes p, p + P, ...
      // in order; step 2: the P parts in order.
      const int nch = nck * 8;
      const int P = nch < kThreads ? kThreads / nch : 1;
      float* parts = fold + kThreads * 8;                     // after the row-lane sums
      // (a slab can hold more channels than the CTA has threads: then P = 1
      // and each thread takes channels t, t + kThreads, ...)
      for (int idx = t; idx < P * nch; idx += kThreads) {
        const int c = idx % nch, pp = idx / nch;
        float sum = fold[pp * nch + c];
        for (int l = pp + P; l < RL; l += P) sum = kMax ? fmaxf(sum, fold[l * nch + c]) : sum + fold[l * nch + c];
        parts[pp * nch + c] = sum;
      }
      __syncthreads();
      for (int c = t; c < nch; c += kThreads) {
        float sum = parts[c];
        for (int pp = 1; pp < P; ++pp) sum = kMax ? fmaxf(sum, parts[pp * nch + c]) : sum + parts[pp * nch + c];
        tot[c] = sum;
      }
    }
  }
  // The pair folds in rank order; CTA q writes the channels c with c % 2 == q.
  const int nch = nck * 8;
  cluster.sync();
  const float* part0 = cluster.map_shared_rank(tot, 0);
  const float* part1 = cluster.map_shared_rank(tot, 1);
  for (int c = rank + kCluster * t; c < nch; c += kCluster * kThreads) {
    const float sum = kMax ? fmaxf(part0[c], part1[c]) : part0[c] + part1[c];
    a[c0 + c] = kMax ? sum : __fdiv_rn(sum, static_cast<float>(N));
  }
  cluster.sync();   // each CTA's shared memory stays alive until the other has read it
}

}  // namespace

cudaError_t launch_act_stats_batched(const uint16_t* const* X, const int64_t* N, const int64_t* D, int n, int stat,
                                     float* const* a, int num_sms, cudaStream_t st) {
  if (n < 1 || n > kMaxStatsInputs) return cudaErrorInvalidValue;
  static SmemAttrOnce once_mean, once_max;
  cudaError_t e = set_smem_once(act_stats_kernel<false>, kSmemBytes, once_mean);
  if (e == cudaSuccess) e = set_smem_once(act_stats_kernel<true>, kSmemBytes, once_max);
  if (e != cudaSuccess) return e;
  // The pairs that fit in one wave are shared out in proportion to the
  // inputs' bytes (at least one each); an input's slab width is its D over
  // its pairs, rounded up to whole lines, at most kMaxSlabChunks chunks.
  const int64_t pairs = num_sms >= 2 ? num_sms / 2 : 1;
  double total = 0.0;
  for (int i = 0; i < n; ++i) total += static_cast<double>(N[i]) * static_cast<double>(D[i]);
  StatsInputs in{};
  in.n = n;
  int slabs_all = 0;
  for (int i = 0; i < n; ++i) {
    int64_t p = static_cast<int64_t>(static_cast<double>(pairs) * static_cast<double>(N[i]) *
                                     static_cast<double>(D[i]) / total);
    if (p < 1) p = 1;
    int64_t slab = (D[i] + p - 1) / p;
    slab = (slab + kSlabAlign - 1) / kSlabAlign * kSlabAlign;
    if (slab > static_cast<int64_t>(kMaxSlabChunks) * 8) slab = static_cast<int64_t>(kMaxSlabChunks) * 8;
    in.X[i] = X[i];
    in.a[i] = a[i];
    in.N[i] = N[i];
    in.D[i] = D[i];
    in.slab_ch[i] = slab;
    in.first_slab[i] = slabs_all;
    slabs_all += static_cast<int>((D[i] + slab - 1) / slab);
  }
  in.first_slab[n] = slabs_all;
  const dim3 grid(static_cast<unsigned>(slabs_all * kCluster));
  if (stat == 1)
    act_stats_kernel<true><<<grid, kThreads, kSmemBytes, st>>>(in);
  else
    act_stats_kernel<false><<<grid, kThreads, kSmemBytes, st>>>(in);
  return cudaGetLastError();
}

cudaError_t launch_act_stats(const uint16_t* X, int64_t N, int64_t D, int stat, float* a, int num_sms,
                             cudaStream_t st) {
  return launch_act_stats_batched(&X, &N, &D, 1, stat, &a, num_sms, st);
}

}  // namespace awq
