// clip.cu -- the weight-clipping search that follows the scale search.
//
// mudrobot.github.io AWQ notes, "searching the optimal scale": after the
// scale search, weight clipping is applied to minimise the quantisation MSE.
// For every group g, output column n and clip ratio c of a grid, the group
// maximum is replaced by c * max before delta is formed (codes clamped), and
// the objective is the squared error of the group's share of the layer output
//     L_c(g, n) = || X_g e_g,n(c) ||^2 = e^T H_g e,    H_g = X_g^T X_g,
// where X_g is the N x G slab of the calibration activations that meets the
// group's rows.  The Gram form is exact algebra; it costs G^2 instead of N G
// multiply-adds per (g, n, c).
//
// Kernels:
//   xt_kernel         X [N][D_in] bf16 -> XT [D_in][Np] bf16 (tokens padded to 8)
//   recip_kernel      r_k = 1 / s_k (IEEE)
//   gram_kernel       per 128-channel block b: D = XT_b XT_b^T on the tensor
//                     cores (one TMA tile is both operands), the diagonal
//                     G x G group blocks written as bf16 Hb[g][G][G]
//   clip_loss_kernel  per (group, 128 columns) unit: H_g loaded once; for each
//                     c, D = E_c H_g (E_c the clipping operand, from
//                     launch_clip_operand in quant.cu) and the epilogue forms
//                     L = sum_j D[n][j] E[n][j], keeping a running argmin over c.
//
// Every mbarrier wait is bounded (the status word records a timeout), and
// every role leaves its loop after a timeout.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace awq {
namespace {

enum ClipSite { kSiteGramFull = 16, kSiteGramEmpty, kSiteGramAcc, kSiteLossAFull, kSiteLossAEmpty, kSiteLossHFull,
                kSiteLossHEmpty, kSiteLossAccFull, kSiteLossAccEmpty };

// ---------------------------------------------------------------- transpose, reciprocal
__global__ void __launch_bounds__(256)
    xt_kernel(const uint16_t* __restrict__ X, int64_t N, int64_t D, int64_t Np, uint16_t* __restrict__ XT) {
  __shared__ uint16_t tile[64][66];
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * 64, k0 = static_cast<int64_t>(blockIdx.y) * 64;
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int r = i >> 6, c = i & 63;
    const int64_t t = t0 + r, k = k0 + c;
    tile[r][c] = (t < N && k < D) ? X[t * D + k] : static_cast<uint16_t>(0);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int r = i >> 6, c = i & 63;
    const int64_t k = k0 + r, t = t0 + c;
    if (k < D && t < Np) XT[k * Np + t] = tile[c][r];
  }
}

__global__ void recip_kernel(const float* __restrict__ s, int64_t D, float* __restrict__ r) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k < D) r[k] = __frcp_rn(s[k]);
}

// ---------------------------------------------------------------- Gram blocks
constexpr int kGramStages = 4;
constexpr int kGramTile = 128 * 64 * 2;                 // 128 channels x 64 tokens, bf16
constexpr int kGramSmem = kGramStages * kGramTile + 1024 + 1024;

// CTA b: channels [128 b, 128 b + 128).  Hb[g][i][j] = (X_g^T X_g)[i][j] in
// bf16 for the groups g inside the block.
template <int G>
__global__ void __launch_bounds__(192, 1)
    gram_kernel(const __grid_constant__ CUtensorMap tmXT, int64_t D_in, int64_t Np, uint16_t* __restrict__ Hb,
                int* status, unsigned long long timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGramStages * kGramTile);
  uint64_t* full = bars;
  uint64_t* empty = full + kGramStages;
  uint64_t* acc_full = empty + kGramStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = static_cast<int>((Np + 63) / 64);
  const int row0 = blockIdx.x * 128;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGramStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  bool aborted = false;
  if (warp == 0) {
    if (lane == 0) {
      int last_round[kGramStages] = {-1, -1, -1, -1};
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % kGramStages, r = kb / kGramStages;
        if (!wait_bounded(&empty[s], (r & 1) ^ 1, abort_flag, status, kSiteGramEmpty, timeout_ns)) {
          aborted = true;
          break;
        }
        mbar_arrive_expect_tx(&full[s], kGramTile);
        tma_load_2d(smem + s * kGramTile, &tmXT, &full[s], kb * 64, row0);
        last_round[s] = r;
      }
      volatile int no_abort = 0;
      for (int s = 0; s < kGramStages; ++s)
        if (last_round[s] >= 0) wait_bounded(&full[s], last_round[s] & 1, &no_abort, status, kSiteGramFull, timeout_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % kGramStages;
        if (!wait_bounded(&full[s], (kb / kGramStages) & 1, abort_flag, status, kSiteGramFull, timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t desc = sw128_kmajor_desc(smem_u32(smem + s * kGramTile));
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_ss_f16_cta(tbase, desc + 2 * j, desc + 2 * j, idesc, (kb | j) != 0 ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      aborted = !ok;
      mma_commit(acc_full);      // arrives once every MMA issued above has completed
      volatile int no_abort = 0;
      wait_bounded(acc_full, 0, &no_abort, status, kSiteGramAcc, timeout_ns);
    }
    __syncwarp();
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 = channel rows of the block
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool got = wait_bounded(acc_full, 0, abort_flag, status, kSiteGramAcc, timeout_ns);
    if (__all_sync(0xffffffffu, got)) {
      tc_fence_after();
      const int gi = row / G;                                    // group inside the block
      const int64_t g = static_cast<int64_t>(row0) / G + gi;
      const bool valid = row0 + row < D_in;
#pragma unroll 1
      for (int c32 = 0; c32 < 128 / 32; ++c32) {
        uint32_t v[32];
        tmem_ld32(tbase + (static_cast<uint32_t>(q * 32) << 16) + c32 * 32, v);
        tmem_wait_ld();
        const int col0 = c32 * 32;
        if (valid && col0 / G == gi) {                           // the diagonal block of this row's group
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          uint4* dst = reinterpret_cast<uint4*>(Hb + (g * G + row % G) * G + col0 % G);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    } else {
      aborted = true;
    }
  }
  if (aborted || *abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 128);
}

// ---------------------------------------------------------------- clip losses
constexpr int kLossStages = 4;
constexpr int kLossThreads = 192;

template <int G>
struct LossLayout {
  static constexpr int kABytes = 128 * G * 2;           // 128 columns x G rows of the operand, bf16
  static constexpr int kHBytes = G * G * 2;
  static constexpr int kSmem = kLossStages * kABytes + kHBytes + 1024 + 1024;
};

struct ClipParams {
  int64_t D_in, D_out;
  int n_clip, groups, nblocks, units;
  AlphaList clips;
  float* clip_out;          // [groups][D_out] chosen ratio
  int* idx_out;             // [groups][D_out] or null
  float* loss_out;          // [n_clip][groups][D_out] or null
  int* status;
  unsigned long long timeout_ns;
};

// Element (n, k) of a 128-row, 64-column bf16 box in the 128-byte swizzled
// K-major layout: 16-byte chunk c of row n sits at chunk c ^ (n % 8).
__device__ __forceinline__ uint4 sw128_row_chunk(const uint8_t* box, int n, int c) {
  return *reinterpret_cast<const uint4*>(box + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4));
}

template <int G>
__global__ void __launch_bounds__(kLossThreads, 1)
    clip_loss_kernel(const __grid_constant__ CUtensorMap tmOp, const __grid_constant__ CUtensorMap tmH,
                     const ClipParams p) {
  using L = LossLayout<G>;
  constexpr int kBoxes = G / 64;                          // 64-wide k boxes per operand tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_sm = smem;
  uint8_t* h_sm = smem + kLossStages * L::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(h_sm + L::kHBytes);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + kLossStages;
  uint64_t* h_full = a_empty + kLossStages;
  uint64_t* h_empty = h_full + 1;
  uint64_t* acc_full = h_empty + 1;                        // [2]
  uint64_t* acc_empty = acc_full + 2;                      // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kLossStages; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 4);
    }
    mbar_init(h_full, 1);
    mbar_init(h_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * G < 32 ? 32 : 2 * G);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;
  bool aborted = false;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t it = 0, ui = 0;
      int last_a[kLossStages] = {-1, -1, -1, -1};
      int last_h = -1;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
        const int g = u / p.nblocks, nb = u % p.nblocks;
        if (!wait_bounded(h_empty, (ui & 1) ^ 1, abort_flag, p.status, kSiteLossHEmpty, tmo)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(h_full, L::kHBytes);
#pragma unroll
        for (int b = 0; b < kBoxes; ++b) tma_load_3d(h_sm + b * (G * 64 * 2), &tmH, h_full, b * 64, 0, g);
        last_h = static_cast<int>(ui);
        for (int c = 0; c < p.n_clip; ++c, ++it) {
          const int s = it % kLossStages, r = it / kLossStages;
          if (!wait_bounded(&a_empty[s], (r & 1) ^ 1, abort_flag, p.status, kSiteLossAEmpty, tmo)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&a_full[s], L::kABytes);
#pragma unroll
          for (int b = 0; b < kBoxes; ++b)
            tma_load_3d(a_sm + s * L::kABytes + b * (128 * 64 * 2), &tmOp, &a_full[s], g * G + b * 64, nb * 128, c);
          last_a[s] = r;
        }
      }
      aborted = !ok;
      volatile int no_abort = 0;
      for (int s = 0; s < kLossStages; ++s)
        if (last_a[s] >= 0) wait_bounded(&a_full[s], last_a[s] & 1, &no_abort, p.status, kSiteLossAFull, tmo);
      if (last_h >= 0) wait_bounded(h_full, last_h & 1, &no_abort, p.status, kSiteLossHFull, tmo);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, G);
      uint32_t it = 0, ui = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ui) {
        if (!wait_bounded(h_full, ui & 1, abort_flag, p.status, kSiteLossHFull, tmo)) {
          ok = false;
          break;
        }
        for (int c = 0; c < p.n_clip; ++c, ++it) {
          const int s = it % kLossStages, b = it & 1;
          if (!wait_bounded(&acc_empty[b], ((it >> 1) & 1) ^ 1, abort_flag, p.status, kSiteLossAccEmpty, tmo) ||
              !wait_bounded(&a_full[s], (it / kLossStages) & 1, abort_flag, p.status, kSiteLossAFull, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kb = 0; kb < kBoxes; ++kb) {
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(a_sm + s * L::kABytes + kb * (128 * 64 * 2)));
            const uint64_t bdesc = sw128_kmajor_desc(smem_u32(h_sm + kb * (G * 64 * 2)));
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_ss_f16_cta(tbase + b * G, adesc + 2 * j, bdesc + 2 * j, idesc, (kb | j) != 0 ? 1u : 0u);
          }
          mma_commit(&acc_full[b]);
        }
        if (!ok) break;
        mma_commit(h_empty);     // the unit's MMAs are done with H_g
      }
      aborted = !ok;
      mma_commit(mma_done);      // arrives once every MMA issued above has completed
      volatile int no_abort = 0;
      wait_bounded(mma_done, 0, &no_abort, p.status, kSiteLossAccFull, tmo);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int nl = q * 32 + lane;                          // column inside the 128-column block
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
      const int g = u / p.nblocks, nb = u % p.nblocks;
      const int64_t n = static_cast<int64_t>(nb) * 128 + nl;
      float best = 0.0f;
      int bi = 0;
      for (int c = 0; c < p.n_clip; ++c, ++it) {
        const int s = it % kLossStages, b = it & 1;
        const bool got = wait_bounded(&acc_full[b], (it >> 1) & 1, abort_flag, p.status, kSiteLossAccFull, tmo);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
        for (int kb = 0; kb < kBoxes; ++kb) {
          const uint8_t* box = a_sm + s * L::kABytes + kb * (128 * 64 * 2);
#pragma unroll 1
          for (int h32 = 0; h32 < 2; ++h32) {
            uint32_t v[32];
            tmem_ld32(tbase + (static_cast<uint32_t>(q * 32) << 16) + b * G + kb * 64 + h32 * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint4 e4 = sw128_row_chunk(box, nl, h32 * 4 + cc);
              const uint32_t ew[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(ew[e] << 16), hi = __uint_as_float(ew[e] & 0xFFFF0000u);
                acc0 = fmaf(__uint_as_float(v[cc * 8 + 2 * e]), lo, acc0);
                acc1 = fmaf(__uint_as_float(v[cc * 8 + 2 * e + 1]), hi, acc1);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acc_empty[b]);
          mbar_arrive(&a_empty[s]);
        }
        const float loss = acc0 + acc1;
        if (c == 0 || loss < best) {
          best = loss;
          bi = c;
        }
        if (p.loss_out && n < p.D_out) p.loss_out[(static_cast<int64_t>(c) * p.groups + g) * p.D_out + n] = loss;
      }
      if (!ok) break;
      if (n < p.D_out) {
        p.clip_out[static_cast<int64_t>(g) * p.D_out + n] = p.clips.v[bi];
        if (p.idx_out) p.idx_out[static_cast<int64_t>(g) * p.D_out + n] = bi;
      }
    }
    aborted = !ok;
  }
  if (aborted || *abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 2 * G < 32 ? 32 : 2 * G);
}

}  // namespace

cudaError_t launch_xt(const uint16_t* X, int64_t N, int64_t D, int64_t Np, uint16_t* XT, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>((Np + 63) / 64), static_cast<unsigned>((D + 63) / 64));
  xt_kernel<<<grid, 256, 0, st>>>(X, N, D, Np, XT);
  return cudaGetLastError();
}

namespace {
// dst [n] bf16 = round-to-nearest of src [n] fp32 (the Gram matrix as the
// search GEMM's operand).
__global__ void __launch_bounds__(256) to_bf16_kernel(const float* __restrict__ src, int64_t n,
                                                      uint16_t* __restrict__ dst) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = __bfloat16_as_ushort(__float2bfloat16_rn(src[i]));
}
}  // namespace

cudaError_t launch_to_bf16(const float* src, int64_t n, uint16_t* dst, cudaStream_t st) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(src, n, dst);
  return cudaGetLastError();
}

cudaError_t launch_recip(const float* s, int64_t D, float* r, cudaStream_t st) {
  recip_kernel<<<static_cast<unsigned>((D + 255) / 256), 256, 0, st>>>(s, D, r);
  return cudaGetLastError();
}

int launch_gram(const uint16_t* XT, int64_t D_in, int64_t Np, int group, uint16_t* Hb, int* status,
                uint64_t timeout_ns, cudaStream_t st, cudaError_t* cerr, const char** what) {
  *cerr = cudaSuccess;
  CUtensorMap m;
  if (!make_bf16_map(&m, XT, static_cast<uint64_t>(Np), static_cast<uint64_t>(D_in), 0, 64, 128)) {
    *what = "tensor map for the transposed activations";
    return kECuda;
  }
  const unsigned grid = static_cast<unsigned>((D_in + 127) / 128);
  static SmemAttrOnce dev64, dev128;
  cudaError_t e;
  if (group == 64) {
    e = set_smem_once(gram_kernel<64>, kGramSmem, dev64);
    if (e == cudaSuccess) gram_kernel<64><<<grid, 192, kGramSmem, st>>>(m, D_in, Np, Hb, status, timeout_ns);
  } else {
    e = set_smem_once(gram_kernel<128>, kGramSmem, dev128);
    if (e == cudaSuccess) gram_kernel<128><<<grid, 192, kGramSmem, st>>>(m, D_in, Np, Hb, status, timeout_ns);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "gram_kernel launch";
    return kECuda;
  }
  return kOk;
}

int launch_clip_loss(const uint16_t* op, const uint16_t* Hb, int64_t D_in, int64_t D_out, int group,
                     const AlphaList& clips, int n_clip, float* clip_out, int* idx_out, float* loss_out, int num_sms,
                     int* status, uint64_t timeout_ns, cudaStream_t st, cudaError_t* cerr, const char** what) {
  *cerr = cudaSuccess;
  const int groups = static_cast<int>(D_in / group);
  CUtensorMap mOp, mH;
  if (!make_bf16_map(&mOp, op, static_cast<uint64_t>(D_in), static_cast<uint64_t>(D_out),
                     static_cast<uint64_t>(n_clip), 64, 128) ||
      !make_bf16_map(&mH, Hb, static_cast<uint64_t>(group), static_cast<uint64_t>(group),
                     static_cast<uint64_t>(groups), 64, static_cast<uint32_t>(group))) {
    *what = "tensor maps of the clipping search";
    return kECuda;
  }
  ClipParams p;
  p.D_in = D_in;
  p.D_out = D_out;
  p.n_clip = n_clip;
  p.groups = groups;
  p.nblocks = static_cast<int>((D_out + 127) / 128);
  p.units = groups * p.nblocks;
  p.clips = clips;
  p.clip_out = clip_out;
  p.idx_out = idx_out;
  p.loss_out = loss_out;
  p.status = status;
  p.timeout_ns = timeout_ns;
  const unsigned grid = static_cast<unsigned>(p.units < num_sms ? p.units : num_sms);
  static SmemAttrOnce dev64, dev128;
  cudaError_t e;
  if (group == 64) {
    e = set_smem_once(clip_loss_kernel<64>, LossLayout<64>::kSmem, dev64);
    if (e == cudaSuccess) clip_loss_kernel<64><<<grid, kLossThreads, LossLayout<64>::kSmem, st>>>(mOp, mH, p);
  } else {
    e = set_smem_once(clip_loss_kernel<128>, LossLayout<128>::kSmem, dev128);
    if (e == cudaSuccess) clip_loss_kernel<128><<<grid, kLossThreads, LossLayout<128>::kSmem, st>>>(mOp, mH, p);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "clip_loss_kernel launch";
    return kECuda;
  }
  return kOk;
}

}  // namespace awq
