// w4a16.cu -- the quantised layer applied to activations,
//     Y = X diag(1/s) Dequant(W_q),   Dequant(W_q)[k][n] = (u_kn - 2^(b-1)) delta_{k/G, n},
// straight from the packed offset-binary words of awq_quantize_pack
// (compassingai.com AWQ concept page, "inference-time equivalent": the INT4
// weights with s* kept as metadata and 1/s* folded into the input).
//
// tcgen05 GEMM (cta_group::1): D[n][t] = sum_k A[n][k] B[t][k] with
//   A  the dequantised weight tile (M = 128 output columns, 64 k per stage,
//      K-major bf16, 128-byte swizzle), produced in shared memory by the
//      producer warps: A[n][k] = bf16(q_kn * fl(delta * (1/s_k))), one
//      rounding per weight (the search's reference-form operand);
//   B  the X tile (N = Nt tokens, Nt a multiple of 16 up to 256), by TMA.
// A thread of the producer warps owns one output column: per stage it loads
// the column's eight packed words (coalesced across the columns) and turns
// each into one 16-byte chunk of its row of A.
//
// Split K: with few output tiles (small N), a cluster of KS CTAs shares one
// tile, each CTA a contiguous range of k blocks; the partial tiles fold
// through distributed shared memory in rank order (deterministic).
//
// Roles (192 threads): warp 0 TMA of X, warp 1 TMEM allocation and MMA issue
// (lane 0), warps 2-5 producers and then the epilogue (warp w owns TMEM lane
// quarter w % 4 = columns 32 (w % 4) .. + 31 of the tile).  Every mbarrier
// wait is bounded.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace awq {
namespace {

constexpr int kW4Threads = 192;
constexpr int kW4ABytes = 128 * 64 * 2;          // one A stage
constexpr int kW4MaxFoldTokens = 64;             // split K only for token tiles up to this

enum W4Site { kSiteW4XEmpty = 40, kSiteW4XFull, kSiteW4AEmpty, kSiteW4AFull, kSiteW4Acc };

struct W4Params {
  const uint32_t* packed;   // [D_in/8][D_out]
  const float* scales;      // [D_in/G][D_out]
  const float* s;           // [D_in]
  float* Y;                 // [N][D_out]
  int64_t N, D_in, D_out;
  int bits, Nt, KB, KS, n_tiles, stages;
  int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

template <int G>
__global__ void __launch_bounds__(kW4Threads, 1)
    w4a16_kernel(const __grid_constant__ CUtensorMap tmX, const W4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  const int b_bytes = p.Nt * 64 * 2;
  uint8_t* a_sm = smem;                                        // [S] x 16 KiB
  uint8_t* b_sm = a_sm + S * kW4ABytes;                        // [S] x Nt*128 B
  float* r_sm = reinterpret_cast<float*>(b_sm + S * b_bytes);  // [4 producer warps][64] 1/s of a stage's k
  float* fold = r_sm + 4 * 64;                                 // [Nt][128] (split K)
  uint64_t* bars = reinterpret_cast<uint64_t*>(fold + (p.KS > 1 ? p.Nt * 128 : 0));
  uint64_t* x_full = bars;
  uint64_t* x_empty = x_full + S;
  uint64_t* a_full = x_empty + S;
  uint64_t* a_empty = a_full + S;
  uint64_t* acc_full = a_empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  cg::cluster_group cluster = cg::this_cluster();
  const int ks = p.KS > 1 ? static_cast<int>(cluster.block_rank()) : 0;
  const int tile = blockIdx.x / p.KS;
  const int n_tile = tile % p.n_tiles, t_tile = tile / p.n_tiles;
  const int64_t n0 = static_cast<int64_t>(n_tile) * 128, t0 = static_cast<int64_t>(t_tile) * p.Nt;
  const int kb0 = static_cast<int>(static_cast<int64_t>(p.KB) * ks / p.KS);
  const int kb1 = static_cast<int>(static_cast<int64_t>(p.KB) * (ks + 1) / p.KS);
  const int tcols = p.Nt <= 32 ? 32 : (p.Nt <= 64 ? 64 : (p.Nt <= 128 ? 128 : 256));

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
      mbar_init(&a_full[s], 4);
      mbar_init(&a_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;
  bool aborted = false;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA of X
    if (lane == 0) {
      int last[8] = {-1, -1, -1, -1, -1, -1, -1, -1};
      for (int kb = kb0; kb < kb1; ++kb) {
        const int i = kb - kb0, s = i % S, r = i / S;
        if (!wait_bounded(&x_empty[s], (r & 1) ^ 1, abort_flag, p.status, kSiteW4XEmpty, tmo)) {
          aborted = true;
          break;
        }
        mbar_arrive_expect_tx(&x_full[s], static_cast<uint32_t>(b_bytes));
        tma_load_2d(b_sm + s * b_bytes, &tmX, &x_full[s], kb * 64, static_cast<int>(t0));
        last[s] = r;
      }
      volatile int no_abort = 0;
      for (int s = 0; s < S; ++s)
        if (last[s] >= 0) wait_bounded(&x_full[s], last[s] & 1, &no_abort, p.status, kSiteW4XFull, tmo);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, p.Nt);
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        const int i = kb - kb0, s = i % S, r = i / S;
        if (!wait_bounded(&a_full[s], r & 1, abort_flag, p.status, kSiteW4AFull, tmo) ||
            !wait_bounded(&x_full[s], r & 1, abort_flag, p.status, kSiteW4XFull, tmo)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t adesc = sw128_kmajor_desc(smem_u32(a_sm + s * kW4ABytes));
        const uint64_t bdesc = sw128_kmajor_desc(smem_u32(b_sm + s * b_bytes));
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_ss_f16_cta(tbase, adesc + 2 * j, bdesc + 2 * j, idesc, (i | j) != 0 ? 1u : 0u);
        mma_commit(&a_empty[s]);
        mma_commit(&x_empty[s]);
      }
      aborted = !ok;
      mma_commit(acc_full);       // arrives once every MMA issued above has completed
      volatile int no_abort = 0;
      wait_bounded(acc_full, 0, &no_abort, p.status, kSiteW4Acc, tmo);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- producers, then the epilogue
    const int q = warp & 3;
    const int n = q * 32 + lane;                  // column in the tile
    const int64_t nn = n0 + n;
    const bool valid = nn < p.D_out;
    const float off = static_cast<float>(1 << (p.bits - 1));
    bool ok = true;
    for (int kb = kb0; kb < kb1 && ok; ++kb) {
      const int i = kb - kb0, s = i % S, r = i / S;
      const bool got = wait_bounded(&a_empty[s], (r & 1) ^ 1, abort_flag, p.status, kSiteW4AEmpty, tmo);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      const int64_t k0 = static_cast<int64_t>(kb) * 64;
      // 1/s of the stage's 64 rows (zero past D_in), each warp its own copy
      float* rs = r_sm + q * 64;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t k = k0 + lane + 32 * h;
        rs[lane + 32 * h] = k < p.D_in ? __frcp_rn(__ldg(p.s + k)) : 0.0f;
      }
      __syncwarp();
      uint4* arow = reinterpret_cast<uint4*>(a_sm + s * kW4ABytes + (n >> 3) * 1024 + (n & 7) * 128);
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const int64_t k8 = k0 / 8 + w;
        uint4 chunk = make_uint4(0u, 0u, 0u, 0u);
        if (valid && k8 * 8 < p.D_in) {
          const uint32_t word = __ldg(p.packed + k8 * p.D_out + nn);
          const float delta = __ldg(p.scales + ((k8 * 8) / G) * p.D_out + nn);
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float qv = static_cast<float>((word >> (4 * e)) & 0xFu) - off;        // exact small integer
            v[e] = __fmul_rn(qv, __fmul_rn(delta, rs[w * 8 + e]));
          }
          chunk = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                             pack_bf16(v[6], v[7]));
        }
        arow[w ^ (n & 7)] = chunk;                 // 16-byte chunk w of row n, 128-byte swizzle
      }
      fence_proxy_async_smem();
      __syncwarp();                                // also: every lane is done with rs before it is rewritten
      if (lane == 0) mbar_arrive(&a_full[s]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) {
      const bool got = wait_bounded(acc_full, 0, abort_flag, p.status, kSiteW4Acc, tmo);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after();
      const uint32_t lane_addr = tbase + (static_cast<uint32_t>(q * 32) << 16);
      for (int c = 0; c < p.Nt; c += 16) {
        uint32_t v[16];
        tmem_ld16(lane_addr + c, v);
        tmem_wait_ld();
        if (p.KS > 1) {
#pragma unroll
          for (int e = 0; e < 16; ++e) fold[(c + e) * 128 + n] = __uint_as_float(v[e]);
        } else if (valid) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (t0 + c + e < p.N) p.Y[(t0 + c + e) * p.D_out + nn] = __uint_as_float(v[e]);
        }
      }
    }
    aborted = !ok;
  }
  if (p.KS > 1) {
    // The K split folds in rank order: CTA ks writes tokens t with t % KS == ks.
    cluster.sync();
    if (warp >= 2 && !aborted) {
      const int n = (warp & 3) * 32 + lane;
      const int64_t nn = n0 + n;
      if (nn < p.D_out) {
        for (int t = ks; t < p.Nt; t += p.KS) {
          if (t0 + t >= p.N) break;
          float acc = 0.0f;
          for (int rk = 0; rk < p.KS; ++rk) acc += cluster.map_shared_rank(fold, rk)[t * 128 + n];
          p.Y[(t0 + t) * p.D_out + nn] = acc;
        }
      }
    }
    cluster.sync();
  }
  if (aborted || *abort_flag) {
    const uint64_t tstart = globaltimer_ns();
    while (globaltimer_ns() - tstart < 200000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, tcols);
}

}  // namespace

int launch_w4a16(const void* X, const float* s, const uint32_t* packed, const float* scales, int64_t N, int64_t D_in,
                 int64_t D_out, int bits, int group, float* Y, int num_sms, int* status, uint64_t timeout_ns,
                 cudaStream_t st, cudaError_t* cerr, const char** what) {
  *cerr = cudaSuccess;
  const int Nt = N >= 256 ? 256 : static_cast<int>((N + 15) / 16 * 16);
  const int n_tiles = static_cast<int>((D_out + 127) / 128);
  const int t_tiles = static_cast<int>((N + Nt - 1) / Nt);
  const int KB = static_cast<int>((D_in + 63) / 64);
  const long long tiles = static_cast<long long>(n_tiles) * t_tiles;
  int KS = 1;
  if (Nt <= kW4MaxFoldTokens && tiles < num_sms) {
    long long k = num_sms / tiles;
    if (k > 8) k = 8;
    if (k > KB) k = KB;
    KS = static_cast<int>(k < 1 ? 1 : k);
  }
  const int stages = Nt > 128 ? 3 : 4;
  CUtensorMap mX;
  if (!make_bf16_map(&mX, X, static_cast<uint64_t>(D_in), static_cast<uint64_t>(N), 0, 64,
                     static_cast<uint32_t>(Nt))) {
    *what = "tensor map for X";
    return kECuda;
  }
  W4Params p;
  p.packed = packed;
  p.scales = scales;
  p.s = s;
  p.Y = Y;
  p.N = N;
  p.D_in = D_in;
  p.D_out = D_out;
  p.bits = bits;
  p.Nt = Nt;
  p.KB = KB;
  p.KS = KS;
  p.n_tiles = n_tiles;
  p.stages = stages;
  p.status = status;
  p.timeout_ns = timeout_ns;
  const int smem = 1024 + stages * (kW4ABytes + Nt * 128) + 4 * 64 * 4 + (KS > 1 ? Nt * 128 * 4 : 0) + 256;
  void (*kern)(CUtensorMap, W4Params) = nullptr;
  switch (group) {
    case 32: kern = w4a16_kernel<32>; break;
    case 64: kern = w4a16_kernel<64>; break;
    case 128: kern = w4a16_kernel<128>; break;
    default:
      *what = "group";
      return kEUnsupported;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * KS));
    cfg.blockDim = dim3(kW4Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = KS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mX, p);
  }
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "w4a16_kernel launch";
    return kECuda;
  }
  return kOk;
}

}  // namespace awq
