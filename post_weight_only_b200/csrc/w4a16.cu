// w4a16.cu -- the quantised layer applied to activations,
//     Y = X diag(1/s) Dequant(W_q),   Dequant(W_q)[k][n] = (u_kn - 2^(b-1)) delta_{k/G, n},
// straight from the packed offset-binary words of awq_quantize_pack
// (compassingai.com AWQ concept page, "inference-time equivalent": the INT4
// weights with s* kept as metadata and 1/s* folded into the input; AWQ paper,
// TinyChat section, "on-the-fly weight dequantization": the integers are
// turned into 16-bit floats inside the GEMM's main loop).
//
// Two launches:
//   1. scale_x: X' = bf16(X / s) into scratch, rows padded with zeros to a
//      multiple of 64 columns (so that a k block never crosses a row), each
//      run of 8 columns stored in the order 0,4,1,5,2,6,3,7.  A packed word holds rows 8j..8j+7 as
//      nibbles 0..7; one mask-and-OR of (word >> 4i) with 0x000F000F |
//      0x43004300 gives the bf16 pair {128 + u_{8j+i}, 128 + u_{8j+i+4}}
//      (exact), so with that order of X' the pairs go straight into the
//      K-major A tile (the same reason the paper's GPU packing interleaves
//      the weights; the permutation sits on the activation side here so
//      that the pack format keeps its natural order).
//   2. the GEMM (tcgen05, cta_group::1): D[n][t] = sum_k A[n][k] X'[t][k]
//      with A the dequantised weight tile, 128 output columns x 64 k per
//      k block, bf16((u - 2^(b-1)) * bf16(delta)): the subtraction is exact
//      and the product is rounded once.
//
// A stage holds KPS consecutive k blocks of one unit: the X' planes
// [KPS][Nt][64] (one 3-D box, 128-byte swizzle), the packed words
// [8 KPS][128] (one TMA box) and their scale rows (one box).  On B200 a
// thread that issues TMA loads and waits for them streams at a rate set by
// the number of loads it keeps going rather than their size, so the small
// token tiles (memory-bound) take KPS = 4 (a 16 KiB box of packed words) and
// two issuing warps that fill alternate stages; large token tiles take
// KPS = 1 (the X' box alone is 32 KiB) and one issuing warp.
//
// Roles (480 threads):
//   warps 0-1   TMA issue (lane 0).
//   warp 2      TMEM allocation and MMA issue (lane 0) into one of two
//               accumulators, so that a unit's epilogue overlaps the next
//               unit's main loop.
//   warps 3-10  dequantisers: thread (n, h) owns column n of the tile and
//               half h of each k block; it reads its 4 words per k block from
//               the stage (conflict-free, the words of a k8 row are
//               contiguous over n) and writes chunks 4h..4h+3 of row n of
//               the A tile.
//   warps 11-14 epilogue: TMEM lanes 32 (w % 4) .. + 31 -> Y.
// Decode (N <= 8 tokens) takes a GEMV instead: there the work is a stream of
// packed words with a few multiply-adds per weight, bound by HBM, and a
// tcgen05 tile of 16+ tokens would sit mostly idle.  One or two tokens run on
// the CUDA cores (w4a16_gemv_kernel); 3-8 tokens hand the products to
// warp-level mma.sync tiles of 8 token slots (w4a16_gemv_mma_kernel), since
// from three tokens on the paired FMAs per word and token make the FMA pipe
// the bound.
//
// Work: a unit is a 128-column x Nt-token output tile of KBS = ceil(KB /
// KPS) stage steps.  Large N: units are dealt out to a persistent grid,
// whole.  N <= 64: stream-K -- the units x KBS steps are cut into equal
// contiguous shares, one per CTA, so that every SM streams the same number
// of packed bytes.  A unit split between CTAs is summed from partial tiles
// in the workspace by the CTA that finishes it last (an atomic count per
// unit), always in CTA order: the result does not depend on timing.  Every
// mbarrier wait is bounded.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace awq {
namespace {

constexpr int kW4Threads = 480;
constexpr int kW4TmaWarps = 2;
constexpr int kW4MmaWarp = 2;
constexpr int kW4DqWarp0 = 3;
constexpr int kW4DqWarps = 8;
constexpr int kW4EpiWarp0 = kW4DqWarp0 + kW4DqWarps;   // 11
constexpr int kW4ABytes = 128 * 64 * 2;          // one dequantised A tile
constexpr int kW4PkBytes = 8 * 128 * 4;          // the packed words of one k block
constexpr int kW4MaxStreamTokens = 64;           // stream-K for token tiles up to this
constexpr int kW4MaxStages = 16;
constexpr int kW4MaxGrid = 512;                  // bounds the partial-tile workspace
constexpr uint32_t kW4SleepNs = 20000;           // suspend hint of the waits

enum W4Site {
  kSiteW4WEmpty = 40, kSiteW4WFull, kSiteW4AEmpty, kSiteW4AFull, kSiteW4AccEmpty, kSiteW4AccFull, kSiteW4Done
};

struct W4Params {
  float* Y;                 // [N][D_out]
  float* partial;           // stream-K: [grid][2][N][128] partial tiles
  int* count;               // stream-K: [units] contributions received (zeroed by scale_x)
  int64_t N, D_out;
  int off;                  // 2^(bits-1)
  uint32_t magic;           // 0x43004300, passed at run time so that it lives in a register and each
                            // mask-and-OR is one three-input logic op (an op takes one immediate)
  int Nt, KB, kps, KBS, n_tiles, units;
  int stream;               // 1: stream-K over units x KBS steps, `chunk` steps per CTA
  int issuers;              // TMA warps that fill alternate stages (1 or 2)
  int64_t chunk, total;
  int stages, a_stages, stage_bytes, scale_rows, tcols;
  int* status;
  unsigned long long timeout_ns;
};

// The segments of work of CTA c, in order: (unit, first step, end step).
struct SegCursor {
  int64_t f, f1;
};
__device__ __forceinline__ SegCursor seg_begin(const W4Params& p, int c) {
  if (p.stream) {
    const int64_t f0 = c * p.chunk;
    return {f0, f0 + p.chunk < p.total ? f0 + p.chunk : p.total};
  }
  return {c, p.units};
}
__device__ __forceinline__ bool seg_next(SegCursor& cur, const W4Params& p, int& u, int& ka, int& kb) {
  if (cur.f >= cur.f1) return false;
  if (p.stream) {
    u = static_cast<int>(cur.f / p.KBS);
    ka = static_cast<int>(cur.f - static_cast<int64_t>(u) * p.KBS);
    const int64_t left = cur.f1 - cur.f;
    kb = left < p.KBS - ka ? ka + static_cast<int>(left) : p.KBS;
    cur.f += kb - ka;
  } else {
    u = static_cast<int>(cur.f);
    ka = 0;
    kb = p.KBS;
    cur.f += gridDim.x;
  }
  return true;
}

// ------------------------------------------------------------ X' = X / s
__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// One thread per run of 8 columns of X' [N][P8 * 8]; runs j >= D8 are the zero pad.
__global__ void __launch_bounds__(256) scale_x_kernel(const uint4* __restrict__ X, const float4* __restrict__ s,
                                                      int64_t total, int64_t D8, int64_t P8, uint4* __restrict__ Xs,
                                                      int* count, int n_count) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_count; i += gridDim.x * blockDim.x) count[i] = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / P8, j = i - t * P8;
    if (j >= D8) {
      Xs[i] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4 xv = X[t * D8 + j];
    const float4 s0 = __ldg(s + 2 * j), s1 = __ldg(s + 2 * j + 1);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t h = (e & 1) ? (xw[e >> 1] >> 16) : (xw[e >> 1] & 0xFFFFu);
      v[e] = __fdiv_rn(bf16_bits_to_float(h), sv[e]);
    }
    Xs[i] = make_uint4(pack_bf16(v[0], v[4]), pack_bf16(v[1], v[5]), pack_bf16(v[2], v[6]), pack_bf16(v[3], v[7]));
  }
}

// zb[g][n] = 128 + zeros[g][n] as fp32: the per-(group, column) bias of the
// asymmetric dequantiser, read by TMA beside the deltas.
__global__ void __launch_bounds__(256) zero_bias_kernel(const uint8_t* __restrict__ zeros, int64_t n,
                                                        float* __restrict__ zb) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    zb[i] = 128.0f + static_cast<float>(zeros[i]);
}

// A kernel argument copied into a register the compiler cannot see through.
// Used for the dequantisers' magic constants: read straight from the
// parameter bank, a constant is a second non-register operand of the
// mask-and-OR, which then takes two logic ops instead of one.
__device__ __forceinline__ uint32_t in_register(uint32_t v) {
  uint32_t r;
  asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}

// ------------------------------------------------------------ the GEMM
__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t u) { return *reinterpret_cast<__nv_bfloat162*>(&u); }
__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// kZp: asymmetric codes; each stage also holds the rows of 128 + z (fp32,
// made by zero_bias_kernel) beside the deltas, and the dequantiser subtracts
// that per-(group, column) value instead of 128 + off.
template <int G, bool kZp>
__global__ void __launch_bounds__(kW4Threads, 1)
    w4a16_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                 const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
                 const W4Params p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // 1024-byte aligned base (128-byte swizzle atoms), derived by pointer
  // arithmetic on the shared array so that accesses stay in the shared space.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int S = p.stages, AS = p.a_stages, KPS = p.kps;
  const int xs_bytes = KPS * p.Nt * 128;          // the X' planes of a stage
  const int pk_bytes = KPS * kW4PkBytes;
  uint8_t* a_sm = smem + S * p.stage_bytes;       // [AS] x 16 KiB
  uint64_t* bars = reinterpret_cast<uint64_t*>(a_sm + AS * kW4ABytes);
  uint64_t* w_full = bars;
  uint64_t* w_empty = w_full + S;
  uint64_t* a_full = w_empty + S;
  uint64_t* a_empty = a_full + AS;
  uint64_t* acc_full = a_empty + AS;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* epi_state = abort_flag + 1;      // [0] an epilogue warp failed, [1] this CTA folds the unit

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], kW4DqWarps + 1);      // the dequantiser warps + the MMA commit
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(&a_full[s], kW4DqWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    epi_state[0] = 0;
    epi_state[1] = 0;
    fence_mbar_init();
  }
  if (warp == kW4MmaWarp) {
    tmem_alloc(tmem_slot, 2 * p.tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;
  bool aborted = false;

  if (warp < kW4TmaWarps) {
    // ---------------------------------------------------------- TMA: warp w fills the stages of step index = w mod issuers
    if (lane == 0 && warp < p.issuers) {
      const uint32_t tx = static_cast<uint32_t>(xs_bytes + pk_bytes + (kZp ? 2 : 1) * p.scale_rows * 128 * 4);
      const int step = p.issuers;
      int s = warp;                 // this warp's next stage slot (S is a multiple of `step`)
      uint32_t ph = 0;
      uint32_t i = 0, fills = 0;    // step counter of the CTA, fills issued by this warp
      bool ok = true;
      SegCursor cur = seg_begin(p, c);
      int u, ka, kb1;
      while (ok && seg_next(cur, p, u, ka, kb1)) {
        const int n0 = (u % p.n_tiles) * 128, t0 = (u / p.n_tiles) * p.Nt;
        for (int st = ka; st < kb1; ++st, ++i) {
          if (static_cast<int>(i % static_cast<uint32_t>(step)) != warp) continue;
          if (!wait_bounded_sleep(&w_empty[s], ph ^ 1, abort_flag, p.status, kSiteW4WEmpty, tmo, kW4SleepNs)) {
            ok = false;
            break;
          }
          uint8_t* sp = smem + s * p.stage_bytes;
          const int kb = st * KPS;
          mbar_arrive_expect_tx(&w_full[s], tx);
          tma_load_3d(sp, &tmX, &w_full[s], 0, t0, kb);
          tma_load_2d(sp + xs_bytes, &tmP, &w_full[s], n0, kb * 8);
          tma_load_2d(sp + xs_bytes + pk_bytes, &tmS, &w_full[s], n0, (kb * 64) / G);
          if (kZp) tma_load_2d(sp + xs_bytes + pk_bytes + p.scale_rows * 512, &tmZ, &w_full[s], n0, (kb * 64) / G);
          ++fills;
          s += step;
          if (s >= S) {
            s -= S;
            ph ^= 1;
          }
        }
      }
      aborted = !ok;
      // Every fill issued has landed before the CTA may exit (matters only
      // when another role gave up early): fill j of this warp used slot
      // (warp + step j) mod S in phase ((warp + step j) / S) & 1.
      volatile int no_abort = 0;
      const uint32_t per_round = static_cast<uint32_t>(S / step);
      for (uint32_t j = fills > per_round ? fills - per_round : 0; j < fills; ++j) {
        const uint32_t q = static_cast<uint32_t>(warp) + static_cast<uint32_t>(step) * j;
        wait_bounded(&w_full[q % S], (q / S) & 1, &no_abort, p.status, kSiteW4WFull, tmo);
      }
    }
  } else if (warp == kW4MmaWarp) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      int s = 0, sa = 0, b = 0;
      uint32_t ph = 0, pha = 0, phb = 0;
      bool ok = true;
      SegCursor cur = seg_begin(p, c);
      int u, ka, kb1;
      const uint32_t idesc = idesc_bf16_f32(128, p.Nt);
      while (ok && seg_next(cur, p, u, ka, kb1)) {
        if (!wait_bounded_sleep(&acc_empty[b], phb ^ 1, abort_flag, p.status, kSiteW4AccEmpty, tmo, kW4SleepNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tbase + static_cast<uint32_t>(b * p.tcols);
        for (int st = ka; st < kb1 && ok; ++st) {
          if (!wait_bounded_sleep(&w_full[s], ph, abort_flag, p.status, kSiteW4WFull, tmo, kW4SleepNs)) {
            ok = false;
            break;
          }
          for (int j = 0; j < KPS; ++j) {
            if (!wait_bounded_sleep(&a_full[sa], pha, abort_flag, p.status, kSiteW4AFull, tmo, kW4SleepNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(a_sm + sa * kW4ABytes));
            const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + s * p.stage_bytes + j * p.Nt * 128));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_ss_f16_cta(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (st > ka || j > 0 || k > 0) ? 1u : 0u);
            mma_commit(&a_empty[sa]);
            if (++sa == AS) {
              sa = 0;
              pha ^= 1;
            }
          }
          if (!ok) break;
          mma_commit(&w_empty[s]);     // the MMAs read X' from the stage
          if (++s == S) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[b]);
        b ^= 1;
        if (b == 0) phb ^= 1;
      }
      aborted = !ok;
      mma_commit(done);            // arrives once every MMA issued above has completed
      volatile int no_abort = 0;
      wait_bounded(done, 0, &no_abort, p.status, kSiteW4Done, tmo);
    }
    __syncwarp();
  } else if (warp < kW4EpiWarp0) {
    // ---------------------------------------------------------- dequantisers
    const int n = (warp & 3) * 32 + lane;
    const int h = (warp - kW4DqWarp0) >> 2;       // half of each k block: chunks 4h..4h+3
    const uint32_t bias_bits = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(128.0f + p.off)));
    const uint32_t magic = in_register(p.magic);
    const __nv_bfloat162 bias = as_bf162(bias_bits | (bias_bits << 16));     // 128 + off, exact
    const int swz = n & 7;
    int s = 0, sa = 0;
    uint32_t ph = 0, pha = 0;
    bool ok = true;
    SegCursor cur = seg_begin(p, c);
    int u, ka, kb1;
    while (ok && seg_next(cur, p, u, ka, kb1)) {
      for (int st = ka; st < kb1 && ok; ++st) {
        const bool got = wait_bounded_sleep(&w_full[s], ph, abort_flag, p.status, kSiteW4WFull, tmo, kW4SleepNs);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const uint8_t* sp = smem + s * p.stage_bytes;
        const int kb0 = st * KPS;
        const int row0 = (kb0 * 64) / G;           // first scale row of the stage
        for (int j = 0; j < KPS; ++j) {
          const bool got_a = wait_bounded_sleep(&a_empty[sa], pha ^ 1, abort_flag, p.status, kSiteW4AEmpty, tmo,
                                                kW4SleepNs);
          if (!__all_sync(0xffffffffu, got_a)) {
            ok = false;
            break;
          }
          const uint32_t* pk = reinterpret_cast<const uint32_t*>(sp + xs_bytes) + (8 * j + 4 * h) * 128 + n;
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w[i] = pk[i * 128];
          const int srow = ((kb0 + j) * 64 + 32 * h) / G - row0;
          const float* sc = reinterpret_cast<const float*>(sp + xs_bytes + pk_bytes) + srow * 128 + n;
          const __nv_bfloat162 d2 = __float2bfloat162_rn(sc[0]);
          __nv_bfloat162 zbias = bias;
          if (kZp) zbias = __float2bfloat162_rn(sc[p.scale_rows * 128]);   // 128 + z, exact in bf16
          uint32_t o[16];                           // chunks 4h..4h+3 of row n: 16 bf16 pairs
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t pair = ((w[i] >> (4 * q)) & 0x000F000Fu) | magic;   // {128 + u_q, 128 + u_{q+4}}
              o[4 * i + q] = as_u32(__hmul2(__hsub2(as_bf162(pair), zbias), d2));
            }
          uint4* arow = reinterpret_cast<uint4*>(a_sm + sa * kW4ABytes + (n >> 3) * 1024 + (n & 7) * 128);
#pragma unroll
          for (int i = 0; i < 4; ++i)   // chunk 4h+i of row n, 128-byte swizzle
            arow[(4 * h + i) ^ swz] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[sa]);
          if (++sa == AS) {
            sa = 0;
            pha ^= 1;
          }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&w_empty[s]);
        if (++s == S) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    aborted = !ok;
  } else {
    // ---------------------------------------------------------- epilogue
    // All four warps walk the same segments and meet at the same named
    // barriers; a warp that failed keeps walking (doing no work) so that the
    // barrier counts always match.
    const int q = warp & 3;
    const int n = q * 32 + lane;
    const uint32_t lane_q = static_cast<uint32_t>(q * 32) << 16;
    int b = 0;
    uint32_t phb = 0;
    bool ok = true;
    bool first_seg = true;
    SegCursor cur = seg_begin(p, c);
    int u, ka, kb1;
    while (seg_next(cur, p, u, ka, kb1)) {
      const bool whole = ka == 0 && kb1 == p.KBS;
      const int64_t nn = static_cast<int64_t>(u % p.n_tiles) * 128 + n;
      const int64_t t0 = static_cast<int64_t>(u / p.n_tiles) * p.Nt;
      const int slot = first_seg ? 0 : 1;
      float* part = p.partial + ((static_cast<int64_t>(c) * 2 + slot) * p.N) * 128 + n;
      const bool got = ok && wait_bounded_sleep(&acc_full[b], phb, abort_flag, p.status, kSiteW4AccFull, tmo,
                                                 kW4SleepNs);
      ok = __all_sync(0xffffffffu, got);
      if (ok) {
        tc_fence_after();
        const uint32_t lane_addr = tbase + static_cast<uint32_t>(b * p.tcols) + lane_q;
        for (int cc = 0; cc < p.Nt; cc += 16) {
          uint32_t v[16];
          tmem_ld16(lane_addr + cc, v);
          tmem_wait_ld();
          if (whole) {
            if (nn < p.D_out) {
#pragma unroll
              for (int e = 0; e < 16; ++e)
                if (t0 + cc + e < p.N) p.Y[(t0 + cc + e) * p.D_out + nn] = __uint_as_float(v[e]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (cc + e < p.N) part[(cc + e) * 128] = __uint_as_float(v[e]);     // stream-K: one token tile
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[b]);
      }
      b ^= 1;
      if (b == 0) phb ^= 1;
      if (!whole) {
        // Publish the partial tile; the last of the unit's contributors sums
        // them all in CTA order.
        if (!ok && lane == 0) epi_state[0] = 1;
        __threadfence();
        named_barrier(1, 128);
        if (warp == kW4EpiWarp0 && lane == 0) {
          int fold = 0;
          if (epi_state[0] == 0) {
            const int64_t first = static_cast<int64_t>(u) * p.KBS / p.chunk;
            const int64_t last = (static_cast<int64_t>(u + 1) * p.KBS - 1) / p.chunk;
            const int old = atomicAdd(&p.count[u], 1);
            fold = old == static_cast<int>(last - first);
            if (fold) __threadfence();
          }
          epi_state[1] = fold;
        }
        named_barrier(1, 128);
        if (epi_state[1] && nn < p.D_out) {
          const int64_t first = static_cast<int64_t>(u) * p.KBS / p.chunk;
          const int64_t last = (static_cast<int64_t>(u + 1) * p.KBS - 1) / p.chunk;
          // eight token rows at a time, so that eight loads per contributor are in flight
          for (int t0r = 0; t0r < p.N; t0r += 8) {
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
            for (int64_t cp = first; cp <= last; ++cp) {
              // CTA cp holds unit u in slot 0 unless u is not its first unit
              const int sl = (cp == first && (cp * p.chunk) / p.KBS != u) ? 1 : 0;
              const float* src = p.partial + ((cp * 2 + sl) * p.N + t0r) * 128 + n;
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (t0r + e < p.N) acc[e] += __ldcg(src + e * 128);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (t0r + e < p.N) p.Y[(t0r + e) * p.D_out + nn] = acc[e];
          }
        }
      }
      first_seg = false;
    }
    aborted = !ok;
  }
  if (aborted || *abort_flag) {
    const uint64_t tstart = globaltimer_ns();
    while (globaltimer_ns() - tstart < 200000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kW4MmaWarp) tmem_dealloc(tbase, 2 * p.tcols);
}

// ------------------------------------------------------------ decode: the GEMV
// Y[t][n] = sum_g delta_{g,n} (sum_{k in g} x'_tk u_kn - z_{g,n} sum_{k in g} x'_tk)
// on CUDA cores for one or two tokens (and for three or four on rows longer
// than the mma.sync GEMV below stages), fp32 throughout: x' = x / s rounded once
// (IEEE division), the integer weights exact, delta applied once per group;
// z is 2^(b-1) for the offset-binary codes, the group's zero point for
// asymmetric ones.
//
// Dequantisation with one logic op per weight and no conversion: a float
// whose bit pattern p is below 2^24 (exponent field 0 or 1) has the value
// p 2^-149 -- the subnormals and the smallest normal binade form one linear
// scale.  So for nibble i <= 5 of a 32-bit word (bits 4i .. 4i+3 <= 23),
// (w & (0xF << 4i)) read as a float is exactly 16^i u 2^-149; nibbles 6 and 7
// are the same after w >> 8 (bits 16..23: 16^4 u, 16^5 u).  The power of two
// of each nibble position is folded into the activation side: x~_k =
// x'_k 16^-e(k) 2^64 with e = 0, 1, 2, 3, 4, 5, 4, 5 for k mod 8 = 0..7 (an
// exact scaling), so every product x~ (w & mask) is x' u 2^-85 exactly before
// the one rounding of its FMA.  The offset comes out once per group: the sum
// of x' over the group's rows is staged with x~, and the group's flush adds
// delta (2^85 acc - z sum x').  Per word: one shift, eight logic ops and four
// paired FMAs per token.
//
// Work: the (column tile, 4-row batch) pairs, tile-major, are cut into
// equal contiguous shares, one per CTA of a grid that fills every SM
// (stream-K), and each CTA's share into eight, one per warp; a share may
// end in one tile and go on in the next.  Lane l of a warp owns columns
// 4l..4l+3 of the tile.  Each thread streams its own 16 bytes of each packed
// row through a ring of gv_slots batches in shared memory (cp.async, waited
// on with cp.async.wait_group: nothing to spin on), so the bytes in flight
// do not cost registers.  A warp stages x~ of its rows 32 at a time, in
// chunks aligned to the tile's 8-batch boundaries (one row per lane), and
// with it the sum of x' over each group's rows of the chunk (a fixed
// butterfly over the lanes); the group size is a template argument, so
// group boundaries cost a mask test.
// The warps' sums of a tile are added in warp order, each CTA writes its
// sums of the (at most two) tiles it worked on to the workspace, and
// gemv_reduce_kernel adds, per tile, the sums of the CTAs that share it in
// CTA order: the result does not depend on timing.  A grid of whole tiles
// (as many CTAs as tiles) stores Y itself.  The kernel also clears the
// status word (it has nothing to wait on).
constexpr int kGvThreads = 256;
constexpr int kGvCols = 128;
constexpr int kGvXRows = 32;                     // k8 rows of x~ a warp stages at a time (8 batches)
constexpr int kGvMaxTokens = 4;
constexpr int kGvMaxCtas = 1024;                 // bounds the workspace of CTA sums

// k8 rows per batch (one ring slot): 8 when a group holds 8 or more and the
// registers allow, so that the per-batch bookkeeping is spread over more
// words; else 4.
template <int NT, int G>
constexpr int gv_batch() { return G >= 64 && NT <= 2 ? 8 : 4; }
template <int NT, int G>
constexpr int gv_slot_bytes() { return gv_batch<NT, G>() * kGvCols * 4; }

// Ring slots per warp (two CTAs of 8 warps fit an SM).
template <int NT, int G>
constexpr int gv_slots() {
  return gv_batch<NT, G>() == 8 ? (NT == 1 ? 3 : 2) : (NT == 1 ? 6 : NT == 2 ? 5 : NT == 3 ? 4 : 3);
}

template <int NT, int G>
constexpr size_t gv_smem_bytes() {
  return static_cast<size_t>(8) * gv_slots<NT, G>() * gv_slot_bytes<NT, G>()   // ring (later the warps' sums of the next tile)
         + static_cast<size_t>(8) * NT * kGvXRows * 8 * 4        // x~
         + static_cast<size_t>(8) * NT * 8 * 4                   // sums of x' per group of the chunk
         + static_cast<size_t>(8) * NT * 32 * 16;                // the warps' sums of the CTA's first tile
}

__device__ __forceinline__ float nibf(uint32_t w, uint32_t mask) { return __uint_as_float(w & mask); }

// kZp: asymmetric codes u = q + z with a zero point per (group, column)
// (zeros [D_in/G][D_out] uint8) in place of 2^(b-1).  part: [gridDim.x][2]
// [NT][128] fp32 CTA sums (slot 0: the CTA's first tile, 1: the next), or
// Y itself when `direct` (one CTA per tile).
template <int NT, int G, bool kZp>
__global__ void __launch_bounds__(kGvThreads, 2) w4a16_gemv_kernel(
    const uint4* __restrict__ X, const float4* __restrict__ s, const uint32_t* __restrict__ packed,
    const float4* __restrict__ scales, const uint8_t* __restrict__ zeros, int64_t D_in, int64_t D_out, int off,
    float* __restrict__ part, float* __restrict__ Y, int y16, int direct, int S, int* __restrict__ status) {
  constexpr int U = gv_batch<NT, G>(), P = gv_slots<NT, G>(), XR = kGvXRows, CB = XR / U;
  constexpr int kSlotBytes = gv_slot_bytes<NT, G>();
  constexpr int GB = G / (8 * U);                  // batches per group: 1, 2, 4 or 8
  constexpr int GR = G / 8;                        // k8 rows per group: 4 .. 32
  static_assert(GB >= 1 && CB % GB == 0, "whole groups per chunk");
  extern __shared__ __align__(16) uint8_t gv_sm[];
  uint8_t* ring = gv_sm;
  float* xt_all = reinterpret_cast<float*>(gv_sm + 8 * P * kSlotBytes);
  float* xg_all = xt_all + 8 * NT * XR * 8;
  float4* first = reinterpret_cast<float4*>(xg_all + 8 * NT * 8);   // [8 warps][NT][32 quads]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (status && blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
  const int64_t rows8 = D_in / 8;
  const int64_t D4 = D_out / 4;
  const int NB = static_cast<int>(rows8 / U);      // batches per tile (rows8 is a multiple of G / 8 >= U)
  const int64_t tiles = (D_out + kGvCols - 1) / kGvCols;
  const int64_t W = tiles * NB;
  const int64_t C = gridDim.x, i = blockIdx.x;
  int64_t cs, ce;                                  // this CTA's share
  if (S > 0) {                                     // split S of a tile: cluster rank y of tile i / S
    const int64_t tau = i / S, y = i % S;
    cs = tau * NB + NB * y / S;
    ce = tau * NB + NB * (y + 1) / S;
  } else {
    cs = W * i / C;
    ce = W * (i + 1) / C;
  }
  const int64_t t0 = cs / NB;                      // its first tile
  const int64_t ws = cs + (ce - cs) * warp / 8, we = cs + (ce - cs) * (warp + 1) / 8;   // this warp's
  const int nw = static_cast<int>(we - ws);
  uint8_t* wring = ring + warp * P * kSlotBytes + lane * 16;
  float* xt = xt_all + warp * NT * XR * 8;
  float* xg = xg_all + warp * NT * 8;
  const float fo = static_cast<float>(off);
  const int64_t rstep = U * D_out;                 // words from one batch to the next

  // the ring: this thread's 16 bytes of each row of batch n of the warp's
  // share go to slot n % P
  int n_iss = 0, islot = 0;
  int iss_b = static_cast<int>(ws % NB);           // tile batch of the next copy
  int64_t iss_q4 = (ws / NB) * (kGvCols / 4) + lane;
  bool iss_ok = iss_q4 < D4;
  const uint32_t* isrc = packed + iss_b * rstep + (iss_ok ? 4 * iss_q4 : 0);
  auto issue = [&]() {
    if (n_iss < nw) {
      uint8_t* dst = wring + islot * kSlotBytes;
      const uint32_t bytes = iss_ok ? 16u : 0u;    // columns past D_out: zero fill from a valid address
#pragma unroll
      for (int u = 0; u < U; ++u) cp_async16(dst + u * (kGvCols * 4), isrc + u * D_out, bytes);
      ++n_iss;
      if (++islot == P) islot = 0;
      isrc += rstep;
      if (++iss_b == NB) {                         // on to the next tile
        iss_b = 0;
        iss_q4 += kGvCols / 4;
        iss_ok = iss_q4 < D4;
        isrc = packed + (iss_ok ? 4 * iss_q4 : 0);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int q = 0; q < P - 1; ++q) issue();
  int rslot = 0;                                   // slot of the next batch to use

#pragma unroll
  for (int t = 0; t < NT; ++t) first[(warp * NT + t) * 32 + lane] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  float tt[NT][4];                                 // the current segment's sums (a warp meets a tile once)
  float2 acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tt[t][c] = 0.0f;
      acc[t][c] = make_float2(0.0f, 0.0f);
    }
  bool next_tile = false;                          // tt holds sums of the CTA's second tile
  float dv[4] = {0.0f, 0.0f, 0.0f, 0.0f};          // the current group's deltas and zero points
  float zv[4] = {fo, fo, fo, fo};

  int64_t pos = ws;
  while (pos < we) {                               // one segment: batches [b0, b1) of tile tau
    const int64_t tau = pos / NB;
    const int b0 = static_cast<int>(pos - tau * NB);
    const int b1 = static_cast<int>(we - tau * NB < NB ? we - tau * NB : NB);
    const int64_t q4 = tau * (kGvCols / 4) + lane;
    const bool valid = q4 < D4;
    for (int ch = b0 / CB; ch * CB < b1; ++ch) {   // chunks of 8 batches aligned to the tile
      // stage x~ of the chunk's rows that lie in the segment: lane = row
      __syncwarp();                                // the previous chunk is no longer read
      {
        const int r = ch * XR + lane;              // k8 row
        const bool in = r >= b0 * U && r < b1 * U;
        float4 s0 = make_float4(1.0f, 1.0f, 1.0f, 1.0f), s1 = s0;
        if (in) {
          s0 = __ldg(s + 2 * r);
          s1 = __ldg(s + 2 * r + 1);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float xsum = 0.0f;
          if (in) {
            const uint4 xv = X[t * rows8 + r];
            const float v0 = __fdiv_rn(bf16_bits_to_float(xv.x & 0xFFFFu), s0.x);
            const float v1 = __fdiv_rn(bf16_bits_to_float(xv.x >> 16), s0.y);
            const float v2 = __fdiv_rn(bf16_bits_to_float(xv.y & 0xFFFFu), s0.z);
            const float v3 = __fdiv_rn(bf16_bits_to_float(xv.y >> 16), s0.w);
            const float v4 = __fdiv_rn(bf16_bits_to_float(xv.z & 0xFFFFu), s1.x);
            const float v5 = __fdiv_rn(bf16_bits_to_float(xv.z >> 16), s1.y);
            const float v6 = __fdiv_rn(bf16_bits_to_float(xv.w & 0xFFFFu), s1.z);
            const float v7 = __fdiv_rn(bf16_bits_to_float(xv.w >> 16), s1.w);
            // x' 16^-e 2^64: e = 0, 1, 2, 3, 4, 5, 4, 5 (exact powers of two)
            float4* dst = reinterpret_cast<float4*>(xt + (t * XR + lane) * 8);
            dst[0] = make_float4(__fmul_rn(v0, 0x1p64f), __fmul_rn(v1, 0x1p60f), __fmul_rn(v2, 0x1p56f),
                                 __fmul_rn(v3, 0x1p52f));
            dst[1] = make_float4(__fmul_rn(v4, 0x1p48f), __fmul_rn(v5, 0x1p44f), __fmul_rn(v6, 0x1p48f),
                                 __fmul_rn(v7, 0x1p44f));
            xsum = ((v0 + v1) + (v2 + v3)) + ((v4 + v5) + (v6 + v7));
          }
          // the sum of x' over each group's rows of the chunk (rows outside the
          // segment count 0), by a butterfly over the group's GR lanes
#pragma unroll
          for (int o = 1; o < GR; o <<= 1) xsum += __shfl_xor_sync(0xffffffffu, xsum, o);
          if (lane % GR == 0) xg[t * 8 + lane / GR] = xsum;
        }
      }
      __syncwarp();
      const int k0 = b0 > ch * CB ? b0 - ch * CB : 0;
      const int k1 = b1 - ch * CB < CB ? b1 - ch * CB : CB;
#pragma unroll 1
      for (int k = k0; k < k1; ++k) {              // not unrolled: the loop body stays in the instruction cache
        const int b = ch * CB + k;
        if ((k & (GB - 1)) == 0 || b == b0) {      // a group's first batch here: its deltas (and zero points)
          if (valid) {
            const int64_t g = b / GB;
            const float4 d = __ldg(scales + g * D4 + q4);
            dv[0] = d.x;
            dv[1] = d.y;
            dv[2] = d.z;
            dv[3] = d.w;
            if (kZp) {                             // the four columns' zero points, one 32-bit load
              const uint32_t z4 = __ldg(reinterpret_cast<const uint32_t*>(zeros + g * D_out) + q4);
#pragma unroll
              for (int c = 0; c < 4; ++c) zv[c] = static_cast<float>((z4 >> (8 * c)) & 0xFFu);
            }
          }
        }
        issue();                                   // the batch P - 1 ahead, into the slot used last
        cp_async_wait<P - 1>();                    // this thread's copies of this batch have landed
        const uint8_t* slot = wring + rslot * kSlotBytes;
        if (++rslot == P) rslot = 0;
        uint4 pw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) pw[u] = *reinterpret_cast<const uint4*>(slot + u * (kGvCols * 4));
        const float* xk = xt + k * U * 8;          // x~ of the batch's first row
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float4 xa[NT], xb[NT];
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float4* src = reinterpret_cast<const float4*>(xk + (t * XR + u) * 8);
            xa[t] = src[0];
            xb[t] = src[1];
          }
          const uint32_t wv[4] = {pw[u].x, pw[u].y, pw[u].z, pw[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t w = wv[c], w8 = w >> 8;
            const float2 v01 = make_float2(nibf(w, 0xFu), nibf(w, 0xF0u));
            const float2 v23 = make_float2(nibf(w, 0xF00u), nibf(w, 0xF000u));
            const float2 v45 = make_float2(nibf(w, 0xF0000u), nibf(w, 0xF00000u));
            const float2 v67 = make_float2(nibf(w8, 0xF0000u), nibf(w8, 0xF00000u));
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              float2 a2 = __ffma2_rn(v01, make_float2(xa[t].x, xa[t].y), acc[t][c]);
              a2 = __ffma2_rn(v23, make_float2(xa[t].z, xa[t].w), a2);
              a2 = __ffma2_rn(v45, make_float2(xb[t].x, xb[t].y), a2);
              acc[t][c] = __ffma2_rn(v67, make_float2(xb[t].z, xb[t].w), a2);
            }
          }
        }
        if (((k + 1) & (GB - 1)) == 0 || b == b1 - 1) {   // a group's last batch here: delta (sum x' u - z sum x')
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float xs = xg[t * 8 + k / GB];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float a = __fmul_rn(acc[t][c].x + acc[t][c].y, 0x1p85f);   // sum of x' u over the group
              tt[t][c] = __fmaf_rn(dv[c], __fmaf_rn(-zv[c], xs, a), tt[t][c]);
              acc[t][c] = make_float2(0.0f, 0.0f);
            }
          }
        }
      }
    }
    pos += b1 - b0;
    if (tau == t0) {                               // the CTA's first tile: to shared memory
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        first[(warp * NT + t) * 32 + lane] = make_float4(tt[t][0], tt[t][1], tt[t][2], tt[t][3]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tt[t][c] = 0.0f;
      }
    } else {
      next_tile = true;                            // the second tile: the warp's last segment
    }
  }
  cp_async_wait<0>();
  __syncthreads();                                 // the ring is free: the warps' sums of the next tile there
  float4* second = reinterpret_cast<float4*>(ring);   // [8 warps][NT][32 quads]
#pragma unroll
  for (int t = 0; t < NT; ++t)
    second[(warp * NT + t) * 32 + lane] = next_tile ? make_float4(tt[t][0], tt[t][1], tt[t][2], tt[t][3])
                                                    : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  __syncthreads();
  if (S > 0) {                                     // a cluster of S splits of one tile
    float4* fin = second + 8 * NT * 32;            // this CTA's sums, read by rank 0 (DSMEM)
    const int t = threadIdx.x >> 5, qd = threadIdx.x & 31;
    float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (threadIdx.x < NT * 32) {
      a = first[t * 32 + qd];
#pragma unroll
      for (int w = 1; w < 8; ++w) {
        const float4 b = first[(w * NT + t) * 32 + qd];
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
      }
      fin[threadIdx.x] = a;
    }
    cluster_sync_all();                            // every rank's sums are in its shared memory
    const bool rank0 = cluster_ctarank() == 0;
    if (rank0 && threadIdx.x < NT * 32) {
      const uint32_t local = smem_u32(&fin[threadIdx.x]);
      for (int r = 1; r < S; ++r) {
        const float4 b = ld_shared_cluster_f4(mapa_shared(local, static_cast<uint32_t>(r)));
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
      }
      const int64_t m4 = t0 * (kGvCols / 4) + qd;
      if (m4 < D4) {
        if (y16) {
          reinterpret_cast<float4*>(Y)[t * D4 + m4] = a;
        } else {
          float* yo = Y + t * D_out + 4 * m4;
          yo[0] = a.x;
          yo[1] = a.y;
          yo[2] = a.z;
          yo[3] = a.w;
        }
      }
    }
    cluster_sync_all();                            // no rank leaves while rank 0 may read its sums
    return;
  }
  if (threadIdx.x < 2 * NT * 32) {                 // (tile k, token t, quad) in warp order
    const int k = threadIdx.x / (NT * 32), t = (threadIdx.x / 32) % NT, qd = threadIdx.x & 31;
    const float4* red = k == 0 ? first : second;
    float4 a = red[t * 32 + qd];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
      const float4 b = red[(w * NT + t) * 32 + qd];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    if (direct) {                                  // one CTA per tile: this CTA's sums are Y
      const int64_t m4 = t0 * (kGvCols / 4) + qd;
      if (k == 0 && m4 < D4) {
        if (y16) {
          reinterpret_cast<float4*>(Y)[t * D4 + m4] = a;
        } else {
          float* yo = Y + t * D_out + 4 * m4;
          yo[0] = a.x;
          yo[1] = a.y;
          yo[2] = a.z;
          yo[3] = a.w;
        }
      }
    } else {
      reinterpret_cast<float4*>(part)[((i * 2 + k) * NT + t) * 32 + qd] = a;
    }
  }
  pdl_launch_dependents();
}

// Y[t][n] = the sums of tile n / 128 of the CTAs whose shares touch it, in
// CTA order (the shares of the GEMV's partition, recomputed).  Launched as a
// programmatic dependent of the GEMV: it waits for the GEMV's writes.
template <int NT>
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float4* __restrict__ part, int64_t D_out,
                                                          int64_t NB, int64_t C, float* __restrict__ Y, int y16) {
  pdl_wait_primary();
  const int64_t D4 = D_out / 4;
  const int64_t tiles = (D_out + kGvCols - 1) / kGvCols;
  const int64_t W = tiles * NB;
  for (int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; o < NT * D4;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = o / D4, m4 = o - t * D4;
    const int64_t tau = m4 / (kGvCols / 4), qd = m4 % (kGvCols / 4);
    // the first CTA whose share ends past the tile's first batch
    int64_t c = tau * NB * C / W;
    while (c > 0 && W * c / C > tau * NB) --c;
    while (W * (c + 1) / C <= tau * NB) ++c;
    float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    bool first = true;
    for (; c < C && W * c / C < (tau + 1) * NB; ++c) {
      const int64_t k = tau - (W * c / C) / NB;    // 0: the CTA's first tile, 1: the next
      const float4 b = part[((c * 2 + k) * NT + t) * 32 + qd];
      if (first) {
        a = b;
        first = false;
      } else {
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
      }
    }
    if (y16) {
      reinterpret_cast<float4*>(Y)[t * D4 + m4] = a;
    } else {
      float* yo = Y + t * D_out + 4 * m4;
      yo[0] = a.x;
      yo[1] = a.y;
      yo[2] = a.z;
      yo[3] = a.w;
    }
  }
}


// ------------------------------------------------------------ decode, 3-8 tokens, on the tensor cores
//
// With three or more tokens the GEMV above spends four paired FMAs per packed
// word and token and the FMA pipe sets its time; up to 16 tokens the tcgen05
// GEMM below pads them to one 16-token tile.  This form keeps the
// dequantisation on the CUDA cores and hands the products to the tensor cores
// through warp-level mma.sync m16n8k16 (bf16 operands, fp32 accumulation;
// N = 8 token slots, of which 3-8 carry tokens).
//
// Operands.  A packed word holds rows r0..r0+7 of one column.  The mask-and-OR
// of (word >> 4i) with 0x000F000F | 0x43004300 is the exact bf16 pair
// {128 + u_(r0+i), 128 + u_(r0+i+4)}; one bf16x2 FMA subtracts 128 + off,
// leaving the exact codes q = u - off.  The k index of an MMA can stand for
// the rows in any order as long as its A and B fragments agree, so lane
// (g = lane / 4, j = lane % 4) takes its word from k8 row base + j and feeds
// the pairs i = 0, 1 as fragments a0, a2 of the first MMA and i = 2, 3 of the
// second: MMA k indices 2j, 2j+1, 2j+8, 2j+9 are rows r0, r0+4, r0+1, r0+5
// (first MMA) or r0+2, r0+6, r0+3, r0+7 (second).  Its B fragments are X' of
// token g at the same rows, staged in shared memory in that pair order.  A
// lane loads 16 bytes, the words of four consecutive columns c0..c0+3: c0 and
// c0+1 are A rows g and g+8 of one accumulator, c0+2 and c0+3 of another, so
// each lane ends with the sums of its own four columns for tokens 2j and 2j+1.
//
// Work: a CTA takes 32 cw columns (cw = mm_slices(NT) warp slices of 32: 4
// for 3-4 tokens, 8 for 5-8) and a range of whole groups, split between the
// 8 / cw warps of a slice; the S CTAs that split one tile's groups form a
// cluster, and rank 0 adds their sums in rank order from their shared memory
// (DSMEM), so the result does not depend on timing.  Each lane keeps 7 steps
// of 16 bytes in flight (a ring of cp.async copies in shared memory); the loop
// runs over the warp's groups with the group's steps unrolled (the group size
// is a template argument), which cut the time by a sixth at four tokens.  At
// four tokens on a 28672 x 8192 layer, 256-column tiles and a ring of 16 steps
// were both measured slower.  A group's delta is applied once, after its last
// step; the zero-point form adds (off - z) times the group's sum of X' at the
// same point.  No waits on other CTAs beyond the cluster barrier, no
// workspace.
constexpr int kMmThreads = 256;
constexpr int kMmRing = 8;                       // 16-byte steps per lane in the ring (7 in flight)
constexpr int kMmMaxSplit = 8;                   // CTAs per tile: a portable cluster
constexpr int kMmMaxTokens = 8;                  // the MMA's token slots
// Rows of one CTA's range (X' of all tokens in shared memory) and warp slices
// of 32 columns per CTA: 5-8 tokens take half the rows and twice the columns,
// so that two CTAs still fit an SM and the tiles x splits still fill one wave.
__host__ __device__ constexpr int mm_max_rows(int nt) { return nt <= 4 ? 8192 : 4096; }
__host__ __device__ constexpr int mm_slices(int nt) { return nt <= 4 ? 4 : 8; }

// Shared memory: X', the zero-point form's group sums of X', the ring; after
// the main loop the ring holds the warps' sums (red) and the CTA's (fin).
struct MmLayout {
  int ts;                                        // bytes per token of X': k8 rows x 16, = 64 mod 128
  int xs, xg, ring, red, fin, total;
};
__host__ __device__ inline MmLayout mm_layout(int nt, int k8max, int gmax) {
  MmLayout L;
  L.ts = (k8max * 16 + 127) / 128 * 128 + 64;    // lanes g, g+1 of a quarter warp hit different banks
  L.xs = 0;
  L.xg = nt * L.ts;
  L.ring = (L.xg + nt * gmax * 4 + 127) / 128 * 128;
  L.red = L.ring;                                // [8 / cw][nt][32 cw] <= 2 nt 256 floats
  L.fin = L.red + 2 * nt * 256 * 4;              // [nt][32 cw]
  L.total = L.ring + kMmRing * kMmThreads * 16;
  return L;
}
static_assert(2 * kMmMaxTokens * 256 * 4 + kMmMaxTokens * 256 * 4 <= kMmRing * kMmThreads * 16,
              "the sums fit in the ring");

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The code pair of nibbles i and i+4 of w: exact bf16 {u_i - off, u_(i+4) - off}
// (bias2 = the pair -(128 + off), exact in bf16).
__device__ __forceinline__ uint32_t code_pair(uint32_t w, int i, uint32_t bias2) {
  const uint32_t p = ((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
  uint32_t q;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(q) : "r"(p), "r"(0x3F803F80u), "r"(bias2));
  return q;
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// Y [NT][D_out] fp32 (any 4-byte alignment).  Grid: tiles x S CTAs, clusters
// of S along x; a tile is 32 cw columns.  k8max / gmax: k8 rows / groups of
// the largest CTA range.
template <int NT, int G, bool kZp>
__global__ void __launch_bounds__(kMmThreads, 2) w4a16_gemv_mma_kernel(
    const uint4* __restrict__ X, const float4* __restrict__ s, const uint32_t* __restrict__ packed,
    const float4* __restrict__ scales, const uint8_t* __restrict__ zeros, int64_t D_in, int64_t D_out,
    int off, int S, int cw, int k8max, int gmax, float* __restrict__ Y, int* __restrict__ status) {
  static_assert(NT >= 2 && NT <= kMmMaxTokens, "2-8 token slots");
  extern __shared__ __align__(16) uint8_t mm_sm[];
  const MmLayout Lm = mm_layout(NT, k8max, gmax);
  uint8_t* xs = mm_sm + Lm.xs;
  uint4* ring = reinterpret_cast<uint4*>(mm_sm + Lm.ring);
  float* red = reinterpret_cast<float*>(mm_sm + Lm.red);
  float* fin = reinterpret_cast<float*>(mm_sm + Lm.fin);
  float* xg = reinterpret_cast<float*>(mm_sm + Lm.xg);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (status && blockIdx.x == 0 && tid == 0) *status = 0;
  const int rank = static_cast<int>(cluster_ctarank());
  const int64_t tile = blockIdx.x / S;
  const int64_t ng = D_in / G, rows8 = D_in / 8;
  constexpr int gr8 = G / 8, spg = G / 32;        // k8 rows and steps (4 k8 rows each) per group
  const int64_t ga = ng * rank / S, gb = ng * (rank + 1) / S;   // this CTA's groups
  const int kw = 8 / cw, cols = 32 * cw;          // warps per slice, columns per tile
  const int part = warp / cw, slice = warp % cw;
  const int64_t wa = ga + (gb - ga) * part / kw, wb = ga + (gb - ga) * (part + 1) / kw;   // this warp's
  const int nsteps = static_cast<int>(wb - wa) * spg;
  const int g = lane >> 2, j = lane & 3;
  const int64_t c0 = tile * cols + slice * 32 + 4 * g;
  const bool valid = c0 < D_out;                  // D_out % 4 == 0: the four columns all in or all out
  const int64_t D4 = D_out / 4;

  // The lane's ring: entry e at ring[e * 256 + tid] (a quarter warp reads 128
  // contiguous bytes).  Step st reads k8 row wa * gr8 + 4 st + j.
  uint4* my_ring = ring + tid;
  const uint32_t* src = packed + (wa * gr8 + j) * D_out + (valid ? c0 : 0);
  const int64_t step_words = 4 * D_out;
  int n_iss = 0;
  auto issue = [&]() {
    if (n_iss < nsteps) {
      cp_async16(my_ring + (n_iss & (kMmRing - 1)) * kMmThreads, src, valid ? 16u : 0u);
      src += step_words;
    }
    ++n_iss;
    cp_async_commit();
  };
#pragma unroll
  for (int e = 0; e < kMmRing - 1; ++e) issue();

  // X' = bf16(x / s) of the CTA's rows, token t at xs + t ts, k8 row r at
  // + 16 r as the pairs (0,4) (1,5) (2,6) (3,7); 1/s by the hardware
  // reciprocal (relative error ~2^-23, far below the bf16 rounding).
  const int64_t k8a = ga * gr8;
  const int k8n = static_cast<int>((gb - ga) * gr8);
  for (int r = tid; r < k8n; r += kMmThreads) {
    const float4 s0 = s[2 * (k8a + r)], s1 = s[2 * (k8a + r) + 1];
    float rs[8];
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rs[e]) : "f"(sv[e]));
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const uint4 xv = X[t * rows8 + k8a + r];
      const uint32_t hv[4] = {xv.x, xv.y, xv.z, xv.w};
      float x[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[2 * e] = __fmul_rn(bf16_bits_to_float(hv[e] & 0xFFFFu), rs[2 * e]);
        x[2 * e + 1] = __fmul_rn(bf16_bits_to_float(hv[e] >> 16), rs[2 * e + 1]);
      }
      *reinterpret_cast<uint4*>(xs + t * Lm.ts + r * 16) =
          make_uint4(pack_bf16(x[0], x[4]), pack_bf16(x[1], x[5]), pack_bf16(x[2], x[6]), pack_bf16(x[3], x[7]));
    }
  }
  __syncthreads();
  if (kZp) {                                      // per token and group: the sum of its X' (as bf16), in row order
    const int ngc = static_cast<int>(gb - ga);
    for (int it = tid; it < NT * ngc; it += kMmThreads) {
      const int t = it / ngc, gl = it % ngc;
      float sum = 0.0f;
      for (int r = gl * gr8; r < (gl + 1) * gr8; ++r) {
        const uint4 v = *reinterpret_cast<const uint4*>(xs + t * Lm.ts + r * 16);
        const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) sum += bf16_bits_to_float(pv[e] & 0xFFFFu) + bf16_bits_to_float(pv[e] >> 16);
      }
      xg[t * gmax + gl] = sum;
    }
    __syncthreads();
  }

  const uint32_t bias = pack_bf16(-(128.0f + static_cast<float>(off)), -(128.0f + static_cast<float>(off)));
  const bool xin = g < NT;                        // lanes g >= NT feed the unused token slots zeros
  const uint8_t* xrow = xs + (xin ? g : 0) * Lm.ts + ((wa - ga) * gr8 + j) * 16;
  float acc[2][4], tot[4][2];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    acc[c >> 1][2 * (c & 1)] = acc[c >> 1][2 * (c & 1) + 1] = 0.0f;
    tot[c][0] = tot[c][1] = 0.0f;
  }
  // the delta (and zero points) of the current group, loaded one group ahead
  float4 dcur = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  uint32_t zcur = 0;
  int64_t gi = wa;
  if (valid && nsteps > 0) {
    dcur = __ldg(scales + wa * D4 + c0 / 4);
    if (kZp) zcur = __ldg(reinterpret_cast<const uint32_t*>(zeros + wa * D_out + c0));
  }
#pragma unroll 1
  for (int gl = 0; gl < nsteps / spg; ++gl) {     // one group of this warp: spg steps, then its delta
#pragma unroll
    for (int q = 0; q < spg; ++q) {
      const int st = gl * spg + q;
      issue();                                    // the step kMmRing - 1 ahead, into the entry used last
      cp_async_wait<kMmRing - 1>();               // this lane's copy of step st has landed
      const uint4 w = my_ring[(st & (kMmRing - 1)) * kMmThreads];
      uint4 xb = make_uint4(0u, 0u, 0u, 0u);
      if (xin) xb = *reinterpret_cast<const uint4*>(xrow + st * 64);
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {               // columns c0 + 2h (A row g) and c0 + 2h + 1 (A row g + 8)
        const uint32_t lo = wv[2 * h], hi = wv[2 * h + 1];
        mma_bf16_16816(acc[h], code_pair(lo, 0, bias), code_pair(hi, 0, bias), code_pair(lo, 1, bias),
                       code_pair(hi, 1, bias), xb.x, xb.y);
        mma_bf16_16816(acc[h], code_pair(lo, 2, bias), code_pair(hi, 2, bias), code_pair(lo, 3, bias),
                       code_pair(hi, 3, bias), xb.z, xb.w);
      }
    }
    // the group's delta (and, with zero points, (off - z) sum x')
    const float dv[4] = {dcur.x, dcur.y, dcur.z, dcur.w};
    float corr[4][2];
#pragma unroll
    for (int c = 0; c < 4; ++c) corr[c][0] = corr[c][1] = 0.0f;
    if (kZp) {
      const int gc = static_cast<int>(gi - ga);
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int t = 2 * j + tt;
        const float xsum = t < NT ? xg[t * gmax + gc] : 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          corr[c][tt] = __fmul_rn(static_cast<float>(off - static_cast<int>((zcur >> (8 * c)) & 0xFFu)), xsum);
      }
    }
    ++gi;
    if (valid && gi < wb) {                       // the next group's delta, a group's steps ahead of its use
      dcur = __ldg(scales + gi * D4 + c0 / 4);
      if (kZp) zcur = __ldg(reinterpret_cast<const uint32_t*>(zeros + gi * D_out + c0));
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        float& a = acc[c >> 1][2 * (c & 1) + tt];
        tot[c][tt] = __fmaf_rn(dv[c], kZp ? a + corr[c][tt] : a, tot[c][tt]);
        a = 0.0f;
      }
    }
  }
  cp_async_wait<0>();

  // the warps' sums (in the ring, free once every lane's copies have landed),
  // then the CTA's [NT][cols] sums: the parts of a slice added in order
  __syncthreads();
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int t = 2 * j + tt;
      if (t < NT) red[(part * NT + t) * cols + slice * 32 + 4 * g + c] = tot[c][tt];
    }
  __syncthreads();
  for (int i = tid; i < NT * cols; i += kMmThreads) {
    float v = red[i];
    for (int q = 1; q < kw; ++q) v += red[q * NT * cols + i];
    fin[i] = v;
  }
  cluster_sync_all();                             // every rank's sums are in its shared memory
  if (rank == 0) {
    for (int i = tid; i < NT * cols; i += kMmThreads) {
      float v = fin[i];
      const uint32_t local = smem_u32(&fin[i]);
      for (int r = 1; r < S; ++r) v += ld_shared_cluster_f32(mapa_shared(local, static_cast<uint32_t>(r)));
      const int t = i / cols;
      const int64_t n = tile * cols + (i % cols);
      if (n < D_out) Y[t * D_out + n] = v;
    }
  }
  cluster_sync_all();                             // no rank leaves while rank 0 may read its sums
}

}  // namespace

namespace {

struct W4Layout {
  size_t xs, count, partial, zb, total;
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

int w4_token_tile(int64_t N) { return N >= 256 ? 256 : static_cast<int>((N + 15) / 16 * 16); }

// zrows: rows of zero points (D_in / group) of the asymmetric consumer, else 0.
W4Layout w4_layout(int64_t N, int64_t D_in, int64_t D_out, int64_t zrows = 0) {
  W4Layout l;
  if (N <= kGvMaxTokens) {                        // the GEMV: two tiles of sums per CTA
    l.xs = l.count = l.partial = l.zb = 0;
    l.total = round256(static_cast<size_t>(kGvMaxCtas) * 2 * N * kGvCols * 4);
    return l;
  }
  const int Nt = w4_token_tile(N);
  const int64_t units = ((D_out + 127) / 128) * ((N + Nt - 1) / Nt);
  l.xs = 0;
  const int64_t Dp = (D_in + 63) / 64 * 64;     // X' rows padded to whole k blocks
  l.count = round256(static_cast<size_t>(N) * static_cast<size_t>(Dp) * 2);
  l.partial = l.count + round256(static_cast<size_t>(units) * 4);
  const size_t part = Nt <= kW4MaxStreamTokens ? static_cast<size_t>(kW4MaxGrid) * 2 * N * 128 * 4 : 0;
  l.zb = l.partial + round256(part);
  l.total = l.zb + round256(static_cast<size_t>(zrows) * D_out * 4);
  return l;
}

// CTAs of the (NT, G, kZp) GEMV resident on one SM, and clusters of c
// CTAs resident on the GPU, per device (0: not yet asked).
constexpr int kGvMaxDevices = 64;
constexpr int kGvMaxCluster = 8;                 // portable cluster size
std::atomic<int> g_gv_occ[kGvMaxDevices][kGvMaxTokens][2][4];
std::atomic<int> g_gv_clusters[kGvMaxDevices][kGvMaxTokens][2][4][kGvMaxCluster + 1];

template <typename K>
cudaError_t gemv_resident_clusters(K kern, int dev, int NT, bool zp, int G, int c, int smem, int* n) {
  std::atomic<int>& slot =
      g_gv_clusters[dev][NT - 1][zp ? 1 : 0][G == 32 ? 0 : G == 64 ? 1 : G == 128 ? 2 : 3][c];
  *n = slot.load(std::memory_order_relaxed);
  if (*n > 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(c), 1, 1);
  cfg.blockDim = dim3(kGvThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(c);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaOccupancyMaxActiveClusters(n, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (*n < 1) *n = 1;
  slot.store(*n, std::memory_order_relaxed);
  return cudaSuccess;
}

template <int NT, int G, bool kZp>
int launch_gemv_k(const void* X, const float* s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                  int64_t D_in, int64_t D_out, int bits, float* Y, void* ws, int num_sms, int* status,
                  cudaStream_t st, cudaError_t* cerr, const char** what) {
  auto kern = w4a16_gemv_kernel<NT, G, kZp>;
  const int smem = static_cast<int>(gv_smem_bytes<NT, G>());
  static SmemAttrOnce once;
  cudaError_t e = set_smem_once(kern, smem, once);
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "cudaFuncSetAttribute(w4a16_gemv_kernel)";
    return kECuda;
  }
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kGvMaxDevices) {
    *cerr = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    *what = "cudaGetDevice";
    return kECuda;
  }
  std::atomic<int>& occ_slot = g_gv_occ[dev][NT - 1][kZp ? 1 : 0][G == 32 ? 0 : G == 64 ? 1 : G == 128 ? 2 : 3];
  int occ = occ_slot.load(std::memory_order_relaxed);
  if (occ <= 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGvThreads, smem);
    if (e != cudaSuccess) {
      *cerr = e;
      *what = "cudaOccupancyMaxActiveBlocksPerMultiprocessor";
      return kECuda;
    }
    if (occ < 1) occ = 1;
    occ_slot.store(occ, std::memory_order_relaxed);
  }
  const int64_t NB = D_in / 8 / gv_batch<NT, G>();
  const int64_t tiles = (D_out + kGvCols - 1) / kGvCols;
  const int off = 1 << (bits - 1);
  const int y16 = (reinterpret_cast<uintptr_t>(Y) & 15u) == 0 ? 1 : 0;
  // One launch of S splits per tile, a cluster each, when all clusters are
  // resident at once (the most splits, at least 8 batches per split): no
  // second launch, which costs more than the uneven load of the SMs that
  // clusters of S bring.  Else stream-K and a reduction launch.
  {
    int S = 0;
    for (int c = kGvMaxCluster; c >= 2 && S == 0; --c) {
      if (NB < 8 * c) continue;
      int n = 0;
      e = gemv_resident_clusters(kern, dev, NT, kZp, G, c, smem, &n);
      if (e != cudaSuccess) {
        *cerr = e;
        *what = "cudaOccupancyMaxActiveClusters";
        return kECuda;
      }
      if (n >= tiles) S = c;
    }
    if (S > 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(tiles * S), 1, 1);
      cfg.blockDim = dim3(kGvThreads, 1, 1);
      cfg.dynamicSmemBytes = static_cast<size_t>(smem);
      cfg.stream = st;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = static_cast<unsigned>(S);
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, kern, static_cast<const uint4*>(X), reinterpret_cast<const float4*>(s), packed,
                             reinterpret_cast<const float4*>(scales), zeros, D_in, D_out, off,
                             static_cast<float*>(nullptr), Y, y16, 0, S, status);
      if (e != cudaSuccess) {
        *cerr = e;
        *what = "w4a16_gemv_kernel launch (clusters)";
        return kECuda;
      }
      return kOk;
    }
  }
  // Every SM full; as many CTAs as tiles (each a whole tile, Y stored
  // directly) when the tiles alone fill the GPU.
  int64_t C = static_cast<int64_t>(occ) * (num_sms > 0 ? num_sms : 1);
  if (C > kGvMaxCtas) C = kGvMaxCtas;
  if (C > tiles * NB) C = tiles * NB;              // at least one batch per CTA
  const bool direct = tiles >= C;
  if (direct) C = tiles;
  float* part = static_cast<float*>(ws);
  kern<<<static_cast<unsigned>(C), kGvThreads, smem, st>>>(
      static_cast<const uint4*>(X), reinterpret_cast<const float4*>(s), packed,
      reinterpret_cast<const float4*>(scales), zeros, D_in, D_out, off, part, Y, y16, direct ? 1 : 0, 0, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "w4a16_gemv_kernel launch";
    return kECuda;
  }
  if (direct) return kOk;
  const int64_t outs = NT * (D_out / 4);
  int64_t blocks = (outs + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 4) blocks = static_cast<int64_t>(num_sms) * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemv_reduce_kernel<NT>, static_cast<const float4*>(ws), D_out, NB, C, Y, y16);
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "gemv_reduce_kernel launch";
    return kECuda;
  }
  return kOk;
}

template <int NT, int G>
int launch_gemv_g(const void* X, const float* s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                  int64_t D_in, int64_t D_out, int bits, float* Y, void* ws, int num_sms, int* status,
                  cudaStream_t st, cudaError_t* cerr, const char** what) {
  if (zeros)
    return launch_gemv_k<NT, G, true>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, ws, num_sms, status, st,
                                      cerr, what);
  return launch_gemv_k<NT, G, false>(X, s, packed, scales, nullptr, D_in, D_out, bits, Y, ws, num_sms, status, st,
                                     cerr, what);
}

template <int NT>
int launch_gemv_nt(const void* X, const float* s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                   int64_t D_in, int64_t D_out, int bits, int group, float* Y, void* ws, int num_sms, int* status,
                   cudaStream_t st, cudaError_t* cerr, const char** what) {
  switch (group) {
    case 32: return launch_gemv_g<NT, 32>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, ws, num_sms, status, st, cerr, what);
    case 64: return launch_gemv_g<NT, 64>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, ws, num_sms, status, st, cerr, what);
    case 128: return launch_gemv_g<NT, 128>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, ws, num_sms, status, st, cerr, what);
    case 256: return launch_gemv_g<NT, 256>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, ws, num_sms, status, st, cerr, what);
    default: *what = "gemv group"; return kEUnsupported;
  }
}

// The tensor-core GEMV for 3-8 tokens (w4a16_gemv_mma_kernel): tiles of
// 32 mm_slices(NT) columns; S CTAs per tile, as many as keep two CTAs on every
// SM (at most 8, at least enough that no CTA's range of groups exceeds
// mm_max_rows(NT) rows), in clusters of S.
template <int NT, int G, bool kZp>
int launch_gemv_mma_k(const void* X, const float* s, const uint32_t* packed, const float* scales,
                      const uint8_t* zeros, int64_t D_in, int64_t D_out, int bits, int group, float* Y, int num_sms,
                      int* status, cudaStream_t st, cudaError_t* cerr, const char** what) {
  const int64_t ng = D_in / group;
  const int64_t sms = num_sms > 0 ? num_sms : 1;
  const int64_t smin = (D_in + mm_max_rows(NT) - 1) / mm_max_rows(NT);
  const int cw = mm_slices(NT);
  const int64_t tiles = (D_out + 32 * cw - 1) / (32 * cw);
  int64_t S = 2 * sms / tiles;
  if (S > kMmMaxSplit) S = kMmMaxSplit;
  if (S < smin) S = smin;
  if (S > ng) S = ng;
  if (S < 1) S = 1;
  const int gmax = static_cast<int>((ng + S - 1) / S);
  const int k8max = gmax * (group / 8);
  const MmLayout Lm = mm_layout(NT, k8max, gmax);
  // the attribute covers the largest layout any call can ask for
  const MmLayout Lmax = mm_layout(NT, (mm_max_rows(NT) + 256) / 8, (mm_max_rows(NT) + 256) / 32);
  auto kern = w4a16_gemv_mma_kernel<NT, G, kZp>;
  static SmemAttrOnce once;
  cudaError_t e = set_smem_once(kern, Lmax.total, once);
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "cudaFuncSetAttribute(w4a16_gemv_mma_kernel)";
    return kECuda;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * S), 1, 1);
  cfg.blockDim = dim3(kMmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(Lm.total);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(S);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const uint4*>(X), reinterpret_cast<const float4*>(s), packed,
                         reinterpret_cast<const float4*>(scales), zeros, D_in, D_out, 1 << (bits - 1),
                         static_cast<int>(S), cw, k8max, gmax, Y, status);
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "w4a16_gemv_mma_kernel launch";
    return kECuda;
  }
  return kOk;
}

template <int NT, int G>
int launch_gemv_mma_g(const void* X, const float* s, const uint32_t* packed, const float* scales,
                      const uint8_t* zeros, int64_t D_in, int64_t D_out, int bits, float* Y, int num_sms, int* status,
                      cudaStream_t st, cudaError_t* cerr, const char** what) {
  if (zeros)
    return launch_gemv_mma_k<NT, G, true>(X, s, packed, scales, zeros, D_in, D_out, bits, G, Y, num_sms, status, st,
                                          cerr, what);
  return launch_gemv_mma_k<NT, G, false>(X, s, packed, scales, nullptr, D_in, D_out, bits, G, Y, num_sms, status,
                                         st, cerr, what);
}

template <int NT>
int launch_gemv_mma(const void* X, const float* s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                    int64_t D_in, int64_t D_out, int bits, int group, float* Y, int num_sms, int* status,
                    cudaStream_t st, cudaError_t* cerr, const char** what) {
  switch (group) {
    case 32: return launch_gemv_mma_g<NT, 32>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, num_sms, status, st, cerr, what);
    case 64: return launch_gemv_mma_g<NT, 64>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, num_sms, status, st, cerr, what);
    case 128: return launch_gemv_mma_g<NT, 128>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, num_sms, status, st, cerr, what);
    case 256: return launch_gemv_mma_g<NT, 256>(X, s, packed, scales, zeros, D_in, D_out, bits, Y, num_sms, status, st, cerr, what);
    default: *what = "gemv group"; return kEUnsupported;
  }
}

int launch_w4a16_gemv(const void* X, const float* s, const uint32_t* packed, const float* scales,
                      const uint8_t* zeros, int64_t N, int64_t D_in, int64_t D_out, int bits, int group, float* Y,
                      void* ws, int num_sms, int* status, cudaStream_t st, cudaError_t* cerr, const char** what) {
  // 3-4 tokens on the tensor cores while a CTA's share of the rows fits its
  // shared memory.  Two tokens stay on the CUDA cores: measured faster there
  // (41.8 against ~44.5 us on a 28672 x 8192 layer; at four tokens 73.2
  // against 45.3 us).
  if (N >= 3 && D_in <= static_cast<int64_t>(kMmMaxSplit) * mm_max_rows(static_cast<int>(N))) {
    switch (N) {
      case 3: return launch_gemv_mma<3>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, num_sms, status, st, cerr, what);
      case 4: return launch_gemv_mma<4>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, num_sms, status, st, cerr, what);
      default: break;
    }
  }
  switch (N) {
    case 1: return launch_gemv_nt<1>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, ws, num_sms, status, st, cerr, what);
    case 2: return launch_gemv_nt<2>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, ws, num_sms, status, st, cerr, what);
    case 3: return launch_gemv_nt<3>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, ws, num_sms, status, st, cerr, what);
    case 4: return launch_gemv_nt<4>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, ws, num_sms, status, st, cerr, what);
    default: *what = "gemv token count"; return kEUnsupported;
  }
}

}  // namespace

size_t w4a16_scratch_bytes(int64_t N, int64_t D_in, int64_t D_out, int64_t zrows) {
  return w4_layout(N, D_in, D_out, zrows).total;
}

bool w4a16_clears_status(int64_t N) { return N <= kGvMaxTokens; }

int launch_w4a16(const void* X, const float* s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                 int64_t N, int64_t D_in, int64_t D_out, int bits, int group, float* Y, void* ws, int num_sms,
                 int* status, uint64_t timeout_ns, cudaStream_t st, cudaError_t* cerr, const char** what) {
  *cerr = cudaSuccess;
  if (N <= kGvMaxTokens)
    return launch_w4a16_gemv(X, s, packed, scales, zeros, N, D_in, D_out, bits, group, Y, ws, num_sms, status, st,
                             cerr, what);
  // 5-8 tokens fill the token slots of the GEMV's MMA tiles: one launch and
  // no workspace, where a tcgen05 tile of 16 tokens would sit half idle.
  if (N <= kMmMaxTokens && D_in <= static_cast<int64_t>(kMmMaxSplit) * mm_max_rows(static_cast<int>(N))) {
    switch (N) {
      case 5: return launch_gemv_mma<5>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, num_sms, status, st, cerr, what);
      case 6: return launch_gemv_mma<6>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, num_sms, status, st, cerr, what);
      case 7: return launch_gemv_mma<7>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, num_sms, status, st, cerr, what);
      case 8: return launch_gemv_mma<8>(X, s, packed, scales, zeros, D_in, D_out, bits, group, Y, num_sms, status, st, cerr, what);
      default: break;
    }
  }
  const bool zp = zeros != nullptr;
  const W4Layout lay = w4_layout(N, D_in, D_out, zp ? D_in / group : 0);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  void* xs = wsb + lay.xs;
  int* count = reinterpret_cast<int*>(wsb + lay.count);
  float* partial = reinterpret_cast<float*>(wsb + lay.partial);

  const int Nt = w4_token_tile(N);
  const int n_tiles = static_cast<int>((D_out + 127) / 128);
  const int t_tiles = static_cast<int>((N + Nt - 1) / Nt);
  const int KB = static_cast<int>((D_in + 63) / 64);
  const int units = n_tiles * t_tiles;
  const bool stream = Nt <= kW4MaxStreamTokens;

  // 1. X' = X / s, rows padded to KB * 64 columns, columns permuted within
  //    runs of 8; clears the unit counts
  const int64_t Dp = static_cast<int64_t>(KB) * 64;
  {
    const int64_t total = N * (Dp / 8);
    int64_t blocks = (total + 255) / 256;
    if (blocks > static_cast<int64_t>(num_sms) * 16) blocks = static_cast<int64_t>(num_sms) * 16;
    scale_x_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint4*>(X), reinterpret_cast<const float4*>(s), total, D_in / 8, Dp / 8,
        static_cast<uint4*>(xs), count, stream ? units : 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *cerr = e;
      *what = "scale_x_kernel launch";
      return kECuda;
    }
  }
  // 2. the GEMM
  const int tcols = Nt <= 32 ? 32 : (Nt <= 64 ? 64 : (Nt <= 128 ? 128 : 256));
  // k blocks per stage: fat stages, two issuing warps for the memory-bound small token tiles
  const int kps = Nt <= 32 ? 4 : (Nt <= 64 ? 2 : 1);
  const int issuers = kps > 1 ? 2 : 1;
  const int KBS = (KB + kps - 1) / kps;
  const int scale_rows = kps * 64 >= group ? kps * 64 / group : 1;
  const int stage_bytes = (kps * Nt * 128 + kps * kW4PkBytes + (zp ? 2 : 1) * scale_rows * 512 + 1023) / 1024 * 1024;
  // One CTA per SM; its shared memory goes to deep rings.
  const int budget = 220 * 1024;
  const int a_stages = Nt <= 32 ? 4 : 3;
  const int fixed = a_stages * kW4ABytes + 1024 + 512;   // alignment slack, barriers
  int stages = (budget - fixed) / stage_bytes;
  if (stages > kW4MaxStages) stages = kW4MaxStages;
  stages -= stages % issuers;                    // each issuing warp owns every issuers-th stage
  if (stages < 2) stages = 2;
  const int smem = fixed + stages * stage_bytes;

  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, W4Params) = nullptr;
  switch (group) {
    case 32: kern = zp ? w4a16_kernel<32, true> : w4a16_kernel<32, false>; break;
    case 64: kern = zp ? w4a16_kernel<64, true> : w4a16_kernel<64, false>; break;
    case 128: kern = zp ? w4a16_kernel<128, true> : w4a16_kernel<128, false>; break;
    case 256: kern = zp ? w4a16_kernel<256, true> : w4a16_kernel<256, false>; break;
    default:
      *what = "group";
      return kEUnsupported;
  }
  float* zb = reinterpret_cast<float*>(wsb + lay.zb);
  if (zp) {
    const int64_t nz = (D_in / group) * D_out;
    int64_t blocks = (nz + 255) / 256;
    if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
    zero_bias_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(zeros, nz, zb);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *cerr = e;
      *what = "zero_bias_kernel launch";
      return kECuda;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "w4a16_kernel attributes";
    return kECuda;
  }
  int64_t slots = num_sms;
  if (slots > kW4MaxGrid) slots = kW4MaxGrid;

  // X' as [KB][N][64]: dimension 1 (tokens) has stride Dp, dimension 2
  // (k blocks) stride 64 elements; one box = the X' planes of a stage.
  CUtensorMap mX, mP, mS, mZ;
  const uint64_t xdims[3] = {64, static_cast<uint64_t>(N), static_cast<uint64_t>(KB)};
  const uint64_t xstr[2] = {static_cast<uint64_t>(Dp) * 2, 128};
  const uint32_t xbox[3] = {64, static_cast<uint32_t>(Nt), static_cast<uint32_t>(kps)};
  if (!make_bf16_map_3d(&mX, xs, xdims, xstr, xbox) ||
      !make_word_map(&mP, packed, false, static_cast<uint64_t>(D_out), static_cast<uint64_t>(D_in / 8), 128,
                     static_cast<uint32_t>(8 * kps)) ||
      !make_word_map(&mS, scales, true, static_cast<uint64_t>(D_out), static_cast<uint64_t>(D_in / group), 128,
                     static_cast<uint32_t>(scale_rows)) ||
      !make_word_map(&mZ, zp ? static_cast<const void*>(zb) : static_cast<const void*>(scales), true,
                     static_cast<uint64_t>(D_out), static_cast<uint64_t>(D_in / group), 128,
                     static_cast<uint32_t>(scale_rows))) {
    *what = "tensor maps for the W4A16 GEMM";
    return kECuda;
  }
  W4Params p;
  p.Y = Y;
  p.partial = partial;
  p.count = count;
  p.N = N;
  p.D_out = D_out;
  p.off = 1 << (bits - 1);
  p.magic = 0x43004300u;
  p.Nt = Nt;
  p.KB = KB;
  p.kps = kps;
  p.KBS = KBS;
  p.n_tiles = n_tiles;
  p.units = units;
  p.stream = stream ? 1 : 0;
  p.issuers = issuers;
  p.total = static_cast<int64_t>(units) * KBS;
  p.stages = stages;
  p.a_stages = a_stages;
  p.stage_bytes = stage_bytes;
  p.scale_rows = scale_rows;
  p.tcols = tcols;
  p.status = status;
  p.timeout_ns = timeout_ns;
  int64_t grid;
  if (stream) {
    // equal shares of the units x KBS stage steps, one per CTA slot
    const int64_t want = p.total < slots ? p.total : slots;
    p.chunk = (p.total + want - 1) / want;
    grid = (p.total + p.chunk - 1) / p.chunk;
  } else {
    p.chunk = KBS;
    grid = units < slots ? units : slots;
  }
  kern<<<static_cast<unsigned>(grid), kW4Threads, smem, st>>>(mX, mP, mS, mZ, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "w4a16_kernel launch";
    return kECuda;
  }
  return kOk;
}

}  // namespace awq
