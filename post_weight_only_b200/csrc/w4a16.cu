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
// Decode (N <= 4 tokens) takes a CUDA-core GEMV instead (see
// w4a16_gemv_kernel): there the work is a stream of packed words with a few
// FMAs per weight, bound by HBM, and a tensor-core tile of 16+ tokens would
// sit mostly idle.
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
// on CUDA cores for N <= 4 tokens, fp32 throughout: x' = x / s rounded once
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
// Work: CTA (column tile, split) owns 128 columns (lane l: columns 4l..4l+3,
// one 16-byte load per k8 row) and a contiguous range of k8 rows (a multiple
// of 32), cut into eight contiguous runs of whole 4-row batches, one per
// warp.  x~ and the per-row sums of x' of the range are staged in shared
// memory in chunks of kGvChunk8 rows; each row's 8 values are a warp-wide
// broadcast.  A warp keeps the next batch of packed words in flight while it
// works on the current one (the first batch is issued before the staging).
// The warps' sums are added in warp order, and with several splits the
// partial rows [split][N][D_out] are summed in split order by
// gemv_reduce_kernel: the result does not depend on timing.  No waits between
// CTAs.
constexpr int kGvThreads = 256;
constexpr int kGvCols = 128;
constexpr int kGvChunk8 = 256;                   // k8 rows of x~ staged at a time, 1-2 tokens (a multiple of 32)
constexpr int kGvBatch = 4;                      // k8 rows per batch of loads
constexpr int kGvMaxSplit = 32;
constexpr int kGvMaxTokens = 4;

__device__ __forceinline__ float nibf(uint32_t w, uint32_t mask) { return __uint_as_float(w & mask); }

// kZp: asymmetric codes u = q + z with a zero point per (group, column)
// (zeros [D_in/G][D_out] uint8) in place of 2^(b-1).
template <int NT, bool kZp>
__global__ void __launch_bounds__(kGvThreads, NT == 1 ? 3 : 2) w4a16_gemv_kernel(const uint4* __restrict__ X,
                                                                const float4* __restrict__ s,
                                                                const uint4* __restrict__ packed,
                                                                const float4* __restrict__ scales,
                                                                const uint8_t* __restrict__ zeros, int64_t D_in,
                                                                int64_t D_out, int gshift, int off, int R8,
                                                                float* __restrict__ out) {
  constexpr int U = kGvBatch;
  constexpr int CH = NT <= 2 ? kGvChunk8 : kGvChunk8 / 2;       // chunk rows (static shared memory <= 48 KiB)
  __shared__ __align__(16) float xt[NT * CH * 8];               // x~ [NT][chunk rows * 8]
  __shared__ float xr[NT * CH];                                 // sum of x' over each row's 8 values
  __shared__ __align__(16) float red[8 * NT * kGvCols];         // per-warp sums
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rows8 = D_in / 8;
  const int64_t D4 = D_out / 4;
  const int64_t rb = static_cast<int64_t>(blockIdx.y) * R8;      // first k8 row of this split
  const int64_t re = rb + R8 < rows8 ? rb + R8 : rows8;
  const int64_t n4 = static_cast<int64_t>(blockIdx.x) * (kGvCols / 4) + lane;   // column quad
  const bool valid = n4 < D4;
  const float fo = static_cast<float>(off);
  float tot[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int c = 0; c < 4; ++c) tot[t][c] = 0.0f;

  for (int64_t cb = rb; cb < re; cb += CH) {
    const int nr = static_cast<int>(re - cb < CH ? re - cb : CH);   // a multiple of 4
    // this warp's rows of the chunk: whole batches
    const int q = (((nr + 7) >> 3) + U - 1) / U * U;
    const int r0 = warp * q, r1 = r0 + q < nr ? r0 + q : nr;
    // the first batch of packed words, before the staging
    uint4 pw[U];
    const uint4* pp = packed + (cb + r0) * D4 + n4;
    if (valid && r0 < r1) {
#pragma unroll
      for (int u = 0; u < U; ++u) pw[u] = __ldcs(pp + u * D4);
    }
    if (cb != rb) __syncthreads();                 // the previous chunk's x~ is no longer read
    for (int i = threadIdx.x; i < NT * nr; i += kGvThreads) {
      const int t = i / nr, r = i - t * nr;
      const uint4 xv = X[t * rows8 + cb + r];
      const float4 s0 = __ldg(s + 2 * (cb + r)), s1 = __ldg(s + 2 * (cb + r) + 1);
      const float v0 = __fdiv_rn(bf16_bits_to_float(xv.x & 0xFFFFu), s0.x);
      const float v1 = __fdiv_rn(bf16_bits_to_float(xv.x >> 16), s0.y);
      const float v2 = __fdiv_rn(bf16_bits_to_float(xv.y & 0xFFFFu), s0.z);
      const float v3 = __fdiv_rn(bf16_bits_to_float(xv.y >> 16), s0.w);
      const float v4 = __fdiv_rn(bf16_bits_to_float(xv.z & 0xFFFFu), s1.x);
      const float v5 = __fdiv_rn(bf16_bits_to_float(xv.z >> 16), s1.y);
      const float v6 = __fdiv_rn(bf16_bits_to_float(xv.w & 0xFFFFu), s1.z);
      const float v7 = __fdiv_rn(bf16_bits_to_float(xv.w >> 16), s1.w);
      // x' 16^-e 2^64: e = 0, 1, 2, 3, 4, 5, 4, 5 (exact powers of two)
      float4* dst = reinterpret_cast<float4*>(xt + (t * CH + r) * 8);
      dst[0] = make_float4(__fmul_rn(v0, 0x1p64f), __fmul_rn(v1, 0x1p60f), __fmul_rn(v2, 0x1p56f),
                           __fmul_rn(v3, 0x1p52f));
      dst[1] = make_float4(__fmul_rn(v4, 0x1p48f), __fmul_rn(v5, 0x1p44f), __fmul_rn(v6, 0x1p48f),
                           __fmul_rn(v7, 0x1p44f));
      xr[t * CH + r] = ((v0 + v1) + (v2 + v3)) + ((v4 + v5) + (v6 + v7));
    }
    __syncthreads();
    if (!valid || r0 >= r1) continue;
    // rows [r0, r1) in batches of U; a group boundary falls only between
    // batches (g8 and every batch start are multiples of U)
    float2 acc[NT][4];
    float xs[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      xs[t] = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[t][c] = make_float2(0.0f, 0.0f);
    }
    int64_t g_cur = ((cb + r0) * 8) >> gshift;
    auto flush = [&](int64_t g) {
      const float4 d = __ldg(scales + g * D4 + n4);
      float z[4] = {fo, fo, fo, fo};
      if (kZp) {                                     // the four columns' zero points, one 32-bit load
        const uint32_t z4 = __ldg(reinterpret_cast<const uint32_t*>(zeros + g * D_out) + n4);
#pragma unroll
        for (int c = 0; c < 4; ++c) z[c] = static_cast<float>((z4 >> (8 * c)) & 0xFFu);
      }
      const float dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
      for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float a = __fmul_rn(acc[t][c].x + acc[t][c].y, 0x1p85f);   // sum of x' u over the group
          tot[t][c] = __fmaf_rn(dv[c], __fmaf_rn(-z[c], xs[t], a), tot[t][c]);
          acc[t][c] = make_float2(0.0f, 0.0f);
        }
        xs[t] = 0.0f;
      }
    };
    for (int r = r0; r < r1; r += U) {
      const int64_t g = ((cb + r) * 8) >> gshift;
      if (g != g_cur) {                              // uniform over the warp
        flush(g_cur);
        g_cur = g;
      }
      uint4 pn[U];                                   // the next batch, in flight during this one
      const bool more = r + U < r1;
      if (more) {
#pragma unroll
        for (int u = 0; u < U; ++u) pn[u] = __ldcs(pp + (U + u) * D4);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int rr = r + u;
        float4 xa[NT], xb[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float4* src = reinterpret_cast<const float4*>(xt + (t * CH + rr) * 8);
          xa[t] = src[0];
          xb[t] = src[1];
          xs[t] += xr[t * CH + rr];
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
      if (more) {
#pragma unroll
        for (int u = 0; u < U; ++u) pw[u] = pn[u];
      }
      pp += U * D4;
    }
    flush(g_cur);
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
    reinterpret_cast<float4*>(red)[(warp * NT + t) * (kGvCols / 4) + lane] =
        make_float4(tot[t][0], tot[t][1], tot[t][2], tot[t][3]);
  __syncthreads();
  if (threadIdx.x < NT * 32) {
    const int t = threadIdx.x >> 5, qd = threadIdx.x & 31;
    const int64_t m4 = static_cast<int64_t>(blockIdx.x) * (kGvCols / 4) + qd;
    if (m4 < D4) {
      const float4* rv = reinterpret_cast<const float4*>(red);
      float4 a = rv[t * (kGvCols / 4) + qd];
#pragma unroll
      for (int w = 1; w < 8; ++w) {
        const float4 b = rv[(w * NT + t) * (kGvCols / 4) + qd];
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
      }
      reinterpret_cast<float4*>(out)[(static_cast<int64_t>(blockIdx.y) * NT + t) * D4 + m4] = a;
    }
  }
}

// Y = sum over splits of the partial rows, in split order.  y16: Y is 16-byte
// aligned (else four scalar stores; the API asks only 4-byte alignment of Y).
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float4* __restrict__ part, int splits, int64_t n4,
                                                          float* __restrict__ Y, int y16) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = part[i];
    for (int k = 1; k < splits; ++k) {
      const float4 b = part[k * n4 + i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    if (y16) {
      reinterpret_cast<float4*>(Y)[i] = a;
    } else {
      Y[4 * i] = a.x;
      Y[4 * i + 1] = a.y;
      Y[4 * i + 2] = a.z;
      Y[4 * i + 3] = a.w;
    }
  }
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
  if (N <= kGvMaxTokens) {                        // the GEMV: partial rows of up to kGvMaxSplit splits
    l.xs = l.count = l.partial = l.zb = 0;
    l.total = round256(static_cast<size_t>(kGvMaxSplit) * N * D_out * 4);
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

template <int NT>
cudaError_t launch_gemv_nt(dim3 grid, cudaStream_t st, const void* X, const float* s, const uint32_t* packed,
                           const float* scales, const uint8_t* zeros, int64_t D_in, int64_t D_out, int gshift, int off,
                           int R8, float* out) {
  if (zeros)
    w4a16_gemv_kernel<NT, true><<<grid, kGvThreads, 0, st>>>(
        static_cast<const uint4*>(X), reinterpret_cast<const float4*>(s), reinterpret_cast<const uint4*>(packed),
        reinterpret_cast<const float4*>(scales), zeros, D_in, D_out, gshift, off, R8, out);
  else
    w4a16_gemv_kernel<NT, false><<<grid, kGvThreads, 0, st>>>(
        static_cast<const uint4*>(X), reinterpret_cast<const float4*>(s), reinterpret_cast<const uint4*>(packed),
        reinterpret_cast<const float4*>(scales), nullptr, D_in, D_out, gshift, off, R8, out);
  return cudaGetLastError();
}

int launch_w4a16_gemv(const void* X, const float* s, const uint32_t* packed, const float* scales,
                      const uint8_t* zeros, int64_t N, int64_t D_in, int64_t D_out, int bits, int group, float* Y,
                      void* ws, int num_sms, cudaStream_t st, cudaError_t* cerr, const char** what) {
  const int64_t rows8 = D_in / 8;
  const int64_t tiles = (D_out + kGvCols - 1) / kGvCols;
  // About eight CTAs per SM over column tiles x splits; at least 8 k8 rows
  // (one per warp) per split.
  int64_t splits = (static_cast<int64_t>(num_sms > 0 ? num_sms : 1) * 8 + tiles / 2) / tiles;
  if (splits > rows8 / 8) splits = rows8 / 8;
  if (splits > kGvMaxSplit) splits = kGvMaxSplit;
  if (splits < 1) splits = 1;
  int64_t R8 = (rows8 + splits - 1) / splits;
  R8 = (R8 + 31) / 32 * 32;                      // whole 4-row batches for each of the 8 warps
  splits = (rows8 + R8 - 1) / R8;
  const int gshift = group == 32 ? 5 : group == 64 ? 6 : group == 128 ? 7 : 8;
  const int off = 1 << (bits - 1);
  // The GEMV stores 16-byte rows: straight into Y when there is one split and
  // Y is 16-byte aligned, else into the workspace for gemv_reduce_kernel.
  const bool y16 = (reinterpret_cast<uintptr_t>(Y) & 15u) == 0;
  float* out = splits == 1 && y16 ? Y : static_cast<float*>(ws);
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(splits));
  cudaError_t e;
  switch (N) {
    case 1: e = launch_gemv_nt<1>(grid, st, X, s, packed, scales, zeros, D_in, D_out, gshift, off, static_cast<int>(R8), out); break;
    case 2: e = launch_gemv_nt<2>(grid, st, X, s, packed, scales, zeros, D_in, D_out, gshift, off, static_cast<int>(R8), out); break;
    case 3: e = launch_gemv_nt<3>(grid, st, X, s, packed, scales, zeros, D_in, D_out, gshift, off, static_cast<int>(R8), out); break;
    case 4: e = launch_gemv_nt<4>(grid, st, X, s, packed, scales, zeros, D_in, D_out, gshift, off, static_cast<int>(R8), out); break;
    default: *what = "gemv token count"; return kEUnsupported;
  }
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "w4a16_gemv_kernel launch";
    return kECuda;
  }
  if (out != Y) {
    const int64_t n4 = N * D_out / 4;
    int64_t blocks = (n4 + 255) / 256;
    if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
    gemv_reduce_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(static_cast<const float4*>(ws),
                                                                     static_cast<int>(splits), n4, Y, y16 ? 1 : 0);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      *cerr = e;
      *what = "gemv_reduce_kernel launch";
      return kECuda;
    }
  }
  return kOk;
}

}  // namespace

size_t w4a16_scratch_bytes(int64_t N, int64_t D_in, int64_t D_out, int64_t zrows) {
  return w4_layout(N, D_in, D_out, zrows).total;
}

int launch_w4a16(const void* X, const float* s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                 int64_t N, int64_t D_in, int64_t D_out, int bits, int group, float* Y, void* ws, int num_sms,
                 int* status, uint64_t timeout_ns, cudaStream_t st, cudaError_t* cerr, const char** what) {
  *cerr = cudaSuccess;
  if (N <= kGvMaxTokens)
    return launch_w4a16_gemv(X, s, packed, scales, zeros, N, D_in, D_out, bits, group, Y, ws, num_sms, st, cerr,
                             what);
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
