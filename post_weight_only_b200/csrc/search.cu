// search.cu -- the fused per-alpha loss GEMM of the AWQ scale search.
//
// For one linear layer Y = X W (X: N x D_in bf16, W: D_in x D_out) and every
// alpha on the grid this kernel evaluates
//     L(alpha) = || X S^-1 Q(S W) - X W ||^2        S = diag(a^alpha)
// (compassingai.com AWQ concept page, flow step 4c; mudrobot.github.io AWQ
// notes, "searching the optimal scale") on the tensor cores, reducing the
// squared error in the epilogue so that no output matrix and no dequantised
// weight ever reaches global memory.
//
// Two loss forms, identical in exact arithmetic:
//   error form (default)  the MMA operand is the weight error itself,
//       E = S^-1 Q(S W) - W,  E_kn = (q_kn - w'_kn / delta) * delta / s_k,
//       and L = ||X E||^2.  The quantiser's rounding residual
//       e' = q - w'/delta (in [-1/2, 1/2]) arrives as an 8-bit fixed-point code
//       per weight (made once per alpha by quant.cu) and E is formed in fp32
//       and rounded to bf16 once, so the bf16 rounding error is relative to E,
//       not to W.
//   reference form        the literal two-product form: the reference output
//       X W is computed once per tile by the same GEMM (bf16 W), parked in a
//       per-CTA scratch that stays in L2, and every alpha pass computes
//       X S^-1 Q(S W) from 4-bit codes and subtracts it in the epilogue.
//
// Orientation.  The MMA computes the transposed product D = A B with
//   A = weight tile (M = 256 output columns of the layer, K = D_in),
//   B = X^T tile    (N = 256 calibration tokens,          K = D_in),
// so that the operand that changes with alpha is the A operand, which
// tcgen05.mma reads straight from tensor memory.  Weight producer warps decode
// the per-alpha codes into bf16 values and store them into TMEM with
// tcgen05.st: the produced tile never touches shared memory, which stays free
// for the TMA stream of X.  Each produced weight is reused by 256 tokens.
//
// CTA pairs.  Two CTAs of a cluster run one tcgen05.mma.cta_group::2 (M 256,
// N 256, K 16), issued by the leader: each CTA holds 128 of the 256 weight
// columns in its TMEM (A operand and accumulator) and stages 128 of the 256
// tokens of the X tile in its shared memory (B operand), which the pair's
// tensor cores share.  So each SM streams half an X tile per stage, which
// keeps the shared-memory pipe (TMA writes, MMA reads, producer reads) well
// below saturation.  Both CTAs' X copies complete on the leader's barrier; the
// producers and epilogues of both CTAs arrive on the leader's barriers; the
// leader's commits arrive on the barriers of both CTAs (multicast).  No TMA
// load uses cluster multicast.
//
// Roles (480 threads per CTA, one CTA per SM, persistent):
//   warp 0      TMA: this CTA's X half-tile (128 tokens x 64 k, 128B-swizzled)
//   warp 14     TMA of the side data (codes, deltas, 1/s; the bf16 weights for
//               a reference pass), on its own, deeper ring
//   warp 1      allocates TMEM (pair); lane 0 of the leader issues the MMAs
//   warps 2-9   weight producers: two per TMEM lane quarter, taking even and
//               odd stages in turn, so that one's tcgen05.st overlaps the
//               other's decoding
//   warps 10-13 epilogue, one per TMEM lane quarter (256 tokens each)
// TMEM: columns [0, 256) accumulator, [256, 512) eight (error form) or four
// 32-column A stages.
//
// Work: a unit is (128 output columns) x (256 tokens); per unit the passes
// are the alphas (after the reference pass in the reference form).  Units are
// dealt round robin in whole waves, all CTAs advancing through alpha in step
// (so the codes of one alpha are read from HBM once and shared through L2);
// the alpha passes of the last partial wave are split evenly over all CTAs.
// The unit numbering is token-minor or weight-minor, whichever keeps the data
// that concurrent CTAs share smaller than L2.
//
// Every mbarrier wait is bounded: on a timeout the kernel records
// AWQ_ETIMEOUT in the status word, every role leaves its loop, in-flight
// copies and MMAs are waited for (again bounded) and TMEM is released.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace awq {
namespace {

constexpr int kBM = 128;                 // output columns per CTA (TMEM lanes); a pair covers 256
constexpr int kPairM = 256;              // MMA M: output columns per CTA pair
constexpr int kBN = 256;                 // tokens per tile (MMA N); each CTA stages 128
constexpr int kHalfN = kBN / 2;
constexpr int kBK = 64;                  // k per stage: one 128-byte swizzle row of bf16
constexpr int kXStages = 6;              // ring of X half-tiles in shared memory
constexpr int kACol0 = 256;              // first TMEM column of the A stages
constexpr int kTmemCols = 512;
constexpr int kXStageBytes = kHalfN * kBK * 2;   // 16 KiB: this CTA's 128 tokens x 64 k
constexpr int kAuxCodesOff = 0;                  // error form [16][128] u32, reference form [8][128] u32
constexpr int kAuxDeltaOff = 8192;               // [<=2][128] f32
constexpr int kAuxROff = 9216;                   // [64] f32 (1/s of the stage's rows)
constexpr int kThreads = 480;
constexpr int kEpiWarps = 4;
constexpr int kProdWarps = 8;
constexpr int kProdPerStage = 4;         // producer warps of one CTA that fill one stage
constexpr int kAuxTmaWarp = 14;
constexpr uint16_t kPairMask = 0x3;

// The weight (A operand) ring is decoupled from the X ring and deeper: the
// side data of a stage can only be requested once the MMA has released the
// stage, and it then goes through a TMA round trip and the producers' decode
// before the MMA needs it again, so that ring holds eight stages (TMEM columns
// 256..511) in the error form.  The reference form's reference pass needs
// 16 KiB of side data per stage, so it keeps four.
template <int kForm>
struct Ring {
  static constexpr int kAStages = kForm == kFormError ? 8 : 4;
  static constexpr int kAuxBytes = kForm == kFormError ? 10240 : 16384;
  static constexpr int kSmemBytes = kXStages * kXStageBytes + kAStages * kAuxBytes + 1024 /*barriers*/ + 1024 /*align*/;
};

enum Site { kSiteTmaEmpty = 1, kSiteMmaAccEmpty, kSiteMmaFull, kSiteMmaAReady, kSiteProdFull, kSiteEpiAccFull,
            kSiteDrainTma, kSiteDrainMma, kSiteSelfTest };

struct Params {
  int N, D_in, D_out, A, group, off_bf16x2;
  int Tt, Wt, U, KB, gpb, gemm_only, weight_minor;
  float* yref;
  float* partial;
  float* y_out;
  int* status;
  unsigned long long timeout_ns;
};

struct Segment {
  int u, a0, a1;     // unit, alpha range [a0, a1)
};

// The sequence of segments a CTA pair processes.  Every role of both CTAs
// walks the same sequence, so ring positions and barrier phases agree.
struct Schedule {
  int U, A, G, c;
  int full_waves, head;
  long long j, te;
  int i;
  __device__ Schedule(int U_, int A_, int G_, int c_) : U(U_), A(A_), G(G_), c(c_), i(0) {
    if (A == 0) {                       // reference output only: whole units round robin
      full_waves = (U - c + G - 1) / G;
      head = U;
      j = te = 0;
    } else {
      full_waves = U / G;
      head = full_waves * G;
      const long long items = static_cast<long long>(U - head) * A;
      j = items * c / G;
      te = items * (c + 1) / G;
    }
  }
  __device__ bool next(Segment& s) {
    if (i < full_waves) {
      s.u = c + i * G;
      s.a0 = 0;
      s.a1 = A;
      ++i;
      return true;
    }
    if (j < te) {
      s.u = head + static_cast<int>(j / A);
      s.a0 = static_cast<int>(j % A);
      const long long rem = te - j;
      s.a1 = static_cast<int>(rem < static_cast<long long>(A - s.a0) ? s.a0 + rem : A);
      j += s.a1 - s.a0;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ void unit_tiles(const Params& p, int u, int& wt, int& tt) {
  if (p.weight_minor) {
    tt = u / p.Wt;
    wt = u % p.Wt;
  } else {
    wt = u / p.Tt;
    tt = u % p.Tt;
  }
}

// Passes of a segment: the reference form starts with the reference pass,
// numbered a0 - 1.
template <int kForm>
__device__ __forceinline__ int first_pass(const Segment& sg) {
  return kForm == kFormReference ? sg.a0 - 1 : sg.a0;
}
template <int kForm>
__device__ __forceinline__ bool is_ref_pass(const Segment& sg, int pass) {
  return kForm == kFormReference && pass == sg.a0 - 1;
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }
__device__ __forceinline__ __nv_bfloat162 as_bf16x2(uint32_t v) { return *reinterpret_cast<__nv_bfloat162*>(&v); }

// One bf16 pair of reference-form A-operand values, rows (k, k+1) of one
// column: v holds the two 4-bit codes as bf16 values 128 + u (exact small
// integers), off2 the code offset 128 + 2^(b-1) in both halves, so v - off2 is
// the signed code q exactly; c = fl32(delta / s_k) is rounded to bf16 once per
// element and q * c once more.  No rounding error is shared by a whole row or
// a whole group of the operand.
__device__ __forceinline__ uint32_t decode_pair(uint32_t v, uint32_t off2, float c_lo, float c_hi) {
  const __nv_bfloat162 q = __hsub2(as_bf16x2(v), as_bf16x2(off2));
  return bf16x2_bits(__hmul2(q, __floats2bfloat162_rn(c_lo, c_hi)));
}

template <int kForm>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    search_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWp,
                  const __grid_constant__ CUtensorMap tmCodes, const __grid_constant__ CUtensorMap tmDelta,
                  const __grid_constant__ CUtensorMap tmR, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kAS = Ring<kForm>::kAStages;
  constexpr int kAuxStageBytes = Ring<kForm>::kAuxBytes;
  uint8_t* xs = smem;
  uint8_t* aux = smem + kXStages * kXStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux + kAS * kAuxStageBytes);
  // Every CTA holds the full set; xfull, aready and acc_empty are used in the
  // leader (rank 0) only, where both CTAs' copies and warps arrive.
  uint64_t* xfull = bars;                   // both X halves landed (leader)       [kXStages]
  uint64_t* xempty = xfull + kXStages;      // MMAs done with the X stage          [kXStages]
  uint64_t* afull = xempty + kXStages;      // this CTA's side data landed         [kAS]
  uint64_t* aready = afull + kAS;           // both CTAs' A stages written (leader) [kAS]
  uint64_t* aempty = aready + kAS;          // MMAs done with the A stage          [kAS]
  uint64_t* acc_full = aempty + kAS;
  uint64_t* acc_empty = acc_full + 1;       // both CTAs' epilogues drained (leader)
  uint64_t* mma_done = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < kAS; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aready[s], 2 * kProdPerStage);
      mbar_init(&aempty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpiWarps);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    if (kForm == kFormReference) tma_prefetch_desc(&tmWp);
    if (!p.gemm_only) {
      tma_prefetch_desc(&tmCodes);
      tma_prefetch_desc(&tmDelta);
      tma_prefetch_desc(&tmR);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();       // barriers of both CTAs initialised, TMEM of both allocated
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;
  bool aborted = false;

  if (warp == 0 || warp == kAuxTmaWarp) {
    // ------------------------------------------------------------ TMA: X half-tiles (warp 0), side data (warp 14)
    if (lane == 0) {
      const bool is_x = warp == 0;
      const int nst = is_x ? kXStages : kAS;
      uint64_t* emptyb = is_x ? xempty : aempty;
      Schedule sch(p.U, p.A, npairs, pair);
      Segment sg;
      uint32_t it = 0;
      int last_round[kAS > kXStages ? kAS : kXStages];
#pragma unroll
      for (int s = 0; s < (kAS > kXStages ? kAS : kXStages); ++s) last_round[s] = -1;
      bool ok = true;
      const uint32_t ref_bytes = 32 * kBM * 4;
      const uint32_t code_rows = kForm == kFormError ? kBK / 4 : kBK / 8;
      const uint32_t alpha_bytes = code_rows * kBM * 4 + p.gpb * kBM * 4 + kBK * 4;
      while (ok && sch.next(sg)) {
        int wt, tt;
        unit_tiles(p, sg.u, wt, tt);
        const int col0 = wt * kPairM + static_cast<int>(rank) * kBM;     // this CTA's weight columns
        const int tok0 = tt * kBN + static_cast<int>(rank) * kHalfN;     // this CTA's tokens
        for (int pass = first_pass<kForm>(sg); ok && pass < sg.a1; ++pass) {
          const bool ref = is_ref_pass<kForm>(sg, pass);
          for (int kb = 0; kb < p.KB; ++kb, ++it) {
            const int s = it % nst;
            const uint32_t r = it / nst;
            if (!wait_bounded(&emptyb[s], (r & 1) ^ 1, abort_flag, p.status, kSiteTmaEmpty, tmo)) {
              ok = false;
              break;
            }
            if (is_x) {
              // Both halves complete on the leader's barrier, which expects the
              // bytes of both.
              if (leader) mbar_arrive_expect_tx(&xfull[s], 2 * kXStageBytes);
              tma_load_2d_pair(xs + s * kXStageBytes, &tmX, mapa_shared(smem_u32(&xfull[s]), 0), kb * kBK, tok0);
            } else {
              uint8_t* ad = aux + s * kAuxStageBytes;
              if (ref) {
                mbar_arrive_expect_tx(&afull[s], ref_bytes);
                tma_load_2d(ad, &tmWp, &afull[s], col0, kb * (kBK / 2));
              } else {
                mbar_arrive_expect_tx(&afull[s], alpha_bytes);
                tma_load_3d(ad + kAuxCodesOff, &tmCodes, &afull[s], col0, kb * code_rows, pass);
                tma_load_3d(ad + kAuxDeltaOff, &tmDelta, &afull[s], col0, (kb * kBK) / p.group, pass);
                tma_load_2d(ad + kAuxROff, &tmR, &afull[s], kb * kBK, pass);
              }
            }
            last_round[s] = static_cast<int>(r);
          }
        }
      }
      aborted = !ok;
      // Never leave the CTA with a copy still writing into shared memory.
      volatile int no_abort = 0;
      if (!is_x) {
        for (int s = 0; s < nst; ++s)
          if (last_round[s] >= 0) wait_bounded(&afull[s], last_round[s] & 1, &no_abort, p.status, kSiteDrainTma, tmo);
      } else if (leader) {
        // The leader's xfull counts both halves of every round it armed.
        for (int s = 0; s < nst; ++s)
          if (last_round[s] >= 0)
            wait_bounded(&xfull[s], last_round[s] & 1, &no_abort, p.status, kSiteDrainTma, tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      Schedule sch(p.U, p.A, npairs, pair);
      Segment sg;
      uint32_t it = 0, acc_it = 0;
      const uint32_t idesc = idesc_bf16_f32(kPairM, kBN);
      bool ok = true;
      while (ok && sch.next(sg)) {
        for (int pass = first_pass<kForm>(sg); ok && pass < sg.a1; ++pass, ++acc_it) {
          if (!wait_bounded(acc_empty, (acc_it & 1) ^ 1, abort_flag, p.status, kSiteMmaAccEmpty, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = 0; kb < p.KB; ++kb, ++it) {
            const int sx = it % kXStages, sa = it % kAS;
            if (!wait_bounded(&xfull[sx], (it / kXStages) & 1, abort_flag, p.status, kSiteMmaFull, tmo) ||
                !wait_bounded(&aready[sa], (it / kAS) & 1, abort_flag, p.status, kSiteMmaAReady, tmo)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t bdesc = sw128_kmajor_desc(smem_u32(xs + sx * kXStageBytes));
            const uint32_t a_tmem = tbase + kACol0 + sa * (kBK / 2);
#pragma unroll
            for (int j = 0; j < kBK / 16; ++j)
              mma_ts_f16_pair(tbase, a_tmem + j * 8, bdesc + 2 * j, idesc, (kb | j) != 0 ? 1u : 0u);
            mma_commit_pair_multicast(&xempty[sx], kPairMask);
            mma_commit_pair_multicast(&aempty[sa], kPairMask);
          }
          if (!ok) break;
          mma_commit_pair_multicast(acc_full, kPairMask);
        }
      }
      aborted = !ok;
      // All MMAs (which write both CTAs' TMEM) must have finished before
      // either CTA releases its TMEM.
      mma_commit_pair_multicast(mma_done, kPairMask);
    }
    if (lane == 0) {
      volatile int no_abort = 0;
      wait_bounded(mma_done, 0, &no_abort, p.status, kSiteDrainMma, tmo);
    }
    __syncwarp();
  } else if (warp < 2 + kProdWarps) {
    // ------------------------------------------------------------ weight producers
    const int q = warp & 3;
    const uint32_t parity = static_cast<uint32_t>((warp - 2) >> 2);   // this warp fills stages it % 2 == parity
    const int nl = q * 32 + lane;
    Schedule sch(p.U, p.A, npairs, pair);
    Segment sg;
    uint32_t it = 0;
    bool ok = true;
    const uint32_t off2 = static_cast<uint32_t>(p.off_bf16x2);
    const bool two_groups = p.gpb == 2;   // group 32: a 64-k stage spans two groups
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(q * 32) << 16) + kACol0;
    const uint32_t aready_leader = mapa_shared(smem_u32(aready), 0);
    while (ok && sch.next(sg)) {
      for (int pass = first_pass<kForm>(sg); ok && pass < sg.a1; ++pass) {
        const bool ref = is_ref_pass<kForm>(sg, pass);
        for (int kb = 0; kb < p.KB; ++kb, ++it) {
          if ((it & 1u) != parity) continue;
          const int s = it % kAS;
          const uint32_t r = it / kAS;
          // The tcgen05.st below is warp-collective: take the outcome of the
          // wait as a warp, never split the warp on a timeout.
          const bool got = wait_bounded(&afull[s], r & 1, abort_flag, p.status, kSiteProdFull, tmo);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* ad = aux + s * kAuxStageBytes;
          const uint32_t* cw = reinterpret_cast<const uint32_t*>(ad + kAuxCodesOff);
          const float* dl = reinterpret_cast<const float*>(ad + kAuxDeltaOff);
          const float4* rf = reinterpret_cast<const float4*>(ad + kAuxROff);
          const uint32_t st_addr = lane_addr + s * (kBK / 2);
          if (ref) {
            uint32_t out[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) out[i] = cw[i * kBM + nl];
            tmem_st32(st_addr, out);
          } else if (kForm == kFormError) {
            // Word j holds the 8-bit codes u = 256 e' + 128 of rows 4j .. 4j+3.
            // A byte permute places u in the mantissa of the float 2^23 + u;
            // subtracting 2^23 + 128 leaves k = 256 e' exactly, and
            // E = k * (delta 2^-8 / s_k) is formed in fp32 (packed pairs) and
            // rounded to bf16 once.  Two 16-column halves keep the live set
            // small.
            const float2 bias = make_float2(-8388736.0f, -8388736.0f);    // -(2^23 + 128)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t out[16];
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) {
                const int j = hh * 8 + jj;
                const uint32_t word = cw[j * kBM + nl];
                const float d = dl[(two_groups ? hh : 0) * kBM + nl];
                const float4 rv = rf[j];
                const float2 c01 = __fmul2_rn(make_float2(d, d), make_float2(rv.x, rv.y));
                const float2 c23 = __fmul2_rn(make_float2(d, d), make_float2(rv.z, rv.w));
                const float2 k01 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(word, 0x4B000000u, 0x7440u)),
                                                          __uint_as_float(__byte_perm(word, 0x4B000000u, 0x7441u))),
                                              bias);
                const float2 k23 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(word, 0x4B000000u, 0x7442u)),
                                                          __uint_as_float(__byte_perm(word, 0x4B000000u, 0x7443u))),
                                              bias);
                const float2 e01 = __fmul2_rn(k01, c01);
                const float2 e23 = __fmul2_rn(k23, c23);
                out[2 * jj] = bf16x2_bits(__floats2bfloat162_rn(e01.x, e01.y));
                out[2 * jj + 1] = bf16x2_bits(__floats2bfloat162_rn(e23.x, e23.y));
              }
              tmem_st16(st_addr + hh * 16, out);
            }
          } else {
            // Word j holds the 4-bit codes of rows 8j .. 8j+7 in the order
            // 0,2,4,6,1,3,5,7, so that shifting by 4i and masking 0x000F000F
            // yields rows (2i, 2i+1) as the two halves of a bf16 pair.
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t out[16];
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                const int j = hh * 4 + jj;
                const uint32_t word = cw[j * kBM + nl];
                const float d = dl[(two_groups ? hh : 0) * kBM + nl];
                const float4 r0 = rf[2 * j], r1 = rf[2 * j + 1];
                const float c[8] = {__fmul_rn(d, r0.x), __fmul_rn(d, r0.y), __fmul_rn(d, r0.z), __fmul_rn(d, r0.w),
                                    __fmul_rn(d, r1.x), __fmul_rn(d, r1.y), __fmul_rn(d, r1.z), __fmul_rn(d, r1.w)};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const uint32_t v = ((word >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
                  out[4 * jj + i] = decode_pair(v, off2, c[2 * i], c[2 * i + 1]);
                }
              }
              tmem_st16(st_addr + hh * 16, out);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(aready_leader + s * 8);
        }
      }
    }
    aborted = !ok;
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    Schedule sch(p.U, p.A, npairs, pair);
    Segment sg;
    uint32_t acc_it = 0;
    bool ok = true;
    float4* yref = reinterpret_cast<float4*>(p.yref + static_cast<size_t>(blockIdx.x) * (kBM * kBN));
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    const int H = p.Tt;
    while (ok && sch.next(sg)) {
      int wt, tt;
      unit_tiles(p, sg.u, wt, tt);
      const int n = wt * kPairM + static_cast<int>(rank) * kBM + nl;
      for (int pass = first_pass<kForm>(sg); ok && pass < sg.a1; ++pass, ++acc_it) {
        const bool ref = is_ref_pass<kForm>(sg, pass);
        const bool got = wait_bounded(acc_full, acc_it & 1, abort_flag, p.status, kSiteEpiAccFull, tmo);
        if (!__all_sync(0xffffffffu, got)) {   // tcgen05.ld is warp-collective
          ok = false;
          break;
        }
        tc_fence_after();
        if (kForm == kFormError) {
          // Four 64-column quarters: load both chunks of a quarter, then square
          // and sum them; release the accumulator after the last load.  (A
          // thread has at most 128 registers, too few to hold more than 64
          // columns besides the rest of its state.)
          float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 1
          for (int h4 = 0; h4 < 4; ++h4) {
            uint32_t v[2][32];
            tmem_ld32(lane_addr + h4 * 64, v[0]);
            tmem_ld32(lane_addr + h4 * 64 + 32, v[1]);
            tmem_wait_ld();
            if (h4 == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x0 = __uint_as_float(v[0][e]), x1 = __uint_as_float(v[1][e]);
              s0 = fmaf(x0, x0, s0);
              s1 = fmaf(x1, x1, s1);
            }
          }
          if (n < p.D_out) p.partial[(static_cast<size_t>(pass) * H + tt) * p.D_out + n] = s0 + s1;
        } else if (ref) {
#pragma unroll 1
          for (int c = 0; c < kBN / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(lane_addr + c * 32, v);
            tmem_wait_ld();
            if (p.gemm_only) {
              const int t0 = tt * kBN + c * 32;
              if (n < p.D_out) {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                  if (t0 + e < p.N) p.y_out[static_cast<size_t>(t0 + e) * p.D_out + n] = __uint_as_float(v[e]);
              }
            } else {
              // [token chunk of 4][column][4]: a warp stores 512 contiguous bytes
              float4* dst = yref + (c * 8) * kBM + nl;
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                dst[jj * kBM] = make_float4(__uint_as_float(v[4 * jj]), __uint_as_float(v[4 * jj + 1]),
                                            __uint_as_float(v[4 * jj + 2]), __uint_as_float(v[4 * jj + 3]));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
        } else {
          float sum = 0.0f;
#pragma unroll 1
          for (int c = 0; c < kBN / 32; ++c) {
            const float4* src = yref + (c * 8) * kBM + nl;
            float4 y[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) y[jj] = src[jj * kBM];
            uint32_t v[32];
            tmem_ld32(lane_addr + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const float d0 = __uint_as_float(v[4 * jj]) - y[jj].x;
              const float d1 = __uint_as_float(v[4 * jj + 1]) - y[jj].y;
              const float d2 = __uint_as_float(v[4 * jj + 2]) - y[jj].z;
              const float d3 = __uint_as_float(v[4 * jj + 3]) - y[jj].w;
              sum = fmaf(d0, d0, sum);
              sum = fmaf(d1, d1, sum);
              sum = fmaf(d2, d2, sum);
              sum = fmaf(d3, d3, sum);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
          if (n < p.D_out) p.partial[(static_cast<size_t>(pass) * H + tt) * p.D_out + n] = sum;
        }
      }
    }
    aborted = !ok;
  }

  // After a timeout a copy issued by this CTA may still be landing in this
  // CTA's shared memory with no barrier here to show it: give it time (a
  // TMA round trip is a few microseconds) before the pair goes away.
  if (aborted || *abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();       // no CTA of the pair leaves while the other may still use its memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tbase, kTmemCols);
}

__global__ void wait_timeout_selftest_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the wait must give up by itself.
    const bool ok = wait_bounded(&bar, 0, &abort_flag, status, kSiteSelfTest, timeout_ns);
    if (ok) atomicExch(status, -1);   // impossible unless the barrier logic is broken
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int kForm>
cudaError_t launch_form(int grid, const CUtensorMap& mX, const CUtensorMap& mWp, const CUtensorMap& mC,
                        const CUtensorMap& mD, const CUtensorMap& mR, const Params& p, cudaStream_t st) {
  static int attr_set_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_set_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(search_kernel<kForm>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Ring<kForm>::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set_device = dev;
  }
  search_kernel<kForm><<<grid, kThreads, Ring<kForm>::kSmemBytes, st>>>(mX, mWp, mC, mD, mR, p);
  return cudaGetLastError();
}

}  // namespace

int search_token_tiles(int N) { return (N + kBN - 1) / kBN; }

// Number of CTAs (two per pair): one pair per unit of work, at most one CTA
// per SM.
int search_grid_size(const SearchShape& sh, int num_sms) {
  const long long U = static_cast<long long>((sh.D_out + kPairM - 1) / kPairM) * search_token_tiles(sh.N);
  const long long work = sh.A > 0 ? U * sh.A : U;
  const long long pairs = num_sms / 2;
  return 2 * static_cast<int>(work < pairs ? work : pairs);
}

int launch_search(const SearchShape& sh, const SearchBuffers& b, int grid, uint64_t timeout_ns, cudaStream_t st,
                  cudaError_t* cerr, const char** what) {
  *cerr = cudaSuccess;
  const bool gemm_only = sh.A == 0;
  const int form = gemm_only ? kFormReference : sh.form;
  CUtensorMap mX, mWp, mC, mD, mR;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(sh.D_in), static_cast<uint64_t>(sh.N)};
    const uint64_t str[1] = {static_cast<uint64_t>(sh.D_in) * 2};
    const uint32_t box[2] = {kBK, kHalfN};
    if (!make_map(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, b.X, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) {
      *what = "tensor map for X";
      return kECuda;
    }
  }
  if (form == kFormReference) {
    const uint64_t dims[2] = {static_cast<uint64_t>(sh.D_out), static_cast<uint64_t>(sh.D_in / 2)};
    const uint64_t str[1] = {static_cast<uint64_t>(sh.D_out) * 4};
    const uint32_t box[2] = {kBM, kBK / 2};
    if (!make_map(&mWp, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, b.w_pairs, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE)) {
      *what = "tensor map for the bf16 weights";
      return kECuda;
    }
  } else {
    mWp = mX;   // never read by the error form
  }
  const int gpb = sh.group >= kBK ? 1 : kBK / sh.group;
  if (!gemm_only) {
    {
      const uint64_t per_word = form == kFormError ? 4 : 8;       // weights per 32-bit code word
      const uint64_t rows = static_cast<uint64_t>(sh.D_in) / per_word;
      const uint64_t dims[3] = {static_cast<uint64_t>(sh.D_out), rows, static_cast<uint64_t>(sh.A)};
      const uint64_t str[2] = {static_cast<uint64_t>(sh.D_out) * 4, static_cast<uint64_t>(sh.D_out) * 4 * rows};
      const uint32_t box[3] = {kBM, static_cast<uint32_t>(kBK / per_word), 1};
      if (!make_map(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, b.codes, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE)) {
        *what = "tensor map for the codes";
        return kECuda;
      }
    }
    {
      const uint64_t G = static_cast<uint64_t>(sh.D_in / sh.group);
      const uint64_t dims[3] = {static_cast<uint64_t>(sh.D_out), G, static_cast<uint64_t>(sh.A)};
      const uint64_t str[2] = {static_cast<uint64_t>(sh.D_out) * 4, static_cast<uint64_t>(sh.D_out) * 4 * G};
      const uint32_t box[3] = {kBM, static_cast<uint32_t>(gpb), 1};
      if (!make_map(&mD, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, b.delta, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE)) {
        *what = "tensor map for the deltas";
        return kECuda;
      }
    }
    {
      const uint64_t dims[2] = {static_cast<uint64_t>(sh.D_in), static_cast<uint64_t>(sh.A)};
      const uint64_t str[1] = {static_cast<uint64_t>(sh.D_in) * 4};
      const uint32_t box[2] = {kBK, 1};
      if (!make_map(&mR, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, b.r_tab, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE)) {
        *what = "tensor map for 1/s";
        return kECuda;
      }
    }
  } else {
    mC = mWp;
    mD = mWp;
    mR = mWp;
  }
  Params p;
  p.N = sh.N;
  p.D_in = sh.D_in;
  p.D_out = sh.D_out;
  p.A = sh.A;
  p.group = sh.group;
  {
    // Offset of the integer codes as bf16 values: 128 + 2^(b-1) for the 4-bit
    // codes, 128 + 64 for the 7-bit residual codes.
    const int bias = form == kFormError ? 64 : (1 << (sh.bits > 0 ? sh.bits - 1 : 0));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(128.0f + static_cast<float>(bias)));
    p.off_bf16x2 = static_cast<int>(h | (h << 16));
  }
  p.Tt = search_token_tiles(sh.N);
  p.Wt = (sh.D_out + kPairM - 1) / kPairM;
  p.U = p.Wt * p.Tt;
  p.KB = (sh.D_in + kBK - 1) / kBK;
  p.gpb = gpb;
  p.gemm_only = gemm_only ? 1 : 0;
  {
    // Concurrent pairs (one wave) either share token tiles (weight-minor
    // numbering: all of X stays hot, plus the codes of a few weight tiles)
    // or weight tiles (token-minor: the codes of one alpha stay hot, plus a
    // few token tiles of X).  Keep the smaller working set.
    const double x_bytes = 2.0 * sh.N * sh.D_in;
    const double codes_per_alpha = (form == kFormError ? 1.0 : 0.5) * sh.D_in * static_cast<double>(sh.D_out);
    p.weight_minor = (!gemm_only && x_bytes > codes_per_alpha) ? 1 : 0;
  }
  p.yref = b.yref;
  p.partial = b.partial;
  p.y_out = b.y_out;
  p.status = b.status;
  p.timeout_ns = timeout_ns;

  cudaError_t e = form == kFormError ? launch_form<kFormError>(grid, mX, mWp, mC, mD, mR, p, st)
                                     : launch_form<kFormReference>(grid, mX, mWp, mC, mD, mR, p, st);
  if (e != cudaSuccess) {
    *cerr = e;
    *what = "search_kernel launch";
    return kECuda;
  }
  return kOk;
}

cudaError_t launch_wait_timeout_selftest(int* status, uint64_t timeout_ns, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace awq
