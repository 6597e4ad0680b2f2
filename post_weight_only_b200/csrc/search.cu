// search.cu -- the fused per-alpha loss GEMMs of the AWQ scale search.
//
// For one linear layer Y = X W (X: N x D_in bf16, W: D_in x D_out) and every
// alpha on the grid this kernel evaluates
//     L(alpha) = || X S^-1 Q(S W) - X W ||^2        S = diag(a^alpha)
// (compassingai.com AWQ concept page, flow step 4c; mudrobot.github.io AWQ
// notes, "searching the optimal scale") on the tensor cores, reducing the
// squared error in the epilogue so that no output matrix ever reaches global
// memory.
//
// Two loss forms, identical in exact arithmetic:
//   error form (default)  the MMA operand is the weight error itself,
//       E = S^-1 Q(S W) - W,  E_kn = (q_kn - w'_kn / delta) * delta / s_k,
//       formed in fp32 from the quantiser's exact rounding residual and
//       rounded to bf16 once (quant.cu), and L = ||X E||^2: the bf16 rounding
//       error is relative to E, not to W.
//   reference form        the literal two-product form: the reference output
//       X W is computed once per tile by the same GEMM (bf16 W), parked in a
//       per-CTA scratch that stays in L2, and every alpha pass computes
//       X S^-1 Q(S W) and subtracts it in the epilogue.
// The per-alpha operands (bf16, [alpha][D_out][D_in]) are written by the
// operand pre-pass in quant.cu; the per-column sums of squares over each
// 128-token half-tile go to a partials array that reduce.cu sums in fp64.
//
// Orientation.  The MMA computes D = A B^T with
//   A = operand tile (M = 256 output columns of the layer, K = D_in),
//   B = X tile       (N = 256 calibration tokens,          K = D_in),
// both K-major, so that D[n][t] = (X op)[t][n]: TMEM lane = output column,
// TMEM column = token.
//
// CTA pairs.  Two CTAs of a cluster run one tcgen05.mma.cta_group::2 (M 256,
// N 256, K 16), issued by the leader.  Each CTA stages 128 of the 256 operand
// rows and 128 of the 256 tokens per 64-wide k step in its own shared memory
// (16 KiB each, 128-byte swizzled, by TMA) and holds 128 accumulator rows in
// its TMEM; the pair's tensor cores share both CTAs' halves.  The copies of
// both CTAs complete on the leader's barrier; the epilogues of both CTAs
// arrive on the leader's barriers; the leader's commits arrive on the
// barriers of both CTAs (multicast).  No TMA load uses cluster multicast.
//
// Roles (320 threads per CTA, one CTA per SM, persistent):
//   warp 0      TMA producer (one lane): operand and X half-tiles
//   warp 1      allocates TMEM (pair); lane 0 of the leader issues the MMAs
//   warps 2-9   epilogue: warp w reads TMEM lane quarter w % 4 and token half
//               (w - 2) / 4 of the accumulator
// TMEM: two 256-column accumulators, so that the epilogue of one pass runs
// under the MMAs of the next.
//
// Work: a unit is (256 output columns) x (256 tokens) for a pair; per unit the
// passes are the alphas (after the reference pass in the reference form).
// Units are dealt round robin in whole waves, all pairs advancing through
// alpha in step: the producers meet at every pass boundary of the full waves
// (a soft barrier on a global counter, see pass_sync_wait), so that the pairs
// sharing an operand tile read it at about the same time and it is fetched
// from HBM about once and shared through L2.  The alpha passes of the last
// partial wave are dealt round robin over all pairs, alpha-major (see
// Schedule).  Units are numbered in token blocks sized to L2 (see unit_tiles
// and search_token_block).  The TMA loads mark X tiles evict-last and
// operand tiles evict-first in L2.
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

constexpr int kBM = 128;                 // operand rows per CTA (TMEM lanes); a pair covers 256
constexpr int kPairM = 256;              // MMA M: output columns per CTA pair
constexpr int kBN = 256;                 // tokens per tile (MMA N); each CTA stages 128
constexpr int kHalfN = kBN / 2;
constexpr int kBK = 64;                  // k per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 6;
constexpr int kTileBytes = kBM * kBK * 2;        // 16 KiB: 128 rows x 64 k (operand half or X half)
constexpr int kStageBytes = 2 * kTileBytes;
constexpr int kAccCols = kBN;                    // fp32 accumulator columns per buffer
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*barriers*/ + 1024 /*align*/;
constexpr uint16_t kPairMask = 0x3;
// L2 budget for the X tiles of one token block of the unit order.
constexpr long long kXBlockBudgetBytes = 64ll << 20;
static_assert(kHalfN == kBM, "operand and X half-tiles share one box shape");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

enum Site { kSiteTmaEmpty = 1, kSiteMmaAccEmpty, kSiteMmaFull, kSiteEpiAccFull, kSiteDrainTma, kSiteDrainMma,
            kSiteSelfTest };

struct Params {
  int N, D_in, D_out, A;
  int Tt, Wt, U, KB, H, gemm_only;
  int tb;                     // token tiles per token block of the unit order (see unit_tiles)
  unsigned* sync;             // pass counter of the full waves (see pass_sync_wait), or null
  const uint16_t* op;         // Gram form: the operand E [A][D_out][D_in], read by the epilogue
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
// The (unit, alpha) passes of the last partial wave are shared out evenly
// over all pairs: when alpha_major, numbered alpha-major and dealt round
// robin, one pass per segment, so that at any time the pairs work on one or
// two alphas and each alpha's operand tiles are fetched about once; else as
// contiguous runs of the unit-major numbering (segments of consecutive alphas
// of one unit: the reference form, whose segments each start with a
// reference pass).
struct Schedule {
  int U, A, G, c;
  int full_waves, head;
  long long j, te;
  int i;
  bool alpha_major;
  __device__ Schedule(int U_, int A_, int G_, int c_, bool am)
      : U(U_), A(A_), G(G_), c(c_), i(0), alpha_major(am) {
    if (A == 0) {                       // reference output only: whole units round robin
      full_waves = (U - c + G - 1) / G;
      head = U;
      j = te = 0;
    } else {
      full_waves = U / G;
      head = full_waves * G;
      const long long items = static_cast<long long>(U - head) * A;
      if (alpha_major) {                // every G-th pass: all pairs on the same alpha or two
        j = c;
        te = items;
      } else {
        j = items * c / G;
        te = items * (c + 1) / G;
      }
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
    if (j < te && alpha_major) {
      const int rem = U - head;
      s.u = head + static_cast<int>(j % rem);
      s.a0 = static_cast<int>(j / rem);
      s.a1 = s.a0 + 1;
      j += G;
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

// The producers of all CTAs keep their passes of the full waves in step: at
// the start of pass q (q >= 1) each one adds 1 to *sync (it has issued every
// load of pass q - 1) and waits until all gridDim.x producers have done so.
// The pairs that share an operand tile (one weight tile, a block's token
// tiles) then read each of its k-slices within a short interval, so the
// slice is fetched from DRAM about once and served from L2 to the others;
// left to drift apart by up to a few passes, they fetched it ~10x.  The wait
// is a hint, not a dependency of the result: a producer that has waited
// kSyncPatienceNs (another kernel holding SMs that a CTA of this grid needs,
// say) stops waiting for the rest of the launch and only keeps counting.
constexpr uint64_t kSyncPatienceNs = 2000000;

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* ptr) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

// true: all producers reached `target`; false: gave up (or the CTA aborted).
__device__ bool pass_sync_wait(const unsigned* ctr, unsigned target, volatile int* abort_flag) {
  if (static_cast<int>(ld_relaxed_gpu(ctr) - target) >= 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(64);
    if (static_cast<int>(ld_relaxed_gpu(ctr) - target) >= 0) return true;
    if (*abort_flag || globaltimer_ns() - t0 > kSyncPatienceNs) return false;
  }
}

// Unit order: the token tiles are cut into blocks of tb tiles (the last block
// may be shorter); the units of one block come before the next block's,
// weight tile by weight tile, token tile fastest.  A wave of pairs then covers
// a few weight tiles across the block's token tiles: the block's X tiles stay
// in L2 through all alpha passes of the wave and the next waves of the block,
// and each alpha's operand tile is read by the wave's pairs at about the same
// time.
__device__ __forceinline__ void unit_tiles(const Params& p, int u, int& wt, int& tt) {
  const int per_block = p.tb * p.Wt;
  const int b = u / per_block;
  const int t0 = b * p.tb;
  const int tc = min(p.tb, p.Tt - t0);          // token tiles in this block
  const int r = u - b * per_block;
  wt = r / tc;
  tt = t0 + r % tc;
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

template <int kForm>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    search_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWt,
                  const __grid_constant__ CUtensorMap tmOp, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  // Every CTA holds the full set; full and acc_empty are used in the leader
  // (rank 0) only, where both CTAs' copies and warps arrive.
  uint64_t* full = bars;                    // both CTAs' halves of the stage landed (leader) [kStages]
  uint64_t* empty = full + kStages;         // MMAs done with the stage                       [kStages]
  uint64_t* acc_full = empty + kStages;     // accumulator b complete                         [2]
  uint64_t* acc_empty = acc_full + 2;       // both CTAs' epilogues drained b (leader)        [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    if (kForm == kFormReference) tma_prefetch_desc(&tmWt);
    if (!p.gemm_only) tma_prefetch_desc(&tmOp);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      Schedule sch(p.U, p.A, npairs, pair, kForm != kFormReference);
      Segment sg;
      uint32_t it = 0;
      int last_round[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last_round[s] = -1;
      bool ok = true;
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      unsigned q = 0;                   // passes of the full waves begun
      bool in_step = p.sync != nullptr;
      while (ok && sch.next(sg)) {
        int wt, tt;
        unit_tiles(p, sg.u, wt, tt);
        const int row0 = wt * kPairM + static_cast<int>(rank) * kBM;     // this CTA's output columns
        const int tok0 = tt * kBN + static_cast<int>(rank) * kHalfN;     // this CTA's tokens
        for (int pass = first_pass<kForm>(sg); ok && pass < sg.a1; ++pass) {
          const bool ref = is_ref_pass<kForm>(sg, pass);
          if (p.sync && sg.u < sch.head) {
            if (q > 0) {
              atomicAdd(p.sync, 1u);
              if (in_step) in_step = pass_sync_wait(p.sync, q * gridDim.x, abort_flag);
            }
            ++q;
          }
          for (int kb = 0; kb < p.KB; ++kb, ++it) {
            const int s = it % kStages;
            const uint32_t r = it / kStages;
            if (!wait_bounded(&empty[s], (r & 1) ^ 1, abort_flag, p.status, kSiteTmaEmpty, tmo)) {
              ok = false;
              break;
            }
            uint8_t* a_sm = smem + s * kStageBytes;
            const uint32_t fb = full_leader + s * 8;
            // All four halves (operand and X of both CTAs) complete on the
            // leader's barrier, which expects the bytes of all four.
            if (leader) mbar_arrive_expect_tx(&full[s], 2 * kStageBytes);
            if (ref)
              tma_load_2d_pair(a_sm, &tmWt, fb, kb * kBK, row0);
            else
              tma_load_3d_pair_hint(a_sm, &tmOp, fb, kb * kBK, row0, pass, l2_policy_evict_first());
            // X tiles evict-last, the operand evict-first: measured on the 70B block,
            // 9% less DRAM traffic and a 2% shorter step than with no policy
            tma_load_2d_pair_hint(a_sm + kTileBytes, &tmX, fb, kb * kBK, tok0, l2_policy_evict_last());
            last_round[s] = static_cast<int>(r);
          }
        }
      }
      aborted = !ok;
      // Never leave the pair with a copy still writing into shared memory:
      // the leader's barrier counts the bytes of both CTAs' copies.
      if (leader) {
        volatile int no_abort = 0;
        for (int s = 0; s < kStages; ++s)
          if (last_round[s] >= 0)
            wait_bounded(&full[s], last_round[s] & 1, &no_abort, p.status, kSiteDrainTma, tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      Schedule sch(p.U, p.A, npairs, pair, kForm != kFormReference);
      Segment sg;
      uint32_t it = 0, acc_it = 0;
      const uint32_t idesc = idesc_bf16_f32(kPairM, kBN);
      bool ok = true;
      while (ok && sch.next(sg)) {
        for (int pass = first_pass<kForm>(sg); ok && pass < sg.a1; ++pass, ++acc_it) {
          const uint32_t b = acc_it & 1, use = acc_it >> 1;
          if (!wait_bounded(&acc_empty[b], (use & 1) ^ 1, abort_flag, p.status, kSiteMmaAccEmpty, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tbase + b * kAccCols;
          for (int kb = 0; kb < p.KB; ++kb, ++it) {
            const int s = it % kStages;
            if (!wait_bounded(&full[s], (it / kStages) & 1, abort_flag, p.status, kSiteMmaFull, tmo)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
            const uint64_t adesc = sw128_kmajor_desc(a_addr);
            const uint64_t bdesc = sw128_kmajor_desc(a_addr + kTileBytes);
#pragma unroll
            for (int j = 0; j < kBK / 16; ++j)
              mma_ss_f16_pair(d_tmem, adesc + 2 * j, bdesc + 2 * j, idesc, (kb | j) != 0 ? 1u : 0u);
            mma_commit_pair_multicast(&empty[s], kPairMask);
          }
          if (!ok) break;
          mma_commit_pair_multicast(&acc_full[b], kPairMask);
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
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;                 // token half of the accumulator
    const int nl = q * 32 + lane;
    Schedule sch(p.U, p.A, npairs, pair, kForm != kFormReference);
    Segment sg;
    uint32_t acc_it = 0;
    bool ok = true;
    float4* yref = reinterpret_cast<float4*>(p.yref + static_cast<size_t>(blockIdx.x) * (kBM * kBN));
    const uint32_t lane_addr = tbase + (static_cast<uint32_t>(q * 32) << 16) + h * kHalfN;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    while (ok && sch.next(sg)) {
      int wt, tt;
      unit_tiles(p, sg.u, wt, tt);
      const int n = wt * kPairM + static_cast<int>(rank) * kBM + nl;
      const int hrow = 2 * tt + h;                 // partials row: this 128-token half-tile
      for (int pass = first_pass<kForm>(sg); ok && pass < sg.a1; ++pass, ++acc_it) {
        const bool ref = is_ref_pass<kForm>(sg, pass);
        const uint32_t b = acc_it & 1, use = acc_it >> 1;
        const bool got = wait_bounded(&acc_full[b], use & 1, abort_flag, p.status, kSiteEpiAccFull, tmo);
        if (!__all_sync(0xffffffffu, got)) {   // tcgen05.ld is warp-collective
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = lane_addr + b * kAccCols;
        const uint32_t release = acc_empty_leader + b * 8;
        if (kForm == kFormError) {
          // Two 64-column quarters; release the accumulator after the last load.
          float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 1
          for (int c2 = 0; c2 < kHalfN / 64; ++c2) {
            uint32_t v[2][32];
            tmem_ld32(acc + c2 * 64, v[0]);
            tmem_ld32(acc + c2 * 64 + 32, v[1]);
            tmem_wait_ld();
            if (c2 == kHalfN / 64 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(release);
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x0 = __uint_as_float(v[0][e]), x1 = __uint_as_float(v[1][e]);
              s0 = fmaf(x0, x0, s0);
              s1 = fmaf(x1, x1, s1);
            }
          }
          if (n < p.D_out) p.partial[(static_cast<size_t>(pass) * p.H + hrow) * p.D_out + n] = s0 + s1;
        } else if (kForm == kFormGram) {
          // "Tokens" are rows t of H = X^T X: the accumulator holds (H e_n)_t
          // for this warp's 128 rows; the partial is sum_t e_nt (H e_n)_t, with
          // e_n read back from the operand (bf16, row n contiguous in t).
          const int t0 = tt * kBN + h * kHalfN;
          const bool col_ok = n < p.D_out;
          const uint16_t* erow = p.op + (static_cast<size_t>(pass) * p.D_out + (col_ok ? n : 0)) * p.D_in;
          float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 1
          for (int c2 = 0; c2 < kHalfN / 64; ++c2) {
            uint32_t v[2][32];
            tmem_ld32(acc + c2 * 64, v[0]);
            tmem_ld32(acc + c2 * 64 + 32, v[1]);
            uint4 ev[8];                                 // e_n at rows t0 + 64 c2 .. + 63
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int t = t0 + c2 * 64 + 8 * j;
              ev[j] = (col_ok && t < p.D_in) ? __ldg(reinterpret_cast<const uint4*>(erow + t))
                                             : make_uint4(0u, 0u, 0u, 0u);
            }
            tmem_wait_ld();
            if (c2 == kHalfN / 64 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(release);
            }
            const uint32_t* ew = reinterpret_cast<const uint32_t*>(ev);
#pragma unroll
            for (int e = 0; e < 16; ++e) {               // bf16 pairs: rows 2e, 2e+1 of each 32-row half
              s0 = fmaf(__uint_as_float(ew[e] << 16), __uint_as_float(v[0][2 * e]), s0);
              s0 = fmaf(__uint_as_float(ew[e] & 0xFFFF0000u), __uint_as_float(v[0][2 * e + 1]), s0);
              s1 = fmaf(__uint_as_float(ew[16 + e] << 16), __uint_as_float(v[1][2 * e]), s1);
              s1 = fmaf(__uint_as_float(ew[16 + e] & 0xFFFF0000u), __uint_as_float(v[1][2 * e + 1]), s1);
            }
          }
          if (col_ok) p.partial[(static_cast<size_t>(pass) * p.H + hrow) * p.D_out + n] = s0 + s1;
        } else if (ref) {
#pragma unroll 1
          for (int c = 0; c < kHalfN / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(acc + c * 32, v);
            tmem_wait_ld();
            const int cc = h * (kHalfN / 32) + c;          // 32-token chunk of the tile
            if (p.gemm_only) {
              const int t0 = tt * kBN + cc * 32;
              if (n < p.D_out) {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                  if (t0 + e < p.N) p.y_out[static_cast<size_t>(t0 + e) * p.D_out + n] = __uint_as_float(v[e]);
              }
            } else {
              // [token chunk of 4][column][4]: a warp stores 512 contiguous bytes
              float4* dst = yref + (cc * 8) * kBM + nl;
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                dst[jj * kBM] = make_float4(__uint_as_float(v[4 * jj]), __uint_as_float(v[4 * jj + 1]),
                                            __uint_as_float(v[4 * jj + 2]), __uint_as_float(v[4 * jj + 3]));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(release);
        } else {
          float sum = 0.0f;
#pragma unroll 1
          for (int c = 0; c < kHalfN / 32; ++c) {
            const int cc = h * (kHalfN / 32) + c;
            const float4* src = yref + (cc * 8) * kBM + nl;
            float4 y[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) y[jj] = src[jj * kBM];
            uint32_t v[32];
            tmem_ld32(acc + c * 32, v);
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
          if (lane == 0) mbar_arrive_cluster(release);
          if (n < p.D_out) p.partial[(static_cast<size_t>(pass) * p.H + hrow) * p.D_out + n] = sum;
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
PFN_cuTensorMapEncodeTiled_v12000 lookup_encode_fn() {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult qres;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
      qres == cudaDriverEntryPointSuccess)
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  return nullptr;
}

// Looked up once (a function-local static is initialised exactly once, even
// with several host threads).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = lookup_encode_fn();
  return fn;
}

template <int kForm>
cudaError_t launch_form(int grid, const CUtensorMap& mX, const CUtensorMap& mWt, const CUtensorMap& mOp,
                        const Params& p, cudaStream_t st) {
  static SmemAttrOnce once;
  const cudaError_t e = set_smem_once(search_kernel<kForm>, kSmemBytes, once);
  if (e != cudaSuccess) return e;
  search_kernel<kForm><<<grid, kThreads, kSmemBytes, st>>>(mX, mWt, mOp, p);
  return cudaGetLastError();
}

}  // namespace

// A bf16 map: rows of `inner` elements (contiguous), `rows` rows, optionally
// `planes` planes of rows x inner; box box_inner x box_rows (x 1), 128-byte
// swizzle (box_inner = 64: one swizzle row).
bool make_bf16_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t planes,
                   uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t dims[3] = {inner, rows, planes};
  const uint64_t str[2] = {inner * 2, inner * 2 * rows};
  const uint32_t box[3] = {box_inner, box_rows, 1};
  const uint32_t estr[3] = {1, 1, 1};
  const cuuint32_t rank = planes > 0 ? 3 : 2;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, str, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A 3-D bf16 map with explicit byte strides for dimensions 1 and 2 (any
// order of strides; each a multiple of 16 bytes), 128-byte swizzle.
bool make_bf16_map_3d(CUtensorMap* m, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                      const uint32_t box[3]) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// An unswizzled TMA map over a row-major 2-D array of 4-byte elements
// (uint32 or fp32): `inner` contiguous elements per row, `rows` rows, box
// box_inner x box_rows.
bool make_word_map(CUtensorMap* m, const void* base, bool is_float, uint64_t inner, uint64_t rows,
                   uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t dims[2] = {inner, rows};
  const uint64_t str[1] = {inner * 4};
  const uint32_t box[2] = {box_inner, box_rows};
  const uint32_t estr[2] = {1, 1};
  CUresult r = fn(m, is_float ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 2,
                  const_cast<void*>(base), dims, str, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int search_token_tiles(int N) { return (N + kBN - 1) / kBN; }

// Token tiles per block of the unit order: as many as keep the block's X tiles
// (256 tokens x D_in bf16 each) within an L2 budget, balanced over the blocks
// (one tile when not even one fits).  Per wave, the operand of every alpha is
// read once for the wave's few weight tiles, and the block's X tiles once for
// all its waves.  Measured on B200 with the pass barrier (21 alphas, N = 4096,
// the 70B block): the 28672 x 8192 down projection took 32.8-34.0 ms with
// blocks of four token tiles against 34.4 with one and 31.6-34.7 with two,
// the whole step 122.7-123.3 ms against 124.6-125.0 and 125.6-126.0.
int search_token_block(const SearchShape& sh, int Tt) {
  const double tile_bytes = 2.0 * kBN * static_cast<double>(sh.D_in);
  const double budget = static_cast<double>(kXBlockBudgetBytes);
  int tmax = static_cast<int>(budget / tile_bytes);
  if (tmax < 1) return 1;
  if (tmax >= Tt) return Tt;
  const int nblk = (Tt + tmax - 1) / tmax;
  return (Tt + nblk - 1) / nblk;
}

int search_partial_rows(int N) { return 2 * search_token_tiles(N); }

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
  CUtensorMap mX, mWt, mOp;
  if (!make_bf16_map(&mX, b.X, static_cast<uint64_t>(sh.D_in), static_cast<uint64_t>(sh.N), 0, kBK, kBM)) {
    *what = "tensor map for X";
    return kECuda;
  }
  if (form == kFormReference) {
    if (!make_bf16_map(&mWt, b.wt, static_cast<uint64_t>(sh.D_in), static_cast<uint64_t>(sh.D_out), 0, kBK, kBM)) {
      *what = "tensor map for the bf16 weights";
      return kECuda;
    }
  } else {
    mWt = mX;   // never read by the error form
  }
  if (!gemm_only) {
    if (!make_bf16_map(&mOp, b.op, static_cast<uint64_t>(sh.D_in), static_cast<uint64_t>(sh.D_out),
                       static_cast<uint64_t>(sh.A), kBK, kBM)) {
      *what = "tensor map for the per-alpha operand";
      return kECuda;
    }
  } else {
    mOp = mX;   // never read in gemm-only mode
  }
  Params p;
  p.N = sh.N;
  p.D_in = sh.D_in;
  p.D_out = sh.D_out;
  p.A = sh.A;
  p.Tt = search_token_tiles(sh.N);
  p.Wt = (sh.D_out + kPairM - 1) / kPairM;
  p.U = p.Wt * p.Tt;
  p.KB = (sh.D_in + kBK - 1) / kBK;
  p.H = search_partial_rows(sh.N);
  p.gemm_only = gemm_only ? 1 : 0;
  p.tb = search_token_block(sh, p.Tt);
  p.op = b.op;
  p.yref = b.yref;
  p.partial = b.partial;
  p.y_out = b.y_out;
  p.status = b.status;
  p.timeout_ns = timeout_ns;
  // the pass counter, for a grid with at least one full wave of units
  const bool sync = b.sync && !gemm_only && p.U >= grid / 2 && grid >= 4;
  p.sync = sync ? b.sync : nullptr;
  if (sync) {
    const cudaError_t e0 = cudaMemsetAsync(b.sync, 0, sizeof(unsigned), st);
    if (e0 != cudaSuccess) {
      *cerr = e0;
      *what = "cudaMemsetAsync(pass counter)";
      return kECuda;
    }
  }

  cudaError_t e = form == kFormError  ? launch_form<kFormError>(grid, mX, mWt, mOp, p, st)
                  : form == kFormGram ? launch_form<kFormGram>(grid, mX, mWt, mOp, p, st)
                                      : launch_form<kFormReference>(grid, mX, mWt, mOp, p, st);
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
