// internal.cuh -- launch helpers shared by the C-ABI layer (api.cu) and the
// kernel files.  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace awq {

constexpr int kMaxAlpha = 64;

// ---- api.cu
// An identifier of the calling thread's current CUDA context, unique for the
// life of the process (a context made after cudaDeviceReset gets a new one);
// 0 when there is no current context yet or the driver cannot tell.
unsigned long long current_context_id();

// Remembers the context in which a kernel's dynamic shared-memory limit was
// last raised, so that it is raised once per context (racing threads may both
// raise it, which is harmless); with no known context it is raised every call.
struct SmemAttrOnce {
  std::atomic<unsigned long long> ctx{0};
};
template <typename K>
inline cudaError_t set_smem_once(K kernel, int bytes, SmemAttrOnce& once) {
  const unsigned long long id = current_context_id();
  if (id != 0 && once.ctx.load(std::memory_order_acquire) == id) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && id != 0) once.ctx.store(id, std::memory_order_release);
  return e;
}

// Quantisers: delta = max / (2^(b-1) - 1), codes +-(2^(b-1) - 1); the
// power-of-two delta = max / 2^(b-1), codes [-2^(b-1), 2^(b-1) - 1]; or the
// asymmetric MinMax delta = (hi - lo) / (2^b - 1) with zero point z, codes
// [-z, 2^b - 1 - z] (stored as u = q + z).
constexpr int kQuantSymmetric = 0;
constexpr int kQuantPow2 = 1;
constexpr int kQuantAsymmetric = 2;

// Loss forms of the search (see search.cu).
constexpr int kFormError = 0;        // L = ||X E||^2 with E = S^-1 Q(S W) - W as the MMA operand
constexpr int kFormReference = 1;    // L = ||X S^-1 Q(S W) - X W||^2, reference output subtracted
constexpr int kFormGram = 2;         // L = sum_n e_n^T H e_n with H = X^T X given in place of X (N = D_in)

struct AlphaList {
  float v[kMaxAlpha];
};

// ---- act_stats.cu
// No scratch: the row split folds through distributed shared memory.
cudaError_t launch_act_stats(const uint16_t* X, int64_t N, int64_t D, int stat, float* a, int num_sms,
                             cudaStream_t st);
// Several inputs (host arrays of n <= kMaxStatsInputs entries) in one launch.
constexpr int kMaxStatsInputs = 16;
cudaError_t launch_act_stats_batched(const uint16_t* const* X, const int64_t* N, const int64_t* D, int n, int stat,
                                     float* const* a, int num_sms, cudaStream_t st);

// ---- scales.cu
// s_tab [A][D] (may be null), r_tab [A][D] = fl32(1 / s) (may be null).
// alpha_dev != null: a single alpha read from device memory (A must be 1).
// b != null: the balanced scale a^alpha / b^(1 - alpha).
cudaError_t launch_scale_table(const float* a, const float* b, int64_t D, const AlphaList& alphas,
                               const float* alpha_dev, int A, float* s_tab, float* r_tab, cudaStream_t st);
// b [D_in] = mean_n |W[j][n]| (fp64 sums, one rounding).
cudaError_t launch_weight_mean(const float* W, int64_t D_in, int64_t D_out, float* b, cudaStream_t st);

// ---- quant.cu
// The search's A operand for every alpha, bf16 [A][D_out][D_in]: error form
// (S^-1 Q(S W) - W)^T, reference form (S^-1 Q(S W))^T.  See quant.cu.
// W rows are ldw elements apart (ldw >= D_out).
cudaError_t launch_search_operand(const float* W, int64_t ldw, const float* s_tab, const float* r_tab, int64_t D_in,
                                  int64_t D_out, int A, int bits, int group, int form, int qmode, uint16_t* op,
                                  cudaStream_t st);
// The clipping search's operand for every clip ratio c of `clips`, bf16
// [n_clip][D_out][D_in]: (S^-1 Q_c(S W) - W)^T with the group maximum scaled
// by c and codes clamped; s and r = 1/s are single rows [D_in].
cudaError_t launch_clip_operand(const float* W, const float* s, const float* r, int64_t D_in, int64_t D_out,
                                const AlphaList& clips, int n_clip, int bits, int group, uint16_t* op,
                                cudaStream_t st);
// bf16 W^T [D_out][D_in] for the reference output X W.
cudaError_t launch_weight_t(const float* W, int64_t ldw, int64_t D_in, int64_t D_out, uint16_t* wt, cudaStream_t st);
// Final quantise + pack for one given scale vector s (natural nibble order);
// clip [D_in/group][D_out] (may be null) scales each group maximum; delta16:
// delta rounded to FP16 before the codes, scales stored as FP16 (else fp32).
// dense3: 3-bit codes as 96-bit strings of 32 rows (words [D_in/32*3][D_out]).
// qmode kQuantAsymmetric: zeros [D_in/group][D_out] receives z (clip must be null).
cudaError_t launch_quantize_pack(const float* W, const float* s, const float* clip, int64_t D_in, int64_t D_out,
                                 int bits, int group, bool delta16, int qmode, bool dense3, uint32_t* packed,
                                 void* scales, uint8_t* zeros, int num_sms, cudaStream_t st);

// ---- reduce.cu
cudaError_t launch_loss_reduce(const float* partial, int A, int H, int64_t D_out, double* L_col, double* blk,
                               int nblk, const AlphaList& alphas, double* L, float* alpha_star, int* alpha_idx,
                               cudaStream_t st);
int loss_reduce_blocks(int64_t D_out);
// Column ranges [off[l], off[l+1]) of the layers of a joint search.
constexpr int kMaxJointLayers = 16;
struct Segments {
  int64_t off[kMaxJointLayers + 1];
};
// out [n_seg][A]: the sums of L_col [A][D] over each range, in a fixed order.
cudaError_t launch_segment_sums(const double* L_col, int A, int64_t D, const Segments& seg, int n_seg, double* out,
                                cudaStream_t st);

// ---- search.cu
struct SearchShape {
  int N, D_in, D_out, A, bits, group, form;
};
struct SearchBuffers {
  const void* X;              // bf16 [N][D_in]
  const uint16_t* wt;         // bf16 W^T [D_out][D_in] (reference pass, gemm-only mode)
  const uint16_t* op;         // bf16 [A][D_out][D_in], the per-alpha operand
  float* yref;                // [grid][128*256]
  float* partial;             // [A][search_partial_rows(N)][D_out]
  float* y_out;               // gemm-only mode: [N][D_out]
  int* status;
  unsigned* sync = nullptr;   // 4 bytes of device memory for the producers' pass counter, or null (no sync)
};
int search_grid_size(const SearchShape& sh, int num_sms);
int search_token_tiles(int N);
// Token tiles per block of the search's unit order (X tiles of a block fit an L2 budget).
int search_token_block(const SearchShape& sh, int Tt);
// Rows of loss partials per alpha: one per 128-token half of a token tile.
int search_partial_rows(int N);
// Returns 0 on success, otherwise an awq error code; *cerr gets the CUDA error.
int launch_search(const SearchShape& sh, const SearchBuffers& b, int grid, uint64_t timeout_ns, cudaStream_t st,
                  cudaError_t* cerr, const char** what);

// bf16 TMA map (128-byte swizzle) over rows of `inner` contiguous elements,
// `rows` rows, `planes` planes (0: a 2-D map); box box_inner x box_rows.
bool make_bf16_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t planes,
                   uint32_t box_inner, uint32_t box_rows);
// 3-D bf16 map (128-byte swizzle) with byte strides of dimensions 1 and 2.
bool make_bf16_map_3d(CUtensorMap* m, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                      const uint32_t box[3]);
// Unswizzled TMA map over rows of `inner` 4-byte elements (fp32 or uint32).
bool make_word_map(CUtensorMap* m, const void* base, bool is_float, uint64_t inner, uint64_t rows,
                   uint32_t box_inner, uint32_t box_rows);

// ---- clip.cu (the weight-clipping search)
// XT [D][Np] = X^T, tokens padded with zeros to Np (a multiple of 8).
cudaError_t launch_xt(const uint16_t* X, int64_t N, int64_t D, int64_t Np, uint16_t* XT, cudaStream_t st);
// r = 1 / s (IEEE).
cudaError_t launch_recip(const float* s, int64_t D, float* r, cudaStream_t st);
// dst [n] = bf16(src [n]), round to nearest even.
cudaError_t launch_to_bf16(const float* src, int64_t n, uint16_t* dst, cudaStream_t st);
// Hb [D_in/group][group][group] bf16: the diagonal Gram blocks X_g^T X_g.
int launch_gram(const uint16_t* XT, int64_t D_in, int64_t Np, int group, uint16_t* Hb, int* status,
                uint64_t timeout_ns, cudaStream_t st, cudaError_t* cerr, const char** what);
// Per (group, column): the clip ratio of `clips` with the smallest e^T H_g e
// (lowest index on ties) -> clip_out [groups][D_out]; idx_out, loss_out
// [n_clip][groups][D_out] may be null.
int launch_clip_loss(const uint16_t* op, const uint16_t* Hb, int64_t D_in, int64_t D_out, int group,
                     const AlphaList& clips, int n_clip, float* clip_out, int* idx_out, float* loss_out, int num_sms,
                     int* status, uint64_t timeout_ns, cudaStream_t st, cudaError_t* cerr, const char** what);

// ---- w4a16.cu (the quantised layer applied to activations)
// Y [N][D_out] fp32 = X diag(1/s) Dequant(packed, scales), tcgen05 with the
// weights dequantised into shared memory; stream-K over the k blocks when
// the token tile is small.  ws: scratch of w4a16_scratch_bytes(N, D_in, D_out,
// zrows) bytes, 256-byte aligned (scaled activations, stream-K partial tiles,
// and with zero points the fp32 rows of 128 + z).  zeros: NULL (offset-binary
// codes u = q + 2^(b-1)) or [D_in/group][D_out] uint8 zero points of
// asymmetric codes u = q + z (zrows = D_in / group).  D_out must be a
// multiple of 4.  For N <= 4 a CUDA-core GEMV takes the place of the
// tensor-core kernel; it has nothing to wait on and clears *status itself
// (w4a16_clears_status), so the caller need not.
size_t w4a16_scratch_bytes(int64_t N, int64_t D_in, int64_t D_out, int64_t zrows);
bool w4a16_clears_status(int64_t N);
int launch_w4a16(const void* X, const float* s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                 int64_t N, int64_t D_in, int64_t D_out, int bits, int group, float* Y, void* ws, int num_sms,
                 int* status, uint64_t timeout_ns, cudaStream_t st, cudaError_t* cerr, const char** what);

// Self-test of the bounded wait: one CTA waits on an mbarrier that nothing
// arrives at, gives up after timeout_ns and records the timeout in *status.
cudaError_t launch_wait_timeout_selftest(int* status, uint64_t timeout_ns, cudaStream_t st);

// Self test of the quantisers' constant divisor and reciprocal on every
// non-negative finite float (quant.cu): bad[0] += mismatches of the division
// by b against the IEEE quotient, bad[1] += reciprocals more than one ulp
// from the correctly rounded one.  bad must be zeroed by the caller.
cudaError_t launch_divide_selftest(float b, unsigned long long* bad, int num_sms, cudaStream_t st);

}  // namespace awq
