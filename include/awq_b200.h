/*
 * awq_b200.h -- C ABI of the B200 (sm_100a) AWQ per-layer scale search.
 *
 * The library evaluates, for ONE linear layer Y = X W, the activation-aware
 * scale search of AWQ and quantises the weights with the chosen scales:
 *   1. a_j = mean_i |X_ij| (or max)                       -> awq_act_stats
 *   2. s_j(alpha) = a_j^alpha for every alpha on a grid    -> awq_scales
 *   3. W' = diag(s) W, symmetric absmax per-group b-bit quantisation along D_in
 *   4. L(alpha) = || X S^-1 Q(S W) - X W ||^2
 *   5. alpha* = argmin L                                   -> awq_search (2-5)
 *   6. the final INT codes + per-group scales for s*       -> awq_quantize_pack
 * Passages: compassingai.com AWQ concept page, "statistical basis of salient
 * channels" (step 1), "full scale-optimisation flow" steps 1-6 (steps 2-5),
 * "quantisation math" (step 3), "inference-time equivalent" (step 6);
 * mudrobot.github.io AWQ notes, "searching the optimal scale" (s = s_X^alpha,
 * alpha* = argmin over [0, 1]).
 *
 * Conventions for every call:
 *   - Matrices are dense row-major.  X: N x D_in bf16 (raw 16-bit patterns),
 *     W: D_in x D_out fp32 (the Y = X W orientation: scales act on the rows of
 *     W, groups run along D_in).
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     its comment says "host".  Device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     only enqueue work; they are asynchronous with respect to the host and
 *     do not synchronise.  Scratch space comes from a caller-provided
 *     workspace whose size is queried (or, for awq_search_noalloc, a fixed
 *     array inside the library).  The library calls no allocator.  A
 *     workspace serves one call at a time: two calls in flight on different
 *     streams need two workspaces.
 *   - The return value is an awq_status.  A non-OK status from argument
 *     checking is returned before any work is enqueued; awq_get_last_error()
 *     then describes it.  Errors found on the device (a wait that timed out)
 *     are written to the caller's device status word (see awq_search).
 *   - Inputs are assumed finite; NaN or Inf inputs give unspecified (but
 *     memory-safe) results.
 *   - Supported bit widths are 2, 3 and 4 (codes are stored as 4-bit
 *     offset-binary values); group sizes are 32, 64, 128 and 256.
 *   - Debug knobs, read once per process from the environment:
 *       AWQ_LOG=1        one stderr line per call that works on the device
 *                        ("[awq] name(sizes)") and one per non-OK status;
 *       AWQ_FAULT=badarg | workspace | alloc | launch
 *                        host-side fault injection at the entry of every such
 *                        call, before any check or launch: AWQ_EINVAL,
 *                        AWQ_EWORKSPACE (on the calls that take a workspace;
 *                        "alloc" is the same, since the library allocates
 *                        nothing), or AWQ_ECUDA as from a failed launch;
 *       AWQ_TIMEOUT_MS   the bounded waits' limit (default 2000).
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AWQ_API __attribute__((visibility("default")))
#else
#define AWQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AWQ_OK = 0,
  AWQ_EINVAL = 1,        /* bad size, null pointer, bad enum value */
  AWQ_EALIGN = 2,        /* a device pointer is not 16-byte aligned */
  AWQ_EUNSUPPORTED = 3,  /* bits/group/n_alpha outside the supported set, or no sm_100 device */
  AWQ_EWORKSPACE = 4,    /* workspace too small or null */
  AWQ_ECUDA = 5,         /* a CUDA call failed; awq_get_last_error() has its message */
  AWQ_ETIMEOUT = 6       /* device only: a pipeline wait gave up (written to the status word) */
} awq_status;

enum { AWQ_STAT_MEAN = 0, AWQ_STAT_MAX = 1 };

/*
 * How awq_search evaluates L(alpha) = || X S^-1 Q(S W) - X W ||^2 on the tensor
 * cores (identical in exact arithmetic):
 *   AWQ_LOSS_ERROR      L = || X E ||^2 with E = S^-1 Q(S W) - W formed per
 *                       weight in fp32 from the quantiser's exact rounding
 *                       residual and rounded to bf16 once; the default, and
 *                       the more accurate form.
 *   AWQ_LOSS_REFERENCE  the reference output X W is computed once per tile by
 *                       the same GEMM (bf16 W) and subtracted from
 *                       X S^-1 Q(S W) (bf16 operands) in the epilogue.
 */
enum { AWQ_LOSS_ERROR = 0, AWQ_LOSS_REFERENCE = 1 };

/* Largest alpha grid accepted by awq_search. */
#define AWQ_MAX_ALPHA 64

/*
 * Activation statistic (compassingai.com AWQ concept page, "statistical basis
 * of salient channels": activation_scale[j] = mean(|X_calib[:, j]|), or max;
 * mudrobot.github.io notes: s_X is the average per-channel magnitude).
 *   X     [N][D_in] bf16, 1 <= N <= 2^24, 8 <= D_in <= 2^20, D_in % 8 == 0
 *   stat  AWQ_STAT_MEAN: a_j = (sum_i |X_ij|) / N, summed in fp32 in a fixed
 *         order (bit-reproducible); AWQ_STAT_MAX: a_j = max_i |X_ij| (exact)
 *   a     [D_in] fp32 output
 * The rows are split over the two CTAs of a cluster pair, which fold their
 * partial rows through distributed shared memory: no scratch is used.
 */
AWQ_API int awq_act_stats(const void* X, int64_t N, int64_t D_in, int stat, float* a, void* stream);

/*
 * The statistic of several inputs in one launch (the distinct inputs of a
 * transformer block: the q/k/v input, the o input, the gate/up input, the down
 * input), each as awq_act_stats defines it (max exact; the mean's fixed fp32
 * summation order can differ from that of a single-input call, within its
 * rounding).  The launch's CTA pairs are shared out over the inputs in
 * proportion to their bytes, so one wave streams them all.
 *   Xs, Ns, D_ins, as  host arrays of n_inputs entries: device pointers X
 *                      [N][D_in] bf16 and a [D_in] fp32 (each 16-byte aligned)
 *   n_inputs           1 .. 16 (AWQ_EUNSUPPORTED beyond)
 * Errors as awq_act_stats, with the failing input's index in the message.
 */
AWQ_API int awq_act_stats_batched(const void* const* Xs, const int64_t* Ns, const int64_t* D_ins, int n_inputs,
                                  int stat, float* const* as, void* stream);

/*
 * Scale vector for one alpha (compassingai.com concept page, flow step 3:
 * s_j = activation_scale[j]^alpha; step 6: s* = activation_scale^alpha*).
 *   s_j = (float) pow((double) max(a_j, 1e-6f * max_i a_i), (double) alpha)
 *   (all ones when every a_j is 0).  alpha = 0 gives exactly 1.
 *   a  [D_in] fp32;  s  [D_in] fp32 output;  alpha is a host value.
 */
AWQ_API int awq_scales(const float* a, int64_t D_in, float alpha, float* s, void* stream);

/* Same, with alpha read from device memory (e.g. the alpha_star output of
 * awq_search), so that search -> scales -> pack needs no host round trip. */
AWQ_API int awq_scales_dev(const float* a, int64_t D_in, const float* alpha_dev, float* s, void* stream);

/*
 * The weight statistic of the balanced scale (zhihu AWQ/GPTQ/SmoothQuant
 * comparison, the per-channel scale s_j = mean|X_j|^alpha / mean|W_j|^(1-alpha)):
 *     w_mean[j] = (sum_n |W[j][n]|) / D_out,
 * summed in fp64 (a fixed order), rounded to fp32 once.
 *   W       [D_in][D_out] fp32, 16-byte aligned;  w_mean [D_in] fp32 output
 */
AWQ_API int awq_weight_mean(const float* W, int64_t D_in, int64_t D_out, float* w_mean, void* stream);

/*
 * Scale vector with an optional weight statistic: s_j = a_j^alpha when w_mean
 * is NULL (as awq_scales), else the balanced s_j = a_j^alpha / w_mean_j^(1-alpha).
 * Both statistics are floored at 1e-6 of their maximum.  The powers are taken
 * in fp64, and the result is rounded to fp32 once.  alpha_dev (device, may be
 * NULL) overrides alpha (HOST, 0 <= alpha <= 1), e.g. the alpha_star of
 * awq_search_ex.
 */
AWQ_API int awq_scales_ex(const float* a, const float* w_mean, int64_t D_in, float alpha, const float* alpha_dev,
                          float* s, void* stream);

/*
 * Bytes of workspace awq_search needs for this shape on the current device
 * (0 if the arguments are invalid).
 */
AWQ_API size_t awq_search_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int n_alpha, int bits, int group,
                                         int loss_form);

/*
 * The grid search (compassingai.com concept page, flow steps 3-5;
 * mudrobot.github.io notes, "searching the optimal scale").  For every alpha
 * in the grid it forms s = a^alpha, quantises diag(s) W per group of `group`
 * rows to `bits` bits (delta = max|w'| / (2^(b-1)-1), round half to even,
 * clamp to +-(2^(b-1)-1)) and evaluates
 *     L(alpha) = || X S^-1 Q(S W) - X W ||^2
 * with bf16 operands and fp32 accumulation on the tensor cores, in the form
 * chosen by loss_form (AWQ_LOSS_ERROR or AWQ_LOSS_REFERENCE); the squared
 * error is summed in fp32 per 128 tokens and in fp64 above that, in a fixed
 * order.
 *   X           [N][D_in] bf16;  W [D_in][D_out] fp32;  a [D_in] fp32
 *   alpha_grid  HOST array of n_alpha fp32 values, 1 <= n_alpha <= 64
 *   bits        2, 3 or 4;  group 32, 64, 128 or 256;  D_in % group == 0,
 *               D_in <= 2^20, D_out % 4 == 0, D_out <= 2^24, 1 <= N <= 2^24
 *   loss_form   AWQ_LOSS_ERROR or AWQ_LOSS_REFERENCE
 *   L           [n_alpha] fp64 output (device)
 *   L_col       [n_alpha][D_out] fp64 output: each column's share of L
 *               (may be NULL)
 *   alpha_star  [1] fp32 output: alpha_grid[argmin L] (smallest index on ties)
 *   alpha_idx   [1] int32 output: argmin L
 *   workspace   at least awq_search_workspace_size(...) bytes, 256-byte aligned
 *   status      [1] int32 device status word (may be NULL): set to 0 by the
 *               call, then AWQ_ETIMEOUT | (site << 8) if a pipeline wait gave
 *               up; the outputs are then invalid.  Read it after the stream
 *               has been synchronised.
 * The kernel's CTAs keep their alpha passes in step through a counter in the
 * workspace (zeroed by the call on `stream`).  A CTA that has waited 2 ms for
 * the others (another kernel holding the SMs some of them need) stops waiting
 * for the rest of the launch; the results never depend on it.
 */
AWQ_API int awq_search(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
                       const float* alpha_grid, int n_alpha, int bits, int group, int loss_form, double* L,
                       double* L_col, float* alpha_star, int32_t* alpha_idx, void* workspace, size_t workspace_bytes,
                       int32_t* status, void* stream);

/*
 * Quantiser and scale variants of the search:
 *   quantizer  AWQ_QUANT_SYMMETRIC: delta = max|w'| / (2^(b-1)-1), codes in
 *              +-(2^(b-1)-1) (as awq_search);
 *              AWQ_QUANT_DELTA_POW2 (mudrobot.github.io notes, "analysing the
 *              quantisation error"): delta = max|w'| / 2^(b-1), codes clamped to
 *              [-2^(b-1), 2^(b-1)-1] (the passage gives no clamp; +max would
 *              need b+1 bits).  Pack with AWQ_PACK_DELTA_POW2.
 *              AWQ_QUANT_ASYMMETRIC (compassingai.com AWQ concept page, "the
 *              AWQ mechanism": MinMax uniform quantisation, symmetric or
 *              asymmetric): lo = min(0, min w'), hi = max(0, max w'),
 *              delta = (hi - lo) / (2^b - 1), zero point
 *              z = clamp(rne(-lo / delta), 0, 2^b - 1), codes
 *              q = clamp(rne(w' / delta), -z, 2^b - 1 - z); the dequantised
 *              weight is q delta.  Pack with awq_quantize_pack_zp.
 *   w_mean     NULL, or [D_in] device fp32 (awq_weight_mean): the candidate
 *              scales are the balanced a^alpha / w_mean^(1-alpha); recover s*
 *              with awq_scales_ex.
 *   gram_form  nonzero: evaluate L(alpha) = sum_n e_n^T H e_n with H = X^T X
 *              (the Gram form of the loss): H is formed once
 *              (tensor cores, fp32, rounded to bf16), then each alpha costs
 *              2 D_in^2 D_out flops instead of 2 N D_in D_out, which is cheaper
 *              when N > D_in.  Error form only.  The workspace is
 *              awq_search_ex_workspace_size(...).
 *   ldw        0, or the row stride of W in elements (ldw >= D_out, a multiple
 *              of 4): row k of W starts at W + k ldw.  It lets a caller search
 *              a slice of output columns of a wider matrix in place (W pointing
 *              at the slice's first column), as the column-sharded multi-GPU
 *              search does; the loss is a sum over output columns (concept
 *              page, flow step 4c), so the slices' losses add up to the layer's.
 */
#define AWQ_QUANT_SYMMETRIC 0
#define AWQ_QUANT_DELTA_POW2 1
#define AWQ_QUANT_ASYMMETRIC 2
typedef struct {
  int quantizer;
  const float* w_mean;
  int gram_form;
  int64_t ldw;
} awq_search_options;

/* Bytes of workspace awq_search_ex needs with these options (0 if invalid). */
AWQ_API size_t awq_search_ex_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int n_alpha, int bits, int group,
                                            int loss_form, const awq_search_options* options);

/*
 * awq_search with options (NULL = awq_search).  Same arguments, outputs and
 * errors; workspace awq_search_ex_workspace_size(...) bytes.
 */
AWQ_API int awq_search_ex(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
                          const float* alpha_grid, int n_alpha, int bits, int group, int loss_form,
                          const awq_search_options* options, double* L, double* L_col, float* alpha_star,
                          int32_t* alpha_idx, void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/* One layer of a batched search (see awq_search for the meaning of each field). */
typedef struct {
  const void* X;
  const float* W;
  const float* a;
  int64_t N, D_in, D_out;
  double* L;          /* [n_alpha] */
  double* L_col;      /* [n_alpha][D_out] or NULL */
  float* alpha_star;  /* [1] */
  int32_t* alpha_idx; /* [1] */
} awq_layer;

/* Bytes of workspace awq_search_batched needs (the largest single layer). */
AWQ_API size_t awq_search_batched_workspace_size(const awq_layer* layers, int n_layers, int n_alpha, int bits,
                                                 int group, int loss_form);

/*
 * Independent searches for several layers with one call (compassingai.com
 * concept page, flow note: each layer is searched independently).  `layers`
 * is a HOST array of n_layers descriptors; every layer gets its own L and
 * alpha*.  The layers run one after another on `stream`, sharing the
 * workspace.
 */
AWQ_API int awq_search_batched(const awq_layer* layers, int n_layers, const float* alpha_grid, int n_alpha,
                               int bits, int group, int loss_form, void* workspace, size_t workspace_bytes,
                               int32_t* status, void* stream);

/*
 * Final quantise + pack for a given scale vector (compassingai.com concept
 * page, "inference-time equivalent": W_quantized = Quantize(diag(s*) W), s*
 * kept as metadata).  Bit-exact IEEE fp32 arithmetic:
 *   w' = fl(s_k w_kn), delta = fl(max|w'| / (2^(b-1)-1)),
 *   q = clamp(rne(fl(w' / delta))), an all-zero group has delta = 0, q = 0.
 *   W       [D_in][D_out] fp32;  s [D_in] fp32
 *   packed  [D_in/8][D_out] uint32 output: word (k8, n) holds rows
 *           8*k8 .. 8*k8+7 of column n, row 8*k8+i in bits 4i..4i+3 as the
 *           offset-binary value u = q + 2^(bits-1)
 *   scales  [D_in/group][D_out] fp32 output: delta of each (group, column)
 */
AWQ_API int awq_quantize_pack(const float* W, const float* s, int64_t D_in, int64_t D_out, int bits, int group,
                      uint32_t* packed, float* scales, void* stream);

/*
 * Joint search of linears that share one input and therefore one scale vector
 * (mudrobot.github.io AWQ notes: 1/s is fused into the previous operator, so
 * q/k/v after one LayerNorm, or gate/up, take the same s).  The objective is
 * the sum of the layers' losses,
 *     L(alpha) = sum_l || X S^-1 Q(S W_l) - X W_l ||^2,
 * and alpha* its argmin.  Since a layer's loss is a sum over its output
 * columns, this is exactly the search of the layers' weights side by side
 * ([D_in][sum_l D_out_l], copied into the workspace).
 *   Ws        HOST array of n_layers device pointers, W_l [D_in][D_outs[l]] fp32
 *   D_outs    HOST array: each a multiple of 4; 1 <= n_layers <= 16
 *   L         [n_alpha] fp64 output: the joint loss
 *   L_layers  [n_layers][n_alpha] fp64 output: each layer's loss (may be NULL)
 *   other arguments and limits as for awq_search; workspace at least
 *   awq_search_joint_workspace_size(...) bytes.
 */
AWQ_API size_t awq_search_joint_workspace_size(int64_t N, int64_t D_in, const int64_t* D_outs, int n_layers,
                                               int n_alpha, int bits, int group, int loss_form);
AWQ_API int awq_search_joint(const void* X, const float* const* Ws, const int64_t* D_outs, int n_layers,
                             const float* a, int64_t N, int64_t D_in, const float* alpha_grid, int n_alpha, int bits,
                             int group, int loss_form, double* L, double* L_layers, float* alpha_star,
                             int32_t* alpha_idx, void* workspace, size_t workspace_bytes, int32_t* status,
                             void* stream);

/*
 * Weight-clipping search, the step after the scale search (mudrobot.github.io
 * AWQ notes, "searching the optimal scale": weight clipping is applied to
 * minimise the quantisation MSE).  For every group g of `group` rows, output
 * column n and clip ratio c = clip_grid[i], the group maximum of
 * W' = diag(s) W is replaced by fl32(c * max) before delta = max / qmax is
 * formed, codes are clamped to +-qmax, and the objective is the squared error
 * of the group's share of the layer output,
 *     L_i(g, n) = || X_g (S^-1 Q_c(S W) - W)_{g,n} ||^2 = e^T (X_g^T X_g) e,
 * evaluated on the tensor cores in the Gram form (bf16 X_g^T X_g blocks, bf16
 * operand, fp32 accumulation).  The chosen ratio is the argmin over i, the
 * lowest index on ties (put c = 1, no clipping, first).
 *   X          [N][D_in] bf16;  W [D_in][D_out] fp32;  s [D_in] fp32 (e.g. s*)
 *   clip_grid  HOST array of n_clip fp32 ratios in (0, 1], 1 <= n_clip <= 64
 *   bits       2, 3 or 4;  group 64 or 128;  D_in % group == 0, D_out % 4 == 0
 *   clip       [D_in/group][D_out] fp32 output: the chosen ratio
 *   clip_idx   [D_in/group][D_out] int32 output: its grid index (may be NULL)
 *   loss       [n_clip][D_in/group][D_out] fp32 output: every L_i (may be NULL)
 *   workspace  at least awq_clip_search_workspace_size(...) bytes, 256-byte aligned
 *   status     as for awq_search (may be NULL)
 */
AWQ_API size_t awq_clip_search_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int n_clip, int bits,
                                              int group);
AWQ_API int awq_clip_search(const void* X, const float* W, const float* s, int64_t N, int64_t D_in, int64_t D_out,
                            const float* clip_grid, int n_clip, int bits, int group, float* clip, int32_t* clip_idx,
                            float* loss, void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/*
 * awq_quantize_pack with a clip ratio per (group, column) (the output of
 * awq_clip_search): the group maximum of diag(s) W is replaced by
 * fl32(clip * max) before delta is formed and codes are clamped to +-qmax;
 * otherwise as awq_quantize_pack.  clip: [D_in/group][D_out] fp32 (device).
 */
AWQ_API int awq_quantize_pack_clip(const float* W, const float* s, const float* clip, int64_t D_in, int64_t D_out,
                                   int bits, int group, uint32_t* packed, float* scales, void* stream);

/*
 * Final quantise + pack with options (the pack of awq_quantize_pack and
 * awq_quantize_pack_clip):
 *   clip    [D_in/group][D_out] fp32 clip ratios, or NULL for none
 *   flags   AWQ_PACK_DELTA_FP16: delta is rounded to FP16 (round to nearest
 *           even; mudrobot.github.io AWQ notes, "analysing the quantisation
 *           error": delta stored in FP16) before the codes are formed, codes
 *           are clamped to +-qmax, and `scales` receives FP16 values
 *           ([D_in/group][D_out] uint16 bit patterns).  Without the flag
 *           `scales` is [D_in/group][D_out] fp32, as in awq_quantize_pack.
 */
#define AWQ_PACK_DELTA_FP16 1
/*   AWQ_PACK_DELTA_POW2: delta = max / 2^(b-1) (with any clip ratio applied
 *           to max first), codes clamped to [-2^(b-1), 2^(b-1)-1]; the
 *           quantiser of awq_search_ex's AWQ_QUANT_DELTA_POW2.  Combines with
 *           AWQ_PACK_DELTA_FP16 (the power-of-two delta then rounded to FP16). */
#define AWQ_PACK_DELTA_POW2 2
/*   AWQ_PACK_DENSE3 (bits = 3 only): codes stored densely, 32 rows of a
 *           column in three words: `packed` is [D_in/32 * 3][D_out] uint32,
 *           word (3j + t, n) holding bits 32t..32t+31 of the 96-bit
 *           little-endian string whose bits 3i..3i+2 are row 32j + i's
 *           u = q + 4 (codes 10 and 21 straddle two words).  With D_out % 4 != 0
 *           it needs group 128 or 256 (AWQ_EUNSUPPORTED otherwise).
 *           awq_w4a16_gemm reads the 4-bit container layout only. */
#define AWQ_PACK_DENSE3 4
AWQ_API int awq_quantize_pack_ex(const float* W, const float* s, const float* clip, int64_t D_in, int64_t D_out,
                                 int bits, int group, int flags, uint32_t* packed, void* scales, void* stream);

/*
 * Final quantise + pack with the asymmetric quantiser (AWQ_QUANT_ASYMMETRIC
 * above): the codes stored are u = q + z in [0, 2^b - 1] in the layout of
 * awq_quantize_pack (nibbles) or, with AWQ_PACK_DENSE3, the dense 3-bit
 * layout; the dequantised weight is (u - z) * scales[g][n].
 *   flags   AWQ_PACK_DELTA_FP16 and/or AWQ_PACK_DENSE3 (AWQ_PACK_DELTA_POW2
 *           is rejected with AWQ_EINVAL).  With AWQ_PACK_DELTA_FP16 delta is
 *           rounded to FP16 before z and the codes are formed.
 *   zeros   [D_in/group][D_out] uint8 output: z (device).
 * No clip ratio (the clipping search is symmetric).  An all-zero group has
 * delta = 0, z = 0 and codes 0.  Errors as awq_quantize_pack_ex.
 * awq_w4a16_gemm_zp applies these codes to activations (fp32 deltas only).
 */
AWQ_API int awq_quantize_pack_zp(const float* W, const float* s, int64_t D_in, int64_t D_out, int bits, int group,
                                 int flags, uint32_t* packed, void* scales, uint8_t* zeros, void* stream);

/*
 * The quantised layer applied to activations, the consumer of the pack
 * format (compassingai.com AWQ concept page, "inference-time equivalent":
 * the INT4 weights with s* kept as metadata and 1/s* folded into the input;
 * AWQ paper, TinyChat section, "on-the-fly weight dequantization"):
 *     Y[t][n] = sum_k x_tk / s_k * (u_kn - 2^(bits-1)) * scales[k/group][n]
 * with u the offset-binary codes of `packed` (the layout of
 * awq_quantize_pack).  N <= 2 (decode): a CUDA-core GEMV in fp32 (x / s
 * rounded once, exact integer weights, delta applied once per group): the
 * splits of each column tile form a thread-block cluster whose first CTA
 * adds the others' sums in a fixed order, or, when the clusters do not fit
 * in one wave, the (column tile, k rows) work is shared out evenly over a
 * grid that fills every SM (stream-K) and a second small launch adds the
 * CTAs' sums of each tile in a fixed order from the workspace.
 * N = 3 to 8 with D_in <= 65536 (N <= 4) or 32768 (N >= 5): one launch of
 * warp-level tensor-core tiles (x / s rounded once to bf16, exact integer
 * codes, fp32 accumulation, the fp32 delta applied once per group), the
 * splits of each column tile summed in a fixed order inside a cluster; no
 * workspace is used.  Longer rows take the CUDA-core GEMV (N <= 4) or the
 * GEMM below.
 * N > 8 (and the longer rows at N 5..8): two launches on `stream`,
 * X' = bf16(X / s) into the workspace, then
 * a tensor-core GEMM that dequantises the weights into shared memory as
 * bf16((u - 2^(bits-1)) * bf16(delta)) (one rounding of the product) and
 * accumulates in fp32.  For N <= 64 the k blocks of all output tiles are
 * shared out evenly over the CTAs (stream-K); a tile split between CTAs is
 * summed from partial tiles in the workspace in a fixed order.  Either way
 * the result is deterministic.
 *   X         [N][D_in] bf16;  s [D_in] fp32 (s*);  packed [D_in/8][D_out] uint32
 *   scales    [D_in/group][D_out] fp32;  bits 2..4;  group 32, 64, 128 or 256
 *   D_out     a multiple of 4 (the rows of packed words are read by TMA)
 *   Y         [N][D_out] fp32 output, 4-byte aligned
 *   workspace at least awq_w4a16_workspace_size(N, D_in, D_out) bytes: for
 *             N <= 4 the CTAs' sums (1024 x 2 x N x 128 fp32); else
 *             the scaled activations (N x D_in bf16) and, for N <= 64, room
 *             for the partial tiles.  No device is needed to compute the size.
 *   status    [1] int32 device status word (required), as for awq_search
 */
AWQ_API size_t awq_w4a16_workspace_size(int64_t N, int64_t D_in, int64_t D_out);
AWQ_API int awq_w4a16_gemm(const void* X, const float* s, const uint32_t* packed, const float* scales, int64_t N,
                           int64_t D_in, int64_t D_out, int bits, int group, float* Y, void* workspace,
                           size_t workspace_bytes, int32_t* status, void* stream);

/*
 * awq_w4a16_gemm for asymmetric codes (the output of awq_quantize_pack_zp:
 * compassingai.com AWQ concept page, "the AWQ mechanism", symmetric or
 * asymmetric quantisation; "inference-time equivalent" for the product):
 *     Y[t][n] = sum_k x_tk / s_k * (u_kn - z[k/group][n]) * scales[k/group][n]
 * with the same paths and roundings: the CUDA-core GEMV subtracts each
 * group's zero point exactly in fp32, the tensor-core GEMV adds
 * (2^(bits-1) - z) times the group's sum of bf16 x / s; the tensor-core path forms bf16((u - z) * bf16(delta))
 * (u - z is exact) from a per-(group, column) fp32 copy of 128 + z that a
 * first small kernel writes into the workspace.
 *   zeros     [D_in/group][D_out] uint8 zero points (device), 16-byte aligned
 *   scales    fp32 deltas (pack without AWQ_PACK_DELTA_FP16)
 *   workspace at least awq_w4a16_zp_workspace_size(N, D_in, D_out, group)
 *             bytes (that of awq_w4a16_gemm plus, for N > 4, 4 bytes per
 *             group and column)
 * Other arguments and errors as awq_w4a16_gemm; zeros NULL is AWQ_EINVAL.
 */
AWQ_API size_t awq_w4a16_zp_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int group);
AWQ_API int awq_w4a16_gemm_zp(const void* X, const float* s, const uint32_t* packed, const float* scales,
                              const uint8_t* zeros, int64_t N, int64_t D_in, int64_t D_out, int bits, int group,
                              float* Y, void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/*
 * The layer's reference output Y = X bf16(W) computed by the search's own
 * tensor-core GEMM (the X W term of the loss, concept page flow step 4c), fp32.
 *   Y          [N][D_out] fp32 output
 *   workspace  at least awq_layer_output_workspace_size(...) bytes
 */
AWQ_API size_t awq_layer_output_workspace_size(int64_t N, int64_t D_in, int64_t D_out);
AWQ_API int awq_layer_output(const void* X, const float* W, int64_t N, int64_t D_in, int64_t D_out, float* Y,
                     void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/*
 * awq_search without a caller-provided workspace, for callers that cannot
 * allocate device memory: code that runs where the allocator must not be
 * called (an engine or plugin host that owns all device memory and hands out
 * only the buffers of a call, a real-time path with a fixed memory budget).
 * The AWQ pages have no counterpart; this is an interface convenience.
 *
 * The scratch space is a file-scope device array of AWQ_NOALLOC_SCRATCH_BYTES
 * (32 MiB) inside the library: every GPU that loads the library holds it until
 * the process exits.  Shapes whose awq_search_workspace_size exceeds it are
 * rejected with AWQ_EWORKSPACE and a message giving both sizes; they need
 * awq_search.  Arguments, outputs and results are those of awq_search, with
 * one difference: `status` is required (AWQ_EINVAL when NULL), because a
 * status word inside the shared array could not be read by the caller.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current, and once more after the device's
 *     context has been torn down and made anew, e.g. by cudaDeviceReset);
 *     make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; each call writes every scratch byte it reads before reading it
 *     and clears the status word it uses.  Calls that may overlap on the GPU
 *     (different streams, or different host threads) race on the array: order
 *     them on one stream.
 *   - Nothing is allocated: no cudaMalloc, no cudaFree, no allocating library
 *     routine (leave stage timing, which creates CUDA events, switched off).
 */
#define AWQ_NOALLOC_SCRATCH_BYTES (32u << 20)
AWQ_API int awq_search_noalloc(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
                               const float* alpha_grid, int n_alpha, int bits, int group, int loss_form, double* L,
                               double* L_col, float* alpha_star, int32_t* alpha_idx, int32_t* status, void* stream);

/*
 * Failure-detection self test: launches one CTA that waits on a barrier no one
 * ever arrives at, with the same bounded wait the search kernel uses.  After
 * about timeout_ns nanoseconds the wait gives up and AWQ_ETIMEOUT | (site << 8)
 * is written to *status (device int32).  Nothing hangs or traps.
 */
AWQ_API int awq_selftest_wait_timeout(int32_t* status, int64_t timeout_ns, void* stream);

/*
 * Self test of the quantisers' arithmetic that is not a plain IEEE operation:
 * delta = fl(m / d) for the constant divisors d (2^(b-1) - 1 and 2^b - 1) is
 * formed by Markstein's FMA correction of m * fl(1/d), and the quotients
 * w'/delta go through a reciprocal within one ulp (hardware approximation
 * plus one Newton step).  This runs both over every non-negative finite float
 * (about two billion values) on the device:
 *   divisor     1 .. 255 (AWQ_EINVAL otherwise)
 *   mismatches  [2] uint64 device output, 8-byte aligned: [0] values whose
 *               quotient differs from the IEEE quotient, [1] normal values up
 *               to 2^125 whose reciprocal is more than one ulp from the
 *               correctly rounded one.  Both are 0 for a correct build.
 * Read the result after the stream has been synchronised.
 */
AWQ_API int awq_selftest_divide(int32_t divisor, uint64_t* mismatches, void* stream);

/*
 * Stage timing.  While enabled, every entry point records a pair of CUDA
 * events on its stream around each kernel it launches; awq_profile_read waits
 * for the recorded events and returns, per stage, the summed device time in
 * milliseconds and the number of launches since the last reset.  Stages:
 */
enum {
  AWQ_STAGE_ACT_STATS = 0,     /* awq_act_stats */
  AWQ_STAGE_SCALE_TABLE = 1,   /* s = a^alpha (and 1/s) for the alpha grid, or one alpha */
  AWQ_STAGE_SEARCH_OPERAND = 2, /* per-alpha bf16 GEMM operand: S^-1 Q(S W) - W, or S^-1 Q(S W) */
  AWQ_STAGE_SEARCH_GEMM = 3,   /* the fused tensor-core loss GEMM */
  AWQ_STAGE_LOSS_REDUCE = 4,   /* L(alpha), argmin */
  AWQ_STAGE_QUANTIZE_PACK = 5, /* awq_quantize_pack */
  AWQ_STAGE_WEIGHT_T = 6,      /* bf16 W^T: reference pass of the search, awq_layer_output */
  AWQ_STAGE_CLIP_GRAM = 7,     /* awq_clip_search: X^T and the group Gram blocks X_g^T X_g */
  AWQ_STAGE_CLIP_OPERAND = 8,  /* awq_clip_search: bf16 operand per clip ratio */
  AWQ_STAGE_CLIP_LOSS = 9,     /* awq_clip_search: e^T H_g e per (ratio, group, column), argmin */
  AWQ_STAGE_W4A16 = 10,        /* awq_w4a16_gemm */
  AWQ_NUM_STAGES = 11
};
AWQ_API int awq_profile_enable(int on);
AWQ_API int awq_profile_reset(void);
AWQ_API int awq_profile_read(int stage, double* total_ms, int32_t* launches);

/* Message describing the last non-OK status returned on this thread. */
AWQ_API const char* awq_get_last_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
AWQ_API int awq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
