// api.cu -- the C ABI (include/awq_b200.h): argument checking, workspace
// layout, and the launch sequence of each entry point.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>

#include "awq_b200.h"
#include "internal.cuh"

namespace {

thread_local std::string g_last_error;

// Debug knobs, read once from the environment:
//   AWQ_LOG=1      one stderr line per entry-point call (its name and sizes),
//                  and one per non-OK status with the message;
//   AWQ_FAULT=...  host-side fault injection at the entry of every call that
//                  works on the device, before any argument check or launch:
//                  "badarg" -> AWQ_EINVAL, "workspace" (or "alloc": the
//                  library allocates nothing, so a caller's failed allocation
//                  reaches it as a short workspace) -> AWQ_EWORKSPACE on the
//                  calls that take one, "launch" -> AWQ_ECUDA as from a
//                  failed kernel launch.  Nothing reaches the GPU.
enum FaultMode { kFaultNone, kFaultBadArg, kFaultWorkspace, kFaultLaunch };

bool log_enabled() {
  static const bool on = [] {
    const char* e = getenv("AWQ_LOG");
    return e != nullptr && e[0] != '\0' && e[0] != '0';
  }();
  return on;
}

FaultMode fault_mode() {
  static const FaultMode m = [] {
    const char* e = getenv("AWQ_FAULT");
    if (e == nullptr) return kFaultNone;
    const std::string v(e);
    if (v == "badarg") return kFaultBadArg;
    if (v == "workspace" || v == "alloc") return kFaultWorkspace;
    if (v == "launch") return kFaultLaunch;
    return kFaultNone;
  }();
  return m;
}

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  if (log_enabled()) fprintf(stderr, "[awq]   -> status %d: %s\n", code, buf);
  return code;
}

enum Workspace { kNoWorkspace = 0, kTakesWorkspace = 1 };

// Entry of a device-side call: the trace line and the injected fault, if any.
int api_entry(const char* name, Workspace ws, const char* fmt, ...) {
  if (log_enabled()) {
    char buf[384];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    fprintf(stderr, "[awq] %s(%s)\n", name, buf);
  }
  switch (fault_mode()) {
    case kFaultBadArg: return fail(AWQ_EINVAL, "%s: AWQ_FAULT=badarg (injected)", name);
    case kFaultWorkspace:
      if (ws == kTakesWorkspace) return fail(AWQ_EWORKSPACE, "%s: AWQ_FAULT=workspace (injected)", name);
      return AWQ_OK;
    case kFaultLaunch:
      return fail(AWQ_ECUDA, "%s: AWQ_FAULT=launch (injected): %s", name, cudaGetErrorName(cudaErrorLaunchFailure));
    default: return AWQ_OK;
  }
}

#define AWQ_ENTRY(name, ws, ...)                                  \
  do {                                                            \
    const int awq_entry_rc_ = api_entry((name), (ws), __VA_ARGS__); \
    if (awq_entry_rc_ != AWQ_OK) return awq_entry_rc_;            \
  } while (0)

int fail_cuda(cudaError_t e, const char* what) {
  return fail(AWQ_ECUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

constexpr int64_t kMaxDim = int64_t(1) << 24;
// Kernels index groups and 64-channel slabs of D_in with gridDim.y (< 65536).
constexpr int64_t kMaxDin = int64_t(1) << 20;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Current device: its SM count, and whether it is an sm_100 part.
int device_info(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute");
  if (major != 10) return fail(AWQ_EUNSUPPORTED, "device %d has compute capability %d.x; this library is built for sm_100a", dev, major);
  e = cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute");
  return AWQ_OK;
}

uint64_t read_timeout_ns() {
  uint64_t ms = 2000;
  if (const char* env = getenv("AWQ_TIMEOUT_MS")) {
    long long v = atoll(env);
    if (v > 0) ms = static_cast<uint64_t>(v);
  }
  return ms * 1000000ull;
}

// The bounded-wait limit of the kernels, read from AWQ_TIMEOUT_MS once (a
// function-local static is initialised exactly once, even with several host
// threads).
uint64_t timeout_ns() {
  static const uint64_t t = read_timeout_ns();
  return t;
}

struct SearchLayout {
  size_t s_tab, r_tab, op, wt, yref, partial, blk, status, sync, total;
  int grid, H, nblk;
};

SearchLayout search_layout(int64_t N, int64_t D_in, int64_t D_out, int A, int group, int form, int num_sms) {
  SearchLayout L{};
  awq::SearchShape sh{static_cast<int>(N), static_cast<int>(D_in), static_cast<int>(D_out), A, 4, group, form};
  const bool ref = form == AWQ_LOSS_REFERENCE;
  L.grid = awq::search_grid_size(sh, num_sms);
  L.H = awq::search_partial_rows(static_cast<int>(N));
  L.nblk = awq::loss_reduce_blocks(D_out);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += round_up(bytes, 256);
    return o;
  };
  const size_t a = static_cast<size_t>(A);
  L.s_tab = take(a * D_in * 4);
  L.r_tab = take(a * D_in * 4);
  L.op = take(a * D_out * D_in * 2);
  L.wt = take(ref ? static_cast<size_t>(D_out) * D_in * 2 : 0);
  L.yref = take(A > 0 && ref ? static_cast<size_t>(L.grid) * 128 * 256 * 4 : 0);
  L.partial = take(a * L.H * D_out * 4);
  L.blk = take(a * L.nblk * 8);
  L.status = take(4);
  L.sync = take(4);
  L.total = off;
  return L;
}

int check_form(int form) {
  if (form != AWQ_LOSS_ERROR && form != AWQ_LOSS_REFERENCE)
    return fail(AWQ_EINVAL, "loss_form = %d: use AWQ_LOSS_ERROR or AWQ_LOSS_REFERENCE", form);
  return AWQ_OK;
}

int check_quant_args(int bits, int group) {
  if (bits < 2 || bits > 4) return fail(AWQ_EUNSUPPORTED, "bits = %d: supported bit widths are 2, 3 and 4", bits);
  if (group != 32 && group != 64 && group != 128 && group != 256)
    return fail(AWQ_EUNSUPPORTED, "group = %d: supported group sizes are 32, 64, 128 and 256", group);
  return AWQ_OK;
}

int check_layer_shape(int64_t N, int64_t D_in, int64_t D_out) {
  if (N < 1 || N > kMaxDim) return fail(AWQ_EINVAL, "N = %lld: need 1 <= N <= 2^24", (long long)N);
  if (D_in < 8 || D_in > kMaxDin || D_in % 8) return fail(AWQ_EINVAL, "D_in = %lld: need a multiple of 8 in [8, 2^20]", (long long)D_in);
  if (D_out < 4 || D_out > kMaxDim || D_out % 4) return fail(AWQ_EINVAL, "D_out = %lld: need a multiple of 4 in [4, 2^24]", (long long)D_out);
  // Tiles of 128 output columns x 256 tokens are numbered with 32-bit ints.
  if (((D_out + 127) / 128) * ((N + 255) / 256) > (int64_t(1) << 30))
    return fail(AWQ_EINVAL, "N x D_out = %lld x %lld is too large", (long long)N, (long long)D_out);
  return AWQ_OK;
}

int check_ptr(const void* p, const char* name, size_t align) {
  if (!p) return fail(AWQ_EINVAL, "%s is NULL", name);
  if (!aligned(p, align)) return fail(AWQ_EALIGN, "%s is not %zu-byte aligned", name, align);
  return AWQ_OK;
}

// ---------------------------------------------------------------- stage timing
struct ProfRec {
  int stage;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_pending;
double g_prof_ms[AWQ_NUM_STAGES] = {};
int g_prof_n[AWQ_NUM_STAGES] = {};

// Brackets one kernel launch with events when profiling is on.
struct StageTimer {
  int stage;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  StageTimer(int stage_, cudaStream_t st_) : stage(stage_), st(st_) {
    if (!g_prof_on) return;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) {
      a = b = nullptr;
      return;
    }
    cudaEventRecord(a, st);
  }
  ~StageTimer() {
    if (!a) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_pending.push_back({stage, a, b});
  }
};

void prof_collect() {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof_pending) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      g_prof_ms[r.stage] += ms;
      g_prof_n[r.stage] += 1;
    }
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_prof_pending.clear();
}

#define AWQ_TRY(expr)            \
  do {                           \
    int _rc = (expr);            \
    if (_rc != AWQ_OK) return _rc; \
  } while (0)

// Quantiser and scale variants of the search (awq_search_ex).
struct SearchOpts {
  int qmode = awq::kQuantSymmetric;
  const float* w_mean = nullptr;    // balanced scale a^alpha / w_mean^(1 - alpha) when set
  bool gram = false;                // L = sum_n e_n^T (X^T X) e_n (error form only)
  int64_t ldw = 0;                  // row stride of W in elements (0: D_out)
};

// Workspace of the Gram form: X^T (tokens padded to 8), H = X^T X in fp32 and
// in bf16, then the search's own layout for D_in "tokens" (the rows of H).
struct GramLayout {
  int64_t Np;
  size_t xt, hf, hb, search, total;
  SearchLayout sl;
};

GramLayout gram_layout(int64_t N, int64_t D_in, int64_t D_out, int A, int group, int num_sms) {
  GramLayout g{};
  g.Np = (N + 7) / 8 * 8;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += round_up(bytes, 256);
    return o;
  };
  g.xt = take(static_cast<size_t>(D_in) * g.Np * 2);
  g.hf = take(static_cast<size_t>(D_in) * D_in * 4);
  g.hb = take(static_cast<size_t>(D_in) * D_in * 2);
  g.sl = search_layout(D_in, D_in, D_out, A, group, awq::kFormGram, num_sms);
  g.search = take(g.sl.total);
  g.total = off;
  return g;
}

// The search for one layer with a workspace already checked; does not reset
// the status word.
int search_one(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
               const awq::AlphaList& alphas, int A, int bits, int group, int form, double* L, double* L_col,
               float* alpha_star, int32_t* alpha_idx, uint8_t* ws, int32_t* status, cudaStream_t st,
               int num_sms, const SearchOpts& opts = SearchOpts()) {
  const SearchLayout lay = search_layout(N, D_in, D_out, A, group, form, num_sms);
  const int64_t ldw = opts.ldw > 0 ? opts.ldw : D_out;
  float* s_tab = reinterpret_cast<float*>(ws + lay.s_tab);
  float* r_tab = reinterpret_cast<float*>(ws + lay.r_tab);
  uint16_t* op = reinterpret_cast<uint16_t*>(ws + lay.op);
  uint16_t* wt = form == AWQ_LOSS_REFERENCE ? reinterpret_cast<uint16_t*>(ws + lay.wt) : nullptr;
  float* yref = reinterpret_cast<float*>(ws + lay.yref);
  float* partial = reinterpret_cast<float*>(ws + lay.partial);
  double* blk = reinterpret_cast<double*>(ws + lay.blk);

  cudaError_t e;
  {
    StageTimer t(AWQ_STAGE_SCALE_TABLE, st);
    e = awq::launch_scale_table(a, opts.w_mean, D_in, alphas, nullptr, A, s_tab, r_tab, st);
  }
  if (e != cudaSuccess) return fail_cuda(e, "scale table kernel");
  {
    StageTimer t(AWQ_STAGE_SEARCH_OPERAND, st);
    const int op_form = form == awq::kFormGram ? awq::kFormError : form;   // the Gram form reads E = S^-1 Q(SW) - W
    e = awq::launch_search_operand(W, ldw, s_tab, r_tab, D_in, D_out, A, bits, group, op_form, opts.qmode, op, st);
  }
  if (e != cudaSuccess) return fail_cuda(e, "search operand kernel");
  if (wt) {
    StageTimer t(AWQ_STAGE_WEIGHT_T, st);
    e = awq::launch_weight_t(W, ldw, D_in, D_out, wt, st);
  }
  if (e != cudaSuccess) return fail_cuda(e, "weight transpose kernel");
  awq::SearchShape sh{static_cast<int>(N), static_cast<int>(D_in), static_cast<int>(D_out), A, bits, group, form};
  awq::SearchBuffers b{X, wt, op, yref, partial, nullptr, status, reinterpret_cast<unsigned*>(ws + lay.sync)};
  const char* what = "search kernel";
  int rc;
  {
    StageTimer t(AWQ_STAGE_SEARCH_GEMM, st);
    rc = awq::launch_search(sh, b, lay.grid, timeout_ns(), st, &e, &what);
  }
  if (rc != AWQ_OK) return e != cudaSuccess ? fail_cuda(e, what) : fail(rc, "%s failed", what);
  {
    StageTimer t(AWQ_STAGE_LOSS_REDUCE, st);
    e = awq::launch_loss_reduce(partial, A, lay.H, D_out, L_col, blk, lay.nblk, alphas, L, alpha_star,
                                alpha_idx, st);
  }
  if (e != cudaSuccess) return fail_cuda(e, "loss reduction kernels");
  return AWQ_OK;
}

int check_search_args(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
                      const float* alpha_grid, int n_alpha, int bits, int group, int form, double* L, double* L_col,
                      float* alpha_star, int32_t* alpha_idx) {
  AWQ_TRY(check_layer_shape(N, D_in, D_out));
  AWQ_TRY(check_quant_args(bits, group));
  AWQ_TRY(check_form(form));
  if (D_in % group) return fail(AWQ_EINVAL, "D_in = %lld is not a multiple of group = %d", (long long)D_in, group);
  if (n_alpha < 1 || n_alpha > AWQ_MAX_ALPHA) return fail(AWQ_EUNSUPPORTED, "n_alpha = %d: need 1..%d", n_alpha, AWQ_MAX_ALPHA);
  if (!alpha_grid) return fail(AWQ_EINVAL, "alpha_grid is NULL");
  AWQ_TRY(check_ptr(X, "X", 16));
  AWQ_TRY(check_ptr(W, "W", 16));
  AWQ_TRY(check_ptr(a, "a", 16));
  AWQ_TRY(check_ptr(L, "L", 8));
  if (L_col) AWQ_TRY(check_ptr(L_col, "L_col", 8));
  AWQ_TRY(check_ptr(alpha_star, "alpha_star", 4));
  AWQ_TRY(check_ptr(alpha_idx, "alpha_idx", 4));
  return AWQ_OK;
}

// ---------------------------------------------------------------- scratch without allocation
// Scratch for awq_search_noalloc: a file-scope device array.  Host code must
// not use its name as a device address; the address comes from
// cudaGetSymbolAddress, once per device (and again if that device's context
// was torn down and made anew, which reloads the module), with that device
// current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[AWQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoallocAddr {
  unsigned long long ctx;   // current_context_id() when the address was looked up
  void* ptr;
};
NoallocAddr g_noalloc[kMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(AWQ_EUNSUPPORTED, "device %d: at most %d devices", dev, kMaxDevices);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  const unsigned long long ctx = awq::current_context_id();
  if (ctx == 0 || g_noalloc[dev].ctx != ctx || !g_noalloc[dev].ptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(no-allocation scratch)");
    // the lookup made the device's context current if it was not yet
    g_noalloc[dev] = {awq::current_context_id(), ptr};
  }
  *out = g_noalloc[dev].ptr;
  return AWQ_OK;
}

}  // namespace

namespace awq {

namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult qres;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
      qres == cudaDriverEntryPointSuccess)
    return reinterpret_cast<F>(ptr);
  return nullptr;
}
}  // namespace

unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace awq

extern "C" {

const char* awq_get_last_error(void) { return g_last_error.c_str(); }

int awq_version(void) { return 100; }

int awq_act_stats(const void* X, int64_t N, int64_t D_in, int stat, float* a, void* stream) {
  AWQ_ENTRY("awq_act_stats", kNoWorkspace, "N=%lld D_in=%lld stat=%d", (long long)N, (long long)D_in, stat);

  if (N < 1 || N > kMaxDim) return fail(AWQ_EINVAL, "N = %lld: need 1 <= N <= 2^24", (long long)N);
  if (D_in < 8 || D_in > kMaxDin || D_in % 8) return fail(AWQ_EINVAL, "D_in = %lld: need a multiple of 8 in [8, 2^20]", (long long)D_in);
  if (stat != AWQ_STAT_MEAN && stat != AWQ_STAT_MAX) return fail(AWQ_EINVAL, "stat = %d: use AWQ_STAT_MEAN or AWQ_STAT_MAX", stat);
  AWQ_TRY(check_ptr(X, "X", 16));
  AWQ_TRY(check_ptr(a, "a", 16));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  cudaError_t e;
  {
    StageTimer t(AWQ_STAGE_ACT_STATS, static_cast<cudaStream_t>(stream));
    e = awq::launch_act_stats(static_cast<const uint16_t*>(X), N, D_in, stat, a, sms, static_cast<cudaStream_t>(stream));
  }
  return e == cudaSuccess ? AWQ_OK : fail_cuda(e, "act_stats kernel");
}

int awq_act_stats_batched(const void* const* Xs, const int64_t* Ns, const int64_t* D_ins, int n_inputs, int stat,
                          float* const* as, void* stream) {
  AWQ_ENTRY("awq_act_stats_batched", kNoWorkspace, "n_inputs=%d stat=%d", n_inputs, stat);
  if (!Xs || !Ns || !D_ins || !as) return fail(AWQ_EINVAL, "Xs, Ns, D_ins and as must not be NULL");
  if (n_inputs < 1 || n_inputs > awq::kMaxStatsInputs)
    return fail(AWQ_EUNSUPPORTED, "n_inputs = %d: need 1..%d", n_inputs, awq::kMaxStatsInputs);
  if (stat != AWQ_STAT_MEAN && stat != AWQ_STAT_MAX) return fail(AWQ_EINVAL, "stat = %d: use AWQ_STAT_MEAN or AWQ_STAT_MAX", stat);
  for (int i = 0; i < n_inputs; ++i) {
    if (Ns[i] < 1 || Ns[i] > kMaxDim) return fail(AWQ_EINVAL, "input %d: N = %lld: need 1 <= N <= 2^24", i, (long long)Ns[i]);
    if (D_ins[i] < 8 || D_ins[i] > kMaxDin || D_ins[i] % 8)
      return fail(AWQ_EINVAL, "input %d: D_in = %lld: need a multiple of 8 in [8, 2^20]", i, (long long)D_ins[i]);
    int rc = check_ptr(Xs[i], "X", 16);
    if (rc == AWQ_OK) rc = check_ptr(as[i], "a", 16);
    if (rc != AWQ_OK) return fail(rc, "input %d: %s", i, g_last_error.c_str());
  }
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  cudaError_t e;
  {
    StageTimer t(AWQ_STAGE_ACT_STATS, static_cast<cudaStream_t>(stream));
    e = awq::launch_act_stats_batched(reinterpret_cast<const uint16_t* const*>(Xs), Ns, D_ins, n_inputs, stat, as,
                                      sms, static_cast<cudaStream_t>(stream));
  }
  return e == cudaSuccess ? AWQ_OK : fail_cuda(e, "act_stats kernel");
}

static int scales_common(const float* a, const float* w_mean, int64_t D_in, float alpha, const float* alpha_dev,
                         float* s, void* stream) {
  if (D_in < 1 || D_in > kMaxDim) return fail(AWQ_EINVAL, "D_in = %lld out of range", (long long)D_in);
  AWQ_TRY(check_ptr(a, "a", 4));
  AWQ_TRY(check_ptr(s, "s", 4));
  if (w_mean) AWQ_TRY(check_ptr(w_mean, "w_mean", 4));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  awq::AlphaList al{};
  al.v[0] = alpha;
  cudaError_t e;
  {
    StageTimer t(AWQ_STAGE_SCALE_TABLE, static_cast<cudaStream_t>(stream));
    e = awq::launch_scale_table(a, w_mean, D_in, al, alpha_dev, 1, s, nullptr, static_cast<cudaStream_t>(stream));
  }
  return e == cudaSuccess ? AWQ_OK : fail_cuda(e, "scale table kernel");
}

int awq_scales(const float* a, int64_t D_in, float alpha, float* s, void* stream) {
  AWQ_ENTRY("awq_scales", kNoWorkspace, "D_in=%lld alpha=%g", (long long)D_in, alpha);

  return scales_common(a, nullptr, D_in, alpha, nullptr, s, stream);
}

int awq_scales_dev(const float* a, int64_t D_in, const float* alpha_dev, float* s, void* stream) {
  AWQ_ENTRY("awq_scales_dev", kNoWorkspace, "D_in=%lld", (long long)D_in);

  AWQ_TRY(check_ptr(alpha_dev, "alpha_dev", 4));
  return scales_common(a, nullptr, D_in, 0.0f, alpha_dev, s, stream);
}

int awq_scales_ex(const float* a, const float* w_mean, int64_t D_in, float alpha, const float* alpha_dev, float* s,
                  void* stream) {
  AWQ_ENTRY("awq_scales_ex", kNoWorkspace, "D_in=%lld alpha=%g weight_statistic=%d", (long long)D_in, alpha, w_mean ? 1 : 0);
  if (alpha_dev) AWQ_TRY(check_ptr(alpha_dev, "alpha_dev", 4));
  if (!alpha_dev && !(alpha >= 0.0f && alpha <= 1.0f)) return fail(AWQ_EINVAL, "alpha = %g: need 0 <= alpha <= 1", alpha);
  return scales_common(a, w_mean, D_in, alpha, alpha_dev, s, stream);
}

int awq_weight_mean(const float* W, int64_t D_in, int64_t D_out, float* w_mean, void* stream) {
  AWQ_ENTRY("awq_weight_mean", kNoWorkspace, "D_in=%lld D_out=%lld", (long long)D_in, (long long)D_out);

  if (D_in < 1 || D_in > kMaxDim || D_out < 1 || D_out > kMaxDim)
    return fail(AWQ_EINVAL, "D_in = %lld, D_out = %lld out of range", (long long)D_in, (long long)D_out);
  AWQ_TRY(check_ptr(W, "W", 16));
  AWQ_TRY(check_ptr(w_mean, "w_mean", 4));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  cudaError_t e = awq::launch_weight_mean(W, D_in, D_out, w_mean, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AWQ_OK : fail_cuda(e, "weight mean kernel");
}

size_t awq_search_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int n_alpha, int bits, int group,
                                 int loss_form) {
  if (check_layer_shape(N, D_in, D_out) != AWQ_OK || check_quant_args(bits, group) != AWQ_OK) return 0;
  if (check_form(loss_form) != AWQ_OK) return 0;
  if (D_in % group || n_alpha < 1 || n_alpha > AWQ_MAX_ALPHA) return 0;
  int sms = 0;
  if (device_info(&sms) != AWQ_OK) return 0;
  return search_layout(N, D_in, D_out, n_alpha, group, loss_form, sms).total;
}

static int search_impl(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
                       const float* alpha_grid, int n_alpha, int bits, int group, int loss_form, double* L,
                       double* L_col, float* alpha_star, int32_t* alpha_idx, void* workspace, size_t workspace_bytes,
                       int32_t* status, void* stream, const SearchOpts& opts) {
  AWQ_TRY(check_search_args(X, W, a, N, D_in, D_out, alpha_grid, n_alpha, bits, group, loss_form, L, L_col,
                            alpha_star, alpha_idx));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  if (opts.gram) {
    // L(alpha) = sum_n e_n^T H e_n with H = X^T X (Gram form): H once, then the
    // search GEMM over the D_in rows of H instead of the N tokens of X.
    if (loss_form != AWQ_LOSS_ERROR) return fail(AWQ_EINVAL, "the Gram form evaluates the error form only");
    const GramLayout gl = gram_layout(N, D_in, D_out, n_alpha, group, sms);
    if (!workspace) return fail(AWQ_EWORKSPACE, "workspace is NULL");
    if (!aligned(workspace, 256)) return fail(AWQ_EALIGN, "workspace is not 256-byte aligned");
    if (workspace_bytes < gl.total)
      return fail(AWQ_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, gl.total);
    if (status && !aligned(status, 4)) return fail(AWQ_EALIGN, "status is not 4-byte aligned");
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* sws = ws + gl.search;
    int32_t* st_word = status ? status : reinterpret_cast<int32_t*>(sws + gl.sl.status);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(st_word, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
    uint16_t* xt = reinterpret_cast<uint16_t*>(ws + gl.xt);
    float* hf = reinterpret_cast<float*>(ws + gl.hf);
    uint16_t* hb = reinterpret_cast<uint16_t*>(ws + gl.hb);
    {
      StageTimer t(AWQ_STAGE_CLIP_GRAM, st);
      e = awq::launch_xt(static_cast<const uint16_t*>(X), N, D_in, gl.Np, xt, st);
      if (e != cudaSuccess) return fail_cuda(e, "transpose of X");
      // H = X^T X by the search GEMM in its output-only mode: "tokens" are the
      // D_in rows of X^T, the reduction runs over the (padded) tokens of X.
      awq::SearchShape shH{static_cast<int>(D_in), static_cast<int>(gl.Np), static_cast<int>(D_in), 0, 4, 128,
                           AWQ_LOSS_REFERENCE};
      awq::SearchBuffers bH{xt, xt, nullptr, nullptr, nullptr, hf, st_word};
      const char* what = "search kernel (Gram matrix)";
      const int rc = awq::launch_search(shH, bH, awq::search_grid_size(shH, sms), timeout_ns(), st, &e, &what);
      if (rc != AWQ_OK) return e != cudaSuccess ? fail_cuda(e, what) : fail(rc, "%s failed", what);
      e = awq::launch_to_bf16(hf, D_in * D_in, hb, st);
      if (e != cudaSuccess) return fail_cuda(e, "bf16 rounding of the Gram matrix");
    }
    awq::AlphaList al{};
    for (int i = 0; i < n_alpha; ++i) al.v[i] = alpha_grid[i];
    return search_one(hb, W, a, D_in, D_in, D_out, al, n_alpha, bits, group, awq::kFormGram, L, L_col, alpha_star,
                      alpha_idx, sws, st_word, st, sms, opts);
  }
  const SearchLayout lay = search_layout(N, D_in, D_out, n_alpha, group, loss_form, sms);
  if (!workspace) return fail(AWQ_EWORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(AWQ_EALIGN, "workspace is not 256-byte aligned");
  if (workspace_bytes < lay.total)
    return fail(AWQ_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, lay.total);
  if (status && !aligned(status, 4)) return fail(AWQ_EALIGN, "status is not 4-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* st_word = status ? status : reinterpret_cast<int32_t*>(ws + lay.status);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(st_word, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  awq::AlphaList al{};
  for (int i = 0; i < n_alpha; ++i) al.v[i] = alpha_grid[i];
  return search_one(X, W, a, N, D_in, D_out, al, n_alpha, bits, group, loss_form, L, L_col, alpha_star, alpha_idx,
                    ws, st_word, st, sms, opts);
}

int awq_search(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
               const float* alpha_grid, int n_alpha, int bits, int group, int loss_form, double* L, double* L_col,
               float* alpha_star, int32_t* alpha_idx, void* workspace, size_t workspace_bytes, int32_t* status,
               void* stream) {
  AWQ_ENTRY("awq_search", kTakesWorkspace, "N=%lld D_in=%lld D_out=%lld n_alpha=%d bits=%d group=%d form=%d", (long long)N, (long long)D_in, (long long)D_out, n_alpha, bits, group, loss_form);
  return search_impl(X, W, a, N, D_in, D_out, alpha_grid, n_alpha, bits, group, loss_form, L, L_col, alpha_star,
                     alpha_idx, workspace, workspace_bytes, status, stream, SearchOpts());
}

int awq_search_ex(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
                  const float* alpha_grid, int n_alpha, int bits, int group, int loss_form,
                  const awq_search_options* options, double* L, double* L_col, float* alpha_star,
                  int32_t* alpha_idx, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  AWQ_ENTRY("awq_search_ex", kTakesWorkspace, "N=%lld D_in=%lld D_out=%lld n_alpha=%d bits=%d group=%d form=%d", (long long)N, (long long)D_in, (long long)D_out, n_alpha, bits, group, loss_form);
  SearchOpts o;
  if (options) {
    switch (options->quantizer) {
      case AWQ_QUANT_SYMMETRIC: o.qmode = awq::kQuantSymmetric; break;
      case AWQ_QUANT_DELTA_POW2: o.qmode = awq::kQuantPow2; break;
      case AWQ_QUANT_ASYMMETRIC: o.qmode = awq::kQuantAsymmetric; break;
      default:
        return fail(AWQ_EINVAL, "quantizer = %d: need AWQ_QUANT_SYMMETRIC, AWQ_QUANT_DELTA_POW2 or AWQ_QUANT_ASYMMETRIC",
                    options->quantizer);
    }
    if (options->w_mean) AWQ_TRY(check_ptr(options->w_mean, "w_mean", 4));
    o.w_mean = options->w_mean;
    o.gram = options->gram_form != 0;
    if (options->ldw != 0 && (options->ldw < D_out || options->ldw % 4 || options->ldw > kMaxDim))
      return fail(AWQ_EINVAL, "ldw = %lld: need 0, or a multiple of 4 with D_out = %lld <= ldw <= 2^24",
                  (long long)options->ldw, (long long)D_out);
    o.ldw = options->ldw;
  }
  return search_impl(X, W, a, N, D_in, D_out, alpha_grid, n_alpha, bits, group, loss_form, L, L_col, alpha_star,
                     alpha_idx, workspace, workspace_bytes, status, stream, o);
}

size_t awq_search_ex_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int n_alpha, int bits, int group,
                                    int loss_form, const awq_search_options* options) {
  if (!options || !options->gram_form) return awq_search_workspace_size(N, D_in, D_out, n_alpha, bits, group, loss_form);
  if (check_layer_shape(N, D_in, D_out) != AWQ_OK || check_quant_args(bits, group) != AWQ_OK) return 0;
  if (loss_form != AWQ_LOSS_ERROR || D_in % group || n_alpha < 1 || n_alpha > AWQ_MAX_ALPHA) return 0;
  int sms = 0;
  if (device_info(&sms) != AWQ_OK) return 0;
  return gram_layout(N, D_in, D_out, n_alpha, group, sms).total;
}

size_t awq_search_batched_workspace_size(const awq_layer* layers, int n_layers, int n_alpha, int bits, int group,
                                         int loss_form) {
  if (!layers || n_layers < 1) return 0;
  size_t m = 0;
  for (int i = 0; i < n_layers; ++i) {
    size_t s = awq_search_workspace_size(layers[i].N, layers[i].D_in, layers[i].D_out, n_alpha, bits, group,
                                         loss_form);
    if (s == 0) return 0;
    if (s > m) m = s;
  }
  return m + 256;   // + the batch's own status word after the largest layout
}

int awq_search_batched(const awq_layer* layers, int n_layers, const float* alpha_grid, int n_alpha, int bits,
                       int group, int loss_form, void* workspace, size_t workspace_bytes, int32_t* status,
                       void* stream) {
  AWQ_ENTRY("awq_search_batched", kTakesWorkspace, "n_layers=%d n_alpha=%d bits=%d group=%d form=%d", n_layers, n_alpha, bits, group, loss_form);
  if (!layers || n_layers < 1) return fail(AWQ_EINVAL, "layers is NULL or n_layers < 1");
  for (int i = 0; i < n_layers; ++i) {
    const awq_layer& l = layers[i];
    int rc = check_search_args(l.X, l.W, l.a, l.N, l.D_in, l.D_out, alpha_grid, n_alpha, bits, group, loss_form,
                               l.L, l.L_col, l.alpha_star, l.alpha_idx);
    if (rc != AWQ_OK) return fail(rc, "layer %d: %s", i, g_last_error.c_str());
  }
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  size_t need = 0;
  for (int i = 0; i < n_layers; ++i) {
    size_t s = search_layout(layers[i].N, layers[i].D_in, layers[i].D_out, n_alpha, group, loss_form, sms).total;
    if (s > need) need = s;
  }
  if (!workspace) return fail(AWQ_EWORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(AWQ_EALIGN, "workspace is not 256-byte aligned");
  if (workspace_bytes < need + 256)
    return fail(AWQ_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need + 256);
  if (status && !aligned(status, 4)) return fail(AWQ_EALIGN, "status is not 4-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Every layer's layout ends at or before `need`; the batch status word sits after it.
  int32_t* st_word = status ? status : reinterpret_cast<int32_t*>(ws + need);
  cudaError_t e = cudaMemsetAsync(st_word, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  awq::AlphaList al{};
  for (int i = 0; i < n_alpha; ++i) al.v[i] = alpha_grid[i];
  for (int i = 0; i < n_layers; ++i) {
    const awq_layer& l = layers[i];
    int rc = search_one(l.X, l.W, l.a, l.N, l.D_in, l.D_out, al, n_alpha, bits, group, loss_form, l.L, l.L_col,
                        l.alpha_star, l.alpha_idx, ws, st_word, st, sms);
    if (rc != AWQ_OK) return rc;
  }
  return AWQ_OK;
}

int awq_quantize_pack(const float* W, const float* s, int64_t D_in, int64_t D_out, int bits, int group,
                      uint32_t* packed, float* scales, void* stream) {
  AWQ_ENTRY("awq_quantize_pack", kNoWorkspace, "D_in=%lld D_out=%lld bits=%d group=%d", (long long)D_in, (long long)D_out, bits, group);
  return awq_quantize_pack_ex(W, s, nullptr, D_in, D_out, bits, group, 0, packed, scales, stream);
}

// ---------------------------------------------------------------- weight-clipping search
struct ClipLayout {
  size_t xt, hb, r, op, status, total;
  int64_t Np;
};

static ClipLayout clip_layout(int64_t N, int64_t D_in, int64_t D_out, int n_clip, int group) {
  ClipLayout L{};
  L.Np = (N + 7) / 8 * 8;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += round_up(bytes, 256);
    return o;
  };
  L.xt = take(static_cast<size_t>(D_in) * L.Np * 2);
  L.hb = take(static_cast<size_t>(D_in) * group * 2);
  L.r = take(static_cast<size_t>(D_in) * 4);
  L.op = take(static_cast<size_t>(n_clip) * D_out * D_in * 2);
  L.status = take(4);
  L.total = off;
  return L;
}

static int check_clip_args(int64_t N, int64_t D_in, int64_t D_out, int n_clip, int bits, int group) {
  AWQ_TRY(check_layer_shape(N, D_in, D_out));
  if (bits < 2 || bits > 4) return fail(AWQ_EUNSUPPORTED, "bits = %d: supported bit widths are 2, 3 and 4", bits);
  if (group != 64 && group != 128)
    return fail(AWQ_EUNSUPPORTED, "group = %d: the clipping search supports groups of 64 and 128", group);
  if (D_in % group) return fail(AWQ_EINVAL, "D_in = %lld is not a multiple of group = %d", (long long)D_in, group);
  if (n_clip < 1 || n_clip > AWQ_MAX_ALPHA) return fail(AWQ_EUNSUPPORTED, "n_clip = %d: need 1..%d", n_clip, AWQ_MAX_ALPHA);
  return AWQ_OK;
}

size_t awq_layer_output_workspace_size(int64_t N, int64_t D_in, int64_t D_out) {
  if (check_layer_shape(N, D_in, D_out) != AWQ_OK) return 0;
  int sms = 0;
  if (device_info(&sms) != AWQ_OK) return 0;
  return search_layout(N, D_in, D_out, 0, 128, AWQ_LOSS_REFERENCE, sms).total;
}

int awq_layer_output(const void* X, const float* W, int64_t N, int64_t D_in, int64_t D_out, float* Y,
                     void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  AWQ_ENTRY("awq_layer_output", kTakesWorkspace, "N=%lld D_in=%lld D_out=%lld", (long long)N, (long long)D_in, (long long)D_out);
  AWQ_TRY(check_layer_shape(N, D_in, D_out));
  AWQ_TRY(check_ptr(X, "X", 16));
  AWQ_TRY(check_ptr(W, "W", 16));
  AWQ_TRY(check_ptr(Y, "Y", 16));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  const SearchLayout lay = search_layout(N, D_in, D_out, 0, 128, AWQ_LOSS_REFERENCE, sms);
  if (!workspace) return fail(AWQ_EWORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(AWQ_EALIGN, "workspace is not 256-byte aligned");
  if (workspace_bytes < lay.total)
    return fail(AWQ_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, lay.total);
  if (status && !aligned(status, 4)) return fail(AWQ_EALIGN, "status is not 4-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* st_word = status ? status : reinterpret_cast<int32_t*>(ws + lay.status);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(st_word, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  uint16_t* wt = reinterpret_cast<uint16_t*>(ws + lay.wt);
  {
    StageTimer t(AWQ_STAGE_WEIGHT_T, st);
    e = awq::launch_weight_t(W, D_out, D_in, D_out, wt, st);
  }
  if (e != cudaSuccess) return fail_cuda(e, "weight transpose kernel");
  awq::SearchShape sh{static_cast<int>(N), static_cast<int>(D_in), static_cast<int>(D_out), 0, 4, 128,
                      AWQ_LOSS_REFERENCE};
  awq::SearchBuffers b{X, wt, nullptr, nullptr, nullptr, Y, st_word};
  const char* what = "search kernel (reference output)";
  int rc;
  {
    StageTimer t(AWQ_STAGE_SEARCH_GEMM, st);
    rc = awq::launch_search(sh, b, lay.grid, timeout_ns(), st, &e, &what);
  }
  if (rc != AWQ_OK) return e != cudaSuccess ? fail_cuda(e, what) : fail(rc, "%s failed", what);
  return AWQ_OK;
}

int awq_profile_enable(int on) {
  g_prof_on = on != 0;
  return AWQ_OK;
}

int awq_profile_reset(void) {
  prof_collect();
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int i = 0; i < AWQ_NUM_STAGES; ++i) {
    g_prof_ms[i] = 0.0;
    g_prof_n[i] = 0;
  }
  return AWQ_OK;
}

int awq_profile_read(int stage, double* total_ms, int32_t* launches) {
  if (stage < 0 || stage >= AWQ_NUM_STAGES) return fail(AWQ_EINVAL, "stage = %d out of range", stage);
  prof_collect();
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (total_ms) *total_ms = g_prof_ms[stage];
  if (launches) *launches = g_prof_n[stage];
  return AWQ_OK;
}

int awq_search_noalloc(const void* X, const float* W, const float* a, int64_t N, int64_t D_in, int64_t D_out,
                       const float* alpha_grid, int n_alpha, int bits, int group, int loss_form, double* L,
                       double* L_col, float* alpha_star, int32_t* alpha_idx, int32_t* status, void* stream) {
  AWQ_ENTRY("awq_search_noalloc", kTakesWorkspace, "N=%lld D_in=%lld D_out=%lld n_alpha=%d bits=%d group=%d form=%d", (long long)N, (long long)D_in, (long long)D_out, n_alpha, bits, group, loss_form);
  AWQ_TRY(check_search_args(X, W, a, N, D_in, D_out, alpha_grid, n_alpha, bits, group, loss_form, L, L_col,
                            alpha_star, alpha_idx));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  const SearchLayout lay = search_layout(N, D_in, D_out, n_alpha, group, loss_form, sms);
  if (lay.total > AWQ_NOALLOC_SCRATCH_BYTES)
    return fail(AWQ_EWORKSPACE,
                "awq_search_noalloc: this shape needs %zu bytes of scratch, the built-in scratch holds %u; "
                "use awq_search with a workspace",
                lay.total, static_cast<unsigned>(AWQ_NOALLOC_SCRATCH_BYTES));
  // The status word is required: inside the shared scratch array a device-side
  // timeout could not be read by the caller and the next call would clear it.
  if (!status) return fail(AWQ_EINVAL, "status is NULL: awq_search_noalloc needs the caller's device status word");
  AWQ_TRY(check_ptr(status, "status", 4));
  void* scratch = nullptr;
  AWQ_TRY(noalloc_scratch(&scratch));
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  int32_t* st_word = status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Every scratch byte the search reads it writes first in the same call;
  // only the status word (the caller's) has to start at zero.
  cudaError_t e = cudaMemsetAsync(st_word, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  awq::AlphaList al{};
  for (int i = 0; i < n_alpha; ++i) al.v[i] = alpha_grid[i];
  return search_one(X, W, a, N, D_in, D_out, al, n_alpha, bits, group, loss_form, L, L_col, alpha_star, alpha_idx,
                    ws, st_word, st, sms);
}

int awq_selftest_wait_timeout(int32_t* status, int64_t timeout_ns_arg, void* stream) {
  AWQ_ENTRY("awq_selftest_wait_timeout", kNoWorkspace, "timeout_ns=%lld", (long long)timeout_ns_arg);

  AWQ_TRY(check_ptr(status, "status", 4));
  if (timeout_ns_arg < 1000 || timeout_ns_arg > 10000000000LL)
    return fail(AWQ_EINVAL, "timeout_ns = %lld: need 1 us .. 10 s", (long long)timeout_ns_arg);
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  e = awq::launch_wait_timeout_selftest(status, static_cast<uint64_t>(timeout_ns_arg), st);
  return e == cudaSuccess ? AWQ_OK : fail_cuda(e, "self-test kernel");
}


int awq_selftest_divide(int32_t divisor, uint64_t* mismatches, void* stream) {
  AWQ_ENTRY("awq_selftest_divide", kNoWorkspace, "divisor=%d", divisor);

  AWQ_TRY(check_ptr(mismatches, "mismatches", 8));
  if (divisor < 1 || divisor > 255) return fail(AWQ_EINVAL, "divisor = %d: need 1 .. 255", divisor);
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(mismatches, 0, 2 * sizeof(uint64_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(mismatches)");
  e = awq::launch_divide_selftest(static_cast<float>(divisor), reinterpret_cast<unsigned long long*>(mismatches), sms,
                                  st);
  return e == cudaSuccess ? AWQ_OK : fail_cuda(e, "divide self-test kernel");
}

size_t awq_clip_search_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int n_clip, int bits, int group) {
  if (check_clip_args(N, D_in, D_out, n_clip, bits, group) != AWQ_OK) return 0;
  return clip_layout(N, D_in, D_out, n_clip, group).total;
}

int awq_clip_search(const void* X, const float* W, const float* s, int64_t N, int64_t D_in, int64_t D_out,
                    const float* clip_grid, int n_clip, int bits, int group, float* clip, int32_t* clip_idx,
                    float* loss, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  AWQ_ENTRY("awq_clip_search", kTakesWorkspace, "N=%lld D_in=%lld D_out=%lld n_clip=%d bits=%d group=%d", (long long)N, (long long)D_in, (long long)D_out, n_clip, bits, group);
  AWQ_TRY(check_clip_args(N, D_in, D_out, n_clip, bits, group));
  if (!clip_grid) return fail(AWQ_EINVAL, "clip_grid is NULL");
  for (int i = 0; i < n_clip; ++i)
    if (!(clip_grid[i] > 0.0f && clip_grid[i] <= 1.0f))
      return fail(AWQ_EINVAL, "clip_grid[%d] = %g: ratios must lie in (0, 1]", i, (double)clip_grid[i]);
  AWQ_TRY(check_ptr(X, "X", 16));
  AWQ_TRY(check_ptr(W, "W", 16));
  AWQ_TRY(check_ptr(s, "s", 16));
  AWQ_TRY(check_ptr(clip, "clip", 4));
  if (clip_idx) AWQ_TRY(check_ptr(clip_idx, "clip_idx", 4));
  if (loss) AWQ_TRY(check_ptr(loss, "loss", 4));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  const ClipLayout lay = clip_layout(N, D_in, D_out, n_clip, group);
  if (!workspace) return fail(AWQ_EWORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(AWQ_EALIGN, "workspace is not 256-byte aligned");
  if (workspace_bytes < lay.total)
    return fail(AWQ_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, lay.total);
  if (status && !aligned(status, 4)) return fail(AWQ_EALIGN, "status is not 4-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* st_word = status ? status : reinterpret_cast<int32_t*>(ws + lay.status);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(st_word, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  uint16_t* xt = reinterpret_cast<uint16_t*>(ws + lay.xt);
  uint16_t* hb = reinterpret_cast<uint16_t*>(ws + lay.hb);
  float* r = reinterpret_cast<float*>(ws + lay.r);
  uint16_t* op = reinterpret_cast<uint16_t*>(ws + lay.op);
  awq::AlphaList clips{};
  for (int i = 0; i < n_clip; ++i) clips.v[i] = clip_grid[i];
  const char* what = "clipping search";
  int rc = AWQ_OK;
  {
    StageTimer t(AWQ_STAGE_CLIP_GRAM, st);
    e = awq::launch_xt(static_cast<const uint16_t*>(X), N, D_in, lay.Np, xt, st);
    if (e == cudaSuccess) e = awq::launch_recip(s, D_in, r, st);
    if (e == cudaSuccess) rc = awq::launch_gram(xt, D_in, lay.Np, group, hb, st_word, timeout_ns(), st, &e, &what);
  }
  if (e != cudaSuccess) return fail_cuda(e, what);
  if (rc != AWQ_OK) return fail(rc, "%s failed", what);
  {
    StageTimer t(AWQ_STAGE_CLIP_OPERAND, st);
    e = awq::launch_clip_operand(W, s, r, D_in, D_out, clips, n_clip, bits, group, op, st);
  }
  if (e != cudaSuccess) return fail_cuda(e, "clipping operand kernel");
  {
    StageTimer t(AWQ_STAGE_CLIP_LOSS, st);
    rc = awq::launch_clip_loss(op, hb, D_in, D_out, group, clips, n_clip, clip, clip_idx, loss, sms, st_word,
                               timeout_ns(), st, &e, &what);
  }
  if (rc != AWQ_OK) return e != cudaSuccess ? fail_cuda(e, what) : fail(rc, "%s failed", what);
  return AWQ_OK;
}

int awq_quantize_pack_clip(const float* W, const float* s, const float* clip, int64_t D_in, int64_t D_out, int bits,
                           int group, uint32_t* packed, float* scales, void* stream) {
  AWQ_ENTRY("awq_quantize_pack_clip", kNoWorkspace, "D_in=%lld D_out=%lld bits=%d group=%d", (long long)D_in, (long long)D_out, bits, group);
  if (!clip) return fail(AWQ_EINVAL, "clip is NULL");
  return awq_quantize_pack_ex(W, s, clip, D_in, D_out, bits, group, 0, packed, scales, stream);
}

static int quantize_pack_impl(const float* W, const float* s, const float* clip, int64_t D_in, int64_t D_out,
                              int bits, int group, int flags, int qmode, uint32_t* packed, void* scales,
                              uint8_t* zeros, void* stream) {
  AWQ_TRY(check_quant_args(bits, group));
  if (flags & ~(AWQ_PACK_DELTA_FP16 | AWQ_PACK_DELTA_POW2 | AWQ_PACK_DENSE3))
    return fail(AWQ_EINVAL, "flags = %#x: unknown bits", flags);
  if ((flags & AWQ_PACK_DENSE3) && bits != 3) return fail(AWQ_EINVAL, "AWQ_PACK_DENSE3 needs bits = 3 (bits = %d)", bits);
  if (D_in < group || D_in > kMaxDin || D_in % group)
    return fail(AWQ_EINVAL, "D_in = %lld: need a positive multiple of group = %d", (long long)D_in, group);
  if (D_out < 1 || D_out > kMaxDim) return fail(AWQ_EINVAL, "D_out = %lld out of range", (long long)D_out);
  if ((flags & AWQ_PACK_DENSE3) && D_out % 4 && group < 128)
    return fail(AWQ_EUNSUPPORTED, "AWQ_PACK_DENSE3 with D_out %% 4 != 0 needs group 128 or 256 (group = %d)", group);
  AWQ_TRY(check_ptr(W, "W", 16));
  AWQ_TRY(check_ptr(s, "s", 16));
  if (clip) AWQ_TRY(check_ptr(clip, "clip", 4));
  AWQ_TRY(check_ptr(packed, "packed", 16));
  AWQ_TRY(check_ptr(scales, "scales", 16));
  if (qmode == awq::kQuantAsymmetric) AWQ_TRY(check_ptr(zeros, "zeros", 1));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  cudaError_t e;
  {
    StageTimer t(AWQ_STAGE_QUANTIZE_PACK, static_cast<cudaStream_t>(stream));
    e = awq::launch_quantize_pack(W, s, clip, D_in, D_out, bits, group, (flags & AWQ_PACK_DELTA_FP16) != 0, qmode,
                                  (flags & AWQ_PACK_DENSE3) != 0, packed, scales, zeros, sms,
                                  static_cast<cudaStream_t>(stream));
  }
  return e == cudaSuccess ? AWQ_OK : fail_cuda(e, "quantize_pack kernel");
}

int awq_quantize_pack_ex(const float* W, const float* s, const float* clip, int64_t D_in, int64_t D_out, int bits,
                         int group, int flags, uint32_t* packed, void* scales, void* stream) {
  AWQ_ENTRY("awq_quantize_pack_ex", kNoWorkspace, "D_in=%lld D_out=%lld bits=%d group=%d flags=%d", (long long)D_in, (long long)D_out, bits, group, flags);
  return quantize_pack_impl(W, s, clip, D_in, D_out, bits, group, flags,
                            (flags & AWQ_PACK_DELTA_POW2) ? awq::kQuantPow2 : awq::kQuantSymmetric, packed, scales,
                            nullptr, stream);
}

int awq_quantize_pack_zp(const float* W, const float* s, int64_t D_in, int64_t D_out, int bits, int group, int flags,
                         uint32_t* packed, void* scales, uint8_t* zeros, void* stream) {
  AWQ_ENTRY("awq_quantize_pack_zp", kNoWorkspace, "D_in=%lld D_out=%lld bits=%d group=%d flags=%d", (long long)D_in, (long long)D_out, bits, group, flags);
  if (flags & AWQ_PACK_DELTA_POW2) return fail(AWQ_EINVAL, "AWQ_PACK_DELTA_POW2 does not apply to the asymmetric quantiser");
  return quantize_pack_impl(W, s, nullptr, D_in, D_out, bits, group, flags, awq::kQuantAsymmetric, packed, scales,
                            zeros, stream);
}

// ---------------------------------------------------------------- joint search over shared-input linears
static int check_joint(const int64_t* D_outs, int n_layers, int64_t* Dsum) {
  if (!D_outs) return fail(AWQ_EINVAL, "D_outs is NULL");
  if (n_layers < 1 || n_layers > awq::kMaxJointLayers)
    return fail(AWQ_EUNSUPPORTED, "n_layers = %d: need 1..%d", n_layers, awq::kMaxJointLayers);
  int64_t s = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (D_outs[l] < 4 || D_outs[l] % 4)
      return fail(AWQ_EINVAL, "D_outs[%d] = %lld: need a multiple of 4, at least 4", l, (long long)D_outs[l]);
    s += D_outs[l];
  }
  *Dsum = s;
  return AWQ_OK;
}

size_t awq_search_joint_workspace_size(int64_t N, int64_t D_in, const int64_t* D_outs, int n_layers, int n_alpha,
                                       int bits, int group, int loss_form) {
  int64_t Dsum = 0;
  if (check_joint(D_outs, n_layers, &Dsum) != AWQ_OK) return 0;
  const size_t base = awq_search_workspace_size(N, D_in, Dsum, n_alpha, bits, group, loss_form);
  if (base == 0) return 0;
  return base + round_up(static_cast<size_t>(D_in) * Dsum * 4, 256) +
         round_up(static_cast<size_t>(n_alpha) * Dsum * 8, 256);
}

int awq_search_joint(const void* X, const float* const* Ws, const int64_t* D_outs, int n_layers, const float* a,
                     int64_t N, int64_t D_in, const float* alpha_grid, int n_alpha, int bits, int group,
                     int loss_form, double* L, double* L_layers, float* alpha_star, int32_t* alpha_idx,
                     void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  AWQ_ENTRY("awq_search_joint", kTakesWorkspace, "N=%lld D_in=%lld n_layers=%d n_alpha=%d bits=%d group=%d form=%d", (long long)N, (long long)D_in, n_layers, n_alpha, bits, group, loss_form);
  int64_t Dsum = 0;
  AWQ_TRY(check_joint(D_outs, n_layers, &Dsum));
  if (!Ws) return fail(AWQ_EINVAL, "Ws is NULL");
  for (int l = 0; l < n_layers; ++l) {
    int rc = check_ptr(Ws[l], "Ws[l]", 16);
    if (rc != AWQ_OK) return fail(rc, "layer %d: %s", l, g_last_error.c_str());
  }
  // The shapes and pointers of the joint layer; W is checked per layer above.
  AWQ_TRY(check_search_args(X, Ws[0], a, N, D_in, Dsum, alpha_grid, n_alpha, bits, group, loss_form, L, nullptr,
                            alpha_star, alpha_idx));
  if (L_layers) AWQ_TRY(check_ptr(L_layers, "L_layers", 8));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  const SearchLayout lay = search_layout(N, D_in, Dsum, n_alpha, group, loss_form, sms);
  const size_t w_off = lay.total;
  const size_t lc_off = w_off + round_up(static_cast<size_t>(D_in) * Dsum * 4, 256);
  const size_t need = lc_off + round_up(static_cast<size_t>(n_alpha) * Dsum * 8, 256);
  if (!workspace) return fail(AWQ_EWORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(AWQ_EALIGN, "workspace is not 256-byte aligned");
  if (workspace_bytes < need) return fail(AWQ_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  if (status && !aligned(status, 4)) return fail(AWQ_EALIGN, "status is not 4-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* Wcat = reinterpret_cast<float*>(ws + w_off);
  double* Lcol = reinterpret_cast<double*>(ws + lc_off);
  int32_t* st_word = status ? status : reinterpret_cast<int32_t*>(ws + lay.status);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(st_word, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  // The layers side by side: [D_in][sum of D_out].  L is a sum over output
  // columns, so the search of the joint matrix gives sum_l L_l(alpha).
  awq::Segments seg{};
  int64_t off = 0;
  for (int l = 0; l < n_layers; ++l) {
    seg.off[l] = off;
    e = cudaMemcpy2DAsync(Wcat + off, static_cast<size_t>(Dsum) * 4, Ws[l], static_cast<size_t>(D_outs[l]) * 4,
                          static_cast<size_t>(D_outs[l]) * 4, static_cast<size_t>(D_in), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemcpy2DAsync(joint weights)");
    off += D_outs[l];
  }
  seg.off[n_layers] = off;
  awq::AlphaList al{};
  for (int i = 0; i < n_alpha; ++i) al.v[i] = alpha_grid[i];
  AWQ_TRY(search_one(X, Wcat, a, N, D_in, Dsum, al, n_alpha, bits, group, loss_form, L, Lcol, alpha_star, alpha_idx,
                     ws, st_word, st, sms));
  if (L_layers) {
    e = awq::launch_segment_sums(Lcol, n_alpha, Dsum, seg, n_layers, L_layers, st);
    if (e != cudaSuccess) return fail_cuda(e, "per-layer loss sums");
  }
  return AWQ_OK;
}

size_t awq_w4a16_workspace_size(int64_t N, int64_t D_in, int64_t D_out) {
  if (N < 1 || D_in < 1 || D_out < 1) return 0;
  return awq::w4a16_scratch_bytes(N, D_in, D_out, 0) + 256;
}

size_t awq_w4a16_zp_workspace_size(int64_t N, int64_t D_in, int64_t D_out, int group) {
  if (N < 1 || D_in < 1 || D_out < 1 || check_quant_args(4, group) != AWQ_OK || D_in % group) return 0;
  return awq::w4a16_scratch_bytes(N, D_in, D_out, D_in / group) + 256;
}

static int w4a16_impl(const void* X, const float* s, const uint32_t* packed, const float* scales,
                      const uint8_t* zeros, int64_t N, int64_t D_in, int64_t D_out, int bits, int group, float* Y,
                      void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  if (N < 1 || N > kMaxDim) return fail(AWQ_EINVAL, "N = %lld: need 1 <= N <= 2^24", (long long)N);
  AWQ_TRY(check_quant_args(bits, group));
  if (D_in < group || D_in > kMaxDin || D_in % group)
    return fail(AWQ_EINVAL, "D_in = %lld: need a positive multiple of group = %d", (long long)D_in, group);
  if (D_out < 4 || D_out > kMaxDim || D_out % 4)
    return fail(AWQ_EINVAL, "D_out = %lld: need a positive multiple of 4 (rows of packed words are read by TMA)",
                (long long)D_out);
  AWQ_TRY(check_ptr(X, "X", 16));
  AWQ_TRY(check_ptr(s, "s", 16));
  AWQ_TRY(check_ptr(packed, "packed", 16));
  AWQ_TRY(check_ptr(scales, "scales", 16));
  AWQ_TRY(check_ptr(Y, "Y", 4));
  if (zeros) AWQ_TRY(check_ptr(zeros, "zeros", 16));
  if (!workspace) return fail(AWQ_EWORKSPACE, "workspace is NULL");
  const size_t need = zeros ? awq_w4a16_zp_workspace_size(N, D_in, D_out, group)
                            : awq_w4a16_workspace_size(N, D_in, D_out);
  if (workspace_bytes < need) return fail(AWQ_EWORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  void* xs = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
  if (!status) return fail(AWQ_EINVAL, "status is NULL");
  AWQ_TRY(check_ptr(status, "status", 4));
  int sms = 0;
  AWQ_TRY(device_info(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (!awq::w4a16_clears_status(N)) {
    e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return fail_cuda(e, "cudaMemsetAsync(status)");
  }
  const char* what = "w4a16 kernel";
  int rc;
  {
    StageTimer t(AWQ_STAGE_W4A16, st);
    rc = awq::launch_w4a16(X, s, packed, scales, zeros, N, D_in, D_out, bits, group, Y, xs, sms, status,
                           timeout_ns(), st, &e, &what);
  }
  if (rc != AWQ_OK) return e != cudaSuccess ? fail_cuda(e, what) : fail(rc, "%s failed", what);
  return AWQ_OK;
}

int awq_w4a16_gemm(const void* X, const float* s, const uint32_t* packed, const float* scales, int64_t N,
                   int64_t D_in, int64_t D_out, int bits, int group, float* Y, void* workspace,
                   size_t workspace_bytes, int32_t* status, void* stream) {
  AWQ_ENTRY("awq_w4a16_gemm", kTakesWorkspace, "N=%lld D_in=%lld D_out=%lld bits=%d group=%d", (long long)N, (long long)D_in, (long long)D_out, bits, group);
  return w4a16_impl(X, s, packed, scales, nullptr, N, D_in, D_out, bits, group, Y, workspace, workspace_bytes,
                    status, stream);
}

int awq_w4a16_gemm_zp(const void* X, const float* s, const uint32_t* packed, const float* scales,
                      const uint8_t* zeros, int64_t N, int64_t D_in, int64_t D_out, int bits, int group, float* Y,
                      void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  AWQ_ENTRY("awq_w4a16_gemm_zp", kTakesWorkspace, "N=%lld D_in=%lld D_out=%lld bits=%d group=%d", (long long)N, (long long)D_in, (long long)D_out, bits, group);
  if (!zeros) return fail(AWQ_EINVAL, "zeros is NULL");
  return w4a16_impl(X, s, packed, scales, zeros, N, D_in, D_out, bits, group, Y, workspace, workspace_bytes, status,
                    stream);
}

}  // extern "C"
