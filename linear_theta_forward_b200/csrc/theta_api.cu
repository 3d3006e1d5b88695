// libtheta C ABI: argument validation, kernel selection and error reporting.
//
// Every entry point validates on the host before it enqueues anything, so a
// rejected call leaves device memory untouched. Kernels run on the caller's
// stream; nothing here allocates device memory or synchronises (except
// theta_device_status, whose job is to synchronise).
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"

#define THETA_API extern "C" __attribute__((visibility("default")))

namespace theta {
namespace {

// Device error words (see common.cuh); kernels receive their address.
__device__ unsigned g_err_words[ERR_WORD_COUNT];

thread_local std::string t_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return status;
}

int fail_cuda(cudaError_t e, const char* where) {
  return fail(THETA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

constexpr int kMaxDevices = 64;
struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  unsigned* err = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

std::atomic<int> g_policy{THETA_POLICY_LATENCY};

int make_ctx(void* stream, LaunchCtx* ctx) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(THETA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
      e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return fail_cuda(e, "cudaDeviceGetAttribute");
      e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_err_words);
      if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(error words)");
      d.ready = true;
    }
    ctx->num_sms = d.num_sms;
    ctx->err = d.err;
  }
  ctx->device = dev;
  ctx->stream = static_cast<cudaStream_t>(stream);
  ctx->policy = g_policy.load(std::memory_order_relaxed);
  return THETA_OK;
}

bool valid_dt(theta_dtype dt) { return dt == THETA_F32 || dt == THETA_BF16; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

size_t forward_ws_bytes(int64_t M, int r, theta_dtype dt) {
  if (r <= 0) return 0;
  // fp32: T = X.V in fp32 [M, r]; bf16: T split into bf16 high and low parts.
  size_t t = dt == THETA_BF16 ? forward_umma_workspace_bytes(M, r) : (size_t)M * r * sizeof(float);
  return align_up(t, 256);
}

#define CHECK_LAUNCH(expr, what)                     \
  do {                                               \
    cudaError_t _e = (expr);                         \
    if (_e != cudaSuccess) return fail_cuda(_e, what); \
  } while (0)

}  // namespace

std::mutex& setup_mutex() {
  static std::mutex mu;
  return mu;
}

// Lets other translation units report through theta_last_error().
int report_error(int status, const char* message) {
  t_last_error = message;
  return status;
}

}  // namespace theta

using namespace theta;

THETA_API int theta_version(void) { return THETA_VERSION; }

THETA_API const char* theta_status_string(int status) {
  switch (status) {
    case THETA_OK: return "THETA_OK";
    case THETA_ERR_INVALID_ARG: return "THETA_ERR_INVALID_ARG";
    case THETA_ERR_UNSUPPORTED: return "THETA_ERR_UNSUPPORTED";
    case THETA_ERR_ALIGNMENT: return "THETA_ERR_ALIGNMENT";
    case THETA_ERR_CUDA: return "THETA_ERR_CUDA";
    case THETA_ERR_TIMEOUT: return "THETA_ERR_TIMEOUT";
    case THETA_ERR_WORKSPACE: return "THETA_ERR_WORKSPACE";
  }
  return "THETA_ERR_UNKNOWN";
}

THETA_API const char* theta_last_error(void) { return t_last_error.c_str(); }

THETA_API int theta_band_index(int num_layers, int G, int32_t* band_of_layer, int32_t* band_start) {
  if (num_layers < 1 || G < 1 || G > num_layers)
    return fail(THETA_ERR_INVALID_ARG, "theta_band_index: need 1 <= G <= num_layers (G=%d, num_layers=%d)",
                G, num_layers);
  if (!band_of_layer) return fail(THETA_ERR_INVALID_ARG, "theta_band_index: band_of_layer is NULL");
  const int q = num_layers / G, m = num_layers % G;
  int first = 0;
  for (int b = 0; b < G; ++b) {
    const int size = q + (b < m ? 1 : 0);
    if (band_start) band_start[b] = first;
    for (int l = first; l < first + size; ++l) band_of_layer[l] = b;
    first += size;
  }
  if (band_start) band_start[G] = num_layers;
  return THETA_OK;
}

THETA_API int theta_band_mean(const void* const* weights, int n, int64_t O, int64_t I,
                              theta_dtype dt, void* W0, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_band_mean: bad dtype %d", (int)dt);
  if (n < 1 || n > THETA_MAX_LAYERS)
    return fail(THETA_ERR_INVALID_ARG, "theta_band_mean: n=%d outside [1, %d]", n, THETA_MAX_LAYERS);
  if (O < 1 || I < 1) return fail(THETA_ERR_INVALID_ARG, "theta_band_mean: O, I must be >= 1");
  if (!weights || !W0) return fail(THETA_ERR_INVALID_ARG, "theta_band_mean: NULL pointer");
  for (int l = 0; l < n; ++l)
    if (!weights[l]) return fail(THETA_ERR_INVALID_ARG, "theta_band_mean: weights[%d] is NULL", l);
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  CHECK_LAUNCH(launch_band_mean(c, dt, weights, n, O, I, W0), "theta_band_mean launch");
  return THETA_OK;
}

THETA_API int theta_row_scale(const void* weight, const void* W0, int64_t O, int64_t I,
                              theta_dtype dt, float* s, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_row_scale: bad dtype %d", (int)dt);
  if (O < 1 || I < 1) return fail(THETA_ERR_INVALID_ARG, "theta_row_scale: O, I must be >= 1");
  if (!weight || !W0 || !s) return fail(THETA_ERR_INVALID_ARG, "theta_row_scale: NULL pointer");
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  const void* w[1] = {weight};
  float* sp[1] = {s};
  void* w0[1] = {const_cast<void*>(W0)};
  const int32_t band_start[2] = {0, 1}, band_of_layer[1] = {0};
  cudaError_t pe = cudaSuccess;
  if (launch_prelude_pipe(c, dt, PRELUDE_ROW, w, 1, 1, band_start, band_of_layer, w0, sp, nullptr, O, I, &pe)) {
    CHECK_LAUNCH(pe, "theta_row_scale launch");
    return THETA_OK;
  }
  CHECK_LAUNCH(launch_rowscale_band(c, dt, W0, w, 1, O, I, sp, nullptr), "theta_row_scale launch");
  return THETA_OK;
}

THETA_API int theta_residual(const void* weight, const void* W0, const float* s, int64_t O,
                             int64_t I, theta_dtype dt, void* R, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_residual: bad dtype %d", (int)dt);
  if (O < 1 || I < 1) return fail(THETA_ERR_INVALID_ARG, "theta_residual: O, I must be >= 1");
  if (!weight || !W0 || !s || !R) return fail(THETA_ERR_INVALID_ARG, "theta_residual: NULL pointer");
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  CHECK_LAUNCH(launch_residual(c, dt, weight, W0, s, O, I, R), "theta_residual launch");
  return THETA_OK;
}

THETA_API int theta_decompose_prelude(const void* const* weights, int num_layers, int G, int64_t O,
                                      int64_t I, theta_dtype dt, void* const* W0, float* const* s,
                                      void* const* residual, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_decompose_prelude: bad dtype %d", (int)dt);
  if (num_layers < 1 || num_layers > THETA_MAX_LAYERS || G < 1 || G > num_layers)
    return fail(THETA_ERR_INVALID_ARG,
                "theta_decompose_prelude: need 1 <= G <= num_layers <= %d (G=%d, num_layers=%d)",
                THETA_MAX_LAYERS, G, num_layers);
  if (O < 1 || I < 1) return fail(THETA_ERR_INVALID_ARG, "theta_decompose_prelude: O, I must be >= 1");
  if (!weights || !W0 || !s) return fail(THETA_ERR_INVALID_ARG, "theta_decompose_prelude: NULL array");
  for (int l = 0; l < num_layers; ++l)
    if (!weights[l] || !s[l] || (residual && !residual[l]))
      return fail(THETA_ERR_INVALID_ARG, "theta_decompose_prelude: NULL pointer for layer %d", l);
  for (int b = 0; b < G; ++b)
    if (!W0[b]) return fail(THETA_ERR_INVALID_ARG, "theta_decompose_prelude: W0[%d] is NULL", b);
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  int32_t band_of_layer[THETA_MAX_LAYERS], band_start[THETA_MAX_LAYERS + 1];
  theta_band_index(num_layers, G, band_of_layer, band_start);
  const int nmax = (num_layers + G - 1) / G;
  cudaError_t pe = cudaSuccess;
  // bands of <= 4 layers: one pass over the family forms W0, s and R
  if (nmax <= 4 && launch_prelude_pipe(c, dt, PRELUDE_BAND, weights, num_layers, G, band_start, band_of_layer, W0,
                                       s, residual, O, I, &pe)) {
    CHECK_LAUNCH(pe, "prelude launch");
    return THETA_OK;
  }
  // longer bands: two passes over each band's rows, the second from L2
  if (nmax > 4 && launch_prelude_pipe(c, dt, PRELUDE_TWO_PASS, weights, num_layers, G, band_start, band_of_layer,
                                      W0, s, residual, O, I, &pe)) {
    CHECK_LAUNCH(pe, "prelude launch");
    return THETA_OK;
  }
  for (int b = 0; b < G; ++b) {
    const int first = band_start[b], n = band_start[b + 1] - band_start[b];
    CHECK_LAUNCH(launch_band_mean(c, dt, weights + first, n, O, I, W0[b]), "band mean launch");
  }
  if (launch_prelude_pipe(c, dt, PRELUDE_ROW, weights, num_layers, G, band_start, band_of_layer, W0, s, residual, O,
                          I, &pe)) {
    CHECK_LAUNCH(pe, "row scale launch");
    return THETA_OK;
  }
  for (int b = 0; b < G; ++b) {
    const int first = band_start[b], n = band_start[b + 1] - band_start[b];
    CHECK_LAUNCH(launch_rowscale_band(c, dt, W0[b], weights + first, n, O, I, s + first,
                                      residual ? residual + first : nullptr),
                 "row scale launch");
  }
  return THETA_OK;
}

THETA_API int theta_reconstruct(const float* s, const void* W0, const void* U, const void* V,
                                int64_t O, int64_t I, int rank, theta_dtype dt, void* W_out,
                                void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct: bad dtype %d", (int)dt);
  if (O < 1 || I < 1 || rank < 0)
    return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct: need O, I >= 1 and rank >= 0");
  if (!s || !W0 || !W_out || (rank > 0 && (!U || !V)))
    return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct: NULL pointer");
  if (dt == THETA_BF16) {
    if (!aligned16(s) || !aligned16(W0) || !aligned16(W_out) || (rank > 0 && (!aligned16(U) || !aligned16(V))) ||
        I % 8 || rank % 8)
      return fail(THETA_ERR_ALIGNMENT, "theta_reconstruct: bf16 needs 16-byte aligned pointers and I, rank multiples of 8");
  } else if (O > kSimtMaxRows) {
    return fail(THETA_ERR_UNSUPPORTED, "theta_reconstruct: fp32 path takes at most %lld rows",
                (long long)kSimtMaxRows);
  }
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  if (dt == THETA_BF16) {
    cudaError_t ce = cudaSuccess;
    st = launch_reconstruct_umma(c, s, W0, U, V, O, I, rank, W_out, &ce);
    if (st == THETA_ERR_CUDA) return fail_cuda(ce, "theta_reconstruct (tensor-core path)");
    if (st) return st;
    return THETA_OK;
  }
  CHECK_LAUNCH(launch_reconstruct_simt(c, dt, s, W0, U, V, O, I, rank, W_out), "theta_reconstruct launch");
  return THETA_OK;
}

THETA_API int theta_reconstruct_band(const float* const* s, const void* W0, const void* const* U,
                                     const void* const* V, int n, int64_t O, int64_t I, int rank, theta_dtype dt,
                                     void* const* W_out, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct_band: bad dtype %d", (int)dt);
  if (n < 1 || n > THETA_MAX_LAYERS)
    return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct_band: n=%d outside [1, %d]", n, THETA_MAX_LAYERS);
  if (O < 1 || I < 1 || rank < 0)
    return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct_band: need O, I >= 1 and rank >= 0");
  if (!s || !W0 || !W_out || (rank > 0 && (!U || !V)))
    return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct_band: NULL array");
  for (int l = 0; l < n; ++l)
    if (!s[l] || !W_out[l] || (rank > 0 && (!U[l] || !V[l])))
      return fail(THETA_ERR_INVALID_ARG, "theta_reconstruct_band: NULL pointer for layer %d", l);
  if (dt == THETA_BF16) {
    bool ok = aligned16(W0) && I % 8 == 0 && rank % 8 == 0;
    for (int l = 0; l < n && ok; ++l)
      ok = aligned16(s[l]) && aligned16(W_out[l]) && (rank == 0 || (aligned16(U[l]) && aligned16(V[l])));
    if (!ok)
      return fail(THETA_ERR_ALIGNMENT,
                  "theta_reconstruct_band: bf16 needs 16-byte aligned pointers and I, rank multiples of 8");
  } else if (O > kSimtMaxRows) {
    return fail(THETA_ERR_UNSUPPORTED, "theta_reconstruct_band: fp32 path takes at most %lld rows",
                (long long)kSimtMaxRows);
  }
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  if (dt == THETA_BF16) {
    cudaError_t ce = cudaSuccess;
    st = launch_reconstruct_band_umma(c, s, W0, rank > 0 ? U : nullptr, rank > 0 ? V : nullptr, n, O, I, rank,
                                      W_out, &ce);
    if (st == THETA_ERR_CUDA) return fail_cuda(ce, "theta_reconstruct_band (tensor-core path)");
    return st;
  }
  for (int l = 0; l < n; ++l)
    CHECK_LAUNCH(launch_reconstruct_simt(c, dt, s[l], W0, rank > 0 ? U[l] : nullptr, rank > 0 ? V[l] : nullptr, O,
                                         I, rank, W_out[l]),
                 "theta_reconstruct_band launch");
  return THETA_OK;
}

THETA_API int theta_frob_error(const void* original, const void* reconstructed, int64_t n,
                               theta_dtype dt, double* out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_frob_error: bad dtype %d", (int)dt);
  if (n < 0) return fail(THETA_ERR_INVALID_ARG, "theta_frob_error: n < 0");
  if ((n > 0 && (!original || !reconstructed)) || !out)
    return fail(THETA_ERR_INVALID_ARG, "theta_frob_error: NULL pointer");
  if (!workspace || workspace_bytes < frob_workspace_bytes() || !aligned16(workspace))
    return fail(THETA_ERR_WORKSPACE, "theta_frob_error: need %zu bytes of 16-byte aligned workspace",
                frob_workspace_bytes());
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  CHECK_LAUNCH(launch_frob(c, dt, original, reconstructed, n, out, workspace), "theta_frob_error launch");
  return THETA_OK;
}

THETA_API int theta_frob_partials(const void* original, const void* reconstructed, int64_t n, theta_dtype dt,
                                  double* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_frob_partials: bad dtype %d", (int)dt);
  if (n < 0) return fail(THETA_ERR_INVALID_ARG, "theta_frob_partials: n < 0");
  if ((n > 0 && (!original || !reconstructed)) || !out)
    return fail(THETA_ERR_INVALID_ARG, "theta_frob_partials: NULL pointer");
  if (reinterpret_cast<uintptr_t>(out) & 7u)
    return fail(THETA_ERR_ALIGNMENT, "theta_frob_partials: out must be 8-byte aligned");
  if (!workspace || workspace_bytes < frob_workspace_bytes() || !aligned16(workspace))
    return fail(THETA_ERR_WORKSPACE, "theta_frob_partials: need %zu bytes of 16-byte aligned workspace",
                frob_workspace_bytes());
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  CHECK_LAUNCH(launch_frob(c, dt, original, reconstructed, n, out, workspace, true), "theta_frob_partials launch");
  return THETA_OK;
}

THETA_API int theta_linear_forward(const void* X, int64_t M, int64_t I, const void* W0, int64_t O,
                                   const float* s, const void* U, const void* V, int rank,
                                   theta_dtype dt, void* Y, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward: bad dtype %d", (int)dt);
  if (M < 1 || I < 1 || O < 1 || rank < 0)
    return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward: need M, I, O >= 1 and rank >= 0");
  if (!X || !W0 || !s || !Y || (rank > 0 && (!U || !V)))
    return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward: NULL pointer");
  const size_t need = forward_ws_bytes(M, rank, dt);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(THETA_ERR_WORKSPACE, "theta_linear_forward: need %zu bytes of 16-byte aligned workspace", need);
  if (dt == THETA_BF16) {
    if (!aligned16(X) || !aligned16(W0) || !aligned16(Y) || !aligned16(s) ||
        (rank > 0 && (!aligned16(U) || !aligned16(V))) || I % 8 || O % 8 || rank % 8)
      return fail(THETA_ERR_ALIGNMENT,
                  "theta_linear_forward: bf16 needs 16-byte aligned pointers and I, O, rank multiples of 8");
    if (rank > 0 && (M + 127) / 128 > 65535)
      return fail(THETA_ERR_UNSUPPORTED, "theta_linear_forward: bf16 with rank > 0 takes at most %lld tokens",
                  (long long)65535 * 128);
  } else if (M > kSimtMaxRows) {
    return fail(THETA_ERR_UNSUPPORTED, "theta_linear_forward: fp32 path takes at most %lld tokens",
                (long long)kSimtMaxRows);
  }
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  if (dt == THETA_BF16) {
    cudaError_t ce = cudaSuccess;
    st = launch_forward_umma(c, X, W0, s, U, V, M, O, I, rank, Y, workspace, &ce);
    if (st == THETA_ERR_CUDA) return fail_cuda(ce, "theta_linear_forward (tensor-core path)");
    return st;
  }
  float* T = rank > 0 ? static_cast<float*>(workspace) : nullptr;
  if (rank > 0) CHECK_LAUNCH(launch_xv_simt(c, dt, X, V, M, I, rank, T), "theta_linear_forward xv launch");
  CHECK_LAUNCH(launch_forward_simt(c, dt, X, W0, s, U, T, M, O, I, rank, Y), "theta_linear_forward launch");
  return THETA_OK;
}

THETA_API int theta_linear_forward_grouped(const theta_forward_problem* problems,
                                           const theta_forward_problem* problems_device, int count, int64_t M,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!problems || !problems_device)
    return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward_grouped: NULL problem table");
  if (count < 1 || count > THETA_MAX_GROUP)
    return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward_grouped: count %d outside [1, %d]", count,
                THETA_MAX_GROUP);
  if (M < 1) return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward_grouped: M < 1");
  if (M > 2) return fail(THETA_ERR_UNSUPPORTED, "theta_linear_forward_grouped: one or two tokens only");
  if (reinterpret_cast<uintptr_t>(problems_device) % alignof(theta_forward_problem))
    return fail(THETA_ERR_ALIGNMENT, "theta_linear_forward_grouped: misaligned device problem table");
  int rmax = 0;
  for (int i = 0; i < count; ++i) {
    const theta_forward_problem& p = problems[i];
    if (p.O < 1 || p.I < 1 || p.rank < 0 || p.rank > 256)
      return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward_grouped: problem %d: need O, I >= 1, 0 <= rank <= 256",
                  i);
    if (!p.X || !p.W0 || !p.s || !p.Y || (p.rank > 0 && (!p.U || !p.V)))
      return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward_grouped: problem %d: NULL pointer", i);
    if (!aligned16(p.X) || !aligned16(p.W0) || !aligned16(p.s) ||
        (p.rank > 0 && (!aligned16(p.U) || !aligned16(p.V))) || p.I % 8 || p.O % 8 || p.rank % 8)
      return fail(THETA_ERR_ALIGNMENT,
                  "theta_linear_forward_grouped: problem %d: 16-byte aligned pointers and I, O, rank multiples of 8",
                  i);
    rmax = std::max(rmax, (int)p.rank);
  }
  const size_t need = forward_grouped_workspace_bytes(count, M, rmax);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(THETA_ERR_WORKSPACE, "theta_linear_forward_grouped: need %zu bytes of 16-byte aligned workspace",
                need);
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  cudaError_t ce = cudaSuccess;
  if (!launch_forward_grouped(c, problems, problems_device, count, M, rmax, workspace, &ce))
    return fail(THETA_ERR_UNSUPPORTED, "theta_linear_forward_grouped: outside the grouped sweep");
  if (ce != cudaSuccess) return fail_cuda(ce, "theta_linear_forward_grouped launch");
  return THETA_OK;
}

THETA_API int theta_linear_gate_up_forward(const void* X, int64_t M, int64_t I, int64_t O, int rank,
                                           theta_dtype dt, const void* W0_gate, const float* s_gate,
                                           const void* U_gate, const void* V_gate, const void* W0_up,
                                           const float* s_up, const void* U_up, const void* V_up, void* Y,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_linear_gate_up_forward: bad dtype %d", (int)dt);
  if (M < 1 || I < 1 || O < 1 || rank < 0)
    return fail(THETA_ERR_INVALID_ARG, "theta_linear_gate_up_forward: need M, I, O >= 1 and rank >= 0");
  if (!X || !W0_gate || !s_gate || !W0_up || !s_up || !Y ||
      (rank > 0 && (!U_gate || !V_gate || !U_up || !V_up)))
    return fail(THETA_ERR_INVALID_ARG, "theta_linear_gate_up_forward: NULL pointer");
  if (dt != THETA_BF16)
    return fail(THETA_ERR_UNSUPPORTED, "theta_linear_gate_up_forward: bf16 only");
  const size_t need = gate_up_umma_workspace_bytes(M, rank);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(THETA_ERR_WORKSPACE, "theta_linear_gate_up_forward: need %zu bytes of 16-byte aligned workspace",
                need);
  for (const void* p : {X, W0_gate, W0_up, static_cast<const void*>(Y), static_cast<const void*>(s_gate),
                        static_cast<const void*>(s_up)})
    if (!aligned16(p))
      return fail(THETA_ERR_ALIGNMENT, "theta_linear_gate_up_forward: bf16 needs 16-byte aligned pointers");
  if ((rank > 0 && (!aligned16(U_gate) || !aligned16(V_gate) || !aligned16(U_up) || !aligned16(V_up))) || I % 8 ||
      O % 8 || rank % 8)
    return fail(THETA_ERR_ALIGNMENT,
                "theta_linear_gate_up_forward: bf16 needs 16-byte aligned pointers and I, O, rank multiples of 8");
  if (rank > 0 && (M + 127) / 128 > 65535)
    return fail(THETA_ERR_UNSUPPORTED, "theta_linear_gate_up_forward: rank > 0 takes at most %lld tokens",
                (long long)65535 * 128);
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  cudaError_t ce = cudaSuccess;
  st = launch_gate_up_umma(c, X, W0_gate, s_gate, U_gate, V_gate, W0_up, s_up, U_up, V_up, M, O, I, rank, Y,
                           workspace, &ce);
  if (st == THETA_ERR_CUDA) return fail_cuda(ce, "theta_linear_gate_up_forward (tensor-core path)");
  return st;
}

THETA_API int theta_residual_svd(const void* R, int64_t O, int64_t I, theta_dtype dt, int rank, int samples,
                                 int power_iters, const float* omega, void* U, void* V, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_residual_svd: bad dtype %d", (int)dt);
  if (O < 1 || I < 1 || rank < 1 || samples < rank || power_iters < 0 || power_iters > 8)
    return fail(THETA_ERR_INVALID_ARG,
                "theta_residual_svd: need O, I >= 1, 1 <= rank <= samples and 0 <= power_iters <= 8");
  if (samples > svd_max_samples() || samples > O || samples > I)
    return fail(THETA_ERR_UNSUPPORTED, "theta_residual_svd: samples must be <= min(%d, O, I)", svd_max_samples());
  // the products' grids tile O and I by 64 along grid y (at most 65535)
  if (O > kSimtMaxRows || I > kSimtMaxRows)
    return fail(THETA_ERR_UNSUPPORTED, "theta_residual_svd: O and I must be <= %lld", (long long)kSimtMaxRows);
  if (!R || !omega || !U || !V) return fail(THETA_ERR_INVALID_ARG, "theta_residual_svd: NULL pointer");
  const size_t need = svd_workspace_bytes(O, I, samples, rank);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(THETA_ERR_WORKSPACE, "theta_residual_svd: need %zu bytes of 16-byte aligned workspace", need);
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  CHECK_LAUNCH(launch_residual_svd(c, dt, R, O, I, rank, samples, power_iters, omega, U, V, workspace),
               "theta_residual_svd launch");
  return THETA_OK;
}

THETA_API int theta_nvfp4_quantize(const void* W0, int64_t O, int64_t I, void* codes, void* scales, float* g,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (O < 1 || I < 1 || I % 32)
    return fail(THETA_ERR_INVALID_ARG, "theta_nvfp4_quantize: need O >= 1 and I a positive multiple of 32");
  if (!W0 || !codes || !scales || !g) return fail(THETA_ERR_INVALID_ARG, "theta_nvfp4_quantize: NULL pointer");
  if (!aligned16(W0) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u) ||
      (reinterpret_cast<uintptr_t>(g) & 3u))
    return fail(THETA_ERR_ALIGNMENT, "theta_nvfp4_quantize: W0 and codes 16-byte, scales 2-byte, g 4-byte aligned");
  if (!workspace || workspace_bytes < 16 || !aligned16(workspace))
    return fail(THETA_ERR_WORKSPACE, "theta_nvfp4_quantize: need 16 bytes of 16-byte aligned workspace");
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  CHECK_LAUNCH(launch_nvfp4_quantize(c, W0, O, I, codes, scales, g, workspace), "theta_nvfp4_quantize launch");
  return THETA_OK;
}

THETA_API int theta_linear_forward_nvfp4(const void* X, int64_t M, int64_t I, const void* codes, const void* scales,
                                         const float* g, int64_t O, const float* s, const void* U, const void* V,
                                         int rank, void* Y, void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 1 || I < 1 || O < 1 || rank < 0 || I % 32)
    return fail(THETA_ERR_INVALID_ARG,
                "theta_linear_forward_nvfp4: need M, O >= 1, rank >= 0 and I a positive multiple of 32");
  if (!X || !codes || !scales || !g || !s || !Y || (rank > 0 && (!U || !V)))
    return fail(THETA_ERR_INVALID_ARG, "theta_linear_forward_nvfp4: NULL pointer");
  if (M > forward_gemv_max_tokens())
    return fail(THETA_ERR_UNSUPPORTED, "theta_linear_forward_nvfp4: at most %d tokens (the decode sweep)",
                forward_gemv_max_tokens());
  if (!aligned16(X) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u) || !aligned16(Y) ||
      (rank > 0 && (!aligned16(U) || !aligned16(V))) || O % 8 || rank % 8)
    return fail(THETA_ERR_ALIGNMENT,
                "theta_linear_forward_nvfp4: X, codes, Y, U, V 16-byte aligned, scales 2-byte; O, rank multiples of 8");
  const size_t need = forward_nvfp4_workspace_bytes(M, I, rank);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(THETA_ERR_WORKSPACE, "theta_linear_forward_nvfp4: need %zu bytes of 16-byte aligned workspace",
                need);
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  cudaError_t ce = cudaSuccess;
  if (!launch_forward_nvfp4(c, X, codes, scales, g, s, U, V, M, O, I, rank, Y, workspace, &ce))
    return fail(THETA_ERR_UNSUPPORTED, "theta_linear_forward_nvfp4: shape outside the decode sweep");
  if (ce != cudaSuccess) return fail_cuda(ce, "theta_linear_forward_nvfp4 launch");
  return THETA_OK;
}

THETA_API int theta_workspace_size(int op, int64_t M, int64_t O, int64_t I, int rank, theta_dtype dt,
                                   size_t* bytes) {
  if (!bytes) return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: bytes is NULL");
  if (!valid_dt(dt)) return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: bad dtype %d", (int)dt);
  switch (op) {
    case THETA_OP_FROB_ERROR: *bytes = frob_workspace_bytes(); return THETA_OK;
    case THETA_OP_LINEAR_FORWARD:
      if (M < 1 || rank < 0) return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: bad M or rank");
      *bytes = forward_ws_bytes(M, rank, dt);
      return THETA_OK;
    case THETA_OP_GATE_UP_FORWARD:
      if (M < 1 || rank < 0) return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: bad M or rank");
      *bytes = gate_up_umma_workspace_bytes(M, rank);
      return THETA_OK;
    case THETA_OP_NVFP4_QUANTIZE:
      *bytes = 16;
      return THETA_OK;
    case THETA_OP_LINEAR_FORWARD_NVFP4:
      if (M < 1 || rank < 0 || I < 1) return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: bad M, I or rank");
      *bytes = forward_nvfp4_workspace_bytes(M, I, rank);
      return THETA_OK;
    case THETA_OP_LINEAR_FORWARD_GROUPED:  // O carries the problem count, rank the largest rank
      if (M < 1 || M > 2 || O < 1 || O > THETA_MAX_GROUP || rank < 0 || rank > 256)
        return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: bad M, count or rank for the grouped forward");
      *bytes = forward_grouped_workspace_bytes((int)O, M, rank);
      return THETA_OK;
    case THETA_OP_RESIDUAL_SVD:  // M carries the number of samples
      if (M < 1 || rank < 1 || M < rank || O < 1 || I < 1)
        return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: bad samples, rank or sizes");
      *bytes = svd_workspace_bytes(O, I, (int)M, rank);
      return THETA_OK;
  }
  return fail(THETA_ERR_INVALID_ARG, "theta_workspace_size: unknown op %d", op);
}

THETA_API int theta_selftest_wait_timeout(unsigned limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000)
    return fail(THETA_ERR_INVALID_ARG, "theta_selftest_wait_timeout: limit %u ms outside [1, 2000]", limit_ms);
  LaunchCtx c;
  int st = make_ctx(stream, &c);
  if (st) return st;
  CHECK_LAUNCH(launch_wait_selftest(c, limit_ms), "theta_selftest_wait_timeout launch");
  return THETA_OK;
}

THETA_API int theta_set_policy(int policy) {
  if (policy != THETA_POLICY_LATENCY && policy != THETA_POLICY_THROUGHPUT)
    return fail(THETA_ERR_INVALID_ARG, "theta_set_policy: unknown policy %d", policy);
  g_policy.store(policy, std::memory_order_relaxed);
  return THETA_OK;
}

THETA_API int theta_get_policy(void) { return g_policy.load(std::memory_order_relaxed); }

THETA_API int theta_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "theta_device_status: stream synchronize");
  unsigned words[ERR_WORD_COUNT] = {};
  e = cudaMemcpyFromSymbol(words, g_err_words, sizeof words);
  if (e != cudaSuccess) return fail_cuda(e, "theta_device_status: read flags");
  const unsigned zero[ERR_WORD_COUNT] = {};
  e = cudaMemcpyToSymbol(g_err_words, zero, sizeof zero);
  if (e != cudaSuccess) return fail_cuda(e, "theta_device_status: clear flags");
  if (words[ERR_WORD_TIMEOUT])
    return fail(THETA_ERR_TIMEOUT, "a kernel's bounded wait ran out (device %d)", 0);
  return THETA_OK;
}
