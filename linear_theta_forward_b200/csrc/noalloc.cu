// theta_linear_forward_noalloc: the theta forward with its scratch memory
// built into the library instead of supplied by the caller.
//
// theta_linear_forward needs device scratch for T = X.V: 4 * M * rank bytes
// (the one- and two-token path keeps 16 fp32 partial sums of T instead,
// 64 * M * rank bytes, at most 32 KB).
// Most callers pass a buffer they allocated once. Some cannot allocate at
// all: engines whose device memory is handed out by their own fixed pool
// with nothing left for a library, and plugins that are given only input and
// output pointers. This entry point serves them from a fixed array compiled
// into the library.
//
// The array below is ordinary device memory of the module: every GPU that
// loads the library holds it, kScratchBytes of it, until the process exits.
// All calls on a device share it, so two calls whose kernels overlap on the
// GPU (different streams, no ordering) race on it; calls ordered on one
// stream are fine. Each call writes the part of the array it reads before it
// reads it, so nothing has to start at zero and the previous call's contents
// do no harm.
#include <cstdio>
#include <mutex>

#include "common.cuh"

#define THETA_API extern "C" __attribute__((visibility("default")))

extern "C" int theta_linear_forward(const void*, int64_t, int64_t, const void*, int64_t, const float*,
                                    const void*, const void*, int, theta_dtype, void*, void*, size_t, void*);
extern "C" int theta_workspace_size(int, int64_t, int64_t, int64_t, int, theta_dtype, size_t*);

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB: M * rank <= 1,048,576 (either dtype)

static __device__ __align__(256) unsigned char g_forward_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

}  // namespace

namespace theta {
int report_error(int status, const char* message);  // sets theta_last_error()
}

THETA_API int theta_linear_forward_noalloc(const void* X, int64_t M, int64_t I, const void* W0, int64_t O,
                                           const float* s, const void* U, const void* V, int rank, theta_dtype dt,
                                           void* Y, void* stream) {
  char msg[320];
  size_t need = 0;
  int st = theta_workspace_size(THETA_OP_LINEAR_FORWARD, M, O, I, rank, dt, &need);
  if (st != THETA_OK) {
    snprintf(msg, sizeof msg, "theta_linear_forward_noalloc: bad sizes (M=%lld, rank=%d)", (long long)M, rank);
    return theta::report_error(st, msg);
  }
  if (need > kScratchBytes) {
    snprintf(msg, sizeof msg,
             "theta_linear_forward_noalloc: needs %zu bytes of scratch for M=%lld, rank=%d; the built-in "
             "scratch holds %zu bytes (M * rank <= %zu); use theta_linear_forward with your own workspace",
             need, (long long)M, rank, kScratchBytes, kScratchBytes / 4);
    return theta::report_error(THETA_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  if (need > 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
      snprintf(msg, sizeof msg, "theta_linear_forward_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
      return theta::report_error(THETA_ERR_CUDA, msg);
    }
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
      // one-time set-up on this device: the host-side name of the array is a
      // stand-in, so ask the runtime for the array's device address
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_forward_scratch);
      if (e != cudaSuccess || p == nullptr) {
        snprintf(msg, sizeof msg, "theta_linear_forward_noalloc: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(e));
        return theta::report_error(THETA_ERR_CUDA, msg);
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  return theta_linear_forward(X, M, I, W0, O, s, U, V, rank, dt, Y, scratch, kScratchBytes, stream);
}
