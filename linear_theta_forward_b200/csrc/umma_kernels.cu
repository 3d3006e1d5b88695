// bf16 forward and reconstruct (bring-up: CUDA-core kernels; the tcgen05
// tensor-core kernels replace these).
#include "common.cuh"
#include "internal.h"

namespace theta {

size_t forward_umma_workspace_bytes(int64_t M, int r) { return (size_t)M * r * sizeof(float); }

int launch_forward_umma(const LaunchCtx& c, const void* X, const void* W0, const float* s,
                        const void* U, const void* V, int64_t M, int64_t O, int64_t I, int r,
                        void* Y, void* ws, cudaError_t* cuda_err) {
  float* T = r > 0 ? static_cast<float*>(ws) : nullptr;
  cudaError_t e = cudaSuccess;
  if (r > 0) e = launch_xv_simt(c, THETA_BF16, X, V, M, I, r, T);
  if (e == cudaSuccess) e = launch_forward_simt(c, THETA_BF16, X, W0, s, U, T, M, O, I, r, Y);
  *cuda_err = e;
  return e == cudaSuccess ? THETA_OK : THETA_ERR_CUDA;
}

int launch_reconstruct_umma(const LaunchCtx& c, const float* s, const void* W0, const void* U,
                            const void* V, int64_t O, int64_t I, int r, void* W_out,
                            cudaError_t* cuda_err) {
  cudaError_t e = launch_reconstruct_simt(c, THETA_BF16, s, W0, U, V, O, I, r, W_out);
  *cuda_err = e;
  return e == cudaSuccess ? THETA_OK : THETA_ERR_CUDA;
}

}  // namespace theta
