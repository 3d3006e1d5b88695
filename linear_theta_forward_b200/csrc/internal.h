// Internal launcher declarations shared by the libtheta translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "theta.h"

namespace theta {

struct LaunchCtx {
  cudaStream_t stream;
  unsigned* err;  // device error words of the current device
  int num_sms;
  int device;
  int policy;  // theta_policy at the time of the call
};

// Held while a kernel's one-time, per-device set-up (attributes, occupancy
// and cluster queries, the caches that remember them) runs, so that threads
// making their first calls at once neither race on a cache nor read one that
// is half written.
std::mutex& setup_mutex();

// ---- streaming kernels (stream_kernels.cu)
cudaError_t launch_band_mean(const LaunchCtx& c, theta_dtype dt, const void* const* w, int n,
                             int64_t O, int64_t I, void* W0);
// Row scale of n layers against one W0 (a band), optionally with residuals.
cudaError_t launch_rowscale_band(const LaunchCtx& c, theta_dtype dt, const void* W0,
                                 const void* const* w, int n, int64_t O, int64_t I,
                                 float* const* s, void* const* R);
cudaError_t launch_residual(const LaunchCtx& c, theta_dtype dt, const void* w, const void* W0,
                            const float* s, int64_t O, int64_t I, void* R);
// ---- prelude pipeline (prelude_kernels.cu): every band of a family in one
// launch. PRELUDE_BAND: bands of <= 4 layers, W0, s and R in one pass;
// PRELUDE_TWO_PASS: longer bands, W0 from a first pass over the band's rows,
// s and R from a second (L2-resident) pass; PRELUDE_ROW: reads the
// already-formed W0 and writes s and R. Returns false without launching when
// the problem does not fit the chosen kernel.
enum { PRELUDE_ROW = 0, PRELUDE_BAND = 1, PRELUDE_TWO_PASS = 2 };
bool launch_prelude_pipe(const LaunchCtx& c, theta_dtype dt, int mode, const void* const* w, int L, int G,
                         const int32_t* band_start, const int32_t* band_of_layer, void* const* W0,
                         float* const* s, void* const* R, int64_t O, int64_t I, cudaError_t* e);
size_t frob_workspace_bytes();
// partials: out[0], out[1] receive the two sums instead of their ratio.
cudaError_t launch_frob(const LaunchCtx& c, theta_dtype dt, const void* a, const void* b,
                        int64_t n, double* out, void* ws, bool partials = false);

// ---- CUDA-core GEMM paths (simt_kernels.cu): fp32 forward / reconstruct.
// Output tiles are 64 x 64; the grid's y extent (tiles of M for the forward,
// of O for reconstruct) is limited to 65535, so callers refuse larger sizes.
constexpr int64_t kSimtMaxRows = (int64_t)65535 * 64;
cudaError_t launch_xv_simt(const LaunchCtx& c, theta_dtype dt, const void* X, const void* V,
                           int64_t M, int64_t I, int r, float* T);
cudaError_t launch_forward_simt(const LaunchCtx& c, theta_dtype dt, const void* X,
                                const void* W0, const float* s, const void* U, const float* T,
                                int64_t M, int64_t O, int64_t I, int r, void* Y);
cudaError_t launch_reconstruct_simt(const LaunchCtx& c, theta_dtype dt, const float* s,
                                    const void* W0, const void* U, const void* V, int64_t O,
                                    int64_t I, int r, void* W_out);

// ---- few-token forward on CUDA cores (gemv_kernels.cu): bf16. Returns false
// without launching when the problem does not fit (the caller takes the tile
// path); launch errors come back in *e.
// It launches its own T = X.V kernel; ws holds that kernel's partial sums.
int forward_gemv_max_tokens();
size_t forward_gemv_workspace_bytes(int64_t M, int r);
bool launch_forward_gemv(const LaunchCtx& c, const void* X, const void* W0, const float* s, const void* U,
                         const void* V, int64_t M, int64_t O, int64_t I, int r, void* Y, void* ws,
                         cudaError_t* e);

// ---- NVFP4 shared block (gemv_kernels.cu): encode W0 [O, I] bf16 into E2M1
// codes [O, I/2], E4M3 block scales [O, I/16] and the tensor scale *g (ws: 4
// bytes of scratch); the forward for one or two tokens from that encoding
// (false: does not fit the sweep; ws of forward_nvfp4_workspace_bytes).
cudaError_t launch_nvfp4_quantize(const LaunchCtx& c, const void* W, int64_t O, int64_t I, void* codes, void* scales,
                                  float* g, void* ws);
size_t forward_nvfp4_workspace_bytes(int64_t M, int64_t I, int r);
// Grouped few-token forward over a problem table (host copy for sizes, device
// copy for the kernels); rmax = the largest rank. false: outside its range.
size_t forward_grouped_workspace_bytes(int count, int64_t M, int rmax);
bool launch_forward_grouped(const LaunchCtx& c, const theta_forward_problem* host, const theta_forward_problem* dev,
                            int count, int64_t M, int rmax, void* ws, cudaError_t* e);
bool launch_forward_nvfp4(const LaunchCtx& c, const void* X, const void* codes, const void* scales, const float* g,
                          const float* s, const void* U, const void* V, int64_t M, int64_t O, int64_t I, int r,
                          void* Y, void* ws, cudaError_t* e);

// ---- randomized SVD of a residual (svd_kernels.cu): R [O, I] in dt, omega
// fp32 [samples, I]; U [O, rank], V [I, rank] in dt; ws of svd_workspace_bytes.
int svd_max_samples();
// Tensor-core products of a bf16 residual R [O, I] with an fp32 factor given
// as three bf16 parts, part_stride elements apart (umma_kernels.cu). r_left:
// part_out[z] = R . F^T [O, k], F parts [k, I] (row pitch I); otherwise
// part_out[z] = F^T . R [k, I], parts of Q^T [k, O] with row pitch
// part_pitch (a multiple of 8). Split z of `splits`
// (at most kSvdMaxSplits, from svd_mma_splits) covers a fixed share of K;
// the caller sums the splits. Needs I % 8 == 0 and 16-byte aligned R.
constexpr int kSvdMaxSplits = 8;
int svd_mma_splits(const LaunchCtx& c, bool r_left, int64_t O, int64_t I, int k);
int launch_svd_mma(const LaunchCtx& c, bool r_left, const void* R, int64_t O, int64_t I, const void* parts,
                   int64_t part_stride, int64_t part_pitch, int k, int splits, float* part_out, cudaError_t* ce);
size_t svd_workspace_bytes(int64_t O, int64_t I, int samples, int rank);
cudaError_t launch_residual_svd(const LaunchCtx& c, theta_dtype dt, const void* R, int64_t O, int64_t I, int rank,
                                int samples, int power_iters, const float* omega, void* U, void* V, void* ws);

// ---- tensor-core paths (umma_kernels.cu): bf16
size_t forward_umma_workspace_bytes(int64_t M, int r);
// Returns THETA_OK or a theta_status; CUDA errors are reported via *cuda_err.
int launch_forward_umma(const LaunchCtx& c, const void* X, const void* W0, const float* s,
                        const void* U, const void* V, int64_t M, int64_t O, int64_t I, int r,
                        void* Y, void* ws, cudaError_t* cuda_err);
// One bounded wait that nothing completes (gives up after limit_ms).
cudaError_t launch_wait_selftest(const LaunchCtx& c, unsigned limit_ms);
// Fused gate/up: Y = gelu_tanh(gate forward) * (up forward), one tile kernel
// after the two T = X.V kernels.
size_t gate_up_umma_workspace_bytes(int64_t M, int r);
int launch_gate_up_umma(const LaunchCtx& c, const void* X, const void* W0g, const float* sg, const void* Ug,
                        const void* Vg, const void* W0u, const float* su, const void* Uu, const void* Vu, int64_t M,
                        int64_t O, int64_t I, int r, void* Y, void* ws, cudaError_t* ce);
int launch_reconstruct_umma(const LaunchCtx& c, const float* s, const void* W0, const void* U,
                            const void* V, int64_t O, int64_t I, int r, void* W_out,
                            cudaError_t* cuda_err);
// The n layers of one band (one shared W0): each W0 tile read once for all of
// them (bands of up to 64 layers per launch; rank <= 128; else per layer).
int launch_reconstruct_band_umma(const LaunchCtx& c, const float* const* s, const void* W0, const void* const* U,
                                 const void* const* V, int n, int64_t O, int64_t I, int r, void* const* W_out,
                                 cudaError_t* cuda_err);

}  // namespace theta
