// The theta forward for a handful of tokens on CUDA cores
// ("The theta bundle" -- approximation formula, applied without forming the
// weight):  Y[m, o] = s[o] * (X[m, :] . W0[o, :]) + T[m, :] . U[o, :]
//
// With one or two tokens the projection is a matrix-vector stream over W0,
// bound by HBM. Each warp owns whole weight rows, two at a time, and
// consecutive warps take consecutive pairs (warp w of nw handles rows 2w and
// 2w + 1, then 2(w + nw) and 2(w + nw) + 1, ...), so at any moment the GPU
// reads one contiguous window of W0: a single sequential
// sweep, the access pattern that sustains the most read bandwidth (tile
// kernels stream 128-row column strips instead). X is read through L1.
//
// The kernel follows its own T = X.V kernel with programmatic dependent
// launch: it streams W0 immediately, keeps each row's X . W0 in registers,
// and waits for the previous grid only before the rank-r term. W0 and X are
// read through L2 only (ld.global.cg), so the stream leaves L1 to the rank
// term; T, U and s are reached through pointers passed through after_wait(),
// which keeps the compiler from scheduling their loads above the wait.
#include "common.cuh"
#include "internal.h"

namespace theta {

namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerIter = 2;  // rows a warp streams together (X vectors serve both)
constexpr int kKeptIters = 4;    // iterations whose results wait in registers for T
constexpr int kMaxRankPerLane = 8;  // rank <= 256

// acc[q][m] = W0[row q] . X[m] for kRowsPerIter consecutive rows
template <int M>
__device__ __forceinline__ void rows_dot(const bf16* __restrict__ W0, int64_t o0, int64_t O,
                                         const bf16* __restrict__ X, int64_t I, int64_t nv, int lane,
                                         float (&acc)[kRowsPerIter][M]) {
  const uint4* w0 = reinterpret_cast<const uint4*>(W0 + o0 * I);
  const uint4* w1 = reinterpret_cast<const uint4*>(W0 + (o0 + 1 < O ? o0 + 1 : o0) * I);
#pragma unroll
  for (int q = 0; q < kRowsPerIter; ++q)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[q][m] = 0.f;
  int64_t v = lane;
  for (; v + 32 < nv; v += 64) {
    uint4 w[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      w[0][u] = __ldcg(w0 + v + 32 * u);
      w[1][u] = __ldcg(w1 + v + 32 * u);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float f0[8], f1[8];
      unpack(w[0][u], f0);
      unpack(w[1][u], f1);
#pragma unroll
      for (int m = 0; m < M; ++m) {
        float fx[8];
        unpack(__ldcg(reinterpret_cast<const uint4*>(X + m * I) + v + 32 * u), fx);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[0][m] = fmaf(f0[e], fx[e], acc[0][m]);
          acc[1][m] = fmaf(f1[e], fx[e], acc[1][m]);
        }
      }
    }
  }
  for (; v < nv; v += 32) {
    float f0[8], f1[8];
    unpack(__ldcg(w0 + v), f0);
    unpack(__ldcg(w1 + v), f1);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float fx[8];
      unpack(__ldcg(reinterpret_cast<const uint4*>(X + m * I) + v), fx);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[0][m] = fmaf(f0[e], fx[e], acc[0][m]);
        acc[1][m] = fmaf(f1[e], fx[e], acc[1][m]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kRowsPerIter; ++q)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[q][m] = warp_sum(acc[q][m]);
}

template <int M>
__global__ void __launch_bounds__(kThreads)
gemv_forward_kernel(const bf16* __restrict__ X, const bf16* __restrict__ W0, const float* __restrict__ s,
                    const bf16* __restrict__ U, const bf16* __restrict__ Thi, const bf16* __restrict__ Tlo,
                    int64_t O, int64_t I, int r, bf16* __restrict__ Y, int early) {
  if (!early) {
    pdl_wait();
    after_wait(X), after_wait(W0), after_wait(s), after_wait(U);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t nw = (int64_t)gridDim.x * (kThreads / 32);
  const int64_t gw = (int64_t)blockIdx.x * (kThreads / 32) + threadIdx.x / 32;
  const int64_t nv = I / 8;
  const int nj = (r + 31) / 32;  // rank entries per lane
  auto first_row = [&](int64_t k) { return (gw + k * nw) * kRowsPerIter; };

  // X . W0 of the first kKeptIters iterations, kept until T is ready
  float kept[kKeptIters][kRowsPerIter][M];
#pragma unroll
  for (int k = 0; k < kKeptIters; ++k) {
    const int64_t o0 = first_row(k);
    if (o0 < O) {
      float acc[kRowsPerIter][M];
      rows_dot<M>(W0, o0, O, X, I, nv, lane, acc);
#pragma unroll
      for (int q = 0; q < kRowsPerIter; ++q)
#pragma unroll
        for (int m = 0; m < M; ++m) kept[k][q][m] = acc[q][m];
    }
  }
  if (early) pdl_wait();  // T is ready from here on
  after_wait(Thi), after_wait(Tlo), after_wait(s), after_wait(U);
  // T = T_hi + T_lo, this lane's rank entries, loaded once
  float t[M][kMaxRankPerLane];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int jj = 0; jj < kMaxRankPerLane; ++jj) {
      const int j = lane + 32 * jj;
      t[m][jj] = (jj < nj && j < r) ? __bfloat162float(Thi[m * r + j]) + __bfloat162float(Tlo[m * r + j]) : 0.f;
    }
  auto finish = [&](int64_t o, const float (&dot)[M]) {
    const float so = __ldg(s + o);
    float rk[M];
#pragma unroll
    for (int m = 0; m < M; ++m) rk[m] = 0.f;
#pragma unroll
    for (int jj = 0; jj < kMaxRankPerLane; ++jj) {
      const int j = lane + 32 * jj;
      if (jj < nj && j < r) {
        const float u = __bfloat162float(U[o * r + j]);
#pragma unroll
        for (int m = 0; m < M; ++m) rk[m] = fmaf(u, t[m][jj], rk[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) rk[m] = warp_sum(rk[m]);
#pragma unroll
    for (int m = 0; m < M; ++m)
      if (lane == m) Y[m * O + o] = __float2bfloat16_rn(fmaf(so, dot[m], rk[m]));
  };
#pragma unroll
  for (int k = 0; k < kKeptIters; ++k) {
#pragma unroll
    for (int q = 0; q < kRowsPerIter; ++q) {
      const int64_t o = first_row(k) + q;
      if (o < O) finish(o, kept[k][q]);
    }
  }
  // iterations beyond what the registers hold (very small grids only)
  for (int64_t k = kKeptIters;; ++k) {
    const int64_t o0 = first_row(k);
    if (o0 >= O) break;
    float acc[kRowsPerIter][M];
    rows_dot<M>(W0, o0, O, X, I, nv, lane, acc);
#pragma unroll
    for (int q = 0; q < kRowsPerIter; ++q)
      if (o0 + q < O) finish(o0 + q, acc[q]);
  }
}

}  // namespace

int forward_gemv_max_tokens() { return 2; }

cudaError_t launch_forward_gemv(const LaunchCtx& c, const void* X, const void* W0, const float* s, const void* U,
                                const void* t_hi, const void* t_lo, int64_t M, int64_t O, int64_t I, int r, void* Y,
                                bool early) {
  int64_t grid = ceil_div(ceil_div(O, kRowsPerIter), kThreads / 32);
  const int64_t cap = (int64_t)c.num_sms * (2048 / kThreads);
  if (grid > cap) grid = cap;
  const bf16* x = static_cast<const bf16*>(X);
  const bf16* w = static_cast<const bf16*>(W0);
  const bf16* u = static_cast<const bf16*>(U);
  const bf16* th = static_cast<const bf16*>(t_hi);
  const bf16* tl = static_cast<const bf16*>(t_lo);
  bf16* y = static_cast<bf16*>(Y);
  const int e = early ? 1 : 0;
  switch (M) {
    case 1: return launch_pdl(gemv_forward_kernel<1>, dim3((unsigned)grid), dim3(kThreads), 0, c.stream, 1, x, w, s, u, th, tl, O, I, r, y, e);
    case 2: return launch_pdl(gemv_forward_kernel<2>, dim3((unsigned)grid), dim3(kThreads), 0, c.stream, 1, x, w, s, u, th, tl, O, I, r, y, e);
  }
  return cudaErrorInvalidValue;
}

}  // namespace theta
