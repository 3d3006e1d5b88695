// CUDA-core (fp32 FMA) kernels of the theta forward and reconstruct_weight.
//
// These serve THETA_F32, where the fp32 tolerance rules out tf32 tensor cores.
// The projection is computed as two accumulations per output element,
//   acc1 = sum_k A1[a,k] B1[b,k]   and   acc2 = sum_j A2[a,j] B2[b,j],
// both "row-major times row-major transposed", followed by an epilogue:
//   forward:      Y[m,o]  = s[o] * acc1(X, W0) + acc2(T, U),  T = X.V
//   reconstruct:  W[o,i]  = s[o] * W0[o,i] + acc1(U, V)
// ("The theta bundle" -- approximation formula; the forward never forms W).
#include "common.cuh"
#include "internal.h"

namespace theta {

namespace {

constexpr int BM = 64, BN = 64, BK = 16, kThreads = 256;

template <typename T>
__device__ __forceinline__ float ldf(const T* p, int64_t i) {
  return to_f32(p[i]);
}

// Loads a BMxBK tile of a row-major [rows, K] matrix into smem as [BK][BM+1]
// (transposed so the inner product loop reads consecutive rows).
template <typename T>
__device__ __forceinline__ void load_tile(float (*dst)[BM + 1], const T* __restrict__ src,
                                          int64_t rows, int64_t K, int64_t row0, int64_t k0) {
  for (int e = threadIdx.x; e < BM * BK; e += kThreads) {
    const int r = e / BK, k = e % BK;
    const int64_t gr = row0 + r, gk = k0 + k;
    dst[k][r] = (gr < rows && gk < K) ? ldf(src, gr * K + gk) : 0.f;
  }
}

// Sums of kChain consecutive products are formed on their own and then added
// to the running total, so no fp32 rounding chain grows beyond about
// kChain + K / kChain additions (a plain running sum over K = 16K drifts past
// the 1e-5 relative tolerance of the fp32 path).
constexpr int kChain = 256;

template <typename TA, typename TB>
__device__ __forceinline__ void accumulate(float (&acc)[4][4], const TA* __restrict__ A,
                                           const TB* __restrict__ B, int64_t Ma, int64_t Nb,
                                           int64_t K, int64_t a0, int64_t b0,
                                           float (*As)[BM + 1], float (*Bs)[BM + 1]) {
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float part[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += BK) {
    if (k0 % kChain == 0 && k0 > 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] += part[i][j];
          part[i][j] = 0.f;
        }
    }
    load_tile(As, A, Ma, K, a0, k0);
    load_tile(Bs, B, Nb, K, b0, k0);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[k][ty + 16 * i];
        bv[i] = Bs[k][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(av[i], bv[j], part[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
}

// Y[M, O] = s (.) (X . W0^T) + T . U^T with T = X . V precomputed in fp32.
template <typename T>
__global__ void __launch_bounds__(kThreads)
forward_simt_kernel(const T* __restrict__ X, const T* __restrict__ W0, const float* __restrict__ s,
                    const T* __restrict__ U, const float* __restrict__ Tm, int64_t M, int64_t O,
                    int64_t I, int r, T* __restrict__ Y) {
  __shared__ float As[BK][BM + 1], Bs[BK][BM + 1];
  const int64_t a0 = (int64_t)blockIdx.y * BM, b0 = (int64_t)blockIdx.x * BN;
  float acc1[4][4] = {}, acc2[4][4] = {};
  accumulate(acc1, X, W0, M, O, I, a0, b0, As, Bs);
  if (r > 0) accumulate(acc2, Tm, U, M, O, (int64_t)r, a0, b0, As, Bs);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t o = b0 + tx + 16 * j;
    if (o >= O) continue;
    const float so = s[o];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t m = a0 + ty + 16 * i;
      if (m < M) Y[m * O + o] = from_f32<T>(fmaf(so, acc1[i][j], acc2[i][j]));
    }
  }
}

// W_out[O, I] = s (.) W0 + U . V^T
template <typename T>
__global__ void __launch_bounds__(kThreads)
reconstruct_simt_kernel(const float* __restrict__ s, const T* __restrict__ W0,
                        const T* __restrict__ U, const T* __restrict__ V, int64_t O, int64_t I,
                        int r, T* __restrict__ W_out) {
  __shared__ float As[BK][BM + 1], Bs[BK][BM + 1];
  const int64_t a0 = (int64_t)blockIdx.y * BM, b0 = (int64_t)blockIdx.x * BN;
  float acc[4][4] = {};
  if (r > 0) accumulate(acc, U, V, O, I, (int64_t)r, a0, b0, As, Bs);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t o = a0 + ty + 16 * i;
    if (o >= O) continue;
    const float so = s[o];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = b0 + tx + 16 * j;
      if (c < I) W_out[o * I + c] = from_f32<T>(fmaf(so, to_f32(W0[o * I + c]), acc[i][j]));
    }
  }
}

// T[M, r] = X[M, I] . V[I, r] in fp32. Block = 32 rank columns x 8 slices of I;
// the 8 slice sums are combined in a fixed order.
template <typename T>
__global__ void __launch_bounds__(kThreads)
xv_simt_kernel(const T* __restrict__ X, const T* __restrict__ V, int64_t M, int64_t I, int r,
               float* __restrict__ Tm) {
  __shared__ float part[8][33];
  const int lane = threadIdx.x & 31, g = threadIdx.x / 32;
  const int j = blockIdx.x * 32 + lane;
  for (int64_t m = blockIdx.y; m < M; m += gridDim.y) {
    float acc = 0.f;
    if (j < r) {
      const T* x = X + m * I;
      for (int64_t i0 = 0; i0 < I; i0 += 8 * kChain) {  // chains of kChain products
        float part = 0.f;
        const int64_t i1 = i0 + 8 * kChain < I ? i0 + 8 * kChain : I;
        for (int64_t i = i0 + g; i < i1; i += 8) part = fmaf(to_f32(x[i]), to_f32(V[i * r + j]), part);
        acc += part;
      }
    }
    part[g][lane] = acc;
    __syncthreads();
    if (g == 0 && j < r) {
      float t = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) t += part[k][lane];
      Tm[m * r + j] = t;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_xv_simt(const LaunchCtx& c, theta_dtype dt, const void* X, const void* V,
                           int64_t M, int64_t I, int r, float* T) {
  dim3 grid((unsigned)ceil_div(r, 32), (unsigned)(M < 65535 ? M : 65535));
  if (dt == THETA_BF16)
    xv_simt_kernel<bf16><<<grid, kThreads, 0, c.stream>>>(static_cast<const bf16*>(X),
                                                          static_cast<const bf16*>(V), M, I, r, T);
  else
    xv_simt_kernel<float><<<grid, kThreads, 0, c.stream>>>(static_cast<const float*>(X),
                                                           static_cast<const float*>(V), M, I, r, T);
  return cudaGetLastError();
}

cudaError_t launch_forward_simt(const LaunchCtx& c, theta_dtype dt, const void* X,
                                const void* W0, const float* s, const void* U, const float* T,
                                int64_t M, int64_t O, int64_t I, int r, void* Y) {
  dim3 grid((unsigned)ceil_div(O, BN), (unsigned)ceil_div(M, BM));
  if (dt == THETA_BF16)
    forward_simt_kernel<bf16><<<grid, kThreads, 0, c.stream>>>(
        static_cast<const bf16*>(X), static_cast<const bf16*>(W0), s, static_cast<const bf16*>(U), T,
        M, O, I, r, static_cast<bf16*>(Y));
  else
    forward_simt_kernel<float><<<grid, kThreads, 0, c.stream>>>(
        static_cast<const float*>(X), static_cast<const float*>(W0), s,
        static_cast<const float*>(U), T, M, O, I, r, static_cast<float*>(Y));
  return cudaGetLastError();
}

cudaError_t launch_reconstruct_simt(const LaunchCtx& c, theta_dtype dt, const float* s,
                                    const void* W0, const void* U, const void* V, int64_t O,
                                    int64_t I, int r, void* W_out) {
  dim3 grid((unsigned)ceil_div(I, BN), (unsigned)ceil_div(O, BM));
  if (dt == THETA_BF16)
    reconstruct_simt_kernel<bf16><<<grid, kThreads, 0, c.stream>>>(
        s, static_cast<const bf16*>(W0), static_cast<const bf16*>(U), static_cast<const bf16*>(V),
        O, I, r, static_cast<bf16*>(W_out));
  else
    reconstruct_simt_kernel<float><<<grid, kThreads, 0, c.stream>>>(
        s, static_cast<const float*>(W0), static_cast<const float*>(U),
        static_cast<const float*>(V), O, I, r, static_cast<float*>(W_out));
  return cudaGetLastError();
}

}  // namespace theta
