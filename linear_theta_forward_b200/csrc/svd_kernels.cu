// Randomized truncated SVD of a residual on the GPU ("The theta bundle" --
// Low-rank residual: U . V^T ~ residual, U absorbing the singular values,
// computed by the randomized algorithm of Halko, Martinsson and Tropp for
// large matrices). With k = rank + oversampling samples:
//
//   Y = R . Omega^T                 [O, k]   range sample (Omega given, [k, I])
//   Q = orth(Y)                              shifted Cholesky QR, then two plain passes
//   repeat power_iters times:                subspace iteration
//     Z^T = Q^T . R  -> orth of its rows     [k, I]
//     Y = R . Z      -> Q = orth(Y)
//   B = Q^T . R                     [k, I]
//   B . B^T = E diag(lambda) E^T             Jacobi eigen-decomposition (one CTA, fp64)
//   U = Q . E_r . diag(sigma_r),  V = B^T . E_r . diag(1 / sigma_r),
//   sigma_j = || B^T e_j ||                  (the singular values of B)
//
// This is decomposition-time work, not the projection hot path: the dense
// products run as fp32 CUDA-core tile GEMMs (64 x 64 tiles, 4 x 4 per thread,
// sums in chains of 256 products), with K split across CTAs and the partial
// tiles added in a fixed order when the output is small; the k x k steps run
// in one CTA in fp64. Every reduction has a fixed order, so the result is
// reproducible run to run.
#include "common.cuh"
#include "internal.h"

namespace theta {

namespace {

constexpr int kT = 256;           // threads of the tile GEMM
constexpr int kBM = 64, kBK = 16;  // output tile edge, K per shared-memory step
constexpr int kChain = 256;        // products per fp32 partial sum
constexpr int kMaxSamples = 96;    // k: the one-CTA fp64 steps hold two k x k matrices
constexpr int kSvdParts3 = 3;      // bf16 parts of an fp32 factor on the tensor-core products

template <typename T>
__device__ __forceinline__ float ldf(const T* p, int64_t i) {
  return to_f32(p[i]);
}

// C[z][m, n] = sum over k in split z of opA(m, k) * opB(n, k), where
// opA(m, k) = A_T ? A[k, m] (A is [K, M]) : A[m, k] (A is [M, K]), and the same
// for B with N. C is fp32 [splits, M, N].
template <typename TA, typename TB, bool A_T, bool B_T>
__global__ void __launch_bounds__(kT)
gemm_kernel(const TA* __restrict__ A, const TB* __restrict__ B, int64_t M, int64_t N, int64_t K, int64_t kchunk,
            float* __restrict__ C) {
  pdl_enter(A, B);
  __shared__ float As[kBK][kBM + 1], Bs[kBK][kBM + 1];
  const int64_t m0 = (int64_t)blockIdx.y * kBM, n0 = (int64_t)blockIdx.x * kBM;
  const int64_t kb = (int64_t)blockIdx.z * kchunk;
  const int64_t ke = kb + kchunk < K ? kb + kchunk : K;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {}, part[4][4] = {};
  for (int64_t k0 = kb; k0 < ke; k0 += kBK) {
    if ((k0 - kb) % kChain == 0 && k0 > kb) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] += part[i][j];
          part[i][j] = 0.f;
        }
    }
    for (int e = threadIdx.x; e < kBM * kBK; e += kT) {
      int r, kk;
      if (A_T) {
        kk = e / kBM, r = e % kBM;  // consecutive threads: consecutive m
      } else {
        r = e / kBK, kk = e % kBK;  // consecutive threads: consecutive k
      }
      const int64_t gm = m0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < ke) ? ldf(A, A_T ? gk * M + gm : gm * K + gk) : 0.f;
    }
    for (int e = threadIdx.x; e < kBM * kBK; e += kT) {
      int r, kk;
      if (B_T) {
        kk = e / kBM, r = e % kBM;
      } else {
        r = e / kBK, kk = e % kBK;
      }
      const int64_t gn = n0 + r, gk = k0 + kk;
      Bs[kk][r] = (gn < N && gk < ke) ? ldf(B, B_T ? gk * N + gn : gn * K + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty + 16 * i];
        bv[i] = Bs[kk][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(av[i], bv[j], part[i][j]);
    }
    __syncthreads();
  }
  float* Cz = C + (int64_t)blockIdx.z * M * N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx + 16 * j;
      if (n < N) Cz[m * N + n] = acc[i][j] + part[i][j];
    }
  }
}

// The exact split of an fp32 value into three bf16 parts, x = p1 + p2 + p3:
// each part is the remainder so far rounded to bf16, and each remainder is
// exact in fp32 (x - p1 and its successor lose no bits).
__device__ __forceinline__ void split3(float x, bf16* p) {
  const bf16 a = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(a);
  const bf16 b = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(b);
  p[0] = a, p[1] = b, p[2] = __float2bfloat16_rn(r2);
}

// F [rows, cols] fp32 -> parts [3][rows, cols] bf16 (each part_elems apart)
__global__ void __launch_bounds__(256) split3_kernel(const float* __restrict__ F, int64_t count,
                                                     bf16* __restrict__ parts, int64_t part_elems) {
  pdl_enter(F, parts);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    bf16 p[3];
    split3(F[i], p);
    parts[i] = p[0], parts[part_elems + i] = p[1], parts[2 * part_elems + i] = p[2];
  }
}

// Q [O, k] fp32 -> parts of Q^T: [3][k, pitch] bf16, element (j, o) = Q[o, j]
__global__ void __launch_bounds__(256) split3_transpose_kernel(const float* __restrict__ Q, int64_t O, int k,
                                                               bf16* __restrict__ parts, int64_t pitch,
                                                               int64_t part_elems) {
  pdl_enter(Q, parts);
  const int64_t count = O * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = i / O, o = i % O;  // consecutive threads write consecutive o
    bf16 p[3];
    split3(Q[o * k + j], p);
    const int64_t d = j * pitch + o;
    parts[d] = p[0], parts[part_elems + d] = p[1], parts[2 * part_elems + d] = p[2];
  }
}

// out[i] = sum over z (in order) of part[z][i], i < count
__global__ void __launch_bounds__(256) sum_splits_kernel(const float* __restrict__ part, int splits, int64_t count,
                                                         float* __restrict__ out) {
  pdl_enter(part);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    float s = 0.f;
    for (int z = 0; z < splits; ++z) s += part[(int64_t)z * count + i];
    out[i] = s;
  }
}

// Cholesky of the k x k Gram matrix G (+ a shift) and the inverse of its
// factor, in fp64, one CTA. shift_rows > 0 adds the shift of shifted
// Cholesky QR (Fukaya, Kannan, Nakatsukasa, Yamamoto, Yanagisawa, 2020),
// 11 c u trace(G): u is the fp32 unit roundoff of the Gram product and c
// bounds its summation error -- here chains of 256 products added across
// rows / 256 chains, c = 256 + rows / 256 (the factorization itself runs in
// fp64, so the paper's k (k + 1) term for it is negligible). The shift makes
// G + shift positive definite for an ill-conditioned sample. A pivot that is
// not positive marks a direction the sample does not have: that row of the
// inverse is set to zero, so the orthonormalized column comes out zero.
// Outputs Linv [k, k] (row j = row j of L^-1) and LinvT = its transpose.
__global__ void __launch_bounds__(256) chol_inv_kernel(const float* __restrict__ G, int k, int64_t shift_rows,
                                                       float* __restrict__ Linv, float* __restrict__ LinvT) {
  pdl_enter(G);
  extern __shared__ double sm[];
  double* A = sm;          // [k][k], lower triangle becomes L
  double* X = sm + k * k;  // [k][k], L^-1
  __shared__ double trace;
  __shared__ int dead[kMaxSamples];
  const int t = threadIdx.x;
  for (int e = t; e < k * k; e += blockDim.x) {
    const int i = e / k, j = e % k;
    A[e] = 0.5 * ((double)G[i * k + j] + (double)G[j * k + i]);  // symmetrize
    X[e] = 0.0;
  }
  __syncthreads();
  if (t == 0) {
    double tr = 0.0;
    for (int i = 0; i < k; ++i) tr += A[i * k + i];
    trace = tr;
  }
  __syncthreads();
  if (shift_rows > 0) {
    const double c = (double)kChain + (double)shift_rows / kChain;
    const double shift = 11.0 * c * 5.960464477539063e-8 * trace;
    for (int i = t; i < k; i += blockDim.x) A[i * k + i] += shift;
  }
  __syncthreads();
  const double tiny = 1e-30 + 1e-14 * trace;
  for (int j = 0; j < k; ++j) {
    if (t == 0) {
      const double piv = A[j * k + j];
      dead[j] = !(piv > tiny);
      A[j * k + j] = dead[j] ? 1.0 : sqrt(piv);
    }
    __syncthreads();
    const double d = A[j * k + j];
    for (int i = j + 1 + t; i < k; i += blockDim.x) A[i * k + j] = dead[j] ? 0.0 : A[i * k + j] / d;
    __syncthreads();
    // trailing update of the lower triangle: A[i][l] -= L[i][j] L[l][j], j < l <= i
    const int n = k - j - 1;
    for (int e = t; e < n * n; e += blockDim.x) {
      const int i = j + 1 + e / n, l = j + 1 + e % n;
      if (l <= i) A[i * k + l] -= A[i * k + j] * A[l * k + j];
    }
    __syncthreads();
  }
  // L^-1 by forward substitution, one column per thread
  for (int c = t; c < k; c += blockDim.x) {
    for (int i = c; i < k; ++i) {
      if (dead[i]) {
        X[i * k + c] = 0.0;
        continue;
      }
      double s = (i == c) ? 1.0 : 0.0;
      for (int p = c; p < i; ++p) s -= A[i * k + p] * X[p * k + c];
      X[i * k + c] = s / A[i * k + i];
    }
  }
  __syncthreads();
  for (int e = t; e < k * k; e += blockDim.x) {
    const int i = e / k, j = e % k;
    Linv[e] = (float)X[e];
    LinvT[j * k + i] = (float)X[e];
  }
}

// Eigen-decomposition of the symmetric k x k matrix S by cyclic Jacobi
// rotations in fp64, one CTA: each round rotates k / 2 disjoint index pairs
// (round-robin order), rows first then columns; sweeps stop when the
// off-diagonal mass is below 1e-28 of the total, or after 40. The r largest
// eigenpairs, in descending order, go out as E [k, r] (column j = eigenvector
// j) and Et [r, k] (its transpose).
__global__ void __launch_bounds__(256) jacobi_eig_kernel(const float* __restrict__ S, int k, int r,
                                                         float* __restrict__ E, float* __restrict__ Et) {
  pdl_enter(S);
  extern __shared__ double sm[];
  const int kp = k + (k & 1);  // even number of indices; the last one is a dummy when k is odd
  double* A = sm;              // [k][k]
  double* W = sm + k * k;      // [k][k] eigenvectors (columns)
  __shared__ double cs[kMaxSamples / 2 + 1][2];
  __shared__ int pp[kMaxSamples / 2 + 1][2];
  __shared__ int order[kMaxSamples];
  __shared__ double off, total;
  const int t = threadIdx.x;
  for (int e = t; e < k * k; e += blockDim.x) {
    const int i = e / k, j = e % k;
    A[e] = 0.5 * ((double)S[i * k + j] + (double)S[j * k + i]);
    W[e] = (i == j) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < 40; ++sweep) {
    if (t == 0) {
      double o = 0.0, a = 0.0;
      for (int i = 0; i < k; ++i)
        for (int j = 0; j < k; ++j) {
          const double v = A[i * k + j] * A[i * k + j];
          a += v;
          if (i != j) o += v;
        }
      off = o;
      total = a;
    }
    __syncthreads();
    if (!(off > 1e-28 * total)) break;
    for (int round = 0; round < kp - 1; ++round) {
      // round-robin (circle) pairing: index kp-1 meets index `round`, and
      // round + q meets round - q (mod kp - 1) for q = 1 .. kp/2 - 1
      for (int q = t; q < kp / 2; q += blockDim.x) {
        int a = q == 0 ? round : (round + q) % (kp - 1);
        int b = q == 0 ? kp - 1 : (round - q + (kp - 1)) % (kp - 1);
        if (a > b) {
          const int x = a;
          a = b;
          b = x;
        }
        pp[q][0] = a;
        pp[q][1] = b;
        double c = 1.0, s = 0.0;
        if (b < k) {  // not the dummy
          const double apq = A[a * k + b];
          if (fabs(apq) > 1e-300) {
            const double theta = (A[b * k + b] - A[a * k + a]) / (2.0 * apq);
            const double tt = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
            c = 1.0 / sqrt(tt * tt + 1.0);
            s = tt * c;
          }
        }
        cs[q][0] = c;
        cs[q][1] = s;
      }
      __syncthreads();
      // rows: A <- J^T A
      for (int e = t; e < (kp / 2) * k; e += blockDim.x) {
        const int q = e / k, col = e % k;
        const int a = pp[q][0], b = pp[q][1];
        if (b >= k) continue;
        const double c = cs[q][0], s = cs[q][1];
        const double x = A[a * k + col], y = A[b * k + col];
        A[a * k + col] = c * x - s * y;
        A[b * k + col] = s * x + c * y;
      }
      __syncthreads();
      // columns: A <- A J, W <- W J
      for (int e = t; e < (kp / 2) * k; e += blockDim.x) {
        const int q = e / k, row = e % k;
        const int a = pp[q][0], b = pp[q][1];
        if (b >= k) continue;
        const double c = cs[q][0], s = cs[q][1];
        double x = A[row * k + a], y = A[row * k + b];
        A[row * k + a] = c * x - s * y;
        A[row * k + b] = s * x + c * y;
        x = W[row * k + a], y = W[row * k + b];
        W[row * k + a] = c * x - s * y;
        W[row * k + b] = s * x + c * y;
      }
      __syncthreads();
    }
  }
  if (t == 0) {  // eigenvalues in descending order (stable selection)
    for (int i = 0; i < k; ++i) order[i] = i;
    for (int i = 0; i < k; ++i) {
      int best = i;
      for (int j = i + 1; j < k; ++j)
        if (A[order[j] * k + order[j]] > A[order[best] * k + order[best]]) best = j;
      const int x = order[i];
      order[i] = order[best];
      order[best] = x;
    }
  }
  __syncthreads();
  for (int e = t; e < k * r; e += blockDim.x) {
    const int i = e / r, j = e % r;  // component i of eigenvector j
    const float v = (float)W[i * k + order[j]];
    E[i * r + j] = v;
    Et[j * k + i] = v;
  }
}

// sigma_j = || column j of Vun ||, in a fixed order: one CTA per column.
__global__ void __launch_bounds__(256) col_norm_kernel(const float* __restrict__ Vun, int64_t rows, int r,
                                                       float* __restrict__ sigma) {
  pdl_enter(Vun);
  __shared__ double red[256 / 32];
  const int j = blockIdx.x;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < rows; i += blockDim.x) {
    const double v = Vun[i * r + j];
    s += v * v;
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < 256 / 32; ++w) tot += red[w];
    sigma[j] = (float)sqrt(tot);
  }
}

// out[i, j] = in[i, j] * (scale ? sigma_j : 1 / sigma_j), 0 where sigma_j = 0
template <typename T>
__global__ void __launch_bounds__(256) scale_cols_kernel(const float* __restrict__ in, const float* __restrict__ sigma,
                                                         int64_t rows, int r, int multiply, T* __restrict__ out) {
  pdl_enter(in, sigma);
  const int64_t n = rows * r, stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
    const float sg = sigma[e % r];
    const float f = sg > 0.f ? (multiply ? sg : 1.f / sg) : 0.f;
    out[e] = from_f32<T>(in[e] * f);
  }
}

// ----------------------------------------------------------------- host
// K splits for small outputs, so the grid has about kTargetCtas CTAs; a
// function of the shapes only, so the workspace size is too.
constexpr int64_t kTargetCtas = 512;
int splits_for(int64_t M, int64_t N, int64_t K) {
  const int64_t tiles = ceil_div(M, kBM) * ceil_div(N, kBM);
  int64_t s = ceil_div(kTargetCtas, tiles);
  if (s > 64) s = 64;
  if (s > K / 64) s = K / 64;  // each split keeps at least 64 products per sum
  return s < 1 ? 1 : (int)s;
}

// The k x k one-CTA kernels hold two fp64 k x k matrices in shared memory.
size_t small_smem(int k) { return (size_t)2 * k * k * sizeof(double); }

struct SvdPlan {
  int64_t O, I;
  int k, r;
  int64_t qpitch;  // row pitch (elements) of the parts of Q^T [k, O]
  int64_t part_elems;  // elements per bf16 part of F
  // workspace offsets, in floats
  int64_t y0, y1, z0, z1, bm, g, li, lit, s, e, et, uraw, vun, sig, part, parts, total;
};

SvdPlan plan_svd(int64_t O, int64_t I, int k, int r) {
  SvdPlan p{};
  p.O = O, p.I = I, p.k = k, p.r = r;
  int64_t at = 0;
  auto take = [&](int64_t n) {
    const int64_t o = at;
    at += (n + 63) / 64 * 64;  // 256-byte aligned pieces
    return o;
  };
  p.y0 = take(O * k), p.y1 = take(O * k);
  p.z0 = take(k * I), p.z1 = take(k * I), p.bm = take(k * I);
  p.g = take(k * k), p.li = take(k * k), p.lit = take(k * k), p.s = take(k * k);
  p.e = take(k * r), p.et = take(r * k), p.uraw = take(O * r), p.vun = take(I * r), p.sig = take(r);
  // partial tiles of the split GEMMs (the largest split output below)
  int64_t part = 0;
  auto need = [&](int64_t M, int64_t N, int64_t K) {
    const int sp = splits_for(M, N, K);
    if (sp > 1 && sp * M * N > part) part = sp * M * N;
  };
  need(O, k, I);  // R Omega^T, R Z
  need(k, k, O);  // Y^T Y
  need(O, k, k);  // Y L^-T
  need(k, I, O);  // Q^T R
  need(k, k, I);  // Z^T Z, B B^T
  need(k, I, k);  // L^-1 Z^T
  need(O, r, k);  // Q E_r
  need(I, r, k);  // B^T E_r
  // the tensor-core products with a bf16 R: split partials of C [O, k] or
  // [k, I], and the three bf16 parts of the fp32 factor
  const int64_t mma_part = (int64_t)kSvdMaxSplits * (O * k > k * I ? O * k : k * I);
  if (mma_part > part) part = mma_part;
  p.part = take(part > 0 ? part : 1);
  p.qpitch = (O + 7) / 8 * 8;
  p.part_elems = (int64_t)k * (p.qpitch > I ? p.qpitch : I);
  p.parts = take((kSvdParts3 * p.part_elems + 1) / 2);
  p.total = at;
  return p;
}

// One product of the bf16 residual with an fp32 factor on tensor cores (the
// factor split into three bf16 parts, the K splits summed in order).
// r_left: out [O, k] = R . F^T, F [k, I]; else out [k, I] = Q^T . R, Q [O, k].
cudaError_t product_mma(const LaunchCtx& c, const SvdPlan& p, float* ws, bool r_left, const bf16* R,
                        const float* F, float* out) {
  const int64_t O = p.O, I = p.I;
  const int k = p.k;
  bf16* parts = reinterpret_cast<bf16*>(ws + p.parts);
  const auto blocks = [&](int64_t n) {
    int64_t b = ceil_div(n, 256);
    return (unsigned)(b > 8 * (int64_t)c.num_sms ? 8 * (int64_t)c.num_sms : b);
  };
  cudaError_t e = r_left ? launch_pdl(split3_kernel, dim3(blocks(k * I)), dim3(256), 0, c.stream, 1, F, (int64_t)k * I,
                                      parts, p.part_elems)
                         : launch_pdl(split3_transpose_kernel, dim3(blocks(O * k)), dim3(256), 0, c.stream, 1, F, O,
                                      k, parts, p.qpitch, p.part_elems);
  if (e != cudaSuccess) return e;
  const int sp = svd_mma_splits(c, r_left, O, I, k);
  float* dst = sp > 1 ? ws + p.part : out;
  int st = launch_svd_mma(c, r_left, R, O, I, parts, p.part_elems, r_left ? I : p.qpitch, k, sp, dst, &e);
  if (st != THETA_OK) return e != cudaSuccess ? e : cudaErrorInvalidValue;
  if (sp == 1) return cudaSuccess;
  const int64_t count = r_left ? O * k : (int64_t)k * I;
  int64_t nb = ceil_div(count, 256);
  if (nb > 4 * (int64_t)c.num_sms) nb = 4 * (int64_t)c.num_sms;
  return launch_pdl(sum_splits_kernel, dim3((unsigned)nb), dim3(256), 0, c.stream, 1, (const float*)(ws + p.part), sp,
                    count, out);
}

// C = op(A) . op(B)^T with the split and its fixed-order sum; out fp32 [M, N]
template <typename TA, typename TB, bool A_T, bool B_T>
cudaError_t gemm(const LaunchCtx& c, const TA* A, const TB* B, int64_t M, int64_t N, int64_t K, float* out,
                 float* part) {
  const int sp = splits_for(M, N, K);
  const int64_t kchunk = ceil_div(ceil_div(K, sp), kBK) * kBK;
  const int spz = (int)ceil_div(K, kchunk);
  dim3 grid((unsigned)ceil_div(N, kBM), (unsigned)ceil_div(M, kBM), (unsigned)spz);
  float* dst = spz > 1 ? part : out;
  cudaError_t e = launch_pdl(gemm_kernel<TA, TB, A_T, B_T>, grid, dim3(kT), 0, c.stream, 1, A, B, M, N, K, kchunk, dst);
  if (e != cudaSuccess || spz == 1) return e;
  int64_t blocks = ceil_div(M * N, 256);
  if (blocks > 4 * (int64_t)c.num_sms) blocks = 4 * (int64_t)c.num_sms;
  return launch_pdl(sum_splits_kernel, dim3((unsigned)blocks), dim3(256), 0, c.stream, 1, (const float*)part, spz,
                    M * N, out);
}

cudaError_t small_kernels_ready(int device) {
  std::lock_guard<std::mutex> lk(setup_mutex());
  static bool done[64] = {};
  if (done[device]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)small_smem(kMaxSamples));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(jacobi_eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)small_smem(kMaxSamples));
  if (e == cudaSuccess) done[device] = true;
  return e;
}

// Orthonormal columns of Y [rows, k] (fp32), in place through `tmp`: one
// shifted Cholesky QR pass and two plain ones. Returns the buffer holding Q.
cudaError_t orth_cols(const LaunchCtx& c, const SvdPlan& p, float* ws, int64_t rows, float* Y, float* tmp,
                      float** Q) {
  const int k = p.k;
  float *g = ws + p.g, *li = ws + p.li, *lit = ws + p.lit, *part = ws + p.part;
  cudaError_t e = cudaSuccess;
  for (int pass = 0; pass < 3 && e == cudaSuccess; ++pass) {
    e = gemm<float, float, true, true>(c, Y, Y, k, k, rows, g, part);  // G = Y^T Y
    if (e == cudaSuccess)
      e = launch_pdl(chol_inv_kernel, dim3(1), dim3(256), small_smem(k), c.stream, 1, (const float*)g, k,
                     pass == 0 ? rows : (int64_t)0, li, lit);
    if (e == cudaSuccess) e = gemm<float, float, false, false>(c, Y, li, rows, k, k, tmp, part);  // Y L^-T
    float* x = Y;
    Y = tmp;
    tmp = x;
  }
  *Q = Y;
  return e;
}

// Orthonormal rows of Zt [k, cols] (fp32): the same passes on the transpose.
cudaError_t orth_rows(const LaunchCtx& c, const SvdPlan& p, float* ws, int64_t cols, float* Zt, float* tmp,
                      float** Q) {
  const int k = p.k;
  float *g = ws + p.g, *li = ws + p.li, *lit = ws + p.lit, *part = ws + p.part;
  cudaError_t e = cudaSuccess;
  for (int pass = 0; pass < 3 && e == cudaSuccess; ++pass) {
    e = gemm<float, float, false, false>(c, Zt, Zt, k, k, cols, g, part);  // G = Zt Zt^T
    if (e == cudaSuccess)
      e = launch_pdl(chol_inv_kernel, dim3(1), dim3(256), small_smem(k), c.stream, 1, (const float*)g, k,
                     pass == 0 ? cols : (int64_t)0, li, lit);
    if (e == cudaSuccess) e = gemm<float, float, true, true>(c, lit, Zt, k, cols, k, tmp, part);  // L^-1 Zt
    float* x = Zt;
    Zt = tmp;
    tmp = x;
  }
  *Q = Zt;
  return e;
}

template <typename T>
cudaError_t run_svd(const LaunchCtx& c, const T* R, int64_t O, int64_t I, int r, int k, int power_iters,
                    const float* omega, T* U, T* V, float* ws) {
  const SvdPlan p = plan_svd(O, I, k, r);
  cudaError_t e = small_kernels_ready(c.device);
  if (e != cudaSuccess) return e;
  float* part = ws + p.part;
  float *Y = ws + p.y0, *Ytmp = ws + p.y1, *Zt = ws + p.z0, *Ztmp = ws + p.z1, *Bm = ws + p.bm;
  float* Q;
  // The products that stream R: on tensor cores for a bf16 R whose rows TMA
  // can address (16-byte aligned, I a multiple of 8), else CUDA-core tiles.
  bool mma = false;
  if constexpr (sizeof(T) == 2) mma = I % 8 == 0 && (reinterpret_cast<uintptr_t>(R) & 15u) == 0;
  auto r_times = [&](const float* F, float* out) -> cudaError_t {  // out [O, k] = R . F^T
    if constexpr (sizeof(T) == 2)
      if (mma) return product_mma(c, p, ws, true, R, F, out);
    return gemm<T, float, false, false>(c, R, F, O, k, I, out, part);
  };
  auto qt_times_r = [&](const float* Qm, float* out) -> cudaError_t {  // out [k, I] = Q^T . R
    if constexpr (sizeof(T) == 2)
      if (mma) return product_mma(c, p, ws, false, R, Qm, out);
    return gemm<float, T, true, true>(c, Qm, R, k, I, O, out, part);
  };
  // range sample and its orthonormal basis
  if ((e = r_times(omega, Y))) return e;  // Y = R Omega^T
  if ((e = orth_cols(c, p, ws, O, Y, Ytmp, &Q))) return e;
  for (int it = 0; it < power_iters; ++it) {
    float* Qz;
    if ((e = qt_times_r(Q, Zt))) return e;  // Zt = Q^T R
    if ((e = orth_rows(c, p, ws, I, Zt, Ztmp, &Qz))) return e;
    float* Ynext = (Q == Y) ? Ytmp : Y;
    if ((e = r_times(Qz, Ynext))) return e;  // Y = R Z
    float* other = (Ynext == Y) ? Ytmp : Y;
    if ((e = orth_cols(c, p, ws, O, Ynext, other, &Q))) return e;
  }
  // projection, its small SVD through B B^T, and the lift
  if ((e = qt_times_r(Q, Bm))) return e;  // B = Q^T R
  if ((e = gemm<float, float, false, false>(c, Bm, Bm, k, k, I, ws + p.s, part))) return e;  // B B^T
  if ((e = launch_pdl(jacobi_eig_kernel, dim3(1), dim3(256), small_smem(k), c.stream, 1, (const float*)(ws + p.s), k,
                      r, ws + p.e, ws + p.et)))
    return e;
  if ((e = gemm<float, float, false, false>(c, Q, ws + p.et, O, r, k, ws + p.uraw, part))) return e;  // Q E_r
  if ((e = gemm<float, float, true, true>(c, Bm, ws + p.e, I, r, k, ws + p.vun, part))) return e;    // B^T E_r
  if ((e = launch_pdl(col_norm_kernel, dim3((unsigned)r), dim3(256), 0, c.stream, 1, (const float*)(ws + p.vun), I, r,
                      ws + p.sig)))
    return e;
  const auto blocks = [&](int64_t n) {
    int64_t b = ceil_div(n, 256);
    return (unsigned)(b > 8 * (int64_t)c.num_sms ? 8 * (int64_t)c.num_sms : b);
  };
  if ((e = launch_pdl(scale_cols_kernel<T>, dim3(blocks(O * r)), dim3(256), 0, c.stream, 1, (const float*)(ws + p.uraw),
                      (const float*)(ws + p.sig), O, r, 1, U)))
    return e;
  return launch_pdl(scale_cols_kernel<T>, dim3(blocks(I * r)), dim3(256), 0, c.stream, 1, (const float*)(ws + p.vun),
                    (const float*)(ws + p.sig), I, r, 0, V);
}

}  // namespace

int svd_max_samples() { return kMaxSamples; }

size_t svd_workspace_bytes(int64_t O, int64_t I, int samples, int rank) {
  return (size_t)plan_svd(O, I, samples, rank).total * sizeof(float);
}

cudaError_t launch_residual_svd(const LaunchCtx& c, theta_dtype dt, const void* R, int64_t O, int64_t I, int rank,
                                int samples, int power_iters, const float* omega, void* U, void* V, void* ws) {
  if (dt == THETA_BF16)
    return run_svd<bf16>(c, static_cast<const bf16*>(R), O, I, rank, samples, power_iters, omega,
                         static_cast<bf16*>(U), static_cast<bf16*>(V), static_cast<float*>(ws));
  return run_svd<float>(c, static_cast<const float*>(R), O, I, rank, samples, power_iters, omega,
                        static_cast<float*>(U), static_cast<float*>(V), static_cast<float*>(ws));
}

}  // namespace theta
