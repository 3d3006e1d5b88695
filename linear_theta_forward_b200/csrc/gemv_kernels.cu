// The theta forward for one or two tokens ("The theta bundle" --
// approximation formula, applied without forming the weight):
//   Y[m, o] = s[o] * (X[m, :] . W0[o, :]) + T[m, :] . U[o, :],   T = X . V
//
// With a few tokens the projection streams W0 once and does a few flops per
// byte: the bound is HBM. Each CTA owns a contiguous range of 8 * rpw rows of
// W0 and each of its warps every eighth row of it, so at any moment a CTA
// reads eight consecutive rows -- one compact window of memory that moves
// front to back, the access pattern that sustains the most read bandwidth
// (tile kernels instead walk 128-row column strips). A lane keeps UNR
// 16-byte loads of its row in flight; X (a few KB, shared by every CTA)
// comes through L1. All CTAs are resident at once and every warp has the
// same number of rows, so they finish together.
//
// T = X.V comes first, from a small CUDA-core kernel: kXvParts CTAs each sum
// X . V over one slice of I and write fp32 partial sums (no tensor memory,
// no cluster, so it lets the next grid launch at once). The sweep follows it
// with programmatic dependent launch and starts streaming W0 immediately:
// that kernel waited for all earlier work before letting this grid launch,
// so W0, X and s are complete. Only the rank-r phase at the end waits; it adds
// the partial sums of T in a fixed order. The partial sums, U and s are
// reached through pointers passed through after_wait(), so the compiler
// cannot schedule their loads above the wait.
#include "common.cuh"
#include "internal.h"

namespace theta {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTokens = 2;  // from 3 tokens on, the tensor-core tile path is faster
// Above this many W0 elements the tile path wins too: in a stream of calls
// it overlaps one call's tail with the next call's loads and sustains more
// bandwidth; the sweep pays off where a call is short and its start-up
// latency dominates.
constexpr int64_t kMaxElements = (int64_t)32 << 20;
constexpr int kMaxRank = 256;
constexpr int kMaxRowsPerWarp = 64;
constexpr int kUnroll = 4;  // 16-byte loads in flight per lane
constexpr int kXvParts = 16;  // slices of I in the T = X.V partial sums

struct GemvArgs {
  const bf16* X;
  const bf16* W0;
  const float* s;
  const bf16* U;
  const float* t_parts;  // [kXvParts][M][r] partial sums of T = X.V
  bf16* Y;
  int64_t O, I;
  int r;
  int early;  // launched right after this call's T = X.V kernel
  int rpw;    // rows per warp; a CTA owns 8 * rpw consecutive rows
};

// parts[p][m][j] = sum over i in slice p of I of X[m, i] V[i, j]. A thread
// owns 8 consecutive columns of V (one 16-byte load per row of V) and every
// nslices-th row of the slice, four rows in flight; the row slices are then
// combined in a fixed order. r is a multiple of 8 and at most 256.
template <int M>
__global__ void __launch_bounds__(kThreads)
xv_parts_kernel(const bf16* __restrict__ X, const bf16* __restrict__ V, int64_t I, int r, float* __restrict__ parts) {
  constexpr int kRowsInFlight = 4;
  __shared__ float red[kThreads * 8 * M];  // [slice][m][column]
  pdl_enter(X, V);
  const int p = blockIdx.x;
  const int64_t i0 = (int64_t)p * I / kXvParts, i1 = (int64_t)(p + 1) * I / kXvParts;
  const int groups = r / 8;  // 16-byte column groups per row of V
  const int nslices = kThreads / groups;
  const int t = threadIdx.x, cg = t % groups, slice = t / groups;
  float acc[M][8];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[m][e] = 0.f;
  if (slice < nslices) {
    const uint4* v4 = reinterpret_cast<const uint4*>(V);
    for (int64_t i = i0 + slice; i < i1; i += (int64_t)kRowsInFlight * nslices) {
      uint4 vv[kRowsInFlight];
      float xv[kRowsInFlight][M];
#pragma unroll
      for (int u = 0; u < kRowsInFlight; ++u) {
        const int64_t ii = i + (int64_t)u * nslices;
        const bool in = ii < i1;
        vv[u] = in ? v4[ii * groups + cg] : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int m = 0; m < M; ++m) xv[u][m] = in ? __bfloat162float(X[m * I + ii]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kRowsInFlight; ++u) {
        float f[8];
        unpack(vv[u], f);
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[m][e] = fmaf(xv[u][m], f[e], acc[m][e]);
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int e = 0; e < 8; ++e) red[(slice * M + m) * r + cg * 8 + e] = acc[m][e];
  }
  __syncthreads();
  for (int q = t; q < M * r; q += kThreads) {
    float sum = 0.f;
    for (int sl = 0; sl < nslices; ++sl) sum += red[sl * M * r + q];
    parts[(int64_t)p * M * r + q] = sum;  // q = m * r + j
  }
}

// Packed fp32 pairs (Blackwell fma.rn.f32x2: two fp32 FMAs per instruction).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void fma_f32x2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

__device__ __forceinline__ float sum_f32x2(uint64_t p) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
  return lo + hi;
}

// 8 bf16 -> 4 fp32 pairs (a bf16 is the high half of its fp32 value)
__device__ __forceinline__ void bf16x8_to_f32x2(const uint4& v, uint64_t (&p)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) p[q] = f32x2(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xffff0000u));
}

template <int M>
__global__ void __launch_bounds__(kThreads) gemv_rows_kernel(const __grid_constant__ GemvArgs a) {
  __shared__ float dots[kWarps][kMaxRowsPerWarp][M];
  __shared__ float tsh[M][kMaxRank];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const bf16* X = a.X;
  const bf16* W0 = a.W0;
  const float* s = a.s;
  const bf16* U = a.U;
  if (!a.early) {
    pdl_wait();
    after_wait(X), after_wait(W0), after_wait(s), after_wait(U);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int64_t I = a.I, nv = I / 8;
  const int64_t row_lo = (int64_t)blockIdx.x * kWarps * a.rpw;
  const uint4* x = reinterpret_cast<const uint4*>(X);
  for (int k = 0; k < a.rpw; ++k) {
    const int64_t o = row_lo + warp + (int64_t)k * kWarps;
    if (o >= a.O) break;
    const uint4* w = reinterpret_cast<const uint4*>(W0 + o * I);
    uint64_t acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0;
    for (int64_t v0 = lane; v0 < nv; v0 += 32 * kUnroll) {
      uint4 wv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t v = v0 + 32 * u;
        wv[u] = v < nv ? __ldcs(w + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t v = v0 + 32 * u;
        if (v >= nv) break;
        uint64_t pw[4];
        bf16x8_to_f32x2(wv[u], pw);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          uint64_t px[4];
          bf16x8_to_f32x2(__ldg(x + m * nv + v), px);
#pragma unroll
          for (int q = 0; q < 4; ++q) fma_f32x2(acc[m], pw[q], px[q]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float d = warp_sum(sum_f32x2(acc[m]));
      if (lane == 0) dots[warp][k][m] = d;
    }
  }

  // ---------------------------------------------------------- rank-r phase
  const float* parts = a.t_parts;
  if (a.early) pdl_wait();  // T's partial sums are complete from here on
  after_wait(parts), after_wait(U), after_wait(s);
  const int r = a.r;
  for (int i = threadIdx.x; i < M * r; i += kThreads) {
    float t = 0.f;
    for (int p = 0; p < kXvParts; ++p) t += parts[(int64_t)p * M * r + i];
    tsh[i / r][i % r] = t;
  }
  __syncthreads();
  for (int k = 0; k < a.rpw; ++k) {
    const int64_t o = row_lo + warp + (int64_t)k * kWarps;
    if (o >= a.O) break;
    float rk[M];
#pragma unroll
    for (int m = 0; m < M; ++m) rk[m] = 0.f;
    for (int j = lane; j < r; j += 32) {
      const float u = __bfloat162float(U[o * r + j]);
#pragma unroll
      for (int m = 0; m < M; ++m) rk[m] = fmaf(u, tsh[m][j], rk[m]);
    }
#pragma unroll
    for (int m = 0; m < M; ++m) rk[m] = warp_sum(rk[m]);
    if (lane < M) {
      float y = 0.f;
#pragma unroll
      for (int m = 0; m < M; ++m)
        if (m == lane) y = fmaf(__ldg(s + o), dots[warp][k][m], rk[m]);
      a.Y[(int64_t)lane * a.O + o] = __float2bfloat16_rn(y);
    }
  }
}

// CTAs of this kernel one SM holds at once (registers and threads decide).
template <int M>
int resident_ctas(int device) {
  static int cached[64] = {};
  if (!cached[device]) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_rows_kernel<M>, kThreads, 0) != cudaSuccess || n < 1)
      n = 1;
    cached[device] = n;
  }
  return cached[device];
}

template <int M>
cudaError_t launch_m(const LaunchCtx& c, GemvArgs a, const void* V) {
  if (a.r > 0) {
    cudaError_t e = launch_pdl(xv_parts_kernel<M>, dim3(kXvParts), dim3(kThreads), 0, c.stream, 1, a.X,
                               static_cast<const bf16*>(V), a.I, a.r, const_cast<float*>(a.t_parts));
    if (e != cudaSuccess) return e;
  }
  // the fewest rows per warp that keep every CTA resident in one wave
  const int64_t capacity = (int64_t)c.num_sms * resident_ctas<M>(c.device) * kWarps;
  a.rpw = (int)ceil_div(a.O, capacity);
  const int64_t grid = ceil_div(a.O, (int64_t)kWarps * a.rpw);
  return launch_pdl(gemv_rows_kernel<M>, dim3((unsigned)grid), dim3(kThreads), 0, c.stream, 1, a);
}

}  // namespace

int forward_gemv_max_tokens() { return kMaxTokens; }

size_t forward_gemv_workspace_bytes(int64_t M, int r) {
  return (M >= 1 && M <= kMaxTokens && r > 0) ? (size_t)kXvParts * M * r * sizeof(float) : 0;
}

bool launch_forward_gemv(const LaunchCtx& c, const void* X, const void* W0, const float* s, const void* U,
                         const void* V, int64_t M, int64_t O, int64_t I, int r, void* Y, void* ws,
                         cudaError_t* e) {
  *e = cudaSuccess;
  if (M < 1 || M > kMaxTokens || r > kMaxRank || I % 8 || I < kXvParts || O * I > kMaxElements) return false;
  // rows per warp grow with O beyond what the GPU holds at once
  if (ceil_div(O, (int64_t)c.num_sms * kWarps) > kMaxRowsPerWarp) return false;
  if ((reinterpret_cast<uintptr_t>(W0) & 15u) != 0 || (reinterpret_cast<uintptr_t>(X) & 15u) != 0) return false;
  GemvArgs a = {};
  a.X = static_cast<const bf16*>(X);
  a.W0 = static_cast<const bf16*>(W0);
  a.s = s;
  a.U = static_cast<const bf16*>(U);
  a.t_parts = static_cast<const float*>(ws);
  a.Y = static_cast<bf16*>(Y);
  a.O = O;
  a.I = I;
  a.r = r;
  a.early = r > 0 ? 1 : 0;
  *e = M == 1 ? launch_m<1>(c, a, V) : launch_m<2>(c, a, V);
  return true;
}

}  // namespace theta
