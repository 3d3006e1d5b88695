// The theta forward for one or two tokens ("The theta bundle" --
// approximation formula, applied without forming the weight):
//   Y[m, o] = s[o] * (X[m, :] . W0[o, :]) + T[m, :] . U[o, :],   T = X . V
//
// With a few tokens the projection streams W0 once and does a few flops per
// byte: the bound is HBM. Each CTA owns a contiguous range of 8 * rpw rows of
// W0 and each of its warps every eighth row of it, so at any moment a CTA
// reads eight consecutive rows -- one compact window of memory that moves
// front to back, the access pattern that sustains the most read bandwidth
// (tile kernels instead walk 128-row column strips). A lane keeps kUnroll
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
//
// The same sweep also reads the shared block in NVFP4 (codes, E4M3 block
// scales, fp32 tensor scale; the format the pages weigh in "Quality" -- what
// NVFP4 quantization costs): 0.5625 bytes per weight instead of 2. Its rows
// are split evenly over one full wave of CTAs, each warp taking a
// contiguous range; see the FP4 branch of gemv_rows_kernel. The encoder
// (nvfp4_amax_kernel, nvfp4_quant_kernel) sits at the end.
//
// The grouped kernels (grouped_*_kernel) run many such forwards -- every
// family of every layer of a decode step -- as one sweep over all their rows.
#include <cuda_fp16.h>

#include <algorithm>

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
constexpr int kUnrollFp4 = 4;  // NVFP4: rows a warp takes at a time, one 16-byte load each
constexpr int kXvParts = 16;  // slices of I in the T = X.V partial sums
// With NVFP4 the sweep is 3.56x shorter, so T = X.V must finish sooner:
// more, smaller slices.
constexpr int kXvPartsFp4 = 64;

struct GemvArgs {
  const bf16* X;
  const bf16* W0;
  const float* s;
  const bf16* U;
  const float* t_parts;  // [nparts][M][r] partial sums of T = X.V
  const uint8_t* codes;   // NVFP4 W0: E2M1 pairs [O, I/2], element 2j in the low nibble
  const uint8_t* scales;  // NVFP4 W0: E4M3 block scales [O, I/16]
  const float* g;         // NVFP4 W0: the tensor scale (device scalar)
  int nparts;             // slices of I in the T = X.V partial sums
  bf16* Y;
  int64_t O, I;
  int r;
  int early;  // launched right after this call's T = X.V kernel
  int rpw;    // rows per warp; a CTA owns 8 * rpw consecutive rows
};

// out[m * r + j] = sum over i in [i0, i1) of X[m, i] V[i, j], by one CTA. A
// thread owns 8 consecutive columns of V (one 16-byte load per row of V) and
// every nslices-th row of the range, four rows in flight; the row slices are
// then combined in a fixed order through shared memory. r is a multiple of 8
// and at most 256.
template <int M>
__device__ __forceinline__ void xv_slice(const bf16* __restrict__ X, const bf16* __restrict__ V, int64_t I, int r,
                                         int64_t i0, int64_t i1, float* red, float* __restrict__ out) {
  constexpr int kRowsInFlight = 4;
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
    out[q] = sum;  // q = m * r + j
  }
}

// parts[p][m][j]: the sum over slice p (of gridDim.x) of I.
template <int M>
__global__ void __launch_bounds__(kThreads)
xv_parts_kernel(const bf16* __restrict__ X, const bf16* __restrict__ V, int64_t I, int r, float* __restrict__ parts) {
  __shared__ float red[kThreads * 8 * M];  // [slice][m][column]
  pdl_enter(X, V);
  const int p = blockIdx.x;
  const int64_t i0 = (int64_t)p * I / gridDim.x, i1 = (int64_t)(p + 1) * I / gridDim.x;
  xv_slice<M>(X, V, I, r, i0, i1, red, parts + (int64_t)p * M * r);
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

// Two E2M1 codes (one byte, element 2j in the low nibble) -> two floats,
// and two E4M3 codes (low byte first) -> two floats, by the Blackwell
// conversions to f16x2; every E2M1 and E4M3 value is exact in fp16.
// A word of 8 E2M1 codes (element 2j in the low nibble of byte j) as four
// f16x2: h[q] holds elements 2q (low half) and 2q + 1.
__device__ __forceinline__ void e2m1x8_to_h2(uint32_t w, uint32_t (&h)[4]) {
  asm("{.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two_bytes) {
  uint32_t h;
  asm("{.reg .b16 u; cvt.u16.u32 u, %1; cvt.rn.f16x2.e4m3x2 %0, u;}" : "=r"(h) : "r"(two_bytes));
  return __half22float2(*reinterpret_cast<__half2*>(&h));
}

// 8 bf16 -> 4 fp32 pairs (a bf16 is the high half of its fp32 value)
__device__ __forceinline__ void bf16x8_to_f32x2(const uint4& v, uint64_t (&p)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) p[q] = f32x2(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xffff0000u));
}

template <int M, bool FP4>
__global__ void __launch_bounds__(kThreads) gemv_rows_kernel(const __grid_constant__ GemvArgs a) {
  __shared__ float dots[kWarps][kMaxRowsPerWarp][M];
  __shared__ float tsh[M][kMaxRank];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const bf16* X = a.X;
  const bf16* W0 = a.W0;
  const float* s = a.s;
  const bf16* U = a.U;
  const uint8_t* codes = a.codes;
  const uint8_t* scales = a.scales;
  const float* gp = a.g;
  if (!a.early) {
    pdl_wait();
    after_wait(X), after_wait(W0), after_wait(s), after_wait(U), after_wait(codes), after_wait(scales), after_wait(gp);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int64_t I = a.I, nv = I / 8;
  const int64_t row_lo = (int64_t)blockIdx.x * kWarps * a.rpw;
  const uint4* x = reinterpret_cast<const uint4*>(X);
  // The rows this warp owns: o = rbase + k * rstride for k < nr.
  int64_t rbase, rstride;
  int nr;
  if constexpr (FP4) {
    // one wave of CTAs; each warp a contiguous, balanced range of rows
    const int64_t nw = (int64_t)gridDim.x * kWarps, gw = (int64_t)blockIdx.x * kWarps + warp;
    rbase = gw * a.O / nw;
    rstride = 1;
    nr = (int)((gw + 1) * a.O / nw - rbase);
  } else {
    rbase = row_lo + warp;
    rstride = kWarps;
    nr = rbase < a.O ? (int)min((int64_t)a.rpw, ceil_div(a.O - rbase, kWarps)) : 0;
  }
  if constexpr (FP4) {
    // NVFP4 W0: a lane takes 16-byte chunks of codes (32 weights, two scale
    // blocks) and the two scale bytes beside them. Two weights widen to an
    // f16x2 in one conversion and meet X in fp16, scaled by a power of two
    // per group of 1024 values so that |x| <= 2^9 (a block's 16 products, at
    // most 6 * 2^9 each, then sum far below fp16's limit); a block is summed
    // by packed fp16 FMAs, each rounding once, and added in fp32 after its
    // E4M3 scale and the group's power of two.
    //
    // First the CTA writes X so converted into shared memory: each warp
    // takes groups (32 chunks, one per lane), reduces the group's largest
    // |x| and stores lane l's 32 values at 16-byte slots
    // group * 128 + h * 32 + l, h = 0..3 (conflict-free on both sides).
    // Then a row has only I/32 chunks, a few per lane, so the warp takes its
    // rows kUnrollFp4 at a time and walks them group by group: the group's X
    // comes from shared memory once for every row of the batch, and the
    // batch's code loads are all in flight together.
    extern __shared__ uint4 xsm[];  // [M][cj][128] fp16 X, then float gsc[M][cj]
    const int nch = (int)(I / 32);  // chunks of a row
    const int cj = (nch + 31) / 32;  // groups of a row
    float* gsc = reinterpret_cast<float*>(xsm + (size_t)M * cj * 128);
    for (int it = warp; it < M * cj; it += kWarps) {
      const int m = it / cj, v = 32 * (it - m * cj) + lane;
      float f[4][8];
      float mx = 0.f;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint4 raw = v < nch ? __ldg(x + (int64_t)m * nv + 4 * v + h) : make_uint4(0, 0, 0, 0);
        unpack(raw, f[h]);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[h][e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      int k = 0;
      if (mx > 0.f) frexpf(mx, &k);  // mx <= 2^k
      const int e = max(-120, min(120, k - 9));  // 2^e >= mx / 2^9, both 2^e and 2^-e finite
      const float inv = ldexpf(1.0f, -e);  // exact scaling
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          __half2 hv = __floats2half2_rn(f[h][2 * q] * inv, f[h][2 * q + 1] * inv);
          w[q] = *reinterpret_cast<uint32_t*>(&hv);
        }
        xsm[it * 128 + 32 * h + lane] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (lane == 0) gsc[it] = ldexpf(1.0f, e);
    }
    __syncthreads();

    const float gval = __ldg(gp);
    const int64_t first = rbase;
    const int nrows = nr;
    const int64_t cstep = (int64_t)nch * rstride;  // chunks from one of the warp's rows to the next
    for (int k0 = 0; k0 < nrows; k0 += kUnrollFp4) {
      const uint4* cb = reinterpret_cast<const uint4*>(codes + (first + (int64_t)k0 * rstride) * (I / 2)) + lane;
      const unsigned short* sb =
          reinterpret_cast<const unsigned short*>(scales + (first + (int64_t)k0 * rstride) * (I / 16)) + lane;
      float acc[kUnrollFp4][M];
#pragma unroll
      for (int u = 0; u < kUnrollFp4; ++u)
#pragma unroll
        for (int m = 0; m < M; ++m) acc[u][m] = 0.f;
      for (int G = 0; G < cj; ++G) {
        const bool vok = lane + 32 * G < nch;
        uint4 cv[kUnrollFp4];
        uint32_t sv[kUnrollFp4];
#pragma unroll
        for (int u = 0; u < kUnrollFp4; ++u) {
          const bool ok = vok && k0 + u < nrows;
          cv[u] = ok ? __ldcs(cb + u * cstep + 32 * G) : make_uint4(0, 0, 0, 0);
          sv[u] = ok ? (uint32_t)__ldcs(sb + u * cstep + 32 * G) : 0u;
        }
        if (vok) {
          uint4 xq[M][4];  // this lane's 32 values of X in the group
          float gs[M];
#pragma unroll
          for (int m = 0; m < M; ++m) {
#pragma unroll
            for (int h = 0; h < 4; ++h) xq[m][h] = xsm[(m * cj + G) * 128 + 32 * h + lane];
            gs[m] = gsc[m * cj + G];
          }
#pragma unroll
          for (int u = 0; u < kUnrollFp4; ++u) {
            if (k0 + u >= nrows) break;
            const float2 sc = e4m3x2_to_f32(sv[u]);
            const uint32_t wd[4] = {cv[u].x, cv[u].y, cv[u].z, cv[u].w};
#pragma unroll
            for (int m = 0; m < M; ++m) {
#pragma unroll
              for (int b = 0; b < 2; ++b) {
                __half2 p = __float2half2_rn(0.f);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const uint4 xv = xq[m][2 * b + h];
                  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                  uint32_t wh[4];
                  e2m1x8_to_h2(wd[2 * b + h], wh);
#pragma unroll
                  for (int q = 0; q < 4; ++q)
                    p = __hfma2(*reinterpret_cast<const __half2*>(&wh[q]), *reinterpret_cast<const __half2*>(&xw[q]), p);
                }
                const float2 pf = __half22float2(p);
                acc[u][m] = fmaf(pf.x + pf.y, (b == 0 ? sc.x : sc.y) * gs[m], acc[u][m]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnrollFp4; ++u) {
        if (k0 + u >= nrows) break;
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float d = warp_sum(acc[u][m]) * gval;
          if (lane == 0) dots[warp][k0 + u][m] = d;
        }
      }
    }
  }
  for (int k = 0; k < (FP4 ? 0 : a.rpw); ++k) {
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
    for (int p = 0; p < a.nparts; ++p) t += parts[(int64_t)p * M * r + i];
    tsh[i / r][i % r] = t;
  }
  __syncthreads();
  for (int k = 0; k < nr; ++k) {
    const int64_t o = rbase + (int64_t)k * rstride;
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

// ------------------------------------------------------- grouped decode
// Many independent forwards of one or two tokens in one call (every family
// of every layer, say): three launches instead of two per problem. T = X.V
// for all problems first (kGroupParts slices of I each, then a fixed-order
// sum), then one sweep over the rows of all problems laid end to end, split
// over one wave of CTAs by weight elements (equal bytes per warp, whatever
// the row widths); a warp owns a contiguous range of those rows and takes
// them kGroupRows at a time (dot products, rank terms, Y).
constexpr int kGroupParts = 8;
constexpr int kGroupRows = 2;    // rows of one problem a warp takes at a time
constexpr int kGroupUnroll = 4;  // 16-byte loads per row in flight per lane
constexpr int kMaxGroup = THETA_MAX_GROUP;

struct GroupArgs {
  const theta_forward_problem* P;  // device copy of the problem table
  const float* T;                   // [count][M][rmax]: T = X.V, entry m * r + j
  int64_t elems[kMaxGroup + 1];     // first weight element of each problem (rows end to end)
  int32_t prefix[kMaxGroup + 1];    // first row of each problem; prefix[count] = all rows
  int count;
  int rmax;
};
static_assert(sizeof(GroupArgs) <= 4096, "kernel parameter space");

// The first row (in the rows of all problems end to end) that starts at or
// after weight element e: rows split at element boundaries, so warps given
// equal element ranges stream equal bytes whatever each problem's width.
__device__ __forceinline__ int64_t group_row_at(const GroupArgs& g, int64_t e) {
  if (e >= g.elems[g.count]) return g.prefix[g.count];
  int p = 0;  // the last problem with elems[p] <= e
  for (int lo = 0, hi = g.count - 1; lo < hi;) {
    const int mid = (lo + hi + 1) / 2;
    if (g.elems[mid] <= e) lo = mid; else hi = mid - 1;
    p = lo;
  }
  const int64_t rows = g.prefix[p + 1] - g.prefix[p];
  const int64_t width = (g.elems[p + 1] - g.elems[p]) / rows;
  return g.prefix[p] + min(rows, ceil_div(e - g.elems[p], width));
}

template <int M>
__global__ void __launch_bounds__(kThreads)
grouped_xv_kernel(const theta_forward_problem* __restrict__ P, int rmax, float* __restrict__ parts) {
  __shared__ float red[kThreads * 8 * M];
  pdl_enter(P);
  const theta_forward_problem d = P[blockIdx.y];
  const int r = (int)d.rank;
  if (r == 0) return;
  const int p = blockIdx.x;
  const int64_t i0 = (int64_t)p * d.I / kGroupParts, i1 = (int64_t)(p + 1) * d.I / kGroupParts;
  xv_slice<M>(static_cast<const bf16*>(d.X), static_cast<const bf16*>(d.V), d.I, r, i0, i1, red,
              parts + ((int64_t)blockIdx.y * kGroupParts + p) * M * rmax);
}

template <int M>
__global__ void __launch_bounds__(kThreads)
grouped_t_kernel(const theta_forward_problem* __restrict__ P, int rmax, const float* __restrict__ parts,
                 float* __restrict__ T) {
  pdl_enter(P, parts);
  const int b = blockIdx.x;
  const int r = (int)P[b].rank;
  for (int q = threadIdx.x; q < M * r; q += kThreads) {
    float t = 0.f;
    for (int p = 0; p < kGroupParts; ++p) t += parts[((int64_t)b * kGroupParts + p) * M * rmax + q];
    T[(int64_t)b * M * rmax + q] = t;
  }
}

template <int M>
__global__ void __launch_bounds__(kThreads) grouped_rows_kernel(const __grid_constant__ GroupArgs g) {
  const theta_forward_problem* P = g.P;
  const float* T = g.T;
  pdl_enter(P, T);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int64_t total = g.elems[g.count];
  const int64_t nw = (int64_t)gridDim.x * kWarps, gw = (int64_t)blockIdx.x * kWarps + warp;
  const int64_t r0 = group_row_at(g, gw * total / nw), r1 = group_row_at(g, (gw + 1) * total / nw);
  if (r0 >= r1) return;
  int p = 0;  // the problem holding row r0: the last p with prefix[p] <= r0
  for (int lo = 0, hi = g.count - 1; lo < hi;) {
    const int mid = (lo + hi + 1) / 2;
    if (g.prefix[mid] <= r0) lo = mid; else hi = mid - 1;
    p = lo;
  }
  theta_forward_problem d = P[p];
  // batches of up to kGroupRows consecutive rows of one problem: their W0
  // chunks are in flight together and share each load of X
  for (int64_t row = r0; row < r1;) {
    if (row >= g.prefix[p + 1]) {
      while (row >= g.prefix[p + 1]) ++p;
      d = P[p];
    }
    const int64_t o0 = row - g.prefix[p], I = d.I, nv = I / 8;
    const int nb = (int)min((int64_t)kGroupRows, min(r1, (int64_t)g.prefix[p + 1]) - row);
    const uint4* w = reinterpret_cast<const uint4*>(static_cast<const bf16*>(d.W0) + o0 * I);
    const uint4* x = reinterpret_cast<const uint4*>(d.X);
    const int r = (int)d.rank;
    const bf16* U = static_cast<const bf16*>(d.U);
    const float* Tp = T + (int64_t)p * M * g.rmax;
    // the rank term and the row scales first: their loads overlap the sweep's
    float y[kGroupRows][M], sv[kGroupRows];
#pragma unroll
    for (int k = 0; k < kGroupRows; ++k) {
      sv[k] = k < nb ? __ldg(d.s + o0 + k) : 0.f;
#pragma unroll
      for (int m = 0; m < M; ++m) y[k][m] = 0.f;
    }
    for (int j = lane; j < r; j += 32) {
      float t[M];
#pragma unroll
      for (int m = 0; m < M; ++m) t[m] = Tp[m * r + j];
#pragma unroll
      for (int k = 0; k < kGroupRows; ++k) {
        if (k >= nb) break;
        const float u = __bfloat162float(U[(o0 + k) * r + j]);
#pragma unroll
        for (int m = 0; m < M; ++m) y[k][m] = fmaf(u, t[m], y[k][m]);
      }
    }
    uint64_t acc[kGroupRows][M];
#pragma unroll
    for (int k = 0; k < kGroupRows; ++k)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[k][m] = 0;
    for (int64_t v0 = lane; v0 < nv; v0 += 32 * kGroupUnroll) {
      uint4 wv[kGroupUnroll][kGroupRows];
#pragma unroll
      for (int u = 0; u < kGroupUnroll; ++u) {
        const int64_t v = v0 + 32 * u;
#pragma unroll
        for (int k = 0; k < kGroupRows; ++k)
          wv[u][k] = (v < nv && k < nb) ? __ldcs(w + k * nv + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kGroupUnroll; ++u) {
        const int64_t v = v0 + 32 * u;
        if (v >= nv) break;
#pragma unroll
        for (int m = 0; m < M; ++m) {
          uint64_t px[4];
          bf16x8_to_f32x2(__ldg(x + m * nv + v), px);
#pragma unroll
          for (int k = 0; k < kGroupRows; ++k) {
            uint64_t pw[4];
            bf16x8_to_f32x2(wv[u][k], pw);
#pragma unroll
            for (int q = 0; q < 4; ++q) fma_f32x2(acc[k][m], pw[q], px[q]);
          }
        }
      }
    }
    // Y = s * dot + rank term, one warp reduction per row and token
#pragma unroll
    for (int k = 0; k < kGroupRows; ++k) {
      if (k >= nb) break;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const float yk = warp_sum(fmaf(sv[k], sum_f32x2(acc[k][m]), y[k][m]));
        if (lane == m) static_cast<bf16*>(d.Y)[m * d.O + o0 + k] = __float2bfloat16_rn(yk);
      }
    }
    row += nb;
  }
}

// Dynamic shared memory of the NVFP4 sweep: X in fp16 and its group scales.
constexpr size_t kFp4SmemMax = 200 << 10;
size_t fp4_smem_bytes(int64_t M, int64_t I) {
  const int64_t groups = M * ceil_div(I / 32, 32);
  return (size_t)groups * 2048 + (size_t)ceil_div(groups * 4, 16) * 16;
}

// CTAs of this kernel one SM holds at once with `smem` bytes of dynamic
// shared memory (registers, threads and shared memory decide).
template <int M, bool FP4>
int resident_ctas(int device, size_t smem) {
  std::lock_guard<std::mutex> lk(setup_mutex());
  static int cached[64] = {};
  static size_t cached_smem[64] = {};
  if (!cached[device] || cached_smem[device] != smem) {
    if (FP4) {
      static bool opted[64] = {};
      if (!opted[device]) {
        cudaFuncSetAttribute(gemv_rows_kernel<M, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFp4SmemMax);
        opted[device] = true;
      }
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_rows_kernel<M, FP4>, kThreads, smem) != cudaSuccess ||
        n < 1)
      n = 1;
    cached[device] = n;
    cached_smem[device] = smem;
  }
  return cached[device];
}

template <int M, bool FP4 = false>
cudaError_t launch_m(const LaunchCtx& c, GemvArgs a, const void* V) {
  if (a.r > 0) {
    cudaError_t e = launch_pdl(xv_parts_kernel<M>, dim3((unsigned)a.nparts), dim3(kThreads), 0, c.stream, 1, a.X,
                               static_cast<const bf16*>(V), a.I, a.r, const_cast<float*>(a.t_parts));
    if (e != cudaSuccess) return e;
  }
  const size_t smem = FP4 ? fp4_smem_bytes(M, a.I) : 0;
  // the fewest rows per warp that keep every CTA resident in one wave
  const int64_t capacity = (int64_t)c.num_sms * resident_ctas<M, FP4>(c.device, smem) * kWarps;
  a.rpw = (int)ceil_div(a.O, capacity);
  // NVFP4 splits the rows evenly over one full wave; bf16 gives every warp rpw
  const int64_t grid = FP4 ? std::min(capacity / kWarps, ceil_div(a.O, (int64_t)kWarps))
                           : ceil_div(a.O, (int64_t)kWarps * a.rpw);
  return launch_pdl(gemv_rows_kernel<M, FP4>, dim3((unsigned)grid), dim3(kThreads), smem, c.stream, 1, a);
}

}  // namespace

int forward_gemv_max_tokens() { return kMaxTokens; }

size_t forward_gemv_workspace_bytes(int64_t M, int r) {
  return (M >= 1 && M <= kMaxTokens && r > 0) ? (size_t)kXvParts * M * r * sizeof(float) : 0;
}

size_t forward_grouped_workspace_bytes(int count, int64_t M, int rmax) {
  return rmax > 0 ? (size_t)count * M * rmax * sizeof(float) * (kGroupParts + 1) : 0;
}

bool launch_forward_grouped(const LaunchCtx& c, const theta_forward_problem* host, const theta_forward_problem* dev,
                            int count, int64_t M, int rmax, void* ws, cudaError_t* e) {
  *e = cudaSuccess;
  if (M < 1 || M > kMaxTokens || count < 1 || count > kMaxGroup || rmax > kMaxRank) return false;
  GroupArgs g = {};
  g.P = dev;
  g.count = count;
  g.rmax = rmax;
  g.prefix[0] = 0;
  g.elems[0] = 0;
  for (int i = 0; i < count; ++i) {
    if (g.prefix[i] + host[i].O > INT32_MAX) return false;
    g.prefix[i + 1] = (int32_t)(g.prefix[i] + host[i].O);
    g.elems[i + 1] = g.elems[i] + host[i].O * host[i].I;
  }
  float* parts = static_cast<float*>(ws);
  float* T = parts + (size_t)count * kGroupParts * M * rmax;
  g.T = T;
  if (rmax > 0) {
    *e = M == 1 ? launch_pdl(grouped_xv_kernel<1>, dim3(kGroupParts, (unsigned)count), dim3(kThreads), 0, c.stream, 1,
                             dev, rmax, parts)
                : launch_pdl(grouped_xv_kernel<2>, dim3(kGroupParts, (unsigned)count), dim3(kThreads), 0, c.stream, 1,
                             dev, rmax, parts);
    if (*e != cudaSuccess) return true;
    *e = M == 1 ? launch_pdl(grouped_t_kernel<1>, dim3((unsigned)count), dim3(kThreads), 0, c.stream, 1, dev, rmax,
                             (const float*)parts, T)
                : launch_pdl(grouped_t_kernel<2>, dim3((unsigned)count), dim3(kThreads), 0, c.stream, 1, dev, rmax,
                             (const float*)parts, T);
    if (*e != cudaSuccess) return true;
  }
  auto go = [&](auto kern) {
    static int cached[2][64] = {};
    int n = 0;
    {
      std::lock_guard<std::mutex> lk(setup_mutex());
      int& slot = cached[M - 1][c.device];
      if (!slot && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&slot, kern, kThreads, 0) != cudaSuccess ||
                    slot < 1))
        slot = 1;
      n = slot;
    }
    const int64_t grid = std::min((int64_t)c.num_sms * n, ceil_div((int64_t)g.prefix[count], (int64_t)kWarps));
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), 0, c.stream, 1, g);
  };
  *e = M == 1 ? go(grouped_rows_kernel<1>) : go(grouped_rows_kernel<2>);
  return true;
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
  a.nparts = kXvParts;
  a.Y = static_cast<bf16*>(Y);
  a.O = O;
  a.I = I;
  a.r = r;
  a.early = r > 0 ? 1 : 0;
  *e = M == 1 ? launch_m<1>(c, a, V) : launch_m<2>(c, a, V);
  return true;
}

}  // namespace theta

namespace theta {

namespace {

// ------------------------------------------------------------ NVFP4 encode
// max |w| over the tensor into *amax_bits (fp32 bits; for non-negative
// floats the integer order is the float order, so atomicMax is exact and
// the result independent of the order of the CTAs).
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const bf16* __restrict__ W, int64_t nvec,
                                                         unsigned* __restrict__ amax_bits) {
  pdl_enter(W);
  __shared__ float red[256 / 32];
  float mx = 0.f;
  const uint4* w4 = reinterpret_cast<const uint4*>(W);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    float f[8];
    unpack(__ldcs(w4 + v), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
    for (int i = 0; i < 256 / 32; ++i) b = fmaxf(b, red[i]);
    atomicMax(amax_bits, __float_as_uint(b));
  }
}

// One thread per block of 16 weights. Every decision in fp32 with
// round-to-nearest-even: g = amax / (6 * 448); block scale
// E4M3(blockmax / 6 / g) (saturating); element code E2M1(w * (1 / (E4M3 * g)))
// (saturating, a negative value that rounds to zero is stored as +0).
__global__ void __launch_bounds__(256) nvfp4_quant_kernel(const bf16* __restrict__ W, int64_t nblocks,
                                                          const unsigned* __restrict__ amax_bits,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                          float* __restrict__ g_out) {
  pdl_enter(W, amax_bits);
  const float g = __fdiv_rn(__uint_as_float(*amax_bits), 2688.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
  const uint4* w4 = reinterpret_cast<const uint4*>(W);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    float w[16];
    unpack(w4[2 * b], *reinterpret_cast<float(*)[8]>(w));
    unpack(w4[2 * b + 1], *reinterpret_cast<float(*)[8]>(w + 8));
    float bmax = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) bmax = fmaxf(bmax, fabsf(w[e]));
    const float ratio = g > 0.f ? __fdiv_rn(__fdiv_rn(bmax, 6.0f), g) : 0.f;
    uint16_t sq16;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(sq16) : "f"(0.f), "f"(ratio));
    const uint32_t sq = sq16 & 0xffu;
    const float scale = __fmul_rn(e4m3x2_to_f32(sq).x, g);
    const float inv = scale > 0.f ? __fdiv_rn(1.0f, scale) : 0.f;
    uint32_t word[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint16_t byte;
      asm("{.reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t;}"
          : "=h"(byte)
          : "f"(__fmul_rn(w[2 * j + 1], inv)), "f"(__fmul_rn(w[2 * j], inv)));
      uint32_t lo = byte & 15u, hi = (byte >> 4) & 15u;
      if ((lo & 7u) == 0) lo = 0;  // -0 -> +0
      if ((hi & 7u) == 0) hi = 0;
      word[j / 4] |= (lo | (hi << 4)) << (8 * (j % 4));
    }
    reinterpret_cast<uint2*>(codes)[b] = make_uint2(word[0], word[1]);
    scales[b] = (uint8_t)sq;
  }
}

}  // namespace

cudaError_t launch_nvfp4_quantize(const LaunchCtx& c, const void* W, int64_t O, int64_t I, void* codes, void* scales,
                                  float* g, void* ws) {
  unsigned* amax = static_cast<unsigned*>(ws);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), c.stream);
  if (e != cudaSuccess) return e;
  const int64_t nvec = O * I / 8, nblocks = O * I / 16;
  const auto grid = [&](int64_t n) {
    int64_t b = ceil_div(n, 256);
    return (unsigned)(b > 8 * (int64_t)c.num_sms ? 8 * (int64_t)c.num_sms : b < 1 ? 1 : b);
  };
  e = launch_pdl(nvfp4_amax_kernel, dim3(grid(nvec)), dim3(256), 0, c.stream, 1, static_cast<const bf16*>(W), nvec,
                 amax);
  if (e != cudaSuccess) return e;
  return launch_pdl(nvfp4_quant_kernel, dim3(grid(nblocks)), dim3(256), 0, c.stream, 1, static_cast<const bf16*>(W),
                    nblocks, (const unsigned*)amax, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales), g);
}

size_t forward_nvfp4_workspace_bytes(int64_t M, int64_t I, int r) {
  (void)I;
  return (M >= 1 && M <= kMaxTokens && r > 0) ? (size_t)kXvPartsFp4 * M * r * sizeof(float) : 0;
}

bool launch_forward_nvfp4(const LaunchCtx& c, const void* X, const void* codes, const void* scales, const float* g,
                          const float* s, const void* U, const void* V, int64_t M, int64_t O, int64_t I, int r,
                          void* Y, void* ws, cudaError_t* e) {
  *e = cudaSuccess;
  if (M < 1 || M > kMaxTokens || r > kMaxRank || I % 32 || fp4_smem_bytes(M, I) > kFp4SmemMax) return false;
  if (ceil_div(O, (int64_t)c.num_sms * kWarps) > kMaxRowsPerWarp) return false;
  if ((reinterpret_cast<uintptr_t>(X) & 15u) != 0) return false;
  GemvArgs a = {};
  a.X = static_cast<const bf16*>(X);
  a.s = s;
  a.U = static_cast<const bf16*>(U);
  a.t_parts = static_cast<const float*>(ws);
  a.nparts = (int)std::min<int64_t>(kXvPartsFp4, I);
  a.codes = static_cast<const uint8_t*>(codes);
  a.scales = static_cast<const uint8_t*>(scales);
  a.g = g;
  a.Y = static_cast<bf16*>(Y);
  a.O = O;
  a.I = I;
  a.r = r;
  a.early = r > 0 ? 1 : 0;
  *e = M == 1 ? launch_m<1, true>(c, a, V) : launch_m<2, true>(c, a, V);
  return true;
}

}  // namespace theta
