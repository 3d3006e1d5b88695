// HBM-streaming kernels of the analytic decomposition ("The theta bundle" --
// Analytic decomposition) and of relative_frobenius_error ("Quality" --
// Reconstruction error).
//
// All of them move each byte of their inputs once from HBM with 16-byte
// vector loads (8 bf16 or 4 fp32), accumulate in fp32 and reduce rows with
// warp shuffles. Grids are multiples of the SM count.
#include "common.cuh"
#include "internal.h"

namespace theta {

namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ const typename Vec<T>::raw* vrow(const void* base, int64_t elem) {
  return reinterpret_cast<const typename Vec<T>::raw*>(static_cast<const T*>(base) + elem);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int grid_for(const LaunchCtx& c, int64_t work_items, int per_block, int blocks_per_sm) {
  int64_t want = ceil_div(work_items, per_block);
  int64_t cap = (int64_t)c.num_sms * blocks_per_sm;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return (int)want;
}

// ------------------------------------------------------------- band mean
// W0 = (sum over layers in order, fp32) / n, one rounding to T.
template <typename T>
__global__ void __launch_bounds__(kThreads)
band_mean_kernel(PtrTable src, int n, int64_t nvec, int64_t count, T* __restrict__ out) {
  pdl_enter();
  using V = Vec<T>;
  using R = typename V::raw;
  const DivByCount div_n(n);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t v = tid; v < nvec; v += stride) {
    float acc[V::N];
#pragma unroll
    for (int e = 0; e < V::N; ++e) acc[e] = 0.f;
    int l = 0;
    for (; l + 4 <= n; l += 4) {
      R r[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) r[q] = ld_stream(vrow<T>(src.p[l + q], 0) + v);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float f[V::N];
        unpack(r[q], f);
#pragma unroll
        for (int e = 0; e < V::N; ++e) acc[e] += f[e];
      }
    }
    for (; l < n; ++l) {
      float f[V::N];
      unpack(ld_stream(vrow<T>(src.p[l], 0) + v), f);
#pragma unroll
      for (int e = 0; e < V::N; ++e) acc[e] += f[e];
    }
#pragma unroll
    for (int e = 0; e < V::N; ++e) acc[e] = div_n(acc[e]);
    reinterpret_cast<R*>(out)[v] = pack(acc, (R*)nullptr);
  }
  // scalar tail (count not a multiple of the vector width)
  for (int64_t i = nvec * V::N + tid; i < count; i += stride) {
    float acc = 0.f;
    for (int l = 0; l < n; ++l) acc += to_f32(static_cast<const T*>(src.p[l])[i]);
    out[i] = from_f32<T>(div_n(acc));
  }
}

// ------------------------------------------------- row scale (+ residual)
// One group of TPR threads per output row; the W0 row and one layer's row
// live in registers (VPT 16-byte vectors per thread). For every layer of the
// band: two fp32 dot products with identical operation order, a group
// reduction (warp shuffle, then shared memory across the group's warps),
// s = <w,W0> / <W0,W0>, then R = w - s W0 (residual_elem) from the registers.
template <typename T, int TPR, int VPT>
__global__ void __launch_bounds__(kThreads)
rowscale_band_kernel(const T* __restrict__ W0, PtrTable w, MutPtrTable s_out, MutPtrTable r_out,
                     int n, int64_t O, int64_t I, int write_r) {
  pdl_enter(W0);
  using V = Vec<T>;
  using R = typename V::raw;
  constexpr int GROUPS = kThreads / TPR;
  constexpr int WPR = TPR / 32;
  __shared__ float red[2][GROUPS][WPR][2];
  const int g = threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const int lane = threadIdx.x & 31;
  const int wr = t / 32;
  const int64_t nv = I / V::N;
  int parity = 0;
  const R zero = R{};

  for (int64_t base = (int64_t)blockIdx.x * GROUPS; base < O; base += (int64_t)gridDim.x * GROUPS) {
    const int64_t o = base + g;
    const bool valid = o < O;
    R a[VPT];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const int64_t v = t + (int64_t)j * TPR;
      a[j] = (valid && v < nv) ? ld_stream(vrow<T>(W0, o * I) + v) : zero;
    }
    for (int l = 0; l < n; ++l) {
      R b[VPT];
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        const int64_t v = t + (int64_t)j * TPR;
        b[j] = (valid && v < nv) ? ld_stream(vrow<T>(w.p[l], o * I) + v) : zero;
      }
      float d1 = 0.f, d2 = 0.f;
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        float fw[V::N], f0[V::N];
        unpack(b[j], fw);
        unpack(a[j], f0);
#pragma unroll
        for (int e = 0; e < V::N; ++e) {
          d1 = fmaf(fw[e], f0[e], d1);
          d2 = fmaf(f0[e], f0[e], d2);
        }
      }
      d1 = warp_sum(d1);
      d2 = warp_sum(d2);
      if constexpr (WPR > 1) {
        if (lane == 0) {
          red[parity][g][wr][0] = d1;
          red[parity][g][wr][1] = d2;
        }
        __syncthreads();
        d1 = 0.f;
        d2 = 0.f;
#pragma unroll
        for (int k = 0; k < WPR; ++k) {
          d1 += red[parity][g][k][0];
          d2 += red[parity][g][k][1];
        }
        parity ^= 1;
      }
      const float s = (d2 != 0.f) ? __fdiv_rn(d1, d2) : 0.f;
      if (valid && t == 0) static_cast<float*>(s_out.p[l])[o] = s;
      if (write_r && valid) {
        R* rrow = reinterpret_cast<R*>(static_cast<T*>(r_out.p[l]) + o * I);
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
          const int64_t v = t + (int64_t)j * TPR;
          if (v < nv) {
            float fw[V::N], f0[V::N], r[V::N];
            unpack(b[j], fw);
            unpack(a[j], f0);
#pragma unroll
            for (int e = 0; e < V::N; ++e) r[e] = residual_elem<T>(s, f0[e], fw[e]);
            rrow[v] = pack(r, (R*)nullptr);
          }
        }
      }
    }
  }
}

// Any row length and alignment: one warp per row, scalar loads, the second
// pass re-reads the row (from L2).
template <typename T>
__global__ void __launch_bounds__(kThreads)
rowscale_band_scalar_kernel(const T* __restrict__ W0, PtrTable w, MutPtrTable s_out,
                            MutPtrTable r_out, int n, int64_t O, int64_t I, int write_r) {
  pdl_enter(W0);
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t o = (int64_t)blockIdx.x * (kThreads / 32) + threadIdx.x / 32; o < O; o += warps) {
    const T* w0 = W0 + o * I;
    for (int l = 0; l < n; ++l) {
      const T* wl = static_cast<const T*>(w.p[l]) + o * I;
      float d1 = 0.f, d2 = 0.f;
      for (int64_t i = lane; i < I; i += 32) {
        const float fw = to_f32(wl[i]), f0 = to_f32(w0[i]);
        d1 = fmaf(fw, f0, d1);
        d2 = fmaf(f0, f0, d2);
      }
      d1 = warp_sum(d1);
      d2 = warp_sum(d2);
      const float s = (d2 != 0.f) ? __fdiv_rn(d1, d2) : 0.f;
      if (lane == 0) static_cast<float*>(s_out.p[l])[o] = s;
      if (write_r) {
        T* rl = static_cast<T*>(r_out.p[l]) + o * I;
        for (int64_t i = lane; i < I; i += 32) rl[i] = from_f32<T>(residual_elem<T>(s, to_f32(w0[i]), to_f32(wl[i])));
      }
    }
  }
}

// ------------------------------------------------------------- residual
template <typename T>
__global__ void __launch_bounds__(kThreads)
residual_vec_kernel(const T* __restrict__ w, const T* __restrict__ W0, const float* __restrict__ s,
                    int64_t nv_row, int64_t nvec, T* __restrict__ R) {
  pdl_enter(w, W0, s);
  using V = Vec<T>;
  using Rw = typename V::raw;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    const float sc = __ldg(s + v / nv_row);
    float fw[V::N], f0[V::N], r[V::N];
    unpack(ld_stream(reinterpret_cast<const Rw*>(w) + v), fw);
    unpack(ld_stream(reinterpret_cast<const Rw*>(W0) + v), f0);
#pragma unroll
    for (int e = 0; e < V::N; ++e) r[e] = residual_elem<T>(sc, f0[e], fw[e]);
    reinterpret_cast<Rw*>(R)[v] = pack(r, (Rw*)nullptr);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
residual_scalar_kernel(const T* __restrict__ w, const T* __restrict__ W0, const float* __restrict__ s,
                       int64_t I, int64_t count, T* __restrict__ R) {
  pdl_enter(w, W0, s);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
    R[i] = from_f32<T>(residual_elem<T>(s[i / I], to_f32(W0[i]), to_f32(w[i])));
}

// ------------------------------------------------------- frobenius error
constexpr int kFrobMaxBlocks = 1024;

template <typename T>
__global__ void __launch_bounds__(kThreads)
frob_partial_kernel(const T* __restrict__ A, const T* __restrict__ B, int64_t nvec, int64_t count,
                    double* __restrict__ ws) {
  pdl_enter(A, B);
  using V = Vec<T>;
  using R = typename V::raw;
  double num = 0.0, den = 0.0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t v = tid; v < nvec; v += stride) {
    float fa[V::N], fb[V::N];
    unpack(ld_stream(reinterpret_cast<const R*>(A) + v), fa);
    unpack(ld_stream(reinterpret_cast<const R*>(B) + v), fb);
    float pn = 0.f, pd = 0.f;
#pragma unroll
    for (int e = 0; e < V::N; ++e) {
      const float d = fa[e] - fb[e];
      pn = fmaf(d, d, pn);
      pd = fmaf(fa[e], fa[e], pd);
    }
    num += (double)pn;
    den += (double)pd;
  }
  for (int64_t i = nvec * V::N + tid; i < count; i += stride) {
    const float a = to_f32(A[i]), d = a - to_f32(B[i]);
    num += (double)(d * d);
    den += (double)(a * a);
  }
  __shared__ double red[kThreads / 32][2];
  num = warp_sum(num);
  den = warp_sum(den);
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x / 32][0] = num;
    red[threadIdx.x / 32][1] = den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double n2 = 0.0, d2 = 0.0;
    for (int k = 0; k < kThreads / 32; ++k) {
      n2 += red[k][0];
      d2 += red[k][1];
    }
    ws[2 * blockIdx.x] = n2;
    ws[2 * blockIdx.x + 1] = d2;
  }
}

// Combines the block partials in a fixed order into the ratio, or (partials)
// into the two sums themselves: out[0] = sum (A-B)^2, out[1] = sum A^2.
__global__ void __launch_bounds__(kThreads) frob_final_kernel(const double* __restrict__ ws, int nb,
                                                              double* __restrict__ out, int partials) {
  pdl_enter(ws);
  double num = 0.0, den = 0.0;
  for (int k = threadIdx.x; k < nb; k += blockDim.x) {
    num += ws[2 * k];
    den += ws[2 * k + 1];
  }
  __shared__ double red[kThreads / 32][2];
  num = warp_sum(num);
  den = warp_sum(den);
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x / 32][0] = num;
    red[threadIdx.x / 32][1] = den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double n2 = 0.0, d2 = 0.0;
    for (int k = 0; k < kThreads / 32; ++k) {
      n2 += red[k][0];
      d2 += red[k][1];
    }
    if (partials) {
      out[0] = n2;
      out[1] = d2;
      return;
    }
    double e;
    if (d2 == 0.0)
      e = (n2 == 0.0) ? 0.0 : __longlong_as_double(0x7ff0000000000000ll);
    else
      e = sqrt(n2) / sqrt(d2);
    *out = e;
  }
}

template <typename T>
cudaError_t band_mean_t(const LaunchCtx& c, const void* const* w, int n, int64_t O, int64_t I,
                        void* W0) {
  PtrTable tab{};
  bool ok = aligned16(W0);
  for (int l = 0; l < n; ++l) {
    tab.p[l] = w[l];
    ok = ok && aligned16(w[l]);
  }
  const int64_t count = O * I;
  const int64_t nvec = ok ? count / Vec<T>::N : 0;
  const int grid = grid_for(c, ok ? nvec : count, kThreads, 8);
  return launch_pdl(band_mean_kernel<T>, grid, kThreads, 0, c.stream, 1, tab, n, nvec, count, static_cast<T*>(W0));
}

template <typename T, int TPR, int VPT>
cudaError_t launch_rs(const LaunchCtx& c, int grid, const T* W0, const PtrTable& w, const MutPtrTable& s,
                      const MutPtrTable& r, int n, int64_t O, int64_t I, int write_r) {
  return launch_pdl(rowscale_band_kernel<T, TPR, VPT>, grid, kThreads, 0, c.stream, 1, W0, w, s, r, n, O, I,
                    write_r);
}

// Launches the register-resident row-scale variant for (TPR, vpt); returns
// false if no such variant exists.
template <typename T, int TPR>
bool dispatch_vpt(const LaunchCtx& c, int vpt, int grid, const T* W0, const PtrTable& w,
                  const MutPtrTable& s, const MutPtrTable& r, int n, int64_t O, int64_t I,
                  int write_r, cudaError_t* e) {
  switch (vpt) {
    case 1: *e = launch_rs<T, TPR, 1>(c, grid, W0, w, s, r, n, O, I, write_r); return true;
    case 2: *e = launch_rs<T, TPR, 2>(c, grid, W0, w, s, r, n, O, I, write_r); return true;
    case 3: *e = launch_rs<T, TPR, 3>(c, grid, W0, w, s, r, n, O, I, write_r); return true;
    case 4: *e = launch_rs<T, TPR, 4>(c, grid, W0, w, s, r, n, O, I, write_r); return true;
    case 6: *e = launch_rs<T, TPR, 6>(c, grid, W0, w, s, r, n, O, I, write_r); return true;
    case 8: *e = launch_rs<T, TPR, 8>(c, grid, W0, w, s, r, n, O, I, write_r); return true;
    case 12: *e = launch_rs<T, TPR, 12>(c, grid, W0, w, s, r, n, O, I, write_r); return true;
  }
  return false;
}

int round_vpt(int64_t v) {
  const int opts[] = {1, 2, 3, 4, 6, 8, 12};
  for (int o : opts)
    if (v <= o) return o;
  return -1;
}

// Ring geometry for `rows_per_item` rows of I elements per slot: up to 16
// slots within ~100 KB (two CTAs per SM), at least 2 slots; 0 if it does not fit.
// Threads per row and vectors per thread for a row of nv vectors: the
// fewest threads that keep every thread at <= 4 vectors, else 256 threads.
void row_geometry(int64_t nv, int* tpr, int* vpt) {
  *tpr = 0;
  const int tprs[] = {32, 64, 128, 256};
  for (int cand : tprs) {
    if (ceil_div(nv, cand) <= 4) {
      *tpr = cand;
      break;
    }
  }
  if (!*tpr) *tpr = 256;
  *vpt = round_vpt(ceil_div(nv, *tpr));
}

template <typename T>
cudaError_t rowscale_t(const LaunchCtx& c, const void* W0, const void* const* w, int n, int64_t O,
                       int64_t I, float* const* s, void* const* R) {
  PtrTable wt{};
  MutPtrTable st{}, rt{};
  const int write_r = R != nullptr;
  bool ok = aligned16(W0) && (I % Vec<T>::N == 0);
  for (int l = 0; l < n; ++l) {
    wt.p[l] = w[l];
    st.p[l] = s[l];
    rt.p[l] = write_r ? R[l] : nullptr;
    ok = ok && aligned16(w[l]) && (!write_r || aligned16(R[l]));
  }

  int tpr = 0, vpt = -1;
  if (ok) row_geometry(I / Vec<T>::N, &tpr, &vpt);
  if (vpt > 0) {
    const int groups = kThreads / tpr;
    const int grid = grid_for(c, O, groups, vpt <= 4 ? 8 : 4);
    const T* W0t = static_cast<const T*>(W0);
    bool launched = false;
    cudaError_t e = cudaSuccess;
    switch (tpr) {
      case 32: launched = dispatch_vpt<T, 32>(c, vpt, grid, W0t, wt, st, rt, n, O, I, write_r, &e); break;
      case 64: launched = dispatch_vpt<T, 64>(c, vpt, grid, W0t, wt, st, rt, n, O, I, write_r, &e); break;
      case 128: launched = dispatch_vpt<T, 128>(c, vpt, grid, W0t, wt, st, rt, n, O, I, write_r, &e); break;
      case 256: launched = dispatch_vpt<T, 256>(c, vpt, grid, W0t, wt, st, rt, n, O, I, write_r, &e); break;
    }
    if (launched) return e;
  }
  const int grid = grid_for(c, O, kThreads / 32, 8);
  return launch_pdl(rowscale_band_scalar_kernel<T>, grid, kThreads, 0, c.stream, 1, static_cast<const T*>(W0),
                    wt, st, rt, n, O, I, write_r);
}

template <typename T>
cudaError_t residual_t(const LaunchCtx& c, const void* w, const void* W0, const float* s,
                       int64_t O, int64_t I, void* R) {
  const bool vec = aligned16(w) && aligned16(W0) && aligned16(R) && (I % Vec<T>::N == 0);
  const int64_t count = O * I;
  if (vec) {
    const int64_t nvec = count / Vec<T>::N;
    return launch_pdl(residual_vec_kernel<T>, grid_for(c, nvec, kThreads, 8), kThreads, 0, c.stream, 1,
                      static_cast<const T*>(w), static_cast<const T*>(W0), s, I / Vec<T>::N, nvec,
                      static_cast<T*>(R));
  }
  return launch_pdl(residual_scalar_kernel<T>, grid_for(c, count, kThreads, 8), kThreads, 0, c.stream, 1,
                    static_cast<const T*>(w), static_cast<const T*>(W0), s, I, count, static_cast<T*>(R));
}

template <typename T>
cudaError_t frob_t(const LaunchCtx& c, const void* a, const void* b, int64_t n, double* out,
                   void* ws, bool partials) {
  const bool vec = aligned16(a) && aligned16(b);
  const int64_t nvec = vec ? n / Vec<T>::N : 0;
  int grid = grid_for(c, vec ? nvec : n, kThreads, 4);
  if (grid > kFrobMaxBlocks) grid = kFrobMaxBlocks;
  double* part = static_cast<double*>(ws);
  cudaError_t e = launch_pdl(frob_partial_kernel<T>, grid, kThreads, 0, c.stream, 1, static_cast<const T*>(a),
                             static_cast<const T*>(b), nvec, n, part);
  if (e != cudaSuccess) return e;
  return launch_pdl(frob_final_kernel, 1, kThreads, 0, c.stream, 1, static_cast<const double*>(part), grid, out,
                    partials ? 1 : 0);
}

}  // namespace

cudaError_t launch_band_mean(const LaunchCtx& c, theta_dtype dt, const void* const* w, int n,
                             int64_t O, int64_t I, void* W0) {
  return dt == THETA_BF16 ? band_mean_t<bf16>(c, w, n, O, I, W0) : band_mean_t<float>(c, w, n, O, I, W0);
}

cudaError_t launch_rowscale_band(const LaunchCtx& c, theta_dtype dt, const void* W0,
                                 const void* const* w, int n, int64_t O, int64_t I,
                                 float* const* s, void* const* R) {
  return dt == THETA_BF16 ? rowscale_t<bf16>(c, W0, w, n, O, I, s, R)
                          : rowscale_t<float>(c, W0, w, n, O, I, s, R);
}

cudaError_t launch_residual(const LaunchCtx& c, theta_dtype dt, const void* w, const void* W0,
                            const float* s, int64_t O, int64_t I, void* R) {
  return dt == THETA_BF16 ? residual_t<bf16>(c, w, W0, s, O, I, R)
                          : residual_t<float>(c, w, W0, s, O, I, R);
}

size_t frob_workspace_bytes() { return (size_t)kFrobMaxBlocks * 2 * sizeof(double); }

cudaError_t launch_frob(const LaunchCtx& c, theta_dtype dt, const void* a, const void* b,
                        int64_t n, double* out, void* ws, bool partials) {
  return dt == THETA_BF16 ? frob_t<bf16>(c, a, b, n, out, ws, partials)
                          : frob_t<float>(c, a, b, n, out, ws, partials);
}

}  // namespace theta
