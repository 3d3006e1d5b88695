// The decomposition prelude of one projection family ("The theta bundle" --
// Analytic decomposition: shared block, per-row scale, residual; "Banded
// sharing" for the bands), streamed through a shared-memory ring.
//
// One launch covers every band of the family. A persistent CTA has a
// producer warp and eight consumer warps. The producer keeps up to 16 items
// in flight with 1-D bulk copies (cp.async.bulk) into ring slots; the
// consumers process one item at a time from shared memory and release the
// slot with one mbarrier arrival per warp. An item is ROWS output rows, each
// owned by a group of TPR consumer threads:
//   BAND mode (bands of at most 4 layers): a slot holds the band's rows for
//     each output row; the group forms the W0 row (fp32 sum in layer order,
//     one division by n, one rounding), writes it, and writes s and the
//     residual of every layer of the band. Each weight row crosses HBM once.
//   ROW mode (larger bands, after their band means are formed): an item is
//     (row group, layer); a slot holds each row's W0 row and that layer's row;
//     the group writes s and the residual of that layer.
// Both dot products of a layer (<w,W0> and <W0,W0>) use the same fp32
// operation order, so a layer equal to its W0 gets s == 1 exactly and a zero
// residual. Reductions: warp shuffles, then one named barrier of the 256
// consumer threads per item across a group's warps (its OR-vote also makes a
// timed-out wait abort every consumer together).
#include "common.cuh"
#include "internal.h"
#include "umma_ptx.cuh"

namespace theta {

namespace {

constexpr int kConsumers = 256;            // 8 consumer warps
constexpr int kThreads = kConsumers + 32;  // + 1 producer warp
constexpr int kMaxSlots = 16;
constexpr int kSmemBudget = 100 * 1024;    // two CTAs per SM

struct PreludeArgs {
  PtrTable w;       // L layer weights [O, I]
  MutPtrTable W0;   // G shared blocks (BAND: written; ROW: read)
  MutPtrTable s;    // L row scales, fp32 [O]
  MutPtrTable r;    // L residuals (unused when write_r == 0)
  int16_t band_start[THETA_MAX_LAYERS + 1];
  int16_t band_of_layer[THETA_MAX_LAYERS];
  int L, G, write_r, nmax;  // nmax: largest band (BAND mode slot layout)
  int64_t O, I;
  int slots, slot_bytes;
  int64_t row_groups;  // ceil(O / ROWS)
  int64_t items;
  unsigned* err;
};

__device__ __forceinline__ bool vote_any(bool p) {
  // OR over the 256 consumer threads (named barrier 1); also orders their
  // shared-memory writes before the reads that follow
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "barrier.red.or.pred b, 1, %2, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "n"(kConsumers)
      : "memory");
  return r != 0;
}

template <typename T, bool BAND, int TPR, int VPT>
__global__ void __launch_bounds__(kThreads)
prelude_pipe_kernel(const __grid_constant__ PreludeArgs a) {
  using V = Vec<T>;
  using R = typename V::raw;
  constexpr int ROWS = kConsumers / TPR;
  constexpr int WPR = TPR / 32;
  constexpr int NL = BAND ? 4 : 1;  // layers per row in an item
  constexpr int NR = NL + 1;        // <W0,W0> and one <w,W0> per layer
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)a.slots * a.slot_bytes);
  uint64_t* empty = full + kMaxSlots;
  __shared__ float red[2][ROWS][WPR][NR];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid & 31;
  const int64_t nv = a.I / V::N;
  const uint32_t row_bytes = (uint32_t)(a.I * sizeof(T));
  const uint32_t row_stride = (uint32_t)(a.slot_bytes / ROWS);  // bytes per output row in a slot

  if (tid == 0) {
    for (int i = 0; i < a.slots; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kConsumers / 32);
    }
    abort_flag = prior_timeout(a.err);
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  pdl_enter();

  // item k -> (band or layer, first output row)
  auto decode = [&](int64_t k, int* bl, int64_t* row0) {
    if constexpr (BAND) {
      *bl = (int)(k / a.row_groups);
      *row0 = (k % a.row_groups) * ROWS;
    } else {
      *bl = (int)(k % a.L);
      *row0 = (k / a.L) * ROWS;
    }
  };

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int64_t j = 0;
      for (int64_t k = blockIdx.x; k < a.items; k += gridDim.x, ++j) {
        const int st = (int)(j % a.slots);
        if (!ptx::mbar_wait(&empty[st], (uint32_t)((j / a.slots) & 1) ^ 1u, &abort_flag)) {
          record_timeout(a.err);
          abort_flag = 1;
          break;
        }
        int bl;
        int64_t row0;
        decode(k, &bl, &row0);
        const int nrows = (int)(a.O - row0 < ROWS ? a.O - row0 : ROWS);
        uint8_t* dst = ring + (size_t)st * a.slot_bytes;
        if constexpr (BAND) {
          const int first = a.band_start[bl], n = a.band_start[bl + 1] - first;
          ptx::mbar_arrive_expect_tx(&full[st], row_bytes * (uint32_t)(n * nrows));
          for (int g = 0; g < nrows; ++g)
            for (int l = 0; l < n; ++l)
              ptx::bulk_load(dst + g * row_stride + l * row_bytes,
                             static_cast<const T*>(a.w.p[first + l]) + (row0 + g) * a.I, row_bytes, &full[st]);
        } else {
          const T* w0 = static_cast<const T*>(a.W0.p[a.band_of_layer[bl]]);
          ptx::mbar_arrive_expect_tx(&full[st], 2 * row_bytes * (uint32_t)nrows);
          for (int g = 0; g < nrows; ++g) {
            ptx::bulk_load(dst + g * row_stride, w0 + (row0 + g) * a.I, row_bytes, &full[st]);
            ptx::bulk_load(dst + g * row_stride + row_bytes, static_cast<const T*>(a.w.p[bl]) + (row0 + g) * a.I,
                           row_bytes, &full[st]);
          }
        }
      }
      // let every copy land before the CTA can leave (immediate unless aborted)
      const int64_t issued = j;
      for (int st = 0; st < a.slots && st < issued; ++st) {
        const int64_t last = st + ((issued - 1 - st) / a.slots) * a.slots;
        int never = 0;
        ptx::mbar_wait(&full[st], (uint32_t)((last / a.slots) & 1), &never);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int g = tid / TPR, t = tid % TPR, wr = t / 32;
    int64_t j = 0;
    for (int64_t k = blockIdx.x; k < a.items; k += gridDim.x, ++j) {
      const int st = (int)(j % a.slots);
      const bool ok = ptx::mbar_wait(&full[st], (uint32_t)((j / a.slots) & 1), &abort_flag);
      int bl;
      int64_t row0;
      decode(k, &bl, &row0);
      const int64_t o = row0 + g;
      const bool valid = ok && o < a.O;
      int first = 0, n = 1;
      if constexpr (BAND) {
        first = a.band_start[bl];
        n = a.band_start[bl + 1] - first;
      }
      const uint8_t* rowp = ring + (size_t)st * a.slot_bytes + g * row_stride;
      const DivByCount div_n(n);
      // W0 row (registers); BAND forms it from the band's rows and writes it
      R w0[VPT];
#pragma unroll
      for (int q = 0; q < VPT; ++q) {
        const int64_t v = t + (int64_t)q * TPR;
        if (!valid || v >= nv) {
          w0[q] = R{};
          continue;
        }
        if constexpr (BAND) {
          if (n == 1) {  // the shared block of a one-layer band is that layer
            w0[q] = reinterpret_cast<const R*>(rowp)[v];
            reinterpret_cast<R*>(static_cast<T*>(a.W0.p[bl]) + o * a.I)[v] = w0[q];
            continue;
          }
          float acc[V::N];
#pragma unroll
          for (int e = 0; e < V::N; ++e) acc[e] = 0.f;
#pragma unroll
          for (int l = 0; l < NL; ++l) {
            if (l < n) {
              float f[V::N];
              unpack(reinterpret_cast<const R*>(rowp + l * row_bytes)[v], f);
#pragma unroll
              for (int e = 0; e < V::N; ++e) acc[e] += f[e];
            }
          }
#pragma unroll
          for (int e = 0; e < V::N; ++e) acc[e] = div_n(acc[e]);
          w0[q] = pack(acc, (R*)nullptr);
          reinterpret_cast<R*>(static_cast<T*>(a.W0.p[bl]) + o * a.I)[v] = w0[q];
        } else {
          w0[q] = reinterpret_cast<const R*>(rowp)[v];
        }
      }
      const uint8_t* wbase = rowp + (BAND ? 0 : row_bytes);
      float d[NR];
#pragma unroll
      for (int q = 0; q < NR; ++q) d[q] = 0.f;
#pragma unroll
      for (int q = 0; q < VPT; ++q) {
        const int64_t v = t + (int64_t)q * TPR;
        if (!valid || v >= nv) continue;
        float f0[V::N];
        unpack(w0[q], f0);
#pragma unroll
        for (int e = 0; e < V::N; ++e) d[0] = fmaf(f0[e], f0[e], d[0]);
#pragma unroll
        for (int l = 0; l < NL; ++l) {
          if (l >= n) break;
          float fw[V::N];
          unpack(reinterpret_cast<const R*>(wbase + l * row_bytes)[v], fw);
#pragma unroll
          for (int e = 0; e < V::N; ++e) d[l + 1] = fmaf(fw[e], f0[e], d[l + 1]);
        }
      }
#pragma unroll
      for (int q = 0; q < NR; ++q) d[q] = warp_sum(d[q]);
      const int par = (int)(j & 1);
      if (lane == 0)
#pragma unroll
        for (int q = 0; q < NR; ++q) red[par][g][wr][q] = d[q];
      if (vote_any(!ok)) {
        if (tid == 0) {
          record_timeout(a.err);
          abort_flag = 1;
        }
        break;
      }
#pragma unroll
      for (int q = 0; q < NR; ++q) {
        d[q] = 0.f;
#pragma unroll
        for (int u = 0; u < WPR; ++u) d[q] += red[par][g][u][q];
      }
#pragma unroll
      for (int l = 0; l < NL; ++l) {
        if (l >= n) break;
        const int layer = BAND ? first + l : bl;
        const float sl = (d[0] != 0.f) ? __fdiv_rn(d[l + 1], d[0]) : 0.f;
        if (valid && t == 0) static_cast<float*>(a.s.p[layer])[o] = sl;
        if (a.write_r && valid) {
          R* rrow = reinterpret_cast<R*>(static_cast<T*>(a.r.p[layer]) + o * a.I);
          const R* wl = reinterpret_cast<const R*>(wbase + l * row_bytes);
#pragma unroll
          for (int q = 0; q < VPT; ++q) {
            const int64_t v = t + (int64_t)q * TPR;
            if (v >= nv) continue;
            float fw[V::N], f0[V::N], rr[V::N];
            unpack(wl[v], fw);
            unpack(w0[q], f0);
#pragma unroll
            for (int e = 0; e < V::N; ++e) rr[e] = residual_elem<T>(sl, f0[e], fw[e]);
            rrow[v] = pack(rr, (R*)nullptr);
          }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[st]);
    }
  }
}

// Long bands (more than 4 layers) in one launch, each weight row read from
// HBM once: a unit is (band, ROWS output rows). Pass 1 streams the band's
// layers for those rows through the ring, LPI layers per item, and the
// consumers sum them in fp32 registers; the group divides once, rounds,
// writes the W0 rows and keeps them in registers. Pass 2 streams the same
// items again -- in reverse order, so the most recently read ones come first
// and are still in L2 -- and forms s and the residual of each layer exactly
// as ROW mode does (same fp32 operation order for <w,W0> and <W0,W0>), with
// one reduction barrier per item. The grid is sized so that the rows all
// CTAs hold between the two passes stay well inside L2.
template <typename T, int TPR, int VPT, int LPI>
__global__ void __launch_bounds__(kThreads)
prelude_band2_kernel(const __grid_constant__ PreludeArgs a) {
  using V = Vec<T>;
  using R = typename V::raw;
  constexpr int ROWS = kConsumers / TPR;
  constexpr int WPR = TPR / 32;
  constexpr int NR = LPI + 1;  // <W0,W0> and one <w,W0> per layer of an item
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)a.slots * a.slot_bytes);
  uint64_t* empty = full + kMaxSlots;
  __shared__ float red[2][ROWS][WPR][NR];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid & 31;
  const int64_t nv = a.I / V::N;
  const uint32_t row_bytes = (uint32_t)(a.I * sizeof(T));
  const uint32_t layer_bytes = row_bytes * ROWS;  // one layer's rows in a slot

  if (tid == 0) {
    for (int i = 0; i < a.slots; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kConsumers / 32);
    }
    abort_flag = prior_timeout(a.err);
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  pdl_enter();

  // unit u -> (band, first output row); a unit's items: ni in pass 1, then
  // the same ni in reverse order in pass 2; item i holds layers
  // first + LPI i ... (at most LPI of them)
  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // pass 1 marks the rows it reads to stay in L2; pass 2 reads them for the last time
      const uint64_t keep = ptx::l2_policy_evict_last(), drop = ptx::l2_policy_evict_first();
      int64_t j = 0;
      bool stop = false;
      for (int64_t u = blockIdx.x; u < a.items && !stop; u += gridDim.x) {
        const int b = (int)(u / a.row_groups);
        const int64_t row0 = (u % a.row_groups) * ROWS;
        const int nrows = (int)(a.O - row0 < ROWS ? a.O - row0 : ROWS);
        const int first = a.band_start[b], n = a.band_start[b + 1] - first;
        const int ni = (n + LPI - 1) / LPI;
        for (int k = 0; k < 2 * ni; ++k, ++j) {
          const int st = (int)(j % a.slots);
          if (!ptx::mbar_wait(&empty[st], (uint32_t)((j / a.slots) & 1) ^ 1u, &abort_flag)) {
            record_timeout(a.err);
            abort_flag = 1;
            stop = true;
            break;
          }
          const int i = k < ni ? k : 2 * ni - 1 - k;
          const int l0 = first + i * LPI, nl = min(LPI, n - i * LPI);
          const uint32_t bytes = row_bytes * (uint32_t)nrows;  // the unit's rows of one layer are contiguous
          ptx::mbar_arrive_expect_tx(&full[st], bytes * (uint32_t)nl);
          for (int q = 0; q < nl; ++q)
            ptx::bulk_load_hint(ring + (size_t)st * a.slot_bytes + (size_t)q * layer_bytes,
                                static_cast<const T*>(a.w.p[l0 + q]) + row0 * a.I, bytes, &full[st],
                                k < ni ? keep : drop);
        }
      }
      // let every copy land before the CTA can leave (immediate unless aborted)
      for (int st = 0; st < a.slots && st < j; ++st) {
        const int64_t last = st + ((j - 1 - st) / a.slots) * a.slots;
        int never = 0;
        ptx::mbar_wait(&full[st], (uint32_t)((last / a.slots) & 1), &never);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int g = tid / TPR, t = tid % TPR, wr = t / 32;
    int64_t j = 0;
    bool aborted = false;
    for (int64_t u = blockIdx.x; u < a.items && !aborted; u += gridDim.x) {
      const int b = (int)(u / a.row_groups);
      const int64_t row0 = (u % a.row_groups) * ROWS;
      const int64_t o = row0 + g;
      const bool row_ok = o < a.O;
      const int first = a.band_start[b], n = a.band_start[b + 1] - first;
      const int ni = (n + LPI - 1) / LPI;
      // ---- pass 1: fp32 sum of the band's rows, in layer order
      float acc[VPT][V::N];
#pragma unroll
      for (int q = 0; q < VPT; ++q)
#pragma unroll
        for (int e = 0; e < V::N; ++e) acc[q][e] = 0.f;
      bool ok_all = true;
      for (int i = 0; i < ni; ++i, ++j) {
        const int st = (int)(j % a.slots);
        const bool ok = ptx::mbar_wait(&full[st], (uint32_t)((j / a.slots) & 1), &abort_flag);
        ok_all = ok_all && ok;
        const int nl = min(LPI, n - i * LPI);
        const uint8_t* base = ring + (size_t)st * a.slot_bytes + (size_t)g * row_bytes;
        if (ok && row_ok) {
#pragma unroll
          for (int l = 0; l < LPI; ++l) {
            if (l >= nl) break;
            const R* row = reinterpret_cast<const R*>(base + (size_t)l * layer_bytes);
#pragma unroll
            for (int q = 0; q < VPT; ++q) {
              const int64_t v = t + (int64_t)q * TPR;
              if (v < nv) {
                float f[V::N];
                unpack(row[v], f);
#pragma unroll
                for (int e = 0; e < V::N; ++e) acc[q][e] += f[e];
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[st]);
      }
      if (vote_any(!ok_all)) {
        aborted = true;
        break;
      }
      // W0 row: one division by n, one rounding; kept raw for pass 2
      const DivByCount div_n(n);
      R w0[VPT];
#pragma unroll
      for (int q = 0; q < VPT; ++q) {
        const int64_t v = t + (int64_t)q * TPR;
#pragma unroll
        for (int e = 0; e < V::N; ++e) acc[q][e] = div_n(acc[q][e]);
        w0[q] = pack(acc[q], (R*)nullptr);
        if (row_ok && v < nv) __stcs(reinterpret_cast<R*>(static_cast<T*>(a.W0.p[b]) + o * a.I) + v, w0[q]);
      }
      // ---- pass 2: s and the residual of each layer (last items first)
      for (int k = 0; k < ni; ++k, ++j) {
        const int st = (int)(j % a.slots);
        const bool ok = ptx::mbar_wait(&full[st], (uint32_t)((j / a.slots) & 1), &abort_flag);
        const int i = ni - 1 - k;
        const int l0 = first + i * LPI, nl = min(LPI, n - i * LPI);
        const uint8_t* base = ring + (size_t)st * a.slot_bytes + (size_t)g * row_bytes;
        float d[NR];
#pragma unroll
        for (int q = 0; q < NR; ++q) d[q] = 0.f;
        if (ok && row_ok) {
#pragma unroll
          for (int q = 0; q < VPT; ++q) {
            const int64_t v = t + (int64_t)q * TPR;
            if (v >= nv) continue;
            float f0[V::N];
            unpack(w0[q], f0);
#pragma unroll
            for (int e = 0; e < V::N; ++e) d[0] = fmaf(f0[e], f0[e], d[0]);
#pragma unroll
            for (int l = 0; l < LPI; ++l) {
              if (l >= nl) break;
              float fw[V::N];
              unpack(reinterpret_cast<const R*>(base + (size_t)l * layer_bytes)[v], fw);
#pragma unroll
              for (int e = 0; e < V::N; ++e) d[l + 1] = fmaf(fw[e], f0[e], d[l + 1]);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < NR; ++q) d[q] = warp_sum(d[q]);
        const int par = (int)(j & 1);
        if (lane == 0)
#pragma unroll
          for (int q = 0; q < NR; ++q) red[par][g][wr][q] = d[q];
        if (vote_any(!ok)) {
          aborted = true;
          break;
        }
#pragma unroll
        for (int q = 0; q < NR; ++q) {
          d[q] = 0.f;
#pragma unroll
          for (int w = 0; w < WPR; ++w) d[q] += red[par][g][w][q];
        }
#pragma unroll
        for (int l = 0; l < LPI; ++l) {
          if (l >= nl) break;
          const int layer = l0 + l;
          const float sl = (d[0] != 0.f) ? __fdiv_rn(d[l + 1], d[0]) : 0.f;
          if (row_ok && t == 0) static_cast<float*>(a.s.p[layer])[o] = sl;
          if (a.write_r && row_ok) {
            R* rrow = reinterpret_cast<R*>(static_cast<T*>(a.r.p[layer]) + o * a.I);
            const R* wl = reinterpret_cast<const R*>(base + (size_t)l * layer_bytes);
#pragma unroll
            for (int q = 0; q < VPT; ++q) {
              const int64_t v = t + (int64_t)q * TPR;
              if (v >= nv) continue;
              float fw[V::N], f0[V::N], rr[V::N];
              unpack(wl[v], fw);
              unpack(w0[q], f0);
#pragma unroll
              for (int e = 0; e < V::N; ++e) rr[e] = residual_elem<T>(sl, f0[e], fw[e]);
              __stcs(rrow + v, pack(rr, (R*)nullptr));  // written once, not read here again
            }
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[st]);
      }
    }
    if (aborted && tid == 0) {
      record_timeout(a.err);
      abort_flag = 1;
    }
  }
}

// Threads per output row (32..256, i.e. 8..1 rows per item): the fewest
// that keep each thread at <= 12 vectors of a row and an item's shared
// memory within item_cap, so a CTA has several items in flight and each
// item carries enough bytes to pay for its one reduction barrier. Vectors
// per thread are rounded up to a compiled variant.
bool geometry(int64_t nv, int64_t per_row_bytes, int64_t item_cap, int* tpr, int* vpt) {
  const int tprs[] = {32, 64, 128, 256};
  *tpr = 0;
  for (int c : tprs) {
    if (ceil_div(nv, c) <= 12 && (kConsumers / c) * per_row_bytes <= item_cap) {
      *tpr = c;
      break;
    }
  }
  if (!*tpr) *tpr = 256;
  const int64_t need = ceil_div(nv, *tpr);
  const int opts[] = {1, 2, 3, 4, 6, 8, 12};
  for (int o : opts)
    if (need <= o) {
      *vpt = o;
      return true;
    }
  return false;
}

template <typename T, bool BAND, int TPR, int VPT>
cudaError_t launch_one(const LaunchCtx& c, const PreludeArgs& a, int grid, size_t smem) {
  auto kern = prelude_pipe_kernel<T, BAND, TPR, VPT>;
  static bool opted[64] = {};
  std::unique_lock<std::mutex> lk(setup_mutex());
  if (!opted[c.device]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBudget + 128 + 2 * kMaxSlots * 8);
    if (e != cudaSuccess) return e;
    opted[c.device] = true;
  }
  lk.unlock();
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), smem, c.stream, 1, a);
}

template <typename T, bool BAND, int TPR>
cudaError_t dispatch_vpt(const LaunchCtx& c, const PreludeArgs& a, int vpt, int grid, size_t smem) {
  switch (vpt) {
    case 1: return launch_one<T, BAND, TPR, 1>(c, a, grid, smem);
    case 2: return launch_one<T, BAND, TPR, 2>(c, a, grid, smem);
    case 3: return launch_one<T, BAND, TPR, 3>(c, a, grid, smem);
    case 4: return launch_one<T, BAND, TPR, 4>(c, a, grid, smem);
    case 6: return launch_one<T, BAND, TPR, 6>(c, a, grid, smem);
    case 8: return launch_one<T, BAND, TPR, 8>(c, a, grid, smem);
    case 12: return launch_one<T, BAND, TPR, 12>(c, a, grid, smem);
  }
  return cudaErrorInvalidValue;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Fills PreludeArgs for L layers in G bands; false if the pipeline cannot
// take the problem (alignment, row too long for the slots).
template <typename T, bool BAND>
bool plan(const LaunchCtx& c, const void* const* w, int L, int G, const int32_t* band_start,
          const int32_t* band_of_layer, void* const* W0, float* const* s, void* const* R, int64_t O, int64_t I,
          PreludeArgs* a, int* tpr, int* vpt, int* grid, size_t* smem) {
  if (I % Vec<T>::N) return false;
  int nmax = 1;
  for (int b = 0; b < G; ++b) nmax = max(nmax, band_start[b + 1] - band_start[b]);
  if (BAND && nmax > 4) return false;
  const int64_t row_bytes = I * (int64_t)sizeof(T);
  const int64_t per_row = BAND ? nmax * row_bytes : 2 * row_bytes;
  // Items of up to 32 KB; the row mode takes up to 48 KB: at the 31B width
  // that is two rows per item with 128 threads each instead of one with 256,
  // measured 12% faster (its consumers are issue-bound, and two rows share
  // one reduction barrier). A larger cap would give BAND mode variants whose
  // registers keep two CTAs off an SM.
  if (!geometry(I / Vec<T>::N, per_row, BAND ? 32 * 1024 : 48 * 1024, tpr, vpt)) return false;
  const int rows = kConsumers / *tpr;
  const int64_t slot = ceil_div(rows * per_row, 128) * 128;
  int64_t slots = kSmemBudget / slot;
  if (slots > kMaxSlots) slots = kMaxSlots;
  if (slots < 2) return false;
  if ((slot / rows) % 16) return false;  // each row's copies start 16-byte aligned
  for (int l = 0; l < L; ++l) {
    if (!aligned16(w[l]) || (R && !aligned16(R[l]))) return false;
    a->w.p[l] = w[l];
    a->s.p[l] = s[l];
    a->r.p[l] = R ? R[l] : nullptr;
    a->band_of_layer[l] = (int16_t)band_of_layer[l];
  }
  for (int b = 0; b < G; ++b) {
    if (!aligned16(W0[b])) return false;
    a->W0.p[b] = W0[b];
  }
  for (int b = 0; b <= G; ++b) a->band_start[b] = (int16_t)band_start[b];
  a->L = L;
  a->G = G;
  a->write_r = R != nullptr;
  a->nmax = nmax;
  a->O = O;
  a->I = I;
  a->slots = (int)slots;
  a->slot_bytes = (int)slot;
  a->row_groups = ceil_div(O, rows);
  a->items = (BAND ? G : L) * a->row_groups;
  a->err = c.err;
  *smem = (size_t)slots * slot + 128 + 2 * kMaxSlots * 8;
  const int per_sm = (int)((224 * 1024) / (*smem + 2048));
  int64_t g = (int64_t)c.num_sms * (per_sm < 1 ? 1 : per_sm > 4 ? 4 : per_sm);
  if (g > a->items) g = a->items;
  *grid = (int)g;
  return true;
}

template <typename T, bool BAND>
bool run(const LaunchCtx& c, const void* const* w, int L, int G, const int32_t* band_start,
         const int32_t* band_of_layer, void* const* W0, float* const* s, void* const* R, int64_t O, int64_t I,
         cudaError_t* e) {
  static thread_local PreludeArgs a;  // ~9 KB: kept off the stack
  int tpr, vpt, grid;
  size_t smem;
  if (!plan<T, BAND>(c, w, L, G, band_start, band_of_layer, W0, s, R, O, I, &a, &tpr, &vpt, &grid, &smem))
    return false;
  switch (tpr) {
    case 32: *e = dispatch_vpt<T, BAND, 32>(c, a, vpt, grid, smem); break;
    case 64: *e = dispatch_vpt<T, BAND, 64>(c, a, vpt, grid, smem); break;
    case 128: *e = dispatch_vpt<T, BAND, 128>(c, a, vpt, grid, smem); break;
    default: *e = dispatch_vpt<T, BAND, 256>(c, a, vpt, grid, smem); break;
  }
  return true;
}

// ---------------------------------------------------------------- two-pass
constexpr int64_t kL2Window = 96ll << 20;    // bytes all CTAs hold between the passes
constexpr int64_t kTwoPassMax = 64ll << 20;  // the same with one CTA per SM

// Threads per row: the fewest that keep each thread at <= 4 vectors (<= 8
// for very long rows) with an item of ROWS rows within 32 KB.
bool geometry2(int64_t nv, int64_t row_bytes, int* tpr, int* vpt) {
  *tpr = 0;
  for (int cap : {4, 8})
    for (int c : {32, 64, 128, 256})
      if (!*tpr && ceil_div(nv, c) <= cap && (kConsumers / c) * row_bytes <= 32 * 1024) *tpr = c;
  if (!*tpr) return false;
  const int64_t need = ceil_div(nv, *tpr);
  for (int o : {2, 3, 4, 6, 8})
    if (need <= o) {
      *vpt = o;
      return true;
    }
  return false;
}

template <typename T, int TPR, int VPT, int LPI>
cudaError_t launch_two(const LaunchCtx& c, const PreludeArgs& a, int grid, size_t smem) {
  auto kern = prelude_band2_kernel<T, TPR, VPT, LPI>;
  static int resident[64] = {};  // CTAs per SM (registers and shared memory decide)
  std::unique_lock<std::mutex> lk(setup_mutex());
  if (!resident[c.device]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBudget + 128 + 2 * kMaxSlots * 8);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, kSmemBudget + 128 + 2 * kMaxSlots * 8);
    if (e != cudaSuccess) return e;
    resident[c.device] = n < 1 ? 1 : n;
  }
  const int per_sm = resident[c.device];
  lk.unlock();
  // one wave: a CTA that waited for a slot of the SM would start its units late
  if (grid > c.num_sms * per_sm) grid = c.num_sms * per_sm;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), smem, c.stream, 1, a);
}

template <typename T, int TPR, int LPI>
cudaError_t dispatch_two(const LaunchCtx& c, const PreludeArgs& a, int vpt, int grid, size_t smem) {
  switch (vpt) {
    case 2: return launch_two<T, TPR, 2, LPI>(c, a, grid, smem);
    case 3: return launch_two<T, TPR, 3, LPI>(c, a, grid, smem);
    case 4: return launch_two<T, TPR, 4, LPI>(c, a, grid, smem);
    case 6: return launch_two<T, TPR, 6, LPI>(c, a, grid, smem);
    case 8: return launch_two<T, TPR, 8, LPI>(c, a, grid, smem);
  }
  return cudaErrorInvalidValue;
}

template <typename T, int LPI>
cudaError_t dispatch_two_tpr(const LaunchCtx& c, const PreludeArgs& a, int tpr, int vpt, int grid, size_t smem) {
  switch (tpr) {
    case 32: return dispatch_two<T, 32, LPI>(c, a, vpt, grid, smem);
    case 64: return dispatch_two<T, 64, LPI>(c, a, vpt, grid, smem);
    case 128: return dispatch_two<T, 128, LPI>(c, a, vpt, grid, smem);
    default: return dispatch_two<T, 256, LPI>(c, a, vpt, grid, smem);
  }
}

template <typename T>
bool run_two(const LaunchCtx& c, const void* const* w, int L, int G, const int32_t* band_start,
             const int32_t* band_of_layer, void* const* W0, float* const* s, void* const* R, int64_t O, int64_t I,
             cudaError_t* e) {
  static thread_local PreludeArgs a;
  if (I % Vec<T>::N) return false;
  const int64_t row_bytes = I * (int64_t)sizeof(T);
  int tpr, vpt;
  if (!geometry2(I / Vec<T>::N, row_bytes, &tpr, &vpt)) return false;
  const int rows = kConsumers / tpr;
  // layers per item: as many (4, 2, 1) as keep an item within 32 KB
  int lpi = 4;
  while (lpi > 1 && lpi * rows * row_bytes > 32 * 1024) lpi /= 2;
  const int64_t slot = ceil_div(lpi * rows * row_bytes, 128) * 128;
  int64_t slots = kSmemBudget / slot;
  if (slots > kMaxSlots) slots = kMaxSlots;
  if (slots < 2 || row_bytes % 16) return false;
  int nmax = 1;
  for (int b = 0; b < G; ++b) nmax = max(nmax, band_start[b + 1] - band_start[b]);
  // with one CTA per SM, a unit's rows must leave room in L2 for everything
  // else, or pass 2 goes back to HBM and the band-mean + row-pass route wins
  const int64_t unit_bytes = (int64_t)nmax * rows * row_bytes;
  if (unit_bytes * c.num_sms > kTwoPassMax) return false;
  for (int l = 0; l < L; ++l) {
    if (!aligned16(w[l]) || (R && !aligned16(R[l]))) return false;
    a.w.p[l] = w[l];
    a.s.p[l] = s[l];
    a.r.p[l] = R ? R[l] : nullptr;
    a.band_of_layer[l] = (int16_t)band_of_layer[l];
  }
  for (int b = 0; b < G; ++b) {
    if (!aligned16(W0[b])) return false;
    a.W0.p[b] = W0[b];
  }
  for (int b = 0; b <= G; ++b) a.band_start[b] = (int16_t)band_start[b];
  a.L = L;
  a.G = G;
  a.write_r = R != nullptr;
  a.nmax = nmax;
  a.O = O;
  a.I = I;
  a.slots = (int)slots;
  a.slot_bytes = (int)slot;
  a.row_groups = ceil_div(O, rows);
  a.items = G * a.row_groups;  // units (band, row group)
  a.err = c.err;
  const size_t smem = (size_t)slots * slot + 128 + 2 * kMaxSlots * 8;
  const int per_sm = (int)((224 * 1024) / (smem + 2048));
  int64_t g = (int64_t)c.num_sms * (per_sm < 1 ? 1 : per_sm > 2 ? 2 : per_sm);
  // keep the rows read in pass 1 and read again in pass 2 inside L2
  const int64_t by_l2 = kL2Window / unit_bytes;
  if (g > by_l2) g = by_l2 < 1 ? 1 : by_l2;
  if (g > a.items) g = a.items;
  switch (lpi) {
    case 4: *e = dispatch_two_tpr<T, 4>(c, a, tpr, vpt, (int)g, smem); break;
    case 2: *e = dispatch_two_tpr<T, 2>(c, a, tpr, vpt, (int)g, smem); break;
    default: *e = dispatch_two_tpr<T, 1>(c, a, tpr, vpt, (int)g, smem); break;
  }
  return true;
}

}  // namespace

bool launch_prelude_pipe(const LaunchCtx& c, theta_dtype dt, int mode, const void* const* w, int L, int G,
                         const int32_t* band_start, const int32_t* band_of_layer, void* const* W0,
                         float* const* s, void* const* R, int64_t O, int64_t I, cudaError_t* e) {
  if (mode == PRELUDE_TWO_PASS)
    return dt == THETA_BF16 ? run_two<bf16>(c, w, L, G, band_start, band_of_layer, W0, s, R, O, I, e)
                            : run_two<float>(c, w, L, G, band_start, band_of_layer, W0, s, R, O, I, e);
  const bool band_mode = mode == PRELUDE_BAND;
  if (dt == THETA_BF16)
    return band_mode ? run<bf16, true>(c, w, L, G, band_start, band_of_layer, W0, s, R, O, I, e)
                     : run<bf16, false>(c, w, L, G, band_start, band_of_layer, W0, s, R, O, I, e);
  return band_mode ? run<float, true>(c, w, L, G, band_start, band_of_layer, W0, s, R, O, I, e)
                   : run<float, false>(c, w, L, G, band_start, band_of_layer, W0, s, R, O, I, e);
}

}  // namespace theta
