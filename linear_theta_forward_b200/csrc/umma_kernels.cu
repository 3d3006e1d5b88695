// Tensor-core (tcgen05) kernels of the bf16 theta path on sm_100a.
//
// One warp-specialised kernel template computes a 128 x BN tile of
//     D1 = A1 . B1^T   (phase 1, K = the contraction of the projection)
//     D2 = A2 . (B2 + B3)^T   (phase 2, K = rank; only the forward uses it)
// with fp32 accumulators in tensor memory, operands staged by TMA into a
// ring of 128-byte-swizzled shared-memory stages:
//   warp 0  TMA producer (one lane)
//   warp 1  tensor-memory allocator and MMA issuer (one lane)
//   warps 2-5  epilogue: tcgen05.ld of their 32-lane quarter of D1/D2
// Two epilogues ("The theta bundle" -- approximation formula):
//   FORWARD  Y[m, o] = s[o] * D1[o, m] + D2[o, m]   with A1 = W0, B1 = X,
//            A2 = U, B2/B3 = high/low bf16 parts of T = X.V  (swap-AB: the
//            weight rows fill the 128-row MMA side, tokens are N)
//   XV       T_hi/T_lo[m, j] from D1[m, j]           with A1 = X, B1 = V (MN-major)
// When the tiles alone cannot fill the GPU, K is split across the CTAs of a
// thread-block cluster (up to 16); the partial tiles are summed in a fixed
// order through distributed shared memory (deterministic, no global scratch).
//
// reconstruct_weight has its own kernel (recon_kernel): the K = rank MMA
// U.V^T into tensor memory, the W0 tile brought in by TMA next to U and V,
// s*W0 + U.V^T combined in swizzled shared memory and written back by a TMA
// store, so both HBM streams (W0 in, W out) move as whole tiles.
//
// All kernels are launched with programmatic dependent launch: their
// prologue (barrier init, tensor-memory allocation) overlaps the previous
// kernel, and griddepcontrol.wait precedes every global memory access.
//
// Every wait is bounded (kWaitLimitNs); a wait that gives up records a
// device error flag, raises a CTA-wide abort so the other roles stop, and the
// kernel drains its own TMA loads and MMAs before releasing tensor memory.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "umma_ptx.cuh"

namespace theta {

namespace {

enum Mode { MODE_FORWARD = 0, MODE_XV = 1, MODE_GATE_UP = 2 };

constexpr int kThreads = 192;
constexpr int kBM = 128;       // MMA M (rows of A)
constexpr int kBK = 64;        // K per stage: one 128-byte swizzle atom of bf16
constexpr int kABytes = kBM * kBK * 2;
constexpr int kPitch = 129;    // fp32 pitch of the split-K partial tiles (bank-conflict free)

struct Args {
  int rows;        // valid rows of the A side (O, or M tokens for XV)
  int cols;        // valid columns of the B side (M tokens, or rank)
  int kb1;         // K blocks of phase 1
  int kb2;         // K blocks of phase 2 (0: none)
  int splits;      // cluster size along x (split-K)
  const float* s;  // FORWARD row scale (GATE_UP: of the gate projection)
  const float* s_up;  // GATE_UP: row scale of the up projection
  bf16* out;       // FORWARD, GATE_UP: Y [cols, rows]
  bf16* t_hi;      // XV outputs [rows, r]
  bf16* t_lo;
  int r;
  int early_start;  // FORWARD after its own T = X.V kernel: see the producer
  unsigned* err;
};

template <int BN, int MODE>
struct Cfg {
  static constexpr int kBBytes = BN * kBK * 2;  // XV: BN = padded rank, MN-major atoms of 64 columns
  static constexpr int kNumA = MODE == MODE_GATE_UP ? 2 : 1;  // A tiles per phase-1 stage
  static constexpr int kStageBytes = kNumA * kABytes + kBBytes;
  // small rings for small BN so 2-3 decode CTAs share an SM
  // GATE_UP (two A tiles per stage): two CTAs per SM up to 64 tokens, a deep
  // ring for the one CTA per SM of 128-token tiles
  static constexpr int kStages = MODE == MODE_GATE_UP ? (BN == 128 ? 4 : BN == 64 ? 2 : 3)
                                 : (BN == 128 || (MODE == MODE_XV && BN > 128)) ? 3 : 4;
  // FORWARD: D1, D2; GATE_UP: D1 gate, D1 up, D2 gate, D2 up; XV: D1
  static constexpr int kTmemNeed = MODE == MODE_FORWARD ? 2 * BN : MODE == MODE_GATE_UP ? 4 * BN : BN;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  static_assert(kTmemNeed <= 512, "accumulators must fit in tensor memory");
  // split-K partial tiles: one per output (GATE_UP: gate and up pre-activations)
  static constexpr int kPartialBytes = kNumA * BN * kPitch * 4;
  static_assert(kPartialBytes <= kStages * kStageBytes, "partial tile must fit in the stage ring");
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
};

// GELU in its tanh form, the activation of the Gemma MLPs:
// 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
__device__ __forceinline__ float gelu_tanh(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * x * (1.f + tanhf(k0 * fmaf(0.044715f * x, x * x, x)));
}

template <int BN, int MODE>
__global__ void __launch_bounds__(kThreads)
umma_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
            const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
            const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmA1u,
            const __grid_constant__ CUtensorMap tmA2u, const __grid_constant__ CUtensorMap tmB2u,
            const __grid_constant__ CUtensorMap tmB3u, const Args args) {
  using C = Cfg<BN, MODE>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* accum = empty + S;
  uint64_t* drain = accum + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int split = args.splits > 1 ? (int)ptx::cluster_ctarank() : 0;
  const int n_tile = blockIdx.x / args.splits;
  const int m_tile = blockIdx.y;
  const int kb_begin = (int)((int64_t)split * args.kb1 / args.splits);
  const int kb_end = (int)((int64_t)(split + 1) * args.kb1 / args.splits);
  constexpr bool kFwd = MODE == MODE_FORWARD || MODE == MODE_GATE_UP;
  const bool has_d2 = kFwd && args.kb2 > 0 && split == 0;
  const int n1 = kb_end - kb_begin;
  // phase 2 items: (high, low) parts of T per projection
  const int total = n1 + (has_d2 ? 2 * C::kNumA * args.kb2 : 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(accum, 1);
    ptx::mbar_init(drain, 1);
    *abort_flag = prior_timeout(args.err);
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Programmatic dependent launch. Normally every thread waits here for the
  // previous grid before touching global memory, and only then lets the next
  // grid launch -- so a grid that lets its dependent start has itself seen
  // all earlier work complete. A forward launched right after its own
  // T = X.V kernel relies on exactly that: it starts early, streaming W0, X
  // and s at once (that kernel writes only T), and waits only before the
  // loads of T (the producer's rank phase) and in the epilogue.
  const bool early = kFwd && args.early_start;
  if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  auto give_up = [&]() {
    record_timeout(args.err);
    *abort_flag = 1;
  };

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    ptx::prefetch_tmap(&tmA1);
    ptx::prefetch_tmap(&tmB1);
    int issued = 0;
    for (int i = 0; i < total; ++i) {
      const int st = i % S;
      const uint32_t ph = (uint32_t)(i / S) & 1u;
      if (!ptx::mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
        give_up();
        break;
      }
      uint8_t* a = smem + st * C::kStageBytes;
      uint8_t* b = a + C::kNumA * kABytes;
      // phase 1 brings kNumA A tiles and the B tile; a phase-2 item one of each
      ptx::mbar_arrive_expect_tx(&full[st], i < n1 ? C::kStageBytes : kABytes + C::kBBytes);
      if (i < n1) {
        const int kx = (kb_begin + i) * kBK;
        ptx::tma_load_2d(a, &tmA1, &full[st], kx, m_tile * kBM);
        if constexpr (MODE == MODE_GATE_UP) ptx::tma_load_2d(a + kABytes, &tmA1u, &full[st], kx, m_tile * kBM);
        if constexpr (MODE == MODE_XV) {
          // V [I, r] row-major is MN-major for B: one box of 64 rank columns
          // x 64 rows of I per 64-wide column atom
#pragma unroll
          for (int at = 0; at < BN / 64; ++at) ptx::tma_load_2d(b + at * 64 * 128, &tmB1, &full[st], at * 64, kx);
        } else {
          ptx::tma_load_2d(b, &tmB1, &full[st], kx, n_tile * BN);
        }
      } else {
        const int j = i - n1;
        if (early && j == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        const int jx = (j % args.kb2) * kBK;
        const int part = j / args.kb2;  // 0, 1: gate (or the forward) T high, low; 2, 3: up T high, low
        const CUtensorMap* mA = part < 2 ? &tmA2 : &tmA2u;
        const CUtensorMap* mB = part == 0 ? &tmB2 : part == 1 ? &tmB3 : part == 2 ? &tmB2u : &tmB3u;
        ptx::tma_load_2d(a, mA, &full[st], jx, m_tile * kBM);
        ptx::tma_load_2d(b, mB, &full[st], jx, n_tile * BN);
      }
      ++issued;
    }
    // drain: wait for the last armed phase of every stage (all loads landed)
    for (int st = 0; st < S && st < issued; ++st) {
      const int last = st + ((issued - 1 - st) / S) * S;
      if (!ptx::mbar_wait(&full[st], (uint32_t)(last / S) & 1u, abort_flag)) {
        // loads still in flight after an abort: keep waiting, bounded, without the abort shortcut
        int never = 0;
        ptx::mbar_wait(&full[st], (uint32_t)(last / S) & 1u, &never);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc1 = ptx::idesc_bf16(kBM, BN, MODE == MODE_XV ? 1 : 0);
    constexpr uint32_t idesc2 = ptx::idesc_bf16(kBM, BN, 0);
    int done = 0;
    for (int i = 0; i < total; ++i) {
      const int st = i % S;
      const uint32_t ph = (uint32_t)(i / S) & 1u;
      if (!ptx::mbar_wait(&full[st], ph, abort_flag)) {
        give_up();
        break;
      }
      ptx::tc_fence_after();
      const uint32_t a = ptx::smem_u32(smem + st * C::kStageBytes);
      const uint32_t b = a + C::kNumA * kABytes;
      if (i < n1) {
        // tensor memory: D1 (GATE_UP: D1 gate at 0, D1 up at BN)
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = ptx::sdesc_sw128(a + kk * 32, 16, 1024);
          const uint64_t bd = MODE == MODE_XV ? ptx::sdesc_sw128(b + kk * 16 * 128, 64 * 128, 1024)
                                              : ptx::sdesc_sw128(b + kk * 32, 16, 1024);
          ptx::umma_bf16(tmem, ad, bd, idesc1, (i > 0 || kk > 0) ? 1u : 0u);
          if constexpr (MODE == MODE_GATE_UP)
            ptx::umma_bf16(tmem + BN, ptx::sdesc_sw128(a + kABytes + kk * 32, 16, 1024), bd, idesc1,
                           (i > 0 || kk > 0) ? 1u : 0u);
        }
      } else {
        // D2 after the D1 accumulators (GATE_UP: gate items first, then up)
        const int j = i - n1;
        const int jd = j % (2 * args.kb2);  // item within its accumulator
        const uint32_t d2 = tmem + (uint32_t)(C::kNumA * BN) + (uint32_t)(j / (2 * args.kb2)) * BN;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = ptx::sdesc_sw128(a + kk * 32, 16, 1024);
          const uint64_t bd = ptx::sdesc_sw128(b + kk * 32, 16, 1024);
          ptx::umma_bf16(d2, ad, bd, idesc2, (jd > 0 || kk > 0) ? 1u : 0u);
        }
      }
      ptx::umma_commit(&empty[st]);
      ++done;
    }
    if (done == total) {
      ptx::umma_commit(accum);
    } else if (done > 0) {
      // aborted: make sure the issued MMAs finish before tensor memory is freed
      ptx::umma_commit(drain);
      int never = 0;
      ptx::mbar_wait(drain, 0, &never);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // accumulator row = TMEM lane
    const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
    if (early) asm volatile("griddepcontrol.wait;" ::: "memory");
    bool ok = ptx::mbar_wait(accum, 0, abort_flag);
    if (!ok) give_up();
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    ptx::tc_fence_after();
    const int grow = m_tile * kBM + row;  // global row of A
    const int col0 = n_tile * BN;
    const int ncols = min(BN, args.cols - col0);
    float so = 0.f, su = 0.f;
    if constexpr (kFwd) so = (grow < args.rows) ? __ldg(args.s + grow) : 0.f;
    if constexpr (MODE == MODE_GATE_UP) su = (grow < args.rows) ? __ldg(args.s_up + grow) : 0.f;
    float* part = reinterpret_cast<float*>(smem);
    if (ok && MODE == MODE_GATE_UP) {
      // gate g = s_g D1g + D2g and up u = s_u D1u + D2u; Y = gelu_tanh(g) u
      for (int c0 = 0; c0 < ncols; c0 += 16) {
        float g1[16], u1[16], g2[16], u2[16];
        ptx::tmem_ld16(taddr + c0, g1);
        ptx::tmem_ld16(taddr + BN + c0, u1);
        if (has_d2) {
          ptx::tmem_ld16(taddr + 2 * BN + c0, g2);
          ptx::tmem_ld16(taddr + 3 * BN + c0, u2);
        }
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float g = has_d2 ? fmaf(so, g1[e], g2[e]) : so * g1[e];
          const float u = has_d2 ? fmaf(su, u1[e], u2[e]) : su * u1[e];
          if (args.splits > 1) {
            part[(c0 + e) * kPitch + row] = g;
            part[(BN + c0 + e) * kPitch + row] = u;
          } else {
            const int m = col0 + c0 + e;
            if (grow < args.rows && m < args.cols)
              args.out[(int64_t)m * args.rows + grow] = __float2bfloat16_rn(gelu_tanh(g) * u);
          }
        }
      }
    } else if (ok) {
      for (int c0 = 0; c0 < ncols; c0 += 16) {
        float d1[16], d2[16];
        ptx::tmem_ld16(taddr + c0, d1);
        if (has_d2) ptx::tmem_ld16(taddr + BN + c0, d2);
        ptx::tmem_wait_ld();
        if (args.splits > 1) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float v = d1[e];
            if constexpr (MODE == MODE_FORWARD) v = has_d2 ? fmaf(so, d1[e], d2[e]) : so * d1[e];
            part[(c0 + e) * kPitch + row] = v;
          }
        } else if (grow < args.rows) {
          if constexpr (MODE == MODE_FORWARD) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int m = col0 + c0 + e;
              if (m < args.cols) {
                const float v = has_d2 ? fmaf(so, d1[e], d2[e]) : so * d1[e];
                args.out[(int64_t)m * args.rows + grow] = __float2bfloat16_rn(v);
              }
            }
          } else if constexpr (MODE == MODE_XV) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int j = col0 + c0 + e;
              if (j < args.r) {
                const bf16 hi = __float2bfloat16_rn(d1[e]);
                args.t_hi[(int64_t)grow * args.r + j] = hi;
                args.t_lo[(int64_t)grow * args.r + j] = __float2bfloat16_rn(d1[e] - __bfloat162float(hi));
              }
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ split-K sum
  __syncwarp();
  if (args.splits > 1) {
    ptx::cluster_sync();  // every CTA of the cluster has staged its partial tile
    if (!*abort_flag) {
      const int col0 = n_tile * BN;
      const int ncols = min(BN, args.cols - col0);
      const int E = ncols * kBM;
      const int e0 = (int)((int64_t)split * E / args.splits), e1 = (int)((int64_t)(split + 1) * E / args.splits);
      const uint32_t part_addr = ptx::smem_u32(smem);
      for (int e = e0 + threadIdx.x; e < e1; e += kThreads) {
        const int c = e / kBM, rr = e % kBM;
        const uint32_t off = part_addr + (uint32_t)((c * kPitch + rr) * 4);
        float v = 0.f;
        for (int p = 0; p < args.splits; ++p) v += ptx::ld_dsmem_f32(ptx::mapa(off, (uint32_t)p));
        const int grow = m_tile * kBM + rr;
        if (grow >= args.rows) continue;
        if constexpr (MODE == MODE_FORWARD) {
          args.out[(int64_t)(col0 + c) * args.rows + grow] = __float2bfloat16_rn(v);
        } else if constexpr (MODE == MODE_GATE_UP) {
          // v is the gate pre-activation; the up one is the tile BN columns further
          const uint32_t off_u = off + (uint32_t)(BN * kPitch * 4);
          float u = 0.f;
          for (int p = 0; p < args.splits; ++p) u += ptx::ld_dsmem_f32(ptx::mapa(off_u, (uint32_t)p));
          args.out[(int64_t)(col0 + c) * args.rows + grow] = __float2bfloat16_rn(gelu_tanh(v) * u);
        } else if constexpr (MODE == MODE_XV) {
          const int j = col0 + c;
          if (j < args.r) {
            const bf16 hi = __float2bfloat16_rn(v);
            args.t_hi[(int64_t)grow * args.r + j] = hi;
            args.t_lo[(int64_t)grow * args.r + j] = __float2bfloat16_rn(v - __bfloat162float(hi));
          }
        }
      }
    }
    ptx::cluster_sync();  // no CTA leaves while a peer still reads its tile
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::kTmemCols);
}

// ------------------------------------------------------------ CTA-pair tiles
// The FORWARD and GATE_UP epilogues over 256-row tiles on pairs of SMs: the
// two CTAs of a cluster of two share each tcgen05 MMA of M = 256 weight rows
// (cta_group::2), issued by the even CTA. Each CTA stages its own half of
// both operands -- 128 weight rows (of each projection) and half the tile's
// tokens per 64-wide K block -- and receives its 128 rows of every
// accumulator in its own tensor memory. FORWARD tiles are 256 tokens wide
// (D1, D2: 2 x 256 columns), GATE_UP tiles 128 (D1 and D2 of the gate and of
// the up projection: 4 x 128 columns). Per K block an SM takes in two thirds
// (FORWARD) or five sixths (GATE_UP) of what a one-SM tile of the same
// tensor work does.
//
// The kernel is persistent: a cluster walks the tiles c, c + clusters, ...
// Its producers load the next tile's stages while the epilogue still works
// on the current one, and the epilogue hands tensor memory back as soon as it
// has moved the tile into shared memory (rounded to bf16 as [token][row], the
// layout of Y), before one TMA store writes it out. So between two tiles the
// tensor pipe waits only for that drain, not for a CTA to finish, launch and
// fill its pipeline.
//
// Each CTA's producer signals the even CTA's full barrier (which expects
// both halves); MMA completion is committed to the empty and accumulator
// barriers of both CTAs; the epilogue warps of both CTAs arrive on the even
// CTA's tensor-memory-free barrier.
template <int MODE>
struct PairCfg {
  static constexpr int kNumA = MODE == MODE_GATE_UP ? 2 : 1;  // weight tiles per phase-1 stage
  static constexpr int kN = MODE == MODE_GATE_UP ? 128 : 256;  // tokens per tile: MMA N
  static constexpr int kHalf = kN / 2;                         // tokens staged by each CTA
  static constexpr int kBBytes = kHalf * kBK * 2;
  static constexpr int kStageBytes = kNumA * kABytes + kBBytes;
  static constexpr int kStages = MODE == MODE_GATE_UP ? 4 : 5;
  static constexpr int kOutBytes = kBM * kN * 2;  // a CTA's Y tile, bf16 [token][row]
  static constexpr int kTmemCols = 2 * kNumA * kN;  // D1 (per projection), then D2 (per projection)
  static_assert(kTmemCols == 512, "the accumulators fill tensor memory");
  static constexpr int kSmemBytes = kStages * kStageBytes + kOutBytes + 1024 /*align*/ + 256 /*barriers*/;
  // warps 0 (TMA) and 1 (MMA), then the epilogue: one warp per 32-lane
  // quarter of tensor memory for FORWARD; two for GATE_UP, each draining half
  // of the tile's columns, since its GELU makes the drain several times
  // longer (measured: eight warps slow the forward by 5%, speed gate/up up)
  static constexpr int kEpiWarps = MODE == MODE_GATE_UP ? 8 : 4;
  static constexpr int kEpi = 32 * kEpiWarps;
  static constexpr int kThreads = 64 + kEpi;
};
constexpr uint16_t kPairMask = 0x3;  // both CTAs of the cluster

template <int MODE>
__global__ void __launch_bounds__(PairCfg<MODE>::kThreads)
pair_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
            const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
            const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmA1u,
            const __grid_constant__ CUtensorMap tmA2u, const __grid_constant__ CUtensorMap tmB2u,
            const __grid_constant__ CUtensorMap tmB3u, const __grid_constant__ CUtensorMap tmY, const Args args) {
  using C = PairCfg<MODE>;
  constexpr int S = C::kStages;
  constexpr int N = C::kN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  bf16* sOut = reinterpret_cast<bf16*>(smem + S * C::kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kOutBytes);
  uint64_t* empty = full + S;
  uint64_t* accum = empty + S;
  uint64_t* tmem_free = accum + 1;
  uint64_t* drain = tmem_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t cta = ptx::cluster_ctarank();  // 0 issues the MMAs
  const int cluster = blockIdx.x / 2, n_clusters = gridDim.x / 2;
  const int n_tiles = (args.cols + N - 1) / N;  // token tiles
  const int tiles = n_tiles * ((args.rows + 2 * kBM - 1) / (2 * kBM));
  const bool has_d2 = args.kb2 > 0;
  const int n1 = args.kb1;
  const int per_tile = n1 + (has_d2 ? 2 * C::kNumA * args.kb2 : 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(accum, 1);
    ptx::mbar_init(tmem_free, 2 * C::kEpiWarps);  // one arrival per epilogue warp of both CTAs
    ptx::mbar_init(drain, 1);
    *abort_flag = prior_timeout(args.err);
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // both CTAs' barriers exist before either signals the other's
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // programmatic dependent launch as in umma_kernel: after its own T = X.V
  // kernels the forward streams W0 and X at once and waits before T
  const bool early = args.early_start;
  if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  auto give_up = [&]() {
    record_timeout(args.err);
    *abort_flag = 1;
  };

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer (both CTAs)
    ptx::prefetch_tmap(&tmA1);
    ptx::prefetch_tmap(&tmB1);
    const uint32_t full0 = ptx::mapa(ptx::smem_u32(full), 0);  // the MMA CTA's full barriers
    bool waited = !early, stop = false;
    int g = 0;  // stage items issued, over all tiles
    for (int tile = cluster; tile < tiles && !stop; tile += n_clusters) {
      const int row0 = (tile / n_tiles) * (2 * kBM) + (int)cta * kBM;
      const int tok0 = (tile % n_tiles) * N + (int)cta * C::kHalf;
      for (int i = 0; i < per_tile; ++i, ++g) {
        const int st = g % S;
        const uint32_t ph = (uint32_t)(g / S) & 1u;
        if (!ptx::mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
          give_up();
          stop = true;
          break;
        }
        uint8_t* a = smem + st * C::kStageBytes;
        uint8_t* b = a + C::kNumA * kABytes;
        const uint32_t bar = full0 + (uint32_t)(st * 8);
        if constexpr (MODE == MODE_FORWARD) {
          // both halves; phase-1 and phase-2 items move the same bytes
          if (cta == 0) ptx::mbar_arrive_expect_tx(&full[st], 2 * C::kStageBytes);
          if (i < n1) {
            ptx::tma_load_2d_pair(a, &tmA1, bar, i * kBK, row0);
            ptx::tma_load_2d_pair(b, &tmB1, bar, i * kBK, tok0);
          } else {
            const int j = i - n1;
            if (!waited) {
              asm volatile("griddepcontrol.wait;" ::: "memory");
              waited = true;
            }
            const int jx = (j % args.kb2) * kBK;
            ptx::tma_load_2d_pair(a, &tmA2, bar, jx, row0);
            ptx::tma_load_2d_pair(b, j < args.kb2 ? &tmB2 : &tmB3, bar, jx, tok0);
          }
        } else if (i < n1) {
          // both halves: every weight tile and the token tile of each CTA
          if (cta == 0) ptx::mbar_arrive_expect_tx(&full[st], 2 * C::kStageBytes);
          ptx::tma_load_2d_pair(a, &tmA1, bar, i * kBK, row0);
          ptx::tma_load_2d_pair(a + kABytes, &tmA1u, bar, i * kBK, row0);
          ptx::tma_load_2d_pair(b, &tmB1, bar, i * kBK, tok0);
        } else {
          // one U tile and one part of T: (high, low) of the gate projection,
          // then (high, low) of the up projection
          const int j = i - n1;
          if (!waited) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            waited = true;
          }
          const int jx = (j % args.kb2) * kBK;
          const int part = j / args.kb2;
          if (cta == 0) ptx::mbar_arrive_expect_tx(&full[st], 2 * (kABytes + C::kBBytes));
          ptx::tma_load_2d_pair(a, part < 2 ? &tmA2 : &tmA2u, bar, jx, row0);
          const CUtensorMap* mB = part == 0 ? &tmB2 : part == 1 ? &tmB3 : part == 2 ? &tmB2u : &tmB3u;
          ptx::tma_load_2d_pair(b, mB, bar, jx, tok0);
        }
      }
    }
    // drain: the MMAs that read a stage's last loads complete after those
    // loads landed, and their commit reaches empty[] in both CTAs. After an
    // abort, loads still in flight land within microseconds: wait a bounded
    // tenth of a second for them without the abort shortcut.
    for (int st = 0; st < S && st < g; ++st) {
      const int last = st + ((g - 1 - st) / S) * S;
      if (!ptx::mbar_wait(&empty[st], (uint32_t)(last / S) & 1u, abort_flag)) {
        int never = 0;
        ptx::mbar_wait(&empty[st], (uint32_t)(last / S) & 1u, &never, 100000000ull);
      }
    }
  } else if (warp == 1 && lane == 0 && cta == 0) {
    // ---------------------------------------------------------- MMA issuer (even CTA)
    constexpr uint32_t idesc = ptx::idesc_bf16(2 * kBM, N, 0);
    bool stop = false;
    int g = 0, j = 0, issued = 0;
    for (int tile = cluster; tile < tiles; tile += n_clusters, ++j) {
      // the epilogues of both CTAs have read the previous tile's accumulators
      if (j > 0 && !ptx::mbar_wait(tmem_free, (uint32_t)(j - 1) & 1u, abort_flag)) {
        give_up();
        stop = true;
        break;
      }
      ptx::tc_fence_after();
      for (int i = 0; i < per_tile; ++i, ++g) {
        const int st = g % S;
        const uint32_t ph = (uint32_t)(g / S) & 1u;
        if (!ptx::mbar_wait(&full[st], ph, abort_flag)) {
          give_up();
          stop = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a = ptx::smem_u32(smem + st * C::kStageBytes);
        const uint32_t b = a + C::kNumA * kABytes;
        if constexpr (MODE == MODE_FORWARD) {
          // D1 = W0 . X^T over K = I at column 0; D2 = U . (T_hi + T_lo)^T at N
          const uint32_t d = i < n1 ? tmem : tmem + (uint32_t)N;
          const bool first = i == 0 || i == n1;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            ptx::umma_bf16_pair(d, ptx::sdesc_sw128(a + kk * 32, 16, 1024), ptx::sdesc_sw128(b + kk * 32, 16, 1024),
                                idesc, (!first || kk > 0) ? 1u : 0u);
        } else if (i < n1) {
          // D1 of projection q at column q * N, over K = I
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = ptx::sdesc_sw128(b + kk * 32, 16, 1024);
#pragma unroll
            for (int q = 0; q < C::kNumA; ++q)
              ptx::umma_bf16_pair(tmem + (uint32_t)(q * N), ptx::sdesc_sw128(a + q * kABytes + kk * 32, 16, 1024),
                                  bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
          // D2 of projection q at column (kNumA + q) * N: U . (T_hi + T_lo)^T
          const int jj = i - n1;
          const int q = jj / (2 * args.kb2);
          const int jd = jj % (2 * args.kb2);  // item within its accumulator
          const uint32_t d2 = tmem + (uint32_t)((C::kNumA + q) * N);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            ptx::umma_bf16_pair(d2, ptx::sdesc_sw128(a + kk * 32, 16, 1024), ptx::sdesc_sw128(b + kk * 32, 16, 1024),
                                idesc, (jd > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit_pair(&empty[st], kPairMask);
        ++issued;
      }
      if (stop) break;
      ptx::umma_commit_pair(accum, kPairMask);
    }
    if (stop && issued > 0) {
      // aborted: the issued MMAs finish before tensor memory is released
      ptx::umma_commit_pair(drain, 0x1);
      int never = 0;
      ptx::mbar_wait(drain, 0, &never);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;          // a warp reads lanes 32 * (warp % 4) ...
    const int part = (warp - 2) / 4;       // ... and columns [part * W, (part + 1) * W)
    constexpr int W = N * 4 / C::kEpiWarps;  // columns per epilogue warp
    const int row = quarter * 32 + lane;  // accumulator row = TMEM lane
    const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool storer = threadIdx.x == 64;  // issues the TMA stores of the tile
    const uint32_t free_bar = ptx::mapa(ptx::smem_u32(tmem_free), 0);
    if (early) asm volatile("griddepcontrol.wait;" ::: "memory");
    bool ok = true;
    int j = 0;
    for (int tile = cluster; tile < tiles; tile += n_clusters, ++j) {
      const int row0 = (tile / n_tiles) * (2 * kBM) + (int)cta * kBM;
      const int col0 = (tile % n_tiles) * N;
      const int ncols = min(N, args.cols - col0);
      if (storer) ptx::bulk_wait_read();  // the previous tile's store has read sOut
      const bool got = ptx::mbar_wait(accum, (uint32_t)j & 1u, abort_flag);
      // one decision for all epilogue warps: the barriers below need every one of them
      ok = ptx::bar_red_and(1, C::kEpi, got);
      if (!ok) break;
      ptx::tc_fence_after();
      const int grow = row0 + row;
      const float so = (grow < args.rows) ? __ldg(args.s + grow) : 0.f;
      float su = 0.f;
      if constexpr (MODE == MODE_GATE_UP) su = (grow < args.rows) ? __ldg(args.s_up + grow) : 0.f;
      const int c_begin = C::kEpiWarps == 4 ? 0 : part * W;
      const int c_end = C::kEpiWarps == 4 ? ncols : min(ncols, (part + 1) * W);
      for (int c0 = c_begin; c0 < c_end; c0 += 16) {
        if constexpr (MODE == MODE_GATE_UP) {
          // gate g = s_g D1g + D2g and up u = s_u D1u + D2u; Y = gelu_tanh(g) u
          float g1[16], u1[16], g2[16], u2[16];
          ptx::tmem_ld16(taddr + c0, g1);
          ptx::tmem_ld16(taddr + N + c0, u1);
          if (has_d2) {
            ptx::tmem_ld16(taddr + 2 * N + c0, g2);
            ptx::tmem_ld16(taddr + 3 * N + c0, u2);
          }
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float gv = has_d2 ? fmaf(so, g1[e], g2[e]) : so * g1[e];
            const float uv = has_d2 ? fmaf(su, u1[e], u2[e]) : su * u1[e];
            sOut[(c0 + e) * kBM + row] = __float2bfloat16_rn(gelu_tanh(gv) * uv);
          }
        } else {
          float d1[16], d2[16];
          ptx::tmem_ld16(taddr + c0, d1);
          if (has_d2) ptx::tmem_ld16(taddr + N + c0, d2);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            sOut[(c0 + e) * kBM + row] = __float2bfloat16_rn(has_d2 ? fmaf(so, d1[e], d2[e]) : so * d1[e]);
        }
      }
      // tensor memory read: the next tile's MMAs may start
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(free_bar);
      ptx::fence_proxy_async_smem();
      asm volatile("bar.sync 1, %0;" ::"n"(C::kEpi) : "memory");
      if (storer) {
        // rows past O and tokens past M fall outside Y and are not written
        ptx::tma_store_2d(&tmY, sOut, row0, col0);
        ptx::bulk_commit();
      }
    }
    if (!ok && !*abort_flag) give_up();
    if (storer) ptx::bulk_wait_all();
  }

  __syncwarp();
  ptx::tc_fence_before();
  ptx::cluster_sync();  // both epilogues have read their accumulators; every MMA has completed
  if (warp == 1) ptx::tmem_dealloc_pair(tmem, C::kTmemCols);
}

// s (.) W0 for rank 0 (no tensor-core work).
__global__ void __launch_bounds__(256) scale_rows_kernel(const float* __restrict__ s, const bf16* __restrict__ W0,
                                                         int64_t I, int64_t nvec, bf16* __restrict__ out) {
  pdl_enter(s, W0);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t per_row = I / 8;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    const float sc = __ldg(s + v / per_row);
    float w[8], o[8];
    unpack(__ldg(reinterpret_cast<const uint4*>(W0) + v), w);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = sc * w[e];
    reinterpret_cast<uint4*>(out)[v] = pack(o, (uint4*)nullptr);
  }
}

// ------------------------------------------------------------- reconstruct
// One 128 x kRecN tile of W = diag(s).W0 + U.V^T. 128 threads: thread 0 issues
// the TMA loads (U and V rank blocks on one barrier, the W0 tile on another)
// and the final TMA store; thread 32 issues the K = rank MMAs; then all four
// warps read their 32-lane quarter of U.V^T from tensor memory, combine it
// with s * W0 in place in the swizzled W0 tile, and the tile is stored.
constexpr int kRecThreads = 128;
constexpr int kRecN = 128;  // columns of W per tile

template <int KB>
struct RecCfg {
  static constexpr int kUBlock = kBM * 128;              // U: 128 rows x 64 rank columns (bf16)
  static constexpr int kVBlock = kRecN * 128;            // V: kRecN rows x 64 rank columns
  static constexpr int kUBytes = KB * kUBlock;
  static constexpr int kVBytes = KB * kVBlock;
  static constexpr int kWBytes = (kRecN / kBK) * kABytes;  // W0 / output tile: kRecN / 64 column boxes
  static constexpr int kSmemBytes = kUBytes + kVBytes + kWBytes + 1024 + 128;
};

template <int KB>
__global__ void __launch_bounds__(kRecThreads)
recon_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmV,
             const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmOut,
             const float* __restrict__ s, int O, int I, unsigned* err) {
  using C = RecCfg<KB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sU = smem;
  uint8_t* sV = smem + C::kUBytes;
  uint8_t* sW = sV + C::kVBytes;
  uint64_t* bar_uv = reinterpret_cast<uint64_t*>(sW + C::kWBytes);
  uint64_t* bar_w = bar_uv + 1;
  uint64_t* bar_acc = bar_w + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_acc + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i0 = blockIdx.x * kRecN, o0 = blockIdx.y * kBM;
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_uv, 1);
    ptx::mbar_init(bar_w, 1);
    ptx::mbar_init(bar_acc, 1);
    *abort_flag = prior_timeout(err);
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kRecN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_enter(s);

  if (threadIdx.x == 0) {
    ptx::mbar_arrive_expect_tx(bar_uv, C::kUBytes + C::kVBytes);
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
      ptx::tma_load_2d(sU + kb * C::kUBlock, &tmU, bar_uv, kb * kBK, o0);
      ptx::tma_load_2d(sV + kb * C::kVBlock, &tmV, bar_uv, kb * kBK, i0);
    }
    ptx::mbar_arrive_expect_tx(bar_w, C::kWBytes);
#pragma unroll
    for (int bx = 0; bx < kRecN / kBK; ++bx) ptx::tma_load_2d(sW + bx * kABytes, &tmW0, bar_w, i0 + bx * kBK, o0);
  }
  bool mma_issued = false;
  if (threadIdx.x == 32) {
    if (ptx::mbar_wait(bar_uv, 0, abort_flag)) {
      ptx::tc_fence_after();
      constexpr uint32_t idesc = ptx::idesc_bf16(kBM, kRecN, 0);
      const uint32_t ua = ptx::smem_u32(sU), va = ptx::smem_u32(sV);
#pragma unroll
      for (int kb = 0; kb < KB; ++kb)
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          ptx::umma_bf16(tmem, ptx::sdesc_sw128(ua + kb * C::kUBlock + kk * 32, 16, 1024),
                         ptx::sdesc_sw128(va + kb * C::kVBlock + kk * 32, 16, 1024), idesc, (kb | kk) ? 1u : 0u);
      ptx::umma_commit(bar_acc);
      mma_issued = true;
    } else {
      record_timeout(err);
      *abort_flag = 1;
    }
  }

  // epilogue: warp w owns tensor-memory lanes (rows) 32w .. 32w+31; the row
  // scale is loaded before the waits, off the critical path
  const int row = warp * 32 + lane;
  const float so = (o0 + row < O) ? __ldg(s + o0 + row) : 0.f;
  bool ok = ptx::mbar_wait(bar_acc, 0, abort_flag) && ptx::mbar_wait(bar_w, 0, abort_flag);
  if (!ok && !*abort_flag) {
    record_timeout(err);
    *abort_flag = 1;
  }
  ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
  ptx::tc_fence_after();
  const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
  if (ok) {
    // one 64-column box of the tile at a time: four tensor-memory loads in
    // flight, one wait
#pragma unroll 1
    for (int bx = 0; bx < kRecN / kBK; ++bx) {
      float d[kBK];
#pragma unroll
      for (int q = 0; q < kBK / 16; ++q)
        ptx::tmem_ld16(taddr + bx * kBK + q * 16, *reinterpret_cast<float(*)[16]>(d + 16 * q));
      ptx::tmem_wait_ld();
      uint8_t* rowp = sW + bx * kABytes + row * 128;
#pragma unroll
      for (int k = 0; k < kBK / 8; ++k) {
        const int chunk = k ^ (row & 7);  // 128-byte swizzle of 16-byte chunks
        uint4* p = reinterpret_cast<uint4*>(rowp + chunk * 16);
        float w[8], o[8];
        unpack(*p, w);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = fmaf(so, w[e], d[8 * k + e]);
        *p = pack(o, (uint4*)nullptr);
      }
    }
  }
  ptx::fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!*abort_flag) {
#pragma unroll
      for (int bx = 0; bx < kRecN / kBK; ++bx)
        if (i0 + bx * kBK < I) ptx::tma_store_2d(&tmOut, sW + bx * kABytes, i0 + bx * kBK, o0);
      ptx::bulk_commit();
      ptx::bulk_wait_read();
    } else {
      int never = 0;  // drain the loads before shared memory goes away
      ptx::mbar_wait(bar_uv, 0, &never);
      ptx::mbar_wait(bar_w, 0, &never);
    }
  }
  if (mma_issued && *abort_flag) {
    int never = 0;
    ptx::mbar_wait(bar_acc, 0, &never);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) ptx::tmem_dealloc(tmem, kRecN);
}

// --------------------------------------------------------- band reconstruct
// The reconstructions of the n layers of one band, which share W0:
// W_l = diag(s_l).W0 + U_l.V_l^T for l < n. One CTA per 128 x 128 tile of W0
// loads that tile once and loops over the layers:
//   warp 0    TMA: the W0 tile, then layer by layer the U_l and V_l rank
//             blocks into a double buffer
//   warp 1    the K = rank MMAs of layer l into one of two tensor-memory
//             accumulators, once the epilogue has read layer l-2's product
//             from it
//   warps 2-9 the epilogue, two warps per 32-lane quarter of tensor memory
//             (64 columns each): U_l.V_l^T from tensor memory plus s_l * W0
//             from the tile, rounded to bf16 into one of several output tiles
//             that one thread stores by TMA, several stores in flight
// So W0 crosses HBM once per band instead of once per layer, and layer l+1's
// loads and MMAs overlap layer l's epilogue and store. Same arithmetic as
// recon_kernel, element for element.
constexpr int kBandMax = 64;  // layers per launch (their tensor maps travel as kernel parameters)
constexpr int kBandThreads = 320;  // producer, MMA issuer, 8 epilogue warps
constexpr int kBandEpi = 256;      // epilogue threads

struct BandArgs {
  CUtensorMap U[kBandMax], V[kBandMax], Out[kBandMax];
  const float* s[kBandMax];
  int n, O, I;
  unsigned* err;
};

template <int KB>
struct BandCfg {
  static constexpr int kUBlock = kBM * 128;    // 128 rows x 64 rank columns (bf16)
  static constexpr int kVBlock = kRecN * 128;
  static constexpr int kUVBytes = KB * (kUBlock + kVBlock);  // one layer's U and V blocks
  static constexpr int kTileBytes = (kRecN / kBK) * kABytes;  // a 128 x 128 bf16 tile as two 64-column boxes
  // output tiles whose stores may be in flight at once (the writes are the
  // kernel's traffic; each SM needs ~100 KB of them in flight)
  static constexpr int kOutBufs = KB == 1 ? 4 : 2;
  static constexpr int kSmemBytes = kTileBytes + 2 * kUVBytes + kOutBufs * kTileBytes + 1024 + 256;
};

template <int KB>
__global__ void __launch_bounds__(kBandThreads, 1)
recon_band_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ BandArgs a) {
  using C = BandCfg<KB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sUV = sW + C::kTileBytes;                 // [2][U blocks, V blocks]
  uint8_t* sOut = sUV + 2 * C::kUVBytes;             // [kOutBufs] output tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + C::kOutBufs * C::kTileBytes);
  uint64_t* w_full = bars;            // the W0 tile landed
  uint64_t* uv_full = bars + 1;       // [2] a layer's U, V blocks landed
  uint64_t* uv_empty = bars + 3;      // [2] the MMAs reading them are done
  uint64_t* acc_full = bars + 5;      // [2] a layer's product in tensor memory
  uint64_t* acc_free = bars + 7;      // [2] the epilogue has read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int i0 = blockIdx.x * kRecN, o0 = blockIdx.y * kBM;
  const int n = a.n;
  if (threadIdx.x == 0) {
    ptx::mbar_init(w_full, 1);
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&uv_full[b], 1);
      ptx::mbar_init(&uv_empty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_free[b], kBandEpi);
    }
    *abort_flag = prior_timeout(a.err);
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 2 * kRecN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_enter();

  auto give_up = [&]() {
    record_timeout(a.err);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(w_full, C::kTileBytes);
#pragma unroll
      for (int bx = 0; bx < kRecN / kBK; ++bx) ptx::tma_load_2d(sW + bx * kABytes, &tmW0, w_full, i0 + bx * kBK, o0);
      int issued = 0;
      for (int l = 0; l < n; ++l) {
        const int b = l & 1;
        if (l >= 2 && !ptx::mbar_wait(&uv_empty[b], (uint32_t)(((l - 2) >> 1) & 1), abort_flag)) {
          give_up();
          break;
        }
        uint8_t* u = sUV + b * C::kUVBytes;
        uint8_t* v = u + KB * C::kUBlock;
        ptx::mbar_arrive_expect_tx(&uv_full[b], C::kUVBytes);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
          ptx::tma_load_2d(u + kb * C::kUBlock, &a.U[l], &uv_full[b], kb * kBK, o0);
          ptx::tma_load_2d(v + kb * C::kVBlock, &a.V[l], &uv_full[b], kb * kBK, i0);
        }
        ++issued;
      }
      // every load lands before the CTA can leave (immediate unless aborted)
      int never = 0;
      ptx::mbar_wait(w_full, 0, &never);
      for (int b = 0; b < 2 && b < issued; ++b) {
        const int last = b + ((issued - 1 - b) / 2) * 2;
        ptx::mbar_wait(&uv_full[b], (uint32_t)((last >> 1) & 1), &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16(kBM, kRecN, 0);
      int done = 0;
      for (int l = 0; l < n; ++l) {
        const int b = l & 1;
        // buffer b of tensor memory was last read by the epilogue of layer l-2
        if (!ptx::mbar_wait(&uv_full[b], (uint32_t)((l >> 1) & 1), abort_flag) ||
            (l >= 2 && !ptx::mbar_wait(&acc_free[b], (uint32_t)(((l - 2) >> 1) & 1), abort_flag))) {
          give_up();
          break;
        }
        ptx::tc_fence_after();
        const uint32_t ua = ptx::smem_u32(sUV + b * C::kUVBytes), va = ua + KB * C::kUBlock;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            ptx::umma_bf16(tmem + (uint32_t)(b * kRecN), ptx::sdesc_sw128(ua + kb * C::kUBlock + kk * 32, 16, 1024),
                           ptx::sdesc_sw128(va + kb * C::kVBlock + kk * 32, 16, 1024), idesc, (kb | kk) ? 1u : 0u);
        ptx::umma_commit(&acc_full[b]);
        ptx::umma_commit(&uv_empty[b]);
        ++done;
      }
      if (done < n && done > 0) {
        // aborted: the issued MMAs finish before tensor memory is freed
        int never = 0;
        const int last = done - 1;
        ptx::mbar_wait(&acc_full[last & 1], (uint32_t)((last >> 1) & 1), &never);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;         // a warp reads lanes 32 * (warp % 4) ...
    const int half = (warp - 2) / 4;      // ... and columns 64 * half ... + 63
    const int row = quarter * 32 + lane;  // tensor-memory lane = row of the tile
    const uint32_t taddr0 = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * 64);
    const bool leader = threadIdx.x == 64;  // issues the stores
    // Every decision to stop is taken by all eight epilogue warps together
    // (bar.red.and): the named barriers below need every one of them, and
    // tcgen05.ld is warp-collective. A wait can succeed in one warp and give
    // up in another when an abort lands just as the barrier completes.
    bool ok = ptx::bar_red_and(1, kBandEpi, ptx::mbar_wait(w_full, 0, abort_flag));
    // this thread's 64 W0 values, unpacked once for all the band's layers
    const uint8_t* wbox = sW + half * kABytes + row * 128;
    float w0f[64];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int chunk = k ^ (row & 7);  // 128-byte swizzle of 16-byte chunks
      unpack(*reinterpret_cast<const uint4*>(wbox + chunk * 16), *reinterpret_cast<float(*)[8]>(w0f + 8 * k));
    }
    // each layer's row scale is loaded one layer ahead, off the critical path
    const bool in_rows = o0 + row < a.O;
    float s_next = (n > 0 && in_rows) ? __ldg(a.s[0] + o0 + row) : 0.f;
    for (int l = 0; l < n && ok; ++l) {
      const int b = l & 1;
      const uint32_t taddr = taddr0 + (uint32_t)(b * kRecN);
      const float so = s_next;
      if (l + 1 < n) s_next = in_rows ? __ldg(a.s[l + 1] + o0 + row) : 0.f;
      const bool got = ptx::mbar_wait(&acc_full[b], (uint32_t)((l >> 1) & 1), abort_flag);
      // the store of layer l - kOutBufs read its buffer before this layer rewrites it
      if (leader) ptx::bulk_wait_read_n<C::kOutBufs - 1>();
      ok = ptx::bar_red_and(1, kBandEpi, got);
      if (!ok) break;
      ptx::tc_fence_after();
      // this warp's 64 columns (one swizzled box of the tile): all four loads
      // in flight, one wait
      float d[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) ptx::tmem_ld16(taddr + q * 16, *reinterpret_cast<float(*)[16]>(d + 16 * q));
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&acc_free[b]);  // tensor memory read: layer l+2's MMAs may start
      uint8_t* obox = sOut + (l % C::kOutBufs) * C::kTileBytes + half * kABytes + row * 128;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int chunk = k ^ (row & 7);
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = fmaf(so, w0f[8 * k + e], d[8 * k + e]);
        *reinterpret_cast<uint4*>(obox + chunk * 16) = pack(o, (uint4*)nullptr);
      }
      ptx::fence_proxy_async_smem();
      asm volatile("bar.sync 1, %0;" ::"n"(kBandEpi) : "memory");
      if (leader) {
        const uint8_t* out = sOut + (l % C::kOutBufs) * C::kTileBytes;
#pragma unroll
        for (int bx = 0; bx < kRecN / kBK; ++bx)
          if (i0 + bx * kBK < a.I) ptx::tma_store_2d(&a.Out[l], out + bx * kABytes, i0 + bx * kBK, o0);
        ptx::bulk_commit();
      }
    }
    if (!ok && !*abort_flag) give_up();
    if (leader) ptx::bulk_wait_read();
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) ptx::tmem_dealloc(tmem, 2 * kRecN);
}

// ------------------------------------------------------------- SVD products
// The randomized SVD's products with a bf16 residual R [O, I] on tensor
// cores ("The theta bundle" -- Low-rank residual, the randomized algorithm of
// Halko, Martinsson and Tropp):
//   R_LEFT   C [O, k] = R . F^T   F [k, I]: the test matrix, or Z^T
//   !R_LEFT  C [k, I] = F^T . R   F = Q [O, k], given here as Q^T [k, O]
// F is fp32; it enters as three bf16 parts F = F1 + F2 + F3 (each the
// rounded remainder of the one before: together the whole 24-bit
// significand), each multiplied into the same fp32 accumulator, so the sums
// are of the exact products of the fp32 operands, in another order than a
// CUDA-core fp32 GEMM. R is bf16, so it enters exactly. K is split over
// grid z; split z writes its partial C to part + z * M * N (fp32, row-major)
// and the caller adds the splits in a fixed order.
// 192 threads as in umma_kernel: TMA warp, MMA warp, four epilogue warps.
constexpr int kSvdParts = 3;

template <bool R_LEFT>
struct SvdCfg {
  static constexpr int kBN = R_LEFT ? 96 : 128;  // N: the samples (k <= 96) / 128 columns of R
  static constexpr int kNumA = R_LEFT ? 1 : kSvdParts;
  static constexpr int kNumB = R_LEFT ? kSvdParts : 1;
  static constexpr int kBBytes = kBN * kBK * 2;
  static constexpr int kStageBytes = kNumA * kABytes + kNumB * kBBytes;
  static constexpr int kStages = 3;
  static constexpr int kTmemCols = 128;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kStageBytes % 1024 == 0 && kBBytes % 1024 == 0, "swizzled tiles start on 1024-byte boundaries");
};

struct SvdArgs {
  int M, N;         // C [M, N]
  int kb;           // K blocks of 64
  int splits;       // grid z
  float* part;      // [splits, M, N]
  unsigned* err;
};

// R_LEFT: m0 = R (A, K-major), m1..m3 = the parts of F (B, K-major [k, I]).
// !R_LEFT: m0..m2 = the parts of Q^T (A, K-major [k, O]), m3 = R (B, MN-major).
template <bool R_LEFT>
__global__ void __launch_bounds__(kThreads)
svd_mma_kernel(const __grid_constant__ CUtensorMap m0, const __grid_constant__ CUtensorMap m1,
               const __grid_constant__ CUtensorMap m2, const __grid_constant__ CUtensorMap m3, const SvdArgs args) {
  using C = SvdCfg<R_LEFT>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* accum = empty + S;
  uint64_t* drain = accum + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int kb_begin = (int)((int64_t)split * args.kb / args.splits);
  const int kb_end = (int)((int64_t)(split + 1) * args.kb / args.splits);
  const int total = kb_end - kb_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(accum, 1);
    ptx::mbar_init(drain, 1);
    *abort_flag = prior_timeout(args.err);
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  auto give_up = [&]() {
    record_timeout(args.err);
    *abort_flag = 1;
  };

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    int issued = 0;
    for (int i = 0; i < total; ++i) {
      const int st = i % S;
      const uint32_t ph = (uint32_t)(i / S) & 1u;
      if (!ptx::mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
        give_up();
        break;
      }
      uint8_t* a = smem + st * C::kStageBytes;
      uint8_t* b = a + C::kNumA * kABytes;
      const int kx = (kb_begin + i) * kBK;
      ptx::mbar_arrive_expect_tx(&full[st], C::kStageBytes);
      if constexpr (R_LEFT) {
        ptx::tma_load_2d(a, &m0, &full[st], kx, m_tile * kBM);
        ptx::tma_load_2d(b, &m1, &full[st], kx, n_tile * C::kBN);
        ptx::tma_load_2d(b + C::kBBytes, &m2, &full[st], kx, n_tile * C::kBN);
        ptx::tma_load_2d(b + 2 * C::kBBytes, &m3, &full[st], kx, n_tile * C::kBN);
      } else {
        ptx::tma_load_2d(a, &m0, &full[st], kx, m_tile * kBM);
        ptx::tma_load_2d(a + kABytes, &m1, &full[st], kx, m_tile * kBM);
        ptx::tma_load_2d(a + 2 * kABytes, &m2, &full[st], kx, m_tile * kBM);
        // R [O, I] as the MN-major B: per 64-column atom of N, 64 rows of K (= O)
#pragma unroll
        for (int at = 0; at < C::kBN / 64; ++at)
          ptx::tma_load_2d(b + at * 64 * 128, &m3, &full[st], n_tile * C::kBN + at * 64, kx);
      }
      ++issued;
    }
    for (int st = 0; st < S && st < issued; ++st) {
      const int last = st + ((issued - 1 - st) / S) * S;
      if (!ptx::mbar_wait(&full[st], (uint32_t)(last / S) & 1u, abort_flag)) {
        int never = 0;
        ptx::mbar_wait(&full[st], (uint32_t)(last / S) & 1u, &never, 100000000ull);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = ptx::idesc_bf16(kBM, C::kBN, R_LEFT ? 0 : 1);
    int done = 0;
    for (int i = 0; i < total; ++i) {
      const int st = i % S;
      const uint32_t ph = (uint32_t)(i / S) & 1u;
      if (!ptx::mbar_wait(&full[st], ph, abort_flag)) {
        give_up();
        break;
      }
      ptx::tc_fence_after();
      const uint32_t a = ptx::smem_u32(smem + st * C::kStageBytes);
      const uint32_t b = a + C::kNumA * kABytes;
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
        for (int p = 0; p < kSvdParts; ++p) {
          const uint64_t ad = R_LEFT ? ptx::sdesc_sw128(a + kk * 32, 16, 1024)
                                     : ptx::sdesc_sw128(a + p * kABytes + kk * 32, 16, 1024);
          const uint64_t bd = R_LEFT ? ptx::sdesc_sw128(b + p * C::kBBytes + kk * 32, 16, 1024)
                                     : ptx::sdesc_sw128(b + kk * 16 * 128, 64 * 128, 1024);
          ptx::umma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0 || p > 0) ? 1u : 0u);
        }
      }
      ptx::umma_commit(&empty[st]);
      ++done;
    }
    if (done == total) {
      ptx::umma_commit(accum);
    } else if (done > 0) {
      ptx::umma_commit(drain);
      int never = 0;
      ptx::mbar_wait(drain, 0, &never);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
    // an empty split (more splits than K blocks) leaves a zero partial
    bool ok = total == 0 || ptx::mbar_wait(accum, 0, abort_flag);
    if (!ok) give_up();
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    ptx::tc_fence_after();
    const int m = m_tile * kBM + row;
    const int n0 = n_tile * C::kBN;
    const int ncols = min(C::kBN, args.N - n0);
    float* out = args.part + (int64_t)split * args.M * args.N + (int64_t)m * args.N + n0;
    if (ok) {
      for (int c0 = 0; c0 < ncols; c0 += 16) {
        float d[16];
        if (total > 0) {
          ptx::tmem_ld16(taddr + c0, d);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) d[e] = 0.f;
        }
        if (m < args.M) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c0 + e < ncols) out[c0 + e] = d[e];
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) ptx::tmem_dealloc(tmem, C::kTmemCols);
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(cudaError_t* e) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  static cudaError_t status = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    status = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (status == cudaSuccess && q != cudaDriverEntryPointSuccess) status = cudaErrorSymbolNotFound;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  *e = status;
  return fn;
}

// 2-D bf16 tensor [rows, cols], row pitch = cols, box [box_rows, box_cols];
// out-of-bounds elements of a box read as zero and are not written.
int make_map_box(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, int box_cols,
                 CUtensorMapSwizzle swizzle, cudaError_t* ce) {
  EncodeTiledFn enc = encode_fn(ce);
  if (!enc) return THETA_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *ce = cudaErrorInvalidValue;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

// The operand layout of the MMA kernels: box [box_rows, 64], 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, cudaError_t* ce) {
  return make_map_box(m, base, rows, cols, box_rows, kBK, CU_TENSOR_MAP_SWIZZLE_128B, ce);
}

// Per-device, per-kernel launch configuration: dynamic shared memory opt-in,
// non-portable cluster sizes, and the number of co-resident CTAs per SM,
// checked against tensor-memory capacity (co-resident CTAs must never need
// more columns than an SM has, or allocation would stall).
struct KernelInfo {
  bool ready = false;
  int blocks_per_sm = 0;
  int max_cluster = 1;
};

template <typename Kern>
cudaError_t prepare_kernel(KernelInfo* info, int device, Kern kern, int threads, int smem, int tmem_cols,
                           bool clusters) {
  std::lock_guard<std::mutex> lk(setup_mutex());
  if (info->ready) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // all of the unified L1/shared array as shared memory: the stage rings are
  // what keeps loads in flight, and the residency count below relies on it
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  if (clusters) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  // Co-resident CTAs per SM, from shared memory (the binding limit for these
  // kernels; the occupancy API under-reports kernels that use cluster
  // instructions). Tensor memory must cover all of them, or allocation
  // would stall.
  int dev_smem = 0, reserved = 0;
  e = cudaDeviceGetAttribute(&dev_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, device);
  if (e != cudaSuccess) return e;
  int blocks = dev_smem / (smem + reserved);
  const int by_threads = 2048 / threads;
  if (blocks > by_threads) blocks = by_threads;
  if (blocks < 1) return cudaErrorInvalidConfiguration;
  if (blocks * tmem_cols > 512) blocks = 512 / tmem_cols;  // never counted on beyond tensor memory
  int api_blocks = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&api_blocks, kern, threads, smem);
  if (e != cudaSuccess) return e;
  if (api_blocks * tmem_cols > 512) return cudaErrorInvalidConfiguration;
  info->blocks_per_sm = blocks;
  info->max_cluster = 1;
  if (clusters) {
    // the largest cluster (16, else 8) that the GPU can place at all; a
    // refused query sets the thread's last error, which is cleared below only
    // when no earlier error was pending (the caller's must not be lost)
    const bool pending = cudaPeekAtLastError() != cudaSuccess;
    bool refused = false;
    for (int cs = 16; cs >= 8 && info->max_cluster == 1; cs /= 2) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(threads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = cs;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      const cudaError_t q = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      if (q == cudaSuccess && n > 0) info->max_cluster = cs;
      if (q != cudaSuccess) refused = true;
    }
    if (refused && !pending) cudaGetLastError();  // a refused query is not an error of this call
    if (info->max_cluster == 1) return cudaErrorInvalidConfiguration;
  }
  info->ready = true;
  return cudaSuccess;
}

// Largest power-of-two split (<= 16) that keeps every CTA resident in one
// wave and leaves each split at least 4 K blocks.
int pick_splits(int64_t tiles, int kb, int capacity, int max_cluster) {
  int s = 1;
  while (2 * s <= max_cluster && tiles * (2 * s) <= capacity && kb / (2 * s) >= 4) s *= 2;
  return s;
}

// The tensor maps of one launch: A1, B1 (phase 1), A2, B2, B3 (phase 2), and
// for GATE_UP the up projection's A1, A2, B2, B3 (other modes repeat A1).
struct Maps {
  CUtensorMap a1, b1, a2, b2, b3, a1u, a2u, b2u, b3u;
};

template <int BN, int MODE>
cudaError_t launch_tile_kernel(const LaunchCtx& c, const Maps& mp, Args args, int m_tiles, int n_tiles) {
  using C = Cfg<BN, MODE>;
  auto kern = umma_kernel<BN, MODE>;
  static KernelInfo info[64];
  cudaError_t e = prepare_kernel(&info[c.device], c.device, kern, kThreads, C::kSmemBytes, C::kTmemCols, true);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (int64_t)m_tiles * n_tiles;
  // Tiles of 64 or more columns keep the tensor pipe busy: a second CTA on
  // the same SM adds no throughput, only split-K reduction work, so they
  // count one CTA per SM. Narrow (decode) tiles are bound by memory latency
  // and count every co-resident CTA.
  const int capacity = c.num_sms * (BN >= 64 ? 1 : info[c.device].blocks_per_sm);
  // The throughput policy gives every CTA of the main projection a whole
  // tile. T = X.V keeps its split under both policies: it has one tile per
  // 128 tokens, so unsplit it is a single CTA walking all of K, a serial
  // latency chain that the forward behind it waits for.
  args.splits = (c.policy == THETA_POLICY_THROUGHPUT && MODE != MODE_XV)
                    ? 1
                    : pick_splits(tiles, args.kb1, capacity, info[c.device].max_cluster);
  return launch_pdl(kern, dim3((unsigned)(n_tiles * args.splits), (unsigned)m_tiles, 1), dim3(kThreads), C::kSmemBytes,
                    c.stream, args.splits, mp.a1, mp.b1, mp.a2, mp.b2, mp.b3, mp.a1u, mp.a2u, mp.b2u, mp.b3u, args);
}

// The persistent CTA-pair kernel: one cluster of two per pair of SMs that
// can hold one (the occupancy query, once per device), at most one per tile.
// Y [M, O] is written by TMA in boxes of 128 rows of W0 (columns of Y) x one
// tile's tokens.
template <int MODE>
cudaError_t launch_pair(const LaunchCtx& c, const Maps& mp, const Args& args, void* Y, cudaError_t* ce_map) {
  using C = PairCfg<MODE>;
  auto kern = pair_kernel<MODE>;
  static KernelInfo info[64];
  static int max_clusters[64];
  CUtensorMap mY;
  if (make_map_box(&mY, Y, args.cols, args.rows, C::kN, kBM, CU_TENSOR_MAP_SWIZZLE_NONE, ce_map))
    return *ce_map;
  cudaError_t e = prepare_kernel(&info[c.device], c.device, kern, C::kThreads, C::kSmemBytes, C::kTmemCols, false);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(setup_mutex());
    if (max_clusters[c.device] == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(C::kThreads, 1, 1);
      cfg.dynamicSmemBytes = C::kSmemBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      const bool pending = cudaPeekAtLastError() != cudaSuccess;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
        if (!pending) cudaGetLastError();  // a refused query is not an error of this call
        n = c.num_sms / 2;                 // one CTA per SM
      }
      max_clusters[c.device] = n;
    }
  }
  const int64_t tiles = ceil_div(args.rows, 2 * kBM) * ceil_div(args.cols, C::kN);
  const int64_t clusters = tiles < max_clusters[c.device] ? tiles : max_clusters[c.device];
  return launch_pdl(kern, dim3((unsigned)(2 * clusters), 1, 1), dim3(C::kThreads), C::kSmemBytes, c.stream, 2, mp.a1,
                    mp.b1, mp.a2, mp.b2, mp.b3, mp.a1u, mp.a2u, mp.b2u, mp.b3u, mY, args);
}

template <int KB>
cudaError_t launch_recon(const LaunchCtx& c, const CUtensorMap& mU, const CUtensorMap& mV, const CUtensorMap& mW0,
                         const CUtensorMap& mOut, const float* s, int O, int I) {
  using C = RecCfg<KB>;
  auto kern = recon_kernel<KB>;
  static KernelInfo info[64];
  cudaError_t e = prepare_kernel(&info[c.device], c.device, kern, kRecThreads, C::kSmemBytes, kRecN, false);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)ceil_div(I, kRecN), (unsigned)ceil_div(O, kBM), 1), dim3(kRecThreads),
                    C::kSmemBytes, c.stream, 1, mU, mV, mW0, mOut, s, O, I, c.err);
}

template <int KB>
cudaError_t launch_band(const LaunchCtx& c, const CUtensorMap& mW0, const BandArgs& a) {
  using C = BandCfg<KB>;
  auto kern = recon_band_kernel<KB>;
  static KernelInfo info[64];
  cudaError_t e = prepare_kernel(&info[c.device], c.device, kern, kBandThreads, C::kSmemBytes, 2 * kRecN, false);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)ceil_div(a.I, kRecN), (unsigned)ceil_div(a.O, kBM), 1), dim3(kBandThreads),
                    C::kSmemBytes, c.stream, 1, mW0, a);
}

// The failure path of every bounded wait, on purpose: one thread waits on an
// mbarrier that nothing will complete, gives up after limit_ns, records the
// timeout flag and returns; the host reads it through theta_device_status.
__global__ void wait_selftest_kernel(unsigned* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int never;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    never = 0;
    ptx::fence_mbarrier_init();
    if (!ptx::mbar_wait(&bar, 0, &never, limit_ns)) record_timeout(err);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(const LaunchCtx& c, unsigned limit_ms) {
  wait_selftest_kernel<<<1, 32, 0, c.stream>>>(c.err, (unsigned long long)limit_ms * 1000000ull);
  return cudaGetLastError();
}

size_t forward_umma_workspace_bytes(int64_t M, int r) {
  const size_t half = ((size_t)M * r * 2 + 255) / 256 * 256;
  const size_t gemv = forward_gemv_workspace_bytes(M, r);
  return 2 * half > gemv ? 2 * half : gemv;
}

namespace {

// T = X . V (fp32 in tensor memory) -> bf16 high and low parts [M, r]
int launch_xv_umma(const LaunchCtx& c, const void* X, const void* V, int64_t M, int64_t I, int r, bf16* t_hi,
                   bf16* t_lo, cudaError_t* ce) {
  Maps mp;
  int st;
  if ((st = make_map(&mp.a1, X, M, I, kBM, ce))) return st;  // 128 token rows per tile
  if ((st = make_map(&mp.b1, V, I, r, kBK, ce))) return st;  // box: 64 rank columns x 64 rows of I
  mp.a2 = mp.b2 = mp.b3 = mp.a1u = mp.a2u = mp.b2u = mp.b3u = mp.b1;
  Args a = {};
  a.rows = (int)M;
  a.cols = r;
  a.kb1 = (int)ceil_div(I, kBK);
  a.kb2 = 0;
  a.t_hi = t_hi;
  a.t_lo = t_lo;
  a.r = r;
  a.err = c.err;
  const int m_tiles = (int)ceil_div(M, kBM);
  cudaError_t e;
  switch ((int)ceil_div(r, 64) * 64) {
    case 64: e = launch_tile_kernel<64, MODE_XV>(c, mp, a, m_tiles, 1); break;
    case 128: e = launch_tile_kernel<128, MODE_XV>(c, mp, a, m_tiles, 1); break;
    case 192: e = launch_tile_kernel<192, MODE_XV>(c, mp, a, m_tiles, 1); break;
    default: e = launch_tile_kernel<256, MODE_XV>(c, mp, a, m_tiles, 1); break;
  }
  if (e != cudaSuccess) {
    *ce = e;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

}  // namespace

int launch_forward_umma(const LaunchCtx& c, const void* X, const void* W0, const float* s, const void* U,
                        const void* V, int64_t M, int64_t O, int64_t I, int r, void* Y, void* ws,
                        cudaError_t* ce) {
  *ce = cudaSuccess;
  if (O > (int64_t)65535 * kBM || M > ((int64_t)1 << 30) || I > ((int64_t)1 << 31) - 64 || r > 256)
    return THETA_ERR_UNSUPPORTED;
  // the T = X.V grid is one CTA row per 128 tokens (grid y <= 65535)
  if (r > 0 && ceil_div(M, kBM) > 65535) return THETA_ERR_UNSUPPORTED;
  cudaError_t e = cudaSuccess;
  // ---- a handful of tokens: a sequential sweep over W0 on CUDA cores
  if (M <= forward_gemv_max_tokens() && launch_forward_gemv(c, X, W0, s, U, V, M, O, I, r, Y, ws, &e)) {
    if (e != cudaSuccess) {
      *ce = e;
      return THETA_ERR_CUDA;
    }
    return THETA_OK;
  }
  const int kb = (int)ceil_div(I, kBK);
  bf16* t_hi = nullptr;
  bf16* t_lo = nullptr;
  int st;
  if (r > 0) {
    t_hi = static_cast<bf16*>(ws);
    t_lo = reinterpret_cast<bf16*>(static_cast<uint8_t*>(ws) + forward_umma_workspace_bytes(M, r) / 2);
    if ((st = launch_xv_umma(c, X, V, M, I, r, t_hi, t_lo, ce))) return st;
  }
  // ---- Y = s * (X . W0^T) + T . U^T, swap-AB: W0 rows are the MMA M side
  const int BN = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 256 ? 128 : 256;
  const int m_tiles = (int)ceil_div(O, kBM);
  const int n_tiles = (int)ceil_div(M, BN);
  // More than 256 tokens: pairs of SMs share 256 x 256 tiles whenever every
  // CTA gets a whole tile -- under the throughput policy, or when the tiles
  // already fill the GPU (the latency policy would not split K then either).
  // 129 to 256 tokens under the throughput policy: one 256-token pair tile
  // per 256 rows instead of two 128-token one-SM tiles (measured 5-8% faster
  // on a stream of Gemma-3-1B-shaped calls).
  const bool pair = (BN == 256 && (c.policy == THETA_POLICY_THROUGHPUT || (int64_t)m_tiles * n_tiles >= c.num_sms)) ||
                    (BN == 128 && M > 128 && c.policy == THETA_POLICY_THROUGHPUT);
  const int box_b = pair ? PairCfg<MODE_FORWARD>::kHalf : BN;  // tokens per B box
  Maps mp;
  if ((st = make_map(&mp.a1, W0, O, I, kBM, ce))) return st;
  if ((st = make_map(&mp.b1, X, M, I, box_b, ce))) return st;
  if (r > 0) {
    if ((st = make_map(&mp.a2, U, O, r, kBM, ce))) return st;
    if ((st = make_map(&mp.b2, t_hi, M, r, box_b, ce))) return st;
    if ((st = make_map(&mp.b3, t_lo, M, r, box_b, ce))) return st;
  } else {
    mp.a2 = mp.a1;
    mp.b2 = mp.b3 = mp.b1;
  }
  mp.a1u = mp.a2u = mp.a1;
  mp.b2u = mp.b3u = mp.b1;
  Args a = {};
  a.rows = (int)O;
  a.cols = (int)M;
  a.kb1 = kb;
  a.kb2 = r > 0 ? (int)ceil_div(r, kBK) : 0;
  a.s = s;
  a.out = static_cast<bf16*>(Y);
  a.early_start = r > 0;  // directly after this call's T = X.V kernel
  a.err = c.err;
  if (pair) {
    a.splits = 1;
    e = launch_pair<MODE_FORWARD>(c, mp, a, Y, ce);
    if (e != cudaSuccess) {
      *ce = e;
      return THETA_ERR_CUDA;
    }
    return THETA_OK;
  }
  switch (BN) {
    case 16: e = launch_tile_kernel<16, MODE_FORWARD>(c, mp, a, m_tiles, n_tiles); break;
    case 32: e = launch_tile_kernel<32, MODE_FORWARD>(c, mp, a, m_tiles, n_tiles); break;
    case 64: e = launch_tile_kernel<64, MODE_FORWARD>(c, mp, a, m_tiles, n_tiles); break;
    case 128: e = launch_tile_kernel<128, MODE_FORWARD>(c, mp, a, m_tiles, n_tiles); break;
    default: e = launch_tile_kernel<256, MODE_FORWARD>(c, mp, a, m_tiles, n_tiles); break;
  }
  if (e != cudaSuccess) {
    *ce = e;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

size_t gate_up_umma_workspace_bytes(int64_t M, int r) {
  if (r <= 0) return 0;
  const size_t half = ((size_t)M * r * 2 + 255) / 256 * 256;
  return 4 * half;  // T high and low parts of the gate, then of the up projection
}

int launch_gate_up_umma(const LaunchCtx& c, const void* X, const void* W0g, const float* sg, const void* Ug,
                        const void* Vg, const void* W0u, const float* su, const void* Uu, const void* Vu, int64_t M,
                        int64_t O, int64_t I, int r, void* Y, void* ws, cudaError_t* ce) {
  *ce = cudaSuccess;
  if (O > (int64_t)65535 * kBM || M > ((int64_t)1 << 30) || I > ((int64_t)1 << 31) - 64 || r > 256)
    return THETA_ERR_UNSUPPORTED;
  if (r > 0 && ceil_div(M, kBM) > 65535) return THETA_ERR_UNSUPPORTED;  // T = X.V grid height
  const size_t half = ((size_t)M * r * 2 + 255) / 256 * 256;
  bf16* t[4] = {};
  int st;
  if (r > 0) {
    for (int q = 0; q < 4; ++q) t[q] = reinterpret_cast<bf16*>(static_cast<uint8_t*>(ws) + q * half);
    if ((st = launch_xv_umma(c, X, Vg, M, I, r, t[0], t[1], ce))) return st;
    if ((st = launch_xv_umma(c, X, Vu, M, I, r, t[2], t[3], ce))) return st;
  }
  // four accumulators of BN columns: at most 128 tokens per tile
  const int BN = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  const int m_tiles = (int)ceil_div(O, kBM);
  const int n_tiles = (int)ceil_div(M, BN);
  // More than 256 tokens: CTA pairs share 256-row x 128-token tiles, on the
  // same condition as the forward's pairs
  const bool pair = M > 256 && (c.policy == THETA_POLICY_THROUGHPUT || (int64_t)m_tiles * n_tiles >= c.num_sms);
  const int box_b = pair ? PairCfg<MODE_GATE_UP>::kHalf : BN;  // tokens per B box
  Maps mp;
  if ((st = make_map(&mp.a1, W0g, O, I, kBM, ce))) return st;
  if ((st = make_map(&mp.a1u, W0u, O, I, kBM, ce))) return st;
  if ((st = make_map(&mp.b1, X, M, I, box_b, ce))) return st;
  if (r > 0) {
    if ((st = make_map(&mp.a2, Ug, O, r, kBM, ce))) return st;
    if ((st = make_map(&mp.b2, t[0], M, r, box_b, ce))) return st;
    if ((st = make_map(&mp.b3, t[1], M, r, box_b, ce))) return st;
    if ((st = make_map(&mp.a2u, Uu, O, r, kBM, ce))) return st;
    if ((st = make_map(&mp.b2u, t[2], M, r, box_b, ce))) return st;
    if ((st = make_map(&mp.b3u, t[3], M, r, box_b, ce))) return st;
  } else {
    mp.a2 = mp.a2u = mp.a1;
    mp.b2 = mp.b3 = mp.b2u = mp.b3u = mp.b1;
  }
  Args a = {};
  a.rows = (int)O;
  a.cols = (int)M;
  a.kb1 = (int)ceil_div(I, kBK);
  a.kb2 = r > 0 ? (int)ceil_div(r, kBK) : 0;
  a.s = sg;
  a.s_up = su;
  a.out = static_cast<bf16*>(Y);
  a.early_start = r > 0;  // directly after the up projection's T = X.V kernel
  a.err = c.err;
  cudaError_t e;
  if (pair) {
    a.splits = 1;
    e = launch_pair<MODE_GATE_UP>(c, mp, a, Y, ce);
    if (e != cudaSuccess) {
      *ce = e;
      return THETA_ERR_CUDA;
    }
    return THETA_OK;
  }
  switch (BN) {
    case 16: e = launch_tile_kernel<16, MODE_GATE_UP>(c, mp, a, m_tiles, n_tiles); break;
    case 32: e = launch_tile_kernel<32, MODE_GATE_UP>(c, mp, a, m_tiles, n_tiles); break;
    case 64: e = launch_tile_kernel<64, MODE_GATE_UP>(c, mp, a, m_tiles, n_tiles); break;
    default: e = launch_tile_kernel<128, MODE_GATE_UP>(c, mp, a, m_tiles, n_tiles); break;
  }
  if (e != cudaSuccess) {
    *ce = e;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

int launch_reconstruct_band_umma(const LaunchCtx& c, const float* const* s, const void* W0, const void* const* U,
                                 const void* const* V, int n, int64_t O, int64_t I, int r, void* const* W_out,
                                 cudaError_t* ce) {
  *ce = cudaSuccess;
  // one layer, rank 0 or a rank beyond two 64-column blocks: one call per layer
  if (n == 1 || r == 0 || r > 2 * kBK) {
    for (int l = 0; l < n; ++l) {
      const int st = launch_reconstruct_umma(c, s[l], W0, r > 0 ? U[l] : nullptr, r > 0 ? V[l] : nullptr, O, I, r,
                                             W_out[l], ce);
      if (st) return st;
    }
    return THETA_OK;
  }
  if (O > (int64_t)65535 * kBM || I > ((int64_t)1 << 31) - 256) return THETA_ERR_UNSUPPORTED;
  static thread_local BandArgs a;  // ~25 KB of tensor maps: kept off the stack
  CUtensorMap mW0;
  int st;
  if ((st = make_map(&mW0, W0, O, I, kBM, ce))) return st;
  for (int l0 = 0; l0 < n; l0 += kBandMax) {
    const int m = n - l0 < kBandMax ? n - l0 : kBandMax;
    for (int j = 0; j < m; ++j) {
      if ((st = make_map(&a.U[j], U[l0 + j], O, r, kBM, ce))) return st;
      if ((st = make_map(&a.V[j], V[l0 + j], I, r, kRecN, ce))) return st;
      if ((st = make_map(&a.Out[j], W_out[l0 + j], O, I, kBM, ce))) return st;
      a.s[j] = s[l0 + j];
    }
    a.n = m;
    a.O = (int)O;
    a.I = (int)I;
    a.err = c.err;
    const cudaError_t e = r > kBK ? launch_band<2>(c, mW0, a) : launch_band<1>(c, mW0, a);
    if (e != cudaSuccess) {
      *ce = e;
      return THETA_ERR_CUDA;
    }
  }
  return THETA_OK;
}

int launch_reconstruct_umma(const LaunchCtx& c, const float* s, const void* W0, const void* U, const void* V,
                            int64_t O, int64_t I, int r, void* W_out, cudaError_t* ce) {
  *ce = cudaSuccess;
  if (r == 0) {
    const int64_t nvec = O * I / 8;
    int64_t grid = ceil_div(nvec, 256);
    if (grid > 8 * (int64_t)c.num_sms) grid = 8 * (int64_t)c.num_sms;
    if (grid < 1) grid = 1;
    *ce = launch_pdl(scale_rows_kernel, dim3((unsigned)grid), dim3(256), 0, c.stream, 1, s,
                     static_cast<const bf16*>(W0), I, nvec, static_cast<bf16*>(W_out));
    return *ce == cudaSuccess ? THETA_OK : THETA_ERR_CUDA;
  }
  if (O > (int64_t)65535 * kBM || I > ((int64_t)1 << 31) - 256 || r > 256) return THETA_ERR_UNSUPPORTED;
  CUtensorMap mU, mV, mW0, mOut;
  int st;
  if ((st = make_map(&mU, U, O, r, kBM, ce))) return st;
  if ((st = make_map(&mV, V, I, r, kRecN, ce))) return st;
  if ((st = make_map(&mW0, W0, O, I, kBM, ce))) return st;
  if ((st = make_map(&mOut, W_out, O, I, kBM, ce))) return st;
  cudaError_t e;
  switch ((int)ceil_div(r, kBK)) {
    case 1: e = launch_recon<1>(c, mU, mV, mW0, mOut, s, (int)O, (int)I); break;
    case 2: e = launch_recon<2>(c, mU, mV, mW0, mOut, s, (int)O, (int)I); break;
    case 3: e = launch_recon<3>(c, mU, mV, mW0, mOut, s, (int)O, (int)I); break;
    default: e = launch_recon<4>(c, mU, mV, mW0, mOut, s, (int)O, (int)I); break;
  }
  if (e != cudaSuccess) {
    *ce = e;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

namespace {

template <bool R_LEFT>
cudaError_t launch_svd_mma_t(const LaunchCtx& c, const CUtensorMap* maps, const SvdArgs& a, int m_tiles,
                             int n_tiles) {
  using C = SvdCfg<R_LEFT>;
  auto kern = svd_mma_kernel<R_LEFT>;
  static KernelInfo info[64];
  cudaError_t e = prepare_kernel(&info[c.device], c.device, kern, kThreads, C::kSmemBytes, C::kTmemCols, false);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)n_tiles, (unsigned)m_tiles, (unsigned)a.splits), dim3(kThreads),
                    C::kSmemBytes, c.stream, 1, maps[0], maps[1], maps[2], maps[3], a);
}

}  // namespace

int svd_mma_splits(const LaunchCtx& c, bool r_left, int64_t O, int64_t I, int k) {
  const int64_t tiles = r_left ? ceil_div(O, kBM) : ceil_div(I, SvdCfg<false>::kBN) * ceil_div(k, kBM);
  const int64_t kb = ceil_div(r_left ? I : O, kBK);
  // one CTA per SM; the split count that finishes the K blocks in the fewest
  // rounds of CTAs, each split keeping at least four K blocks
  int best = 1;
  int64_t best_cost = -1;
  for (int sp = 1; sp <= kSvdMaxSplits; ++sp) {
    if (sp > 1 && kb / sp < 4) break;
    const int64_t cost = ceil_div(tiles * sp, (int64_t)c.num_sms) * ceil_div(kb, (int64_t)sp);
    if (best_cost < 0 || cost < best_cost) best = sp, best_cost = cost;
  }
  return best;
}

int launch_svd_mma(const LaunchCtx& c, bool r_left, const void* R, int64_t O, int64_t I, const void* parts,
                   int64_t part_stride, int64_t part_pitch, int k, int splits, float* part_out, cudaError_t* ce) {
  *ce = cudaSuccess;
  CUtensorMap maps[4];
  int st;
  const bf16* P = static_cast<const bf16*>(parts);
  const int64_t part_elems = part_stride;
  SvdArgs a = {};
  a.splits = splits;
  a.part = part_out;
  a.err = c.err;
  if (r_left) {
    // C [O, k] = R . F^T: R rows by 128, the k samples as one N tile
    if ((st = make_map_box(&maps[0], R, O, I, kBM, kBK, CU_TENSOR_MAP_SWIZZLE_128B, ce))) return st;
    for (int p = 0; p < kSvdParts; ++p)
      if ((st = make_map_box(&maps[1 + p], P + p * part_elems, k, I, SvdCfg<true>::kBN, kBK,
                             CU_TENSOR_MAP_SWIZZLE_128B, ce)))
        return st;
    a.M = (int)O, a.N = k, a.kb = (int)ceil_div(I, kBK);
  } else {
    // C [k, I] = Q^T . R: the parts of Q^T [k, O] (row pitch part_pitch) as A,
    // R as the MN-major B in boxes of 64 columns x 64 rows
    for (int p = 0; p < kSvdParts; ++p) {
      EncodeTiledFn enc = encode_fn(ce);
      if (!enc) return THETA_ERR_CUDA;
      cuuint64_t dims[2] = {(cuuint64_t)O, (cuuint64_t)k};
      cuuint64_t strides[1] = {(cuuint64_t)part_pitch * 2};
      cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
      cuuint32_t estr[2] = {1, 1};
      if (enc(&maps[p], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(P + p * part_elems), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        *ce = cudaErrorInvalidValue;
        return THETA_ERR_CUDA;
      }
    }
    if ((st = make_map_box(&maps[3], R, O, I, kBK, 64, CU_TENSOR_MAP_SWIZZLE_128B, ce))) return st;
    a.M = k, a.N = (int)I, a.kb = (int)ceil_div(O, kBK);
  }
  const int m_tiles = (int)ceil_div(a.M, kBM);
  const int n_tiles = (int)ceil_div(a.N, r_left ? SvdCfg<true>::kBN : SvdCfg<false>::kBN);
  const cudaError_t e = r_left ? launch_svd_mma_t<true>(c, maps, a, m_tiles, n_tiles)
                               : launch_svd_mma_t<false>(c, maps, a, m_tiles, n_tiles);
  if (e != cudaSuccess) {
    *ce = e;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

}  // namespace theta
