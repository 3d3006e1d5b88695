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
// Three epilogues ("The theta bundle" -- approximation formula):
//   FORWARD  Y[m, o] = s[o] * D1[o, m] + D2[o, m]   with A1 = W0, B1 = X,
//            A2 = U, B2/B3 = high/low bf16 parts of T = X.V  (swap-AB: the
//            weight rows fill the 128-row MMA side, tokens are N)
//   XV       T_hi/T_lo[m, j] from D1[m, j]           with A1 = X, B1 = V (MN-major)
//   RECON    W[o, i] = s[o] * W0[o, i] + D1[o, i]   with A1 = U, B1 = V (K = rank)
// Decode-sized problems split K across the CTAs of a thread-block cluster;
// the partial tiles are summed in a fixed order through distributed shared
// memory (deterministic, no global scratch).
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

enum Mode { MODE_FORWARD = 0, MODE_XV = 1, MODE_RECON = 2 };

constexpr int kThreads = 192;
constexpr int kBM = 128;       // MMA M (rows of A)
constexpr int kBK = 64;        // K per stage: one 128-byte swizzle atom of bf16
constexpr int kABytes = kBM * kBK * 2;
constexpr int kPitch = 129;    // fp32 pitch of the split-K partial tiles (bank-conflict free)

struct Args {
  int rows;        // valid rows of the A side (O, or M tokens for XV)
  int cols;        // valid columns of the B side (M tokens, I, or rank)
  int kb1;         // K blocks of phase 1
  int kb2;         // K blocks of phase 2 (0: none)
  int splits;      // cluster size along x (split-K)
  const float* s;  // FORWARD / RECON row scale
  const bf16* W0;  // RECON
  bf16* out;       // FORWARD: Y [cols, rows]; RECON: W [rows, cols]
  bf16* t_hi;      // XV outputs [rows, r]
  bf16* t_lo;
  int r;
  unsigned* err;
};

template <int BN, int MODE>
struct Cfg {
  static constexpr int kBBytes = BN * kBK * 2;  // XV: BN = padded rank, MN-major atoms of 64 columns
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN <= 32 ? 8 : (BN <= 64 ? 6 : 4);
  static constexpr int kTmemNeed = MODE == MODE_FORWARD ? 2 * BN : BN;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kPartialBytes = BN * kPitch * 4;
  static_assert(kPartialBytes <= kStages * kStageBytes, "partial tile must fit in the stage ring");
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
};

template <int BN, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
umma_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
            const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
            const __grid_constant__ CUtensorMap tmB3, const Args args) {
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
  const bool has_d2 = MODE == MODE_FORWARD && args.kb2 > 0 && split == 0;
  const int n1 = kb_end - kb_begin;
  const int total = n1 + (has_d2 ? 2 * args.kb2 : 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(accum, 1);
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
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
      uint8_t* b = a + kABytes;
      ptx::mbar_arrive_expect_tx(&full[st], C::kStageBytes);
      if (i < n1) {
        const int kx = (kb_begin + i) * kBK;
        ptx::tma_load_2d(a, &tmA1, &full[st], kx, m_tile * kBM);
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
        const int jx = (j % args.kb2) * kBK;
        ptx::tma_load_2d(a, &tmA2, &full[st], jx, m_tile * kBM);
        ptx::tma_load_2d(b, j < args.kb2 ? &tmB2 : &tmB3, &full[st], jx, n_tile * BN);
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
      const uint32_t b = a + kABytes;
      if (i < n1) {
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = ptx::sdesc_sw128(a + kk * 32, 16, 1024);
          const uint64_t bd = MODE == MODE_XV ? ptx::sdesc_sw128(b + kk * 16 * 128, 64 * 128, 1024)
                                              : ptx::sdesc_sw128(b + kk * 32, 16, 1024);
          ptx::umma_bf16(tmem, ad, bd, idesc1, (i > 0 || kk > 0) ? 1u : 0u);
        }
      } else {
        const int j = i - n1;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = ptx::sdesc_sw128(a + kk * 32, 16, 1024);
          const uint64_t bd = ptx::sdesc_sw128(b + kk * 32, 16, 1024);
          ptx::umma_bf16(tmem + BN, ad, bd, idesc2, (j > 0 || kk > 0) ? 1u : 0u);
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
    const bool ok = ptx::mbar_wait(accum, 0, abort_flag);
    if (!ok) give_up();
    ptx::tc_fence_after();
    const int grow = m_tile * kBM + row;  // global row of A
    const int col0 = n_tile * BN;
    const int ncols = min(BN, args.cols - col0);
    float so = 0.f;
    if constexpr (MODE != MODE_XV) so = (grow < args.rows) ? __ldg(args.s + grow) : 0.f;
    float* part = reinterpret_cast<float*>(smem);
    if (ok) {
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
          } else {  // RECON: 16 consecutive columns of one weight row
            const int64_t base = (int64_t)grow * args.cols + col0 + c0;
            if (c0 + 16 <= ncols) {
              const uint4* w0v = reinterpret_cast<const uint4*>(args.W0 + base);
              uint4* ov = reinterpret_cast<uint4*>(args.out + base);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                float w[8], o[8];
                unpack(__ldg(w0v + h), w);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = fmaf(so, w[e], d1[8 * h + e]);
                ov[h] = pack(o, (uint4*)nullptr);
              }
            } else {
              for (int e = 0; e < ncols - c0; ++e)
                args.out[base + e] = __float2bfloat16_rn(fmaf(so, __bfloat162float(args.W0[base + e]), d1[e]));
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

// s (.) W0 for rank 0 (no tensor-core work).
__global__ void __launch_bounds__(256) scale_rows_kernel(const float* __restrict__ s, const bf16* __restrict__ W0,
                                                         int64_t I, int64_t nvec, bf16* __restrict__ out) {
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

// 2-D bf16 tensor [rows, cols], row pitch = cols, box [box_rows, 64] with
// 128-byte swizzle; out-of-bounds elements of a box read as zero.
int make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, cudaError_t* ce) {
  EncodeTiledFn enc = encode_fn(ce);
  if (!enc) return THETA_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *ce = cudaErrorInvalidValue;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

template <int BN, int MODE>
cudaError_t launch_tile_kernel(const LaunchCtx& c, const CUtensorMap& a1, const CUtensorMap& b1, const CUtensorMap& a2,
                               const CUtensorMap& b2, const CUtensorMap& b3, const Args& args, int m_tiles,
                               int n_tiles) {
  using C = Cfg<BN, MODE>;
  auto kern = umma_kernel<BN, MODE>;
  static bool configured[64] = {};
  if (!configured[c.device]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    int blocks = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kThreads, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // co-resident CTAs must never need more tensor memory than an SM has
    if (blocks * C::kTmemCols > 512) return cudaErrorInvalidConfiguration;
    configured[c.device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(n_tiles * args.splits), (unsigned)m_tiles, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)args.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a1, b1, a2, b2, b3, args);
}

int pick_splits(int64_t tiles, int kb, int num_sms) {
  int s = 1;
  while (s < 8 && tiles * s < 2 * (int64_t)num_sms && kb / (2 * s) >= 4) s *= 2;
  return s;
}

}  // namespace

size_t forward_umma_workspace_bytes(int64_t M, int r) {
  const size_t half = ((size_t)M * r * 2 + 255) / 256 * 256;
  return 2 * half;
}

int launch_forward_umma(const LaunchCtx& c, const void* X, const void* W0, const float* s, const void* U,
                        const void* V, int64_t M, int64_t O, int64_t I, int r, void* Y, void* ws,
                        cudaError_t* ce) {
  *ce = cudaSuccess;
  if (O > (int64_t)65535 * kBM || M > (int64_t)1 << 30 || I > ((int64_t)1 << 31) - 64 || r > 256)
    return THETA_ERR_UNSUPPORTED;
  const int kb = (int)ceil_div(I, kBK);
  bf16* t_hi = nullptr;
  bf16* t_lo = nullptr;
  CUtensorMap mX, mW0, mU, mThi, mTlo, mV;
  int st;
  if ((st = make_map(&mX, X, M, I, kBM, ce))) return st;  // XV A side (128 token rows)
  if (r > 0) {
    t_hi = static_cast<bf16*>(ws);
    t_lo = reinterpret_cast<bf16*>(static_cast<uint8_t*>(ws) + forward_umma_workspace_bytes(M, r) / 2);
    // ---- T = X . V (fp32 in tensor memory) -> bf16 high and low parts
    if ((st = make_map(&mV, V, I, r, kBK, ce))) return st;  // box: 64 rank columns x 64 rows of I
    Args a = {};
    a.rows = (int)M;
    a.cols = r;
    a.kb1 = kb;
    a.kb2 = 0;
    a.t_hi = t_hi;
    a.t_lo = t_lo;
    a.r = r;
    a.err = c.err;
    const int m_tiles = (int)ceil_div(M, kBM);
    a.splits = pick_splits(m_tiles, kb, c.num_sms);
    const int rp = (int)ceil_div(r, 64) * 64;
    cudaError_t e;
    switch (rp) {
      case 64: e = launch_tile_kernel<64, MODE_XV>(c, mX, mV, mV, mV, mV, a, m_tiles, 1); break;
      case 128: e = launch_tile_kernel<128, MODE_XV>(c, mX, mV, mV, mV, mV, a, m_tiles, 1); break;
      case 192: e = launch_tile_kernel<192, MODE_XV>(c, mX, mV, mV, mV, mV, a, m_tiles, 1); break;
      default: e = launch_tile_kernel<256, MODE_XV>(c, mX, mV, mV, mV, mV, a, m_tiles, 1); break;
    }
    if (e != cudaSuccess) {
      *ce = e;
      return THETA_ERR_CUDA;
    }
  }
  // ---- Y = s * (X . W0^T) + T . U^T, swap-AB: W0 rows are the MMA M side
  const int BN = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  const int m_tiles = (int)ceil_div(O, kBM);
  const int n_tiles = (int)ceil_div(M, BN);
  if ((st = make_map(&mW0, W0, O, I, kBM, ce))) return st;
  CUtensorMap mXb;
  if ((st = make_map(&mXb, X, M, I, BN, ce))) return st;
  if (r > 0) {
    if ((st = make_map(&mU, U, O, r, kBM, ce))) return st;
    if ((st = make_map(&mThi, t_hi, M, r, BN, ce))) return st;
    if ((st = make_map(&mTlo, t_lo, M, r, BN, ce))) return st;
  } else {
    mU = mW0;
    mThi = mTlo = mXb;
  }
  Args a = {};
  a.rows = (int)O;
  a.cols = (int)M;
  a.kb1 = kb;
  a.kb2 = r > 0 ? (int)ceil_div(r, kBK) : 0;
  a.s = s;
  a.out = static_cast<bf16*>(Y);
  a.err = c.err;
  a.splits = pick_splits((int64_t)m_tiles * n_tiles, kb, c.num_sms);
  cudaError_t e;
  switch (BN) {
    case 16: e = launch_tile_kernel<16, MODE_FORWARD>(c, mW0, mXb, mU, mThi, mTlo, a, m_tiles, n_tiles); break;
    case 32: e = launch_tile_kernel<32, MODE_FORWARD>(c, mW0, mXb, mU, mThi, mTlo, a, m_tiles, n_tiles); break;
    case 64: e = launch_tile_kernel<64, MODE_FORWARD>(c, mW0, mXb, mU, mThi, mTlo, a, m_tiles, n_tiles); break;
    default: e = launch_tile_kernel<128, MODE_FORWARD>(c, mW0, mXb, mU, mThi, mTlo, a, m_tiles, n_tiles); break;
  }
  if (e != cudaSuccess) {
    *ce = e;
    return THETA_ERR_CUDA;
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
    scale_rows_kernel<<<(unsigned)grid, 256, 0, c.stream>>>(s, static_cast<const bf16*>(W0), I, nvec,
                                                           static_cast<bf16*>(W_out));
    *ce = cudaGetLastError();
    return *ce == cudaSuccess ? THETA_OK : THETA_ERR_CUDA;
  }
  if (O > (int64_t)65535 * kBM || I > ((int64_t)1 << 31) - 256 || r > ((int64_t)1 << 20)) return THETA_ERR_UNSUPPORTED;
  constexpr int BN = 128;
  CUtensorMap mU, mV;
  int st;
  if ((st = make_map(&mU, U, O, r, kBM, ce))) return st;
  if ((st = make_map(&mV, V, I, r, BN, ce))) return st;
  Args a = {};
  a.rows = (int)O;
  a.cols = (int)I;
  a.kb1 = (int)ceil_div(r, kBK);
  a.kb2 = 0;
  a.splits = 1;
  a.s = s;
  a.W0 = static_cast<const bf16*>(W0);
  a.out = static_cast<bf16*>(W_out);
  a.err = c.err;
  cudaError_t e = launch_tile_kernel<BN, MODE_RECON>(c, mU, mV, mU, mV, mV, a, (int)ceil_div(O, kBM),
                                                     (int)ceil_div(I, BN));
  if (e != cudaSuccess) {
    *ce = e;
    return THETA_ERR_CUDA;
  }
  return THETA_OK;
}

}  // namespace theta
