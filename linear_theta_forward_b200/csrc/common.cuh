// Shared device helpers for libtheta kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "theta.h"

namespace theta {

using bf16 = __nv_bfloat16;

// Device error flags (one word per cause), set by bounded waits that ran out.
enum : unsigned { ERR_WORD_TIMEOUT = 0, ERR_WORD_COUNT = 4 };

// Upper bound of any single device wait, in nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Pointer table passed by value as a kernel parameter.
struct PtrTable {
  const void* p[THETA_MAX_LAYERS];
};
struct MutPtrTable {
  void* p[THETA_MAX_LAYERS];
};

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_timeout(unsigned* err) {
  if (err) atomicExch(err + ERR_WORD_TIMEOUT, 1u);
}

// 1 if some wait on this device ran out since theta_device_status() last
// cleared the flag. Kernels with bounded waits start with their abort flag
// set to this, so after one timeout the rest give up at once (their results
// are undefined until the status is read) instead of each waiting out its
// own limit.
__device__ __forceinline__ int prior_timeout(const unsigned* err) {
  return (err && *reinterpret_cast<const volatile unsigned*>(err + ERR_WORD_TIMEOUT)) ? 1 : 0;
}

// ------------------------------------------------------------- element I/O
// 16-byte vectors: 8 bf16 or 4 fp32 elements.
template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  using raw = float4;
};
template <>
struct Vec<bf16> {
  static constexpr int N = 8;
  using raw = uint4;
};

__device__ __forceinline__ void unpack(const float4& r, float (&f)[4]) {
  f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
}
__device__ __forceinline__ void unpack(const uint4& r, float (&f)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ float4 pack(const float (&f)[4], float4*) {
  return make_float4(f[0], f[1], f[2], f[3]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 pack(const float (&f)[8], uint4*) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// Read-only streaming load of 16 bytes (weights are read once per pass).
template <typename R>
__device__ __forceinline__ R ld_stream(const R* p) {
  return __ldg(p);
}

// One element of the residual w - s*w0 as one fused multiply-add, rounded
// once to fp32. Stored as bf16 it is rounded a second time; the two roundings
// agree with one rounding of the exact value except when the fp32 result
// lands exactly halfway between two bf16 values (every such point is an fp32
// number, so the first rounding can reach one but never cross it), where the
// stored value may be the other neighbour: at most one bf16 ulp from the
// correctly rounded residual.
template <typename T>
__device__ __forceinline__ float residual_elem(float s, float w0, float w) {
  return fmaf(-s, w0, w);
}

// x / n rounded once (IEEE division). For n a power of two the quotient is
// x * 2^-k, which is what the multiplication below computes and rounds
// identically, so the costly division sequence runs only for other n.
struct DivByCount {
  float inv;
  float fn;
  bool pow2;
  __device__ __forceinline__ explicit DivByCount(int n) : inv(1.f / (float)n), fn((float)n), pow2((n & (n - 1)) == 0) {}
  __device__ __forceinline__ float operator()(float x) const { return pow2 ? x * inv : __fdiv_rn(x, fn); }
};

// ------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Programmatic dependent launch (device side): wait for the previous grid's
// results before touching global memory, then let the next grid launch. The
// order matters: a grid that has let its dependent launch has already seen
// every earlier grid complete, which is what a dependent that starts early
// (a forward after its own T = X.V kernel) relies on.
//
// The wait is an opaque asm statement to the compiler, and a load through a
// `const __restrict__` kernel parameter counts as reading memory that nothing
// else writes while the kernel runs, so the compiler may legally schedule such
// a load before the wait -- and then read what the previous grid has not yet
// written. after_wait() hides a pointer's origin behind an asm statement
// ordered after the wait: every load through the returned value depends on it
// and cannot move above the wait. pdl_enter(p, q, ...) does this for the
// pointers it is given; every pointer whose target an earlier grid may write
// must pass through one of the two.
template <typename P>
__device__ __forceinline__ void after_wait(P& p) {
  asm volatile("" : "+l"(p) : : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... P>
__device__ __forceinline__ void pdl_enter(P&... ptrs) {
  pdl_wait();
  (after_wait(ptrs), ...);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches `kern` on `stream` with programmatic stream serialization (the
// kernel must call pdl_enter() or griddepcontrol.wait before its first global
// memory access) and, if cluster > 1, a 1-D thread-block cluster.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace theta
