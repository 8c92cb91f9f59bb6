// common.cuh -- element access, activations and launch bookkeeping shared by the kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr int kHeadDim = 128;   // d_k = d_v supported by the kernels
constexpr int kConvK = 4;       // conv width supported by the kernels

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// 8 consecutive elements <-> fp32 (16-byte aligned for bf16, 32-byte for fp32)
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
// 32 bytes in one read-only load (a whole L2 sector per lane; p 32-byte aligned).
__device__ __forceinline__ void load32_nc(const void* p, uint4& lo, uint4& hi) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y),
                 "=r"(hi.z), "=r"(hi.w)
               : "l"(p));
}
// 32 bytes in one load (p 32-byte aligned).
__device__ __forceinline__ void load32(const void* p, uint4& lo, uint4& hi) {
  asm volatile("ld.global.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y),
                 "=r"(hi.z), "=r"(hi.w)
               : "l"(p)
               : "memory");
}
// 16 values as bf16 (round to nearest even) in one 32-byte store: a whole L2 sector per lane
// (p 32-byte aligned).
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float* v) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sequence index of token t: the n with cu[n] <= t < cu[n+1] (largest such n when sequences
// are empty).  cu has N+1 entries.
__device__ __forceinline__ int seq_of_token(const int32_t* cu, int N, int t) {
  int lo = 0, hi = N;  // answer in [0, N)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  return lo;
}

// Record a device status word (first error wins).
__device__ __forceinline__ void report_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// Index checks of the bounds-check build (-DGDN_BOUNDS_CHECK, libgdn_checked.so): a failed
// check records GDN_ERR_BOUNDS in the caller's status word and the guarded access is skipped.
// In the normal build GDN_IN_BOUNDS is the constant true and costs nothing.
__device__ __forceinline__ bool bounds_ok(bool cond, int32_t* status) {
  if (!cond) report_status(status, GDN_ERR_BOUNDS);
  return cond;
}
#ifdef GDN_BOUNDS_CHECK
#define GDN_IN_BOUNDS(cond, status) (::gdn::bounds_ok((cond), (status)))
#else
#define GDN_IN_BOUNDS(cond, status) (true)
#endif

}  // namespace gdn

// ---------------------------------------------------------------- host-side launch helpers
namespace gdn_host {
// Brackets a launch with trace events when a trace is attached to this host thread.
void trace_begin(const char* name, cudaStream_t s);
void trace_end(cudaStream_t s);
// True while a trace is attached to this host thread (its launches go without programmatic
// dependent launch, so that each kernel's events bracket that kernel alone).
bool trace_attached();
// Debug and test controls set with gdn_debug_set for the calling host thread (defaults: zeros).
const gdn_debug_options& debug_opts();
}  // namespace gdn_host
