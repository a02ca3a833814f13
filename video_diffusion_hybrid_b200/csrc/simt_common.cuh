// Small helpers of the SIMT kernels: typed loads and stores (fp32 or bf16
// storage, fp32 arithmetic), the sigmoid, and the query groups of the read.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "vdn_internal.h"

namespace vdn {
namespace {

template <typename T> __device__ __forceinline__ float ldf(const T* p);
template <> __device__ __forceinline__ float ldf<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void stf(T* p, float x);
template <> __device__ __forceinline__ void stf<float>(float* p, float x) { *p = x; }
template <> __device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float sigm(float x) { return 1.0f / (1.0f + expf(-x)); }

// Query groups: group g < C is the non-anchor frames of chunk g (contiguous);
// groups C and C+1 are the two anchor frames.  Returns false if empty.
__device__ __forceinline__ bool query_group(const Dims& d, int g, int& f0, int& f1, int& ridx) {
  if (g < d.C) {
    f0 = g * d.chunk;
    f1 = min(d.T, f0 + d.chunk);
    if (d.anchors) {
      if (f0 == 0) f0 = 1;
      if (f1 == d.T) f1 = d.T - 1;
    }
    ridx = g;
  } else {
    f0 = (g == d.C) ? 0 : d.T - 1;
    f1 = f0 + 1;
    ridx = d.C;
  }
  return f0 < f1;
}

}  // namespace
}  // namespace vdn
