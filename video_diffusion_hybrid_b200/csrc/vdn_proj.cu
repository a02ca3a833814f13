// Output projection of the hybrid attention layer: one GEMM over the output's
// concat axis.
//
// What it computes (PaperDaily digest section 三: each branch is gated and
// projected; the two outputs of the core sit on a size-2 axis so that one
// projection with the stacked weight [W_o^sm; W_o^lin] equals the sum of the
// two separate projections):
//   out[m, n] = sum_k Y[m, k] W[k, n],   Y = y viewed as [B*T*N, H*2*d_v]
// (row k = (h, slot, i) of the per-token [H, 2, d_v] block), W [H*2*d_v, n].
//
// A plain dense GEMM: cuBLASLt (bf16 operands, fp32 accumulation and scale,
// bf16 or fp32 output), no workspace.  Row-major out = Y W is computed as the
// column-major product out^T = W^T Y^T, which reads both operands as they lie.
// FP8 linear layer (deepmagic post "生成比播放還快", section 實測數據: the
// per-block latency reaches its lowest figure once optimized kernels and FP8
// linear layers are added): e4m3 operands with one dequantisation scale per
// tensor, the weight given transposed ([n, K], both operands K-contiguous as
// FP8 GEMMs need).
#include <cublasLt.h>
#include <cuda_fp8.h>

#include <mutex>

#include "vdn_internal.h"

namespace vdn {
namespace {

std::once_flag g_lt_once;
cublasLtHandle_t g_lt = nullptr;

cublasLtHandle_t lt_handle() {
  std::call_once(g_lt_once, [] {
    if (cublasLtCreate(&g_lt) != CUBLAS_STATUS_SUCCESS) g_lt = nullptr;
  });
  return g_lt;
}

// RAII holders of the cuBLASLt descriptors of one call
struct Desc {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t a = nullptr, b = nullptr, d = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  ~Desc() {
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    if (d) cublasLtMatrixLayoutDestroy(d);
    if (b) cublasLtMatrixLayoutDestroy(b);
    if (a) cublasLtMatrixLayoutDestroy(a);
    if (op) cublasLtMatmulDescDestroy(op);
  }
};

}  // namespace

vdn_status out_proj(int M, int K, int N, int out_dtype, const void* y, const void* w, void* out, cudaStream_t s,
                    const float* scales) {
  cublasLtHandle_t h = lt_handle();
  if (!h) return VDN_ERR_CUDA;
  const cudaDataType_t tout = out_dtype == VDN_BF16 ? CUDA_R_16BF : CUDA_R_32F;
  const bool fp8 = scales != nullptr;
  Desc ds;
  if (cublasLtMatmulDescCreate(&ds.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) return VDN_ERR_CUDA;
  if (fp8) {
    // e4m3 operands, both K-contiguous: A = w given as [N, K] row-major, read
    // transposed (column-major K x N, ld K); the dequantisation scales of w and
    // y multiply the product
    const cublasOperation_t ta = CUBLAS_OP_T;
    const float* sw = scales + 1;
    const float* sy = scales;
    if (cublasLtMatmulDescSetAttribute(ds.op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta)) != CUBLAS_STATUS_SUCCESS ||
        cublasLtMatmulDescSetAttribute(ds.op, CUBLASLT_MATMUL_DESC_A_SCALE_POINTER, &sw, sizeof(sw)) !=
            CUBLAS_STATUS_SUCCESS ||
        cublasLtMatmulDescSetAttribute(ds.op, CUBLASLT_MATMUL_DESC_B_SCALE_POINTER, &sy, sizeof(sy)) !=
            CUBLAS_STATUS_SUCCESS)
      return VDN_ERR_CUDA;
    if (cublasLtMatrixLayoutCreate(&ds.a, CUDA_R_8F_E4M3, K, N, K) != CUBLAS_STATUS_SUCCESS ||
        cublasLtMatrixLayoutCreate(&ds.b, CUDA_R_8F_E4M3, K, M, K) != CUBLAS_STATUS_SUCCESS ||
        cublasLtMatrixLayoutCreate(&ds.d, tout, N, M, N) != CUBLAS_STATUS_SUCCESS)
      return VDN_ERR_CUDA;
  } else {
    // column-major: A = W^T (N x K, ld N), B = Y^T (K x M, ld K), D = out^T (N x M, ld N)
    if (cublasLtMatrixLayoutCreate(&ds.a, CUDA_R_16BF, N, K, N) != CUBLAS_STATUS_SUCCESS ||
        cublasLtMatrixLayoutCreate(&ds.b, CUDA_R_16BF, K, M, K) != CUBLAS_STATUS_SUCCESS ||
        cublasLtMatrixLayoutCreate(&ds.d, tout, N, M, N) != CUBLAS_STATUS_SUCCESS)
      return VDN_ERR_CUDA;
  }
  if (cublasLtMatmulPreferenceCreate(&ds.pref) != CUBLAS_STATUS_SUCCESS) return VDN_ERR_CUDA;
  size_t ws = 0;
  cublasLtMatmulPreferenceSetAttribute(ds.pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws, sizeof(ws));
  cublasLtMatmulHeuristicResult_t res;
  int found = 0;
  if (cublasLtMatmulAlgoGetHeuristic(h, ds.op, ds.a, ds.b, ds.d, ds.d, ds.pref, 1, &res, &found) !=
          CUBLAS_STATUS_SUCCESS ||
      found == 0)
    return VDN_ERR_UNSUPPORTED;
  const float one = 1.f, zero = 0.f;
  if (cublasLtMatmul(h, ds.op, &one, w, ds.a, y, ds.b, &zero, out, ds.d, out, ds.d, &res.algo, nullptr, 0, s) !=
      CUBLAS_STATUS_SUCCESS)
    return VDN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

// ---------------------------------------------------------- FP8 quantisation
// x (bf16 or fp32) -> e4m3 with one scale per tensor: s = amax(|x|) / 448 (the
// largest finite e4m3), q = e4m3(x / s) rounded to nearest even and saturated,
// so x ~ q * s.  Pass 1 reduces amax into *scale (as an unsigned bit pattern,
// which orders non-negative floats like the floats); pass 2 turns it into s
// and converts.  Grid-stride loops over 8-element vectors (16-byte loads).
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// 8 consecutive elements (16-byte aligned) as floats
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

// the first n8 * 8 elements in 8-wide vectors, the tail one by one
template <typename T>
__global__ void k_amax(const T* __restrict__ x, long long n, unsigned* amax_bits) {
  float m = 0.f;
  const long long n8 = n / 8, stride = (long long)gridDim.x * blockDim.x;
  const long long i0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long i = i0; i < n8; i += stride) {
    float v[8];
    load8(x + 8 * i, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
  }
  for (long long i = 8 * n8 + i0; i < n; i += stride) m = fmaxf(m, fabsf(to_f(x[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

template <typename T>
__global__ void k_to_fp8(const T* __restrict__ x, long long n, float* scale, __nv_fp8_storage_t* __restrict__ q) {
  const float amax = __uint_as_float(*reinterpret_cast<const unsigned*>(scale));
  const float s = amax > 0.f ? amax / 448.0f : 1.0f;
  const float inv = 1.0f / s;
  const long long n8 = n / 8, stride = (long long)gridDim.x * blockDim.x;
  const long long i0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long i = i0; i < n8; i += stride) {
    float v[8];
    load8(x + 8 * i, v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j >> 2] |= (uint32_t)__nv_cvt_float_to_fp8(v[j] * inv, __NV_SATFINITE, __NV_E4M3) << (8 * (j & 3));
    *reinterpret_cast<uint2*>(q + 8 * i) = make_uint2(w[0], w[1]);
  }
  for (long long i = 8 * n8 + i0; i < n; i += stride)
    q[i] = __nv_cvt_float_to_fp8(to_f(x[i]) * inv, __NV_SATFINITE, __NV_E4M3);
}

__global__ void k_store_scale(float* scale) {
  const float amax = __uint_as_float(*reinterpret_cast<const unsigned*>(scale));
  *scale = amax > 0.f ? amax / 448.0f : 1.0f;
}

}  // namespace

vdn_status quantize_fp8(const void* x, int dtype, long long n, void* q, float* scale, cudaStream_t s) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return VDN_ERR_CUDA;
  const int blocks = sms * 8, threads = 256;
  if (cudaMemsetAsync(scale, 0, sizeof(float), s) != cudaSuccess) return VDN_ERR_CUDA;
  auto* qq = static_cast<__nv_fp8_storage_t*>(q);
  auto* bits = reinterpret_cast<unsigned*>(scale);
  if (dtype == VDN_BF16) {
    const auto* xx = static_cast<const __nv_bfloat16*>(x);
    k_amax<<<blocks, threads, 0, s>>>(xx, n, bits);
    k_to_fp8<<<blocks, threads, 0, s>>>(xx, n, scale, qq);
  } else {
    const auto* xx = static_cast<const float*>(x);
    k_amax<<<blocks, threads, 0, s>>>(xx, n, bits);
    k_to_fp8<<<blocks, threads, 0, s>>>(xx, n, scale, qq);
  }
  k_store_scale<<<1, 1, 0, s>>>(scale);
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

}  // namespace vdn
