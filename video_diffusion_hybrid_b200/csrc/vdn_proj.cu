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
#include <cublasLt.h>

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

vdn_status out_proj(int M, int K, int N, int out_dtype, const void* y, const void* w, void* out, cudaStream_t s) {
  cublasLtHandle_t h = lt_handle();
  if (!h) return VDN_ERR_CUDA;
  const cudaDataType_t tout = out_dtype == VDN_BF16 ? CUDA_R_16BF : CUDA_R_32F;
  Desc ds;
  if (cublasLtMatmulDescCreate(&ds.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) return VDN_ERR_CUDA;
  // column-major: A = W^T (N x K, ld N), B = Y^T (K x M, ld K), D = out^T (N x M, ld N)
  if (cublasLtMatrixLayoutCreate(&ds.a, CUDA_R_16BF, N, K, N) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&ds.b, CUDA_R_16BF, K, M, K) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&ds.d, tout, N, M, N) != CUBLAS_STATUS_SUCCESS)
    return VDN_ERR_CUDA;
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

}  // namespace vdn
