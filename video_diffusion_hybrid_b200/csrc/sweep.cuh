// The symmetric sweep of a D x D SPD matrix held in registers by 256 threads
// (thread (ty, tx) of a 16 x 16 grid holds the R x R block G[ty R + a][tx R + c],
// R = D / 16), shared by the solve kernels.  On return the registers hold
// -G^-1.  The sweep's special rules for row p, column p and the pivot are
// folded into one rank-one update by broadcasting g_pp - 1 in place of g_pp
// (row and column p come out divided by g_pp, the pivot as 2 - 1 / g_pp; the
// surplus 2 is removed from the diagonal at the end, since later pivots only
// add to it).  Every pivot is a Schur complement of G, >= 1 for G = I + A
// with A positive semidefinite, so no pivoting is needed.
#pragma once
#include <cuda_runtime.h>

namespace vdn {

template <int R>
__device__ __forceinline__ void ld_row(float (&dst)[R], const float* src) {
  if constexpr (R % 4 == 0) {
#pragma unroll
    for (int c = 0; c < R; c += 4) {
      const float4 v = *reinterpret_cast<const float4*>(src + c);
      dst[c] = v.x; dst[c + 1] = v.y; dst[c + 2] = v.z; dst[c + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < R; c += 2) {
      const float2 v = *reinterpret_cast<const float2*>(src + c);
      dst[c] = v.x; dst[c + 1] = v.y;
    }
  }
}

template <int R>
__device__ __forceinline__ void st_row(float* dst, const float (&src)[R], float sgn) {
  if constexpr (R % 4 == 0) {
#pragma unroll
    for (int c = 0; c < R; c += 4)
      *reinterpret_cast<float4*>(dst + c) = make_float4(sgn * src[c], sgn * src[c + 1], sgn * src[c + 2], sgn * src[c + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < R; c += 2) *reinterpret_cast<float2*>(dst + c) = make_float2(sgn * src[c], sgn * src[c + 1]);
  }
}

// rowbuf: 2 * (D + 4) floats of shared memory.  Ends after a barrier-free
// update; the caller synchronises before reusing rowbuf.
template <int D>
__device__ __forceinline__ void sweep_regs(float (&g)[D / 16][D / 16], float* rowbuf) {
  constexpr int R = D / 16;
  constexpr int BP = D + 4;
  static_assert(R % 2 == 0, "pivot buffers alternate with the parity of p");
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int r0 = ty * R, c0 = tx * R;
  for (int pb = 0; pb < 16; ++pb) {
#pragma unroll
    for (int a = 0; a < R; ++a) {
      float* buf = rowbuf + (a & 1) * BP;
      if (ty == pb) {
        float v[R];
#pragma unroll
        for (int c = 0; c < R; ++c) v[c] = g[a][c];
        if (tx == pb) {
          buf[D] = 1.0f / v[a];
          v[a] -= 1.0f;
        }
        st_row<R>(buf + c0, v, 1.0f);
      }
      __syncthreads();  // also orders the reads of this buffer two pivots ago
      const float inv = buf[D];
      float colv[R], rowv[R];
      ld_row<R>(colv, buf + r0);
      ld_row<R>(rowv, buf + c0);
#pragma unroll
      for (int c = 0; c < R; ++c) rowv[c] *= inv;
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int c = 0; c < R; ++c) g[i][c] = fmaf(-colv[i], rowv[c], g[i][c]);
    }
  }
  if (ty == tx) {
#pragma unroll
    for (int a = 0; a < R; ++a) g[a][a] -= 2.0f;
  }

}

}  // namespace vdn
