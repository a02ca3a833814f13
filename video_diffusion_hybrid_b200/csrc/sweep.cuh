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

// Two pivots per step.  Sweeping pivots p and q = p + 1 one after the other
// equals the block sweep on P = {p, q} with Z = G_PP^-1:
//   G_ij - G_iP Z G_Pj,  G_iP Z,  Z G_Pj,  -Z   (i, j not in P / column P / row P / block)
// and the same fold holds: broadcasting rows p and q with 1 taken off their
// entries (p, p) and (q, q) (G' = G with G_PP - I) and updating every entry
// as G_ij - G'_iP Z G'_Pj gives G_iP Z on column P, Z G_Pj on row P and
// 2 I - Z on the block (since (G_PP - I) Z (G_PP - I) = G_PP - 2 I + Z), the
// same surplus 2 on the diagonal.  One barrier per two pivots; the 2 x 2
// block G_PP (a Schur complement of G, symmetric positive definite with
// eigenvalues >= 1) is inverted in closed form by its owner.
//
// rowbuf: 4 * (D + 4) floats of shared memory (two pairs of rows, used on
// alternate steps).  Ends after a barrier-free update; the caller
// synchronises before reusing rowbuf.
template <int D>
__device__ __forceinline__ void sweep_regs(float (&g)[D / 16][D / 16], float* rowbuf) {
  constexpr int R = D / 16;
  constexpr int BP = D + 4;
  static_assert(R % 2 == 0, "pivot pairs stay inside one register block");
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int r0 = ty * R, c0 = tx * R;
  for (int pb = 0; pb < 16; ++pb) {
#pragma unroll
    for (int a = 0; a < R; a += 2) {
      // rows p = pb R + a and q = p + 1; the pair of buffers alternates with
      // the step number pb R / 2 + a / 2
      float* bp = rowbuf + ((pb * (R / 2) + (a >> 1)) & 1) * 2 * BP;
      float* bq = bp + BP;
      if (ty == pb) {
        float vp[R], vq[R];
#pragma unroll
        for (int c = 0; c < R; ++c) {
          vp[c] = g[a][c];
          vq[c] = g[a + 1][c];
        }
        if (tx == pb) {
          // Z = G_PP^-1 of the 2 x 2 block [[x, y], [y, z]]
          const float x = vp[a], y = vp[a + 1], z = vq[a + 1];
          const float idet = 1.0f / (x * z - y * y);
          bp[D] = z * idet;
          bp[D + 1] = -y * idet;
          bq[D + 1] = x * idet;
          vp[a] -= 1.0f;
          vq[a + 1] -= 1.0f;
        }
        st_row<R>(bp + c0, vp, 1.0f);
        st_row<R>(bq + c0, vq, 1.0f);
      }
      __syncthreads();  // also orders the reads of this pair of buffers two steps ago
      const float z00 = bp[D], z01 = bp[D + 1], z11 = bq[D + 1];
      float colp[R], colq[R], rp[R], rq[R];
      ld_row<R>(colp, bp + r0);
      ld_row<R>(colq, bq + r0);
      ld_row<R>(rp, bp + c0);
      ld_row<R>(rq, bq + c0);
      float up[R], uq[R];  // Z G'_Pj for this thread's columns
#pragma unroll
      for (int c = 0; c < R; ++c) {
        up[c] = fmaf(z00, rp[c], z01 * rq[c]);
        uq[c] = fmaf(z01, rp[c], z11 * rq[c]);
      }
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int c = 0; c < R; ++c) g[i][c] = fmaf(-colp[i], up[c], fmaf(-colq[i], uq[c], g[i][c]));
    }
  }
  if (ty == tx) {
#pragma unroll
    for (int a = 0; a < R; ++a) g[a][a] -= 2.0f;
  }
}

}  // namespace vdn
