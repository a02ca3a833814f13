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

// R pivots per round (a panel: the rows of one register block, P = [p R, p R + R)).
// The same fold as above, on the whole panel: with G' = G and G_PP - I in
// place of the panel's diagonal block, Z = G_PP^-1, every entry becomes
//   G_ij - G'_iP Z G'_Pj,
// which is the block sweep on P (G_iP Z on column P, Z G_Pj on row P) and
// 2 I - Z on the block itself, so the same surplus 2 on the diagonal.  A round:
//   1. the row block p writes its rows of G' to shared memory; its diagonal
//      thread, which holds G_PP, writes G_PP - I, inverts G_PP in its
//      registers (the single-thread sweep of an R x R block, eigenvalues >= 1:
//      a Schur complement of I + A), writes Z and keeps 2 I - Z as its result;
//   2. V = Z G'_P (R x D) is formed once, a few entries per thread;
//   3. every other thread subtracts C V from its block, C = its rows of G'_P^T
//      (= G'_iP by symmetry), as R rank-one updates with no barrier between.
// Two barriers per R pivots.  The rows and Z
// alternate between two buffers with the round, V has one.  The block
// inverse takes the hardware reciprocal approximation (relative error below
// 2^-22 on pivots >= 1).  (Forming the inverses one round ahead in a ninth
// warp, off the other threads' path, measured slower: the 288-thread CTA
// leaves 112 registers a thread for two CTAs per SM.)
// buf: sweep_panel_floats<D>() floats of shared memory.
template <int D>
__host__ __device__ constexpr int sweep_panel_floats() {
  return 2 * (D / 16) * (D + 4) + 2 * (D / 16) * (D / 16) + (D / 16) * (D + 4);
}

// Where V's column j lives: for R = 8 the two 4-column halves of every
// thread's 8 columns are stored 64 floats apart, so that the 128-bit loads of
// eight neighbouring threads fall on distinct banks.
template <int D>
__device__ __forceinline__ int vcol(int j) {
  if constexpr (D / 16 == 8) return ((j >> 2) & 1) * 64 + (j >> 3) * 4 + (j & 3);
  return j;
}

template <int D>
__device__ __forceinline__ void sweep_panels(float (&g)[D / 16][D / 16], float* buf) {
  constexpr int R = D / 16;
  constexpr int BP = D + 4;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int r0 = ty * R, c0 = tx * R;
  float* V = buf + 2 * R * BP + 2 * R * R;  // [R][BP]
  for (int pb = 0; pb < 16; ++pb) {
    float* rows = buf + (pb & 1) * R * BP;          // [R][BP]: rows P of G'
    float* Z = buf + 2 * R * BP + (pb & 1) * R * R;  // [R][R]
    const bool diag = ty == pb && tx == pb;
    if (ty == pb) {
      if (diag) {
#pragma unroll
        for (int a = 0; a < R; ++a) g[a][a] -= 1.0f;
      }
#pragma unroll
      for (int a = 0; a < R; ++a) st_row<R>(rows + a * BP + c0, g[a], 1.0f);
      if (diag) {
        // back to G_PP, then the sweep of the block in place: g = -G_PP^-1
#pragma unroll
        for (int a = 0; a < R; ++a) g[a][a] += 1.0f;
#pragma unroll
        for (int k = 0; k < R; ++k) {
          float rk;
          asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rk) : "f"(g[k][k]));
#pragma unroll
          for (int i = 0; i < R; ++i) {
            if (i == k) continue;
            const float f = g[i][k] * rk;
#pragma unroll
            for (int j = 0; j < R; ++j)
              if (j != k) g[i][j] = fmaf(-f, g[k][j], g[i][j]);
          }
#pragma unroll
          for (int i = 0; i < R; ++i) {
            if (i == k) continue;
            g[i][k] *= rk;
            g[k][i] *= rk;
          }
          g[k][k] = -rk;
        }
        // Z = -g to shared memory; this block's result is 2 I - Z = 2 I + g
#pragma unroll
        for (int a = 0; a < R; ++a) {
          st_row<R>(Z + a * R, g[a], -1.0f);
          g[a][a] += 2.0f;
        }
      }
    }
    __syncthreads();  // rows P and Z written; every read of V of the last round done
    for (int e = tid; e < R * D; e += 256) {
      const int k = e / D, j = e - (e / D) * D;
      float v = 0.f;
#pragma unroll
      for (int l = 0; l < R; ++l) v = fmaf(Z[k * R + l], rows[l * BP + j], v);
      V[k * BP + vcol<D>(j)] = v;
    }
    __syncthreads();  // V written
    if (!diag) {
#pragma unroll
      for (int k = 0; k < R; ++k) {
        float cc[R], vv[R];
        ld_row<R>(cc, rows + k * BP + r0);  // G'_{i, P_k} for this thread's rows i (symmetry)
        if constexpr (R == 8) {
          const float4 v0 = *reinterpret_cast<const float4*>(V + k * BP + tx * 4);
          const float4 v1 = *reinterpret_cast<const float4*>(V + k * BP + 64 + tx * 4);
          vv[0] = v0.x; vv[1] = v0.y; vv[2] = v0.z; vv[3] = v0.w;
          vv[4] = v1.x; vv[5] = v1.y; vv[6] = v1.z; vv[7] = v1.w;
        } else {
          ld_row<R>(vv, V + k * BP + c0);
        }
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
          for (int c = 0; c < R; ++c) g[i][c] = fmaf(-cc[i], vv[c], g[i][c]);
      }
    }
  }
  if (ty == tx) {
#pragma unroll
    for (int a = 0; a < R; ++a) g[a][a] -= 2.0f;
  }
}

}  // namespace vdn
