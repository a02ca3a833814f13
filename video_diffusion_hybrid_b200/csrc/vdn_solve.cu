// SPD solve of the frame write: M_t = (I + A_t)^-1 and C_t = B_t M_t, one CTA
// per (batch, frame, head), for the A_t / B_t the tensor-core Gram left in the
// M_t / C_t slots of the workspace (overwritten in place).
//
// The closed form S_t = (alpha S_{t-1} + B_t)(I + A_t)^-1 (deepmagic post
// "用兩條分支取代一條"; PaperDaily digest section 四: the (I+A) inverse is the
// key of the method) needs M_t itself for the state scan, so the inverse is
// formed explicitly.  I + A_t is symmetric positive definite with every
// eigenvalue >= 1, so symmetric Gauss-Jordan elimination (the sweep operator)
// needs no pivoting: each pivot is a Schur complement of I + A_t and is >= 1.
// Sweeping all d pivots turns G = I + A into -G^-1 in d^3 multiply-adds, the
// same work as Cholesky + triangular inverse + W^T W, in one pass: a panel of
// d / 16 pivots per round, two barriers per round (sweep.cuh).
//
// Thread (ty, tx) of a 16 x 16 grid keeps the R x R block G[ty R + a][tx R + c]
// (R = d / 16) in registers.  The only exchange per round is the panel's
// rows (its columns equal them by symmetry).  The sweep's special rules for row p,
// column p and the pivot itself are folded into the one rank-one update by
// broadcasting g_pp - 1 in place of g_pp:
//   g_ij - g_ip (g_pj / g_pp)              (i, j != p)  the ordinary update
//   g_ip - g_ip (g_pp - 1) / g_pp = g_ip / g_pp          column p
//   g_pj - (g_pp - 1) g_pj / g_pp = g_pj / g_pp          row p
//   g_pp - (g_pp - 1)^2 / g_pp    = 2 - 1 / g_pp         pivot: the sweep wants
// -1 / g_pp, and since later pivots only add to this entry the surplus 2 is
// removed from the whole diagonal once, at the end.
#include "vdn_internal.h"
#include "sweep.cuh"

namespace vdn {
namespace {

constexpr int kThreadsS = 256;

// bf16 hi/lo split of 8 consecutive values: hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat16 a = __float2bfloat16_rn(x[2 * j]), b = __float2bfloat16_rn(x[2 * j + 1]);
    const __nv_bfloat16 ra = __float2bfloat16_rn(x[2 * j] - __bfloat162float(a));
    const __nv_bfloat16 rb = __float2bfloat16_rn(x[2 * j + 1] - __bfloat162float(b));
    h[j] = (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
    l[j] = (uint32_t)__bfloat16_as_ushort(ra) | ((uint32_t)__bfloat16_as_ushort(rb) << 16);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// TEXT: A_x, B_x from the text_gram region; writes S_x / 2 = B_x M_x / 2 to
// the half-text state and no M.
template <int D, bool TEXT>
__global__ void __launch_bounds__(kThreadsS, 2)
k_solve_sweep(Dims dm, Work w) {
  constexpr int R = D / 16;   // register tile edge
  constexpr int P = D + 4;    // shared pitch (16-byte rows)
  static_assert(R % 2 == 0, "pivot buffers alternate with the parity of p");
  extern __shared__ float sm[];
  float* rowbuf = sm;                           // the sweep's rows, Z and V
  float* Ms = sm + sweep_panel_floats<D>();     // [D][P]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (!TEXT && is_anchor(dm, t)) return;
  const long long fh = ((long long)b * dm.T + t) * dm.H + h;
  const long long bh = (long long)b * dm.H + h;
  float* gA = TEXT ? w.text_gram + bh * 2 * D * D : w.M + fh * D * D;
  float* gB = TEXT ? gA + D * D : w.Cm + fh * D * D;
  float* outC = TEXT ? w.half_text + bh * D * D : gB;
  const float cscale = TEXT ? 0.5f : 1.0f;
  const int r0 = ty * R, c0 = tx * R;

  float g[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a) {
    ld_row<R>(g[a], gA + (r0 + a) * D + c0);
    if (ty == tx) g[a][a] += 1.0f;
  }

  sweep_panels<D>(g, rowbuf);  // g = -G^-1

  // the tensor-core scan forms (alpha S + B_t) M_t itself: no C_t
  const bool skip_c = !TEXT && w.bform;
  // M = -G_swept: to global and to shared for C = B M
#pragma unroll
  for (int a = 0; a < R; ++a) {
    if (!skip_c) st_row<R>(Ms + (r0 + a) * P + c0, g[a], -1.0f);
    if (!TEXT) st_row<R>(gA + (r0 + a) * D + c0, g[a], -1.0f);
  }
  if constexpr (!TEXT && R == 8) {
    // operand of the tensor-core scan: [hi | lo] bf16 rows of M
    if (w.M16 != nullptr) {
      __nv_bfloat16* mh = static_cast<__nv_bfloat16*>(w.M16) + fh * 2 * D * D;
#pragma unroll
      for (int a = 0; a < R; ++a) {
        float m[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m[c] = -g[a][c];
        uint4 hi, lo;
        split8(m, hi, lo);
        *reinterpret_cast<uint4*>(mh + (r0 + a) * D + c0) = hi;
        *reinterpret_cast<uint4*>(mh + D * D + (r0 + a) * D + c0) = lo;
      }
    }
  }
  if (skip_c) return;  // uniform: B_t stays in the C_t slot
  __syncthreads();
  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int c = 0; c < R; ++c) acc[a][c] = 0.f;
#pragma unroll 1
  for (int k = 0; k < D; k += 4) {
    float4 bv[R];
#pragma unroll
    for (int a = 0; a < R; ++a) bv[a] = *reinterpret_cast<const float4*>(gB + (r0 + a) * D + k);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      float mv[R];
      ld_row<R>(mv, Ms + (k + kk) * P + c0);
#pragma unroll
      for (int a = 0; a < R; ++a) {
        const float bb = kk == 0 ? bv[a].x : kk == 1 ? bv[a].y : kk == 2 ? bv[a].z : bv[a].w;
#pragma unroll
        for (int c = 0; c < R; ++c) acc[a][c] = fmaf(bb, mv[c], acc[a][c]);
      }
    }
  }
  __syncthreads();  // every read of B done before C overwrites it in place
#pragma unroll
  for (int a = 0; a < R; ++a) st_row<R>(outC + (r0 + a) * D + c0, acc[a], cscale);
}

template <int D, bool TEXT>
cudaError_t launch(const Dims& d, const Work& w, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)(sweep_panel_floats<D>() + D * (D + 4));
  auto kern = k_solve_sweep<D, TEXT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(TEXT ? 1 : d.T, d.H, d.B), kThreadsS, smem, s>>>(d, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_solve_inplace(const Dims& d, const Work& w, cudaStream_t s) {
  switch (d.dk) {
    case 32: return launch<32, false>(d, w, s);
    case 64: return launch<64, false>(d, w, s);
    case 128: return launch<128, false>(d, w, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_text_solve_sweep(const Dims& d, const Work& w, cudaStream_t s) {
  switch (d.dk) {
    case 32: return launch<32, true>(d, w, s);
    case 64: return launch<64, true>(d, w, s);
    case 128: return launch<128, true>(d, w, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vdn
