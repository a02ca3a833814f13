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
// same work as Cholesky + triangular inverse + W^T W, in one pass with one
// barrier per pivot and every thread busy: thread (ty, tx) of a 16 x 16 grid
// keeps the (d/16) x (d/16) elements G[ty + 16a][tx + 16b] in registers, and
// the only exchange per pivot is row p (column p equals it by symmetry).
#include "vdn_internal.h"

namespace vdn {
namespace {

constexpr int kThreadsS = 256;

// TEXT: A_x, B_x from the text_gram region; writes S_x / 2 = B_x M_x / 2 to
// the half-text state and no M.
template <int D, bool TEXT>
__global__ void __launch_bounds__(kThreadsS)
k_solve_sweep(Dims dm, Work w) {
  constexpr int R = D / 16;   // register tile edge
  constexpr int P = D + 1;    // shared pitch
  extern __shared__ float sm[];
  float* rowbuf = sm;         // [2][D]  pivot row, double-buffered
  float* Ms = sm + 2 * D;     // [D][P]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (!TEXT && is_anchor(dm, t)) return;
  const long long fh = ((long long)b * dm.T + t) * dm.H + h;
  const long long bh = (long long)b * dm.H + h;
  float* gA = TEXT ? w.text_gram + bh * 2 * D * D : w.M + fh * D * D;
  float* gB = TEXT ? gA + D * D : w.Cm + fh * D * D;
  float* outC = TEXT ? w.half_text + bh * D * D : gB;
  const float cscale = TEXT ? 0.5f : 1.0f;

  float g[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int c = 0; c < R; ++c) {
      const int i = ty + 16 * a, j = tx + 16 * c;
      g[a][c] = gA[i * D + j] + (i == j ? 1.0f : 0.0f);
    }

  for (int p = 0; p < D; ++p) {
    float* buf = rowbuf + (p & 1) * D;
    if (ty == (p & 15)) {
      // row p lives in tile row p / 16 of these threads; select it with
      // register moves (no dynamic indexing of g, which would spill it)
      const int pa = p >> 4;
      float rsel[R];
#pragma unroll
      for (int cc = 0; cc < R; ++cc) rsel[cc] = g[0][cc];
#pragma unroll
      for (int a = 1; a < R; ++a)
#pragma unroll
        for (int cc = 0; cc < R; ++cc) rsel[cc] = (a == pa) ? g[a][cc] : rsel[cc];
#pragma unroll
      for (int cc = 0; cc < R; ++cc) buf[tx + 16 * cc] = rsel[cc];
    }
    __syncthreads();  // also orders the previous reads of this buffer (two pivots ago)
    const float inv = 1.0f / buf[p];
    float colv[R], rowv[R];
#pragma unroll
    for (int a = 0; a < R; ++a) colv[a] = buf[ty + 16 * a];
#pragma unroll
    for (int c = 0; c < R; ++c) rowv[c] = buf[tx + 16 * c] * inv;
    // every element takes the rank-one update ...
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int c = 0; c < R; ++c) g[a][c] = fmaf(-colv[a], rowv[c], g[a][c]);
    // ... then the owners of row p and of column p overwrite those (one tile
    // row / column each, selected by register moves, not dynamic indexing)
    const int pa = p >> 4;
    if (ty == (p & 15)) {
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int c = 0; c < R; ++c) g[a][c] = (a == pa) ? rowv[c] : g[a][c];
    }
    if (tx == (p & 15)) {
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int c = 0; c < R; ++c) g[a][c] = (c == pa) ? ((ty + 16 * a == p) ? -inv : colv[a] * inv) : g[a][c];
    }
  }

  // M = -G_swept: to global and to shared for C = B M
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int c = 0; c < R; ++c) {
      const int i = ty + 16 * a, j = tx + 16 * c;
      Ms[i * P + j] = -g[a][c];
      if (!TEXT) gA[i * D + j] = -g[a][c];
    }
  __syncthreads();
  float acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int c = 0; c < R; ++c) acc[a][c] = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    float bv[R], mv[R];
#pragma unroll
    for (int a = 0; a < R; ++a) bv[a] = gB[(ty + 16 * a) * D + k];  // B read from global (L1)
#pragma unroll
    for (int c = 0; c < R; ++c) mv[c] = Ms[k * P + tx + 16 * c];
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
      for (int c = 0; c < R; ++c) acc[a][c] = fmaf(bv[a], mv[c], acc[a][c]);
  }
  __syncthreads();  // every read of B done before C overwrites it in place
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int c = 0; c < R; ++c) outC[(ty + 16 * a) * D + tx + 16 * c] = cscale * acc[a][c];
}

template <int D, bool TEXT>
cudaError_t launch(const Dims& d, const Work& w, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)(2 * D + D * (D + 1));
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
