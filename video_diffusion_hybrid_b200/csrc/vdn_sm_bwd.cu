// Backward pass of the windowed softmax branch, SIMT fp32.
//
// Forward (PaperDaily digest, section 二; deepmagic post and aimodeling news,
// the windowed softmax with first/last-frame anchors): for a query row q of
// frame t over the keys K of the frames its mask allows (the chunks
// c(t) - 1 .. c(t) + 1, the anchor frames; every frame for an anchor query)
//   o = softmax(s q K^T) V,   y_sm = sigmoid(g_sm) * o.
// Given dy (the gradient of y's softmax slot) the kernels form
//   dg = dy o sigma'(g),  dO = dy sigma(g),  Delta = <dO, o>,
//   P = exp(s q k^T - LSE),  dS = P (dO v^T - Delta),
//   dq = s dS K,  dk = s dS^T Q,  dv = P^T dO,
// the plain derivative of the forward (the pages describe the forward only).
//
//   k_sbwd_q  : one CTA per 64 query rows of a frame and head.  Pass 1 runs the
//               forward again (online softmax) for o and LSE, then dO, Delta
//               and dg; pass 2 accumulates dq.  dO, LSE and Delta go to the
//               scratch for the second kernel.
//   k_sbwd_kv : one CTA per 64 key rows of a frame and head, over every query
//               row that sees that frame (the frame mask is symmetric, so these
//               are the frames the key frame itself would see): dk, dv.
#include <math.h>

#include "vdn_internal.h"
#include "simt_common.cuh"

namespace vdn {
namespace {

constexpr int kRows = 64;   // query or key rows per tile
constexpr int kSBT = 256;   // threads per CTA (16 x 16)

// The frame intervals [lo, hi) a query of frame t may attend to (at most
// three, in increasing order, disjoint).  The mask is symmetric in the two
// frames, so these are also the query frames that see key frame t.
__device__ __forceinline__ int mask_intervals(const Dims& d, int t, int (&lo)[3], int (&hi)[3]) {
  if (is_anchor(d, t)) {
    lo[0] = 0;
    hi[0] = d.T;
    return 1;
  }
  const int c = t / d.chunk;
  const int a = max(0, d.chunk * (c - 1)), b = min(d.T, d.chunk * (c + 2));
  int n = 0;
  if (d.anchors && a > 0) { lo[n] = 0; hi[n] = 1; ++n; }
  lo[n] = a; hi[n] = b; ++n;
  if (d.anchors && b < d.T) { lo[n] = d.T - 1; hi[n] = d.T; ++n; }
  return n;
}

// c[i][j] += <A row (ty + 16 i), B row (tx + 16 j)> over D (rows in shared
// memory with pitch P).
template <int D, int P>
__device__ __forceinline__ void dot_tile(const float* A, const float* B, int ty, int tx, float (&c)[4][4]) {
#pragma unroll 4
  for (int k = 0; k < D; k += 4) {
    float4 a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(A + (ty + 16 * i) * P + k);
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = *reinterpret_cast<const float4*>(B + (tx + 16 * j) * P + k);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        c[i][j] = fmaf(a[i].x, b[j].x, fmaf(a[i].y, b[j].y, fmaf(a[i].z, b[j].z, fmaf(a[i].w, b[j].w, c[i][j]))));
  }
}

// acc[i][cc] += sum_j X[ty + 16 i][j] Y[j][tx + 16 cc] over the 64 rows j of Y.
template <int D, int XP, int YP>
__device__ __forceinline__ void mm_acc(const float* X, const float* Y, int ty, int tx, float (&acc)[4][D / 16]) {
#pragma unroll 2
  for (int j = 0; j < kRows; j += 4) {
    float4 x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const float4*>(X + (ty + 16 * i) * XP + j);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      float y[D / 16];
#pragma unroll
      for (int cc = 0; cc < D / 16; ++cc) y[cc] = Y[(j + jj) * YP + tx + 16 * cc];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float xv = jj == 0 ? x[i].x : jj == 1 ? x[i].y : jj == 2 ? x[i].z : x[i].w;
#pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) acc[i][cc] = fmaf(xv, y[cc], acc[i][cc]);
      }
    }
  }
}

// sum / max over the 16 lanes that share ty (lanes tx = 0..15 of a half warp)
__device__ __forceinline__ float sum16(float x) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float max16(float x) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

struct SmBwdWork {
  float* dO;     // [B,T,N,H,D]  dy * sigmoid(g_sm)
  float* lse;    // [B,T,N,H]    log-sum-exp of the scaled scores of each query row
  float* delta;  // [B,T,N,H]    <dO, o>
};

struct SmGrads {
  const void* dy;
  float *dq, *dk, *dv, *dgate;
};

template <int D> struct SmTile {
  static constexpr int QP = D + 4, PP = kRows + 4, DC = D / 16;
};

// rows [n0, n0 + 64) of `src` ([B, T*N, H, D] token-major, this (b, h)) into
// a [64][QP] fp32 tile; rows at or past `end` are zero.
template <typename T, int D>
__device__ __forceinline__ void load_rows(float* dst, const T* src, long long base_tok, int H, int h, long long n0,
                                          long long end) {
  constexpr int QP = SmTile<D>::QP;
  for (int e = threadIdx.x; e < kRows * D; e += kSBT) {
    const int r = e / D, c = e % D;
    const long long n = n0 + r;
    dst[r * QP + c] = n < end ? to_f(src[((base_tok + n) * H + h) * D + c]) : 0.f;
  }
}

template <typename Ti, typename Ty, int D>
__global__ void __launch_bounds__(kSBT, 1) k_sbwd_q(Dims dm, Inputs in, SmBwdWork ws, SmGrads gr) {
  using TL = SmTile<D>;
  constexpr int QP = TL::QP, PP = TL::PP, DC = TL::DC;
  extern __shared__ float4 sm4[];
  float* Qs = reinterpret_cast<float*>(sm4);
  float* Ds = Qs + kRows * QP;
  float* Ks = Ds + kRows * QP;
  float* Vs = Ks + kRows * QP;
  float* Ps = Vs + kRows * QP;  // [64][PP]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int t = blockIdx.y, bh = blockIdx.z, b = bh / dm.H, h = bh % dm.H;
  const int N = dm.N, H = dm.H;
  const long long seq = (long long)b * dm.T * N;  // first token of batch b
  const long long q0 = (long long)t * N + (long long)blockIdx.x * kRows, qend = (long long)(t + 1) * N;
  const Ti* q = static_cast<const Ti*>(in.q);
  const Ti* k = static_cast<const Ti*>(in.k);
  const Ti* v = static_cast<const Ti*>(in.v);
  const float scale = dm.scale;
  int lo[3], hi[3];
  const int niv = mask_intervals(dm, t, lo, hi);

  load_rows<Ti, D>(Qs, q, seq, H, h, q0, qend);
  // ---- pass 1: the forward again, online, for o and LSE
  float m[4], l[4], o[4][DC];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int c = 0; c < DC; ++c) o[i][c] = 0.f;
  }
  for (int iv = 0; iv < niv; ++iv) {
    const long long kend = (long long)hi[iv] * N;
    for (long long k0 = (long long)lo[iv] * N; k0 < kend; k0 += kRows) {
      __syncthreads();  // previous users of Ks, Vs, Ps
      load_rows<Ti, D>(Ks, k, seq, H, h, k0, kend);
      load_rows<Ti, D>(Vs, v, seq, H, h, k0, kend);
      __syncthreads();
      float s[4][4] = {};
      dot_tile<D, QP>(Qs, Ks, ty, tx, s);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[i][j] = (k0 + tx + 16 * j < kend) ? s[i][j] * scale : -INFINITY;
          mx = fmaxf(mx, s[i][j]);
        }
        const float mn = fmaxf(m[i], max16(mx));  // finite: every tile holds a key
        const float corr = expf(m[i] - mn);
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float p = expf(s[i][j] - mn);
          ls += p;
          Ps[(ty + 16 * i) * PP + tx + 16 * j] = p;
        }
        l[i] = l[i] * corr + sum16(ls);
        m[i] = mn;
#pragma unroll
        for (int c = 0; c < DC; ++c) o[i][c] *= corr;
      }
      __syncthreads();
      mm_acc<D, PP, QP>(Ps, Vs, ty, tx, o);
    }
  }
  // ---- gate backward, dO, Delta, LSE
  const Ti* gs = static_cast<const Ti*>(in.gate_sm);
  const Ty* dy = static_cast<const Ty*>(gr.dy);
  const int ys = dm.out_mode == 0 ? 2 : 1;  // slot 0 of [.., 2, D] or the summed y
  float lse[4], del[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty + 16 * i;
    const long long n = q0 + r;
    const bool valid = n < qend;
    const long long row = (seq + n) * H + h;
    lse[i] = m[i] + logf(l[i]);
    const float inv = 1.0f / l[i];
    float dl = 0.f;
#pragma unroll
    for (int c = 0; c < DC; ++c) {
      const int col = tx + 16 * c;
      float dOv = 0.f;
      if (valid) {
        const float ov = o[i][c] * inv;
        const float g = to_f(gs[row * D + col]);
        const float dyv = to_f(dy[row * ys * D + col]);
        const float sg = sigm(g);
        dOv = dyv * sg;
        gr.dgate[row * D + col] = dyv * ov * sg * (1.0f - sg);
        ws.dO[row * D + col] = dOv;
        dl = fmaf(dOv, ov, dl);
      }
      Ds[r * QP + col] = dOv;
    }
    del[i] = sum16(dl);
    if (valid && tx == 0) {
      ws.lse[row] = lse[i];
      ws.delta[row] = del[i];
    }
  }
  // ---- pass 2: dq = s sum_j P (dP - Delta) k_j
  float dq[4][DC];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < DC; ++c) dq[i][c] = 0.f;
  for (int iv = 0; iv < niv; ++iv) {
    const long long kend = (long long)hi[iv] * N;
    for (long long k0 = (long long)lo[iv] * N; k0 < kend; k0 += kRows) {
      __syncthreads();
      load_rows<Ti, D>(Ks, k, seq, H, h, k0, kend);
      load_rows<Ti, D>(Vs, v, seq, H, h, k0, kend);
      __syncthreads();
      float s[4][4] = {}, dp[4][4] = {};
      dot_tile<D, QP>(Qs, Ks, ty, tx, s);
      dot_tile<D, QP>(Ds, Vs, ty, tx, dp);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float p = (k0 + tx + 16 * j < kend) ? expf(s[i][j] * scale - lse[i]) : 0.f;
          Ps[(ty + 16 * i) * PP + tx + 16 * j] = p * (dp[i][j] - del[i]);
        }
      __syncthreads();
      mm_acc<D, PP, QP>(Ps, Ks, ty, tx, dq);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long n = q0 + ty + 16 * i;
    if (n >= qend) continue;
    float* dst = gr.dq + ((seq + n) * H + h) * D;
#pragma unroll
    for (int c = 0; c < DC; ++c) dst[tx + 16 * c] = dq[i][c] * scale;
  }
}

template <typename Ti, int D>
__global__ void __launch_bounds__(kSBT, 1) k_sbwd_kv(Dims dm, Inputs in, SmBwdWork ws, SmGrads gr) {
  using TL = SmTile<D>;
  constexpr int QP = TL::QP, PP = TL::PP, DC = TL::DC;
  extern __shared__ float4 sm4[];
  float* Ks = reinterpret_cast<float*>(sm4);
  float* Vs = Ks + kRows * QP;
  float* Qs = Vs + kRows * QP;
  float* Ds = Qs + kRows * QP;
  float* Pt = Ds + kRows * QP;  // [64 keys][PP]  P^T
  float* St = Pt + kRows * PP;  // [64 keys][PP]  dS^T
  float* ls = St + kRows * PP;  // [64] LSE of the tile's queries
  float* dl = ls + kRows;       // [64] Delta
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int f = blockIdx.y, bh = blockIdx.z, b = bh / dm.H, h = bh % dm.H;
  const int N = dm.N, H = dm.H;
  const long long seq = (long long)b * dm.T * N;
  const long long k0 = (long long)f * N + (long long)blockIdx.x * kRows, kend = (long long)(f + 1) * N;
  const Ti* q = static_cast<const Ti*>(in.q);
  const float scale = dm.scale;
  int lo[3], hi[3];
  const int niv = mask_intervals(dm, f, lo, hi);

  load_rows<Ti, D>(Ks, static_cast<const Ti*>(in.k), seq, H, h, k0, kend);
  load_rows<Ti, D>(Vs, static_cast<const Ti*>(in.v), seq, H, h, k0, kend);
  float dk[4][DC], dv[4][DC];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < DC; ++c) dk[i][c] = dv[i][c] = 0.f;
  for (int iv = 0; iv < niv; ++iv) {
    const long long qend = (long long)hi[iv] * N;
    for (long long q0 = (long long)lo[iv] * N; q0 < qend; q0 += kRows) {
      __syncthreads();
      load_rows<Ti, D>(Qs, q, seq, H, h, q0, qend);
      load_rows<float, D>(Ds, ws.dO, seq, H, h, q0, qend);
      for (int r = tid; r < kRows; r += kSBT) {
        const long long n = q0 + r;
        const bool valid = n < qend;
        ls[r] = valid ? ws.lse[(seq + n) * H + h] : INFINITY;  // exp(s - inf) = 0
        dl[r] = valid ? ws.delta[(seq + n) * H + h] : 0.f;
      }
      __syncthreads();
      float s[4][4] = {}, dp[4][4] = {};
      dot_tile<D, QP>(Ks, Qs, ty, tx, s);   // keys (ty + 16 i) x queries (tx + 16 j)
      dot_tile<D, QP>(Vs, Ds, ty, tx, dp);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int qc = tx + 16 * j;
          const float p = expf(s[i][j] * scale - ls[qc]);
          Pt[(ty + 16 * i) * PP + qc] = p;
          St[(ty + 16 * i) * PP + qc] = p * (dp[i][j] - dl[qc]);
        }
      __syncthreads();
      mm_acc<D, PP, QP>(Pt, Ds, ty, tx, dv);
      mm_acc<D, PP, QP>(St, Qs, ty, tx, dk);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long n = k0 + ty + 16 * i;
    if (n >= kend) continue;
    const long long row = (seq + n) * H + h;
#pragma unroll
    for (int c = 0; c < DC; ++c) {
      gr.dk[row * D + tx + 16 * c] = dk[i][c] * scale;
      gr.dv[row * D + tx + 16 * c] = dv[i][c];
    }
  }
}

template <int D> constexpr size_t q_smem() { return sizeof(float) * (4 * kRows * (D + 4) + kRows * (kRows + 4)); }
template <int D> constexpr size_t kv_smem() {
  return sizeof(float) * (4 * kRows * (D + 4) + 2 * kRows * (kRows + 4) + 2 * kRows);
}

template <typename Ti, typename Ty, int D>
cudaError_t launch_sm(const Dims& d, const Inputs& in, const SmBwdWork& ws, const SmGrads& g, cudaStream_t s) {
  cudaError_t e;
  const dim3 grid((d.N + kRows - 1) / kRows, d.T, d.B * d.H);
  if ((e = cudaFuncSetAttribute(k_sbwd_q<Ti, Ty, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)q_smem<D>())) != cudaSuccess)
    return e;
  k_sbwd_q<Ti, Ty, D><<<grid, kSBT, q_smem<D>(), s>>>(d, in, ws, g);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_sbwd_kv<Ti, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kv_smem<D>())) != cudaSuccess)
    return e;
  k_sbwd_kv<Ti, D><<<grid, kSBT, kv_smem<D>(), s>>>(d, in, ws, g);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_sm_d(const Dims& d, const Inputs& in, const SmBwdWork& ws, const SmGrads& g, cudaStream_t s) {
  if (d.bf16)
    return d.out_bf16 ? launch_sm<__nv_bfloat16, __nv_bfloat16, D>(d, in, ws, g, s)
                      : launch_sm<__nv_bfloat16, float, D>(d, in, ws, g, s);
  return d.out_bf16 ? launch_sm<float, __nv_bfloat16, D>(d, in, ws, g, s) : launch_sm<float, float, D>(d, in, ws, g, s);
}

}  // namespace

// offsets relative to the scratch handed to launch_sm_bwd; the C ABI places
// it after the 256-byte status region that heads the caller's workspace
size_t sm_bwd_workspace(const Dims& d, size_t* off) {
  const size_t rows = (size_t)d.B * d.T * d.N * d.H;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t sizes[3] = {rows * d.dv * sizeof(float), rows * sizeof(float), rows * sizeof(float)};
  size_t o = 0;
  for (int i = 0; i < 3; ++i) {
    if (off) off[i] = o;
    o += up(sizes[i]);
  }
  return o + 256;
}

cudaError_t launch_sm_bwd(const Dims& d, const Inputs& in, const SmBwdArgs& a, cudaStream_t s) {
  size_t off[3];
  sm_bwd_workspace(d, off);
  char* base = static_cast<char*>(a.workspace);
  SmBwdWork ws{reinterpret_cast<float*>(base + off[0]), reinterpret_cast<float*>(base + off[1]),
               reinterpret_cast<float*>(base + off[2])};
  SmGrads g{a.dy, a.dq, a.dk, a.dv, a.dgate};
  switch (d.dk) {
    case 32: return launch_sm_d<32>(d, in, ws, g, s);
    case 64: return launch_sm_d<64>(d, in, ws, g, s);
    case 128: return launch_sm_d<128>(d, in, ws, g, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vdn
