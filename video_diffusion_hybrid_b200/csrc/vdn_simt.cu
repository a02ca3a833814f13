// SIMT (CUDA-core fp32) kernels of the hybrid attention core.
//
// These are the exact-arithmetic path: every product and sum is an fp32 FFMA,
// so that fp32 mode meets a 1e-4 (relative to output RMS) bound against the
// fp64 oracle.  They also serve any (dtype, d) that has no tensor-core kernel.
//
// Stages (PaperDaily digest sections 二-四; deepmagic post "用兩條分支取代一條";
// aimodeling news "The VDN split"):
//   k_gram_solve : A = K^T diag(beta) K, B = V^T diag(beta) K, Cholesky of I+A,
//                  M = (I+A)^-1, C = B M          (one CTA per frame-head)
//   k_scan       : S <- alpha_t S M_t + C_t forward and backward over frames,
//                  anchors skipped, chunk-boundary snapshots
//   k_read       : R = fwd + bwd snapshot, o = R q, RMSNorm, sigmoid gate
//   k_softmax    : windowed + anchor softmax (online, flash style), gate
#include "vdn_internal.h"
#include "simt_common.cuh"

namespace vdn {
namespace {

constexpr int kThreads = 256;

// Cholesky-based SPD solve in shared memory, 256 threads.  On entry G = I + A
// and Bs = B (pitch D+1); writes M = (I+A)^-1 (to outM when not null) and
// cscale * B M (to outC).  Uses G, Bs and W = sm + 2*D*(D+1) as scratch.
template <int D>
__device__ __forceinline__ void spd_solve(float* sm, float* outM, float* outC, float cscale) {
  constexpr int P = D + 1;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float* G = sm;
  float* Bs = sm + D * P;
  float* W = sm + 2 * D * P;
  for (int j = 0; j < D; ++j) {
    const float piv = sqrtf(G[j * P + j]);
    const float inv = 1.0f / piv;
    __syncthreads();
    for (int i = j + tid; i < D; i += kThreads) G[i * P + j] = (i == j) ? piv : G[i * P + j] * inv;
    __syncthreads();
    const int m = D - j - 1;
    for (int idx = tid; idx < m * m; idx += kThreads) {
      int ii = idx / m, ll = idx - ii * m;
      if (ll <= ii) {
        int i = j + 1 + ii, l = j + 1 + ll;
        G[i * P + l] = fmaf(-G[i * P + j], G[l * P + j], G[i * P + l]);
      }
    }
    __syncthreads();
  }

  // ---- W = L^-1 (lower), row by row; two threads share a column ----------
  for (int idx = tid; idx < D * P; idx += kThreads) W[idx] = 0.f;
  __syncthreads();
  {
    const int c = tid >> 1, part = tid & 1;  // kThreads / 2 >= D for D <= 128
    for (int i = 0; i < D; ++i) {
      const bool active = (c <= i) && (c < D);
      float s = 0.f;
      if (active && c < i) {
        for (int k = c + part; k < i; k += 2) s = fmaf(G[i * P + k], W[k * P + c], s);
      }
      s += __shfl_xor_sync(0xffffffffu, s, 1);  // the pair (2c, 2c+1) shares a warp
      if (active && part == 0) W[i * P + c] = (c == i) ? 1.0f / G[i * P + i] : -s / G[i * P + i];
      __syncthreads();
    }
  }

  // ---- M = W^T W into G's storage -----------------------------------------
  {
    constexpr int MT = D / 16;
    float macc[MT][MT];
#pragma unroll
    for (int x = 0; x < MT; ++x)
#pragma unroll
      for (int y = 0; y < MT; ++y) macc[x][y] = 0.f;
    for (int k = 0; k < D; ++k) {
      float a[MT], r[MT];
#pragma unroll
      for (int x = 0; x < MT; ++x) a[x] = W[k * P + ty + 16 * x];
#pragma unroll
      for (int y = 0; y < MT; ++y) r[y] = W[k * P + tx + 16 * y];
#pragma unroll
      for (int x = 0; x < MT; ++x)
#pragma unroll
        for (int y = 0; y < MT; ++y) macc[x][y] = fmaf(a[x], r[y], macc[x][y]);
    }
    __syncthreads();  // all reads of L done before G is overwritten
#pragma unroll
    for (int x = 0; x < MT; ++x)
#pragma unroll
      for (int y = 0; y < MT; ++y) {
        int i = ty + 16 * x, j = tx + 16 * y;
        G[i * P + j] = macc[x][y];
        if (outM) outM[i * D + j] = macc[x][y];
      }
    __syncthreads();
  }

  // ---- C = B M --------------------------------------------------------------
  {
    constexpr int MT = D / 16;
    float cacc[MT][MT];
#pragma unroll
    for (int x = 0; x < MT; ++x)
#pragma unroll
      for (int y = 0; y < MT; ++y) cacc[x][y] = 0.f;
    for (int k = 0; k < D; ++k) {
      float a[MT], r[MT];
#pragma unroll
      for (int x = 0; x < MT; ++x) a[x] = Bs[(ty + 16 * x) * P + k];
#pragma unroll
      for (int y = 0; y < MT; ++y) r[y] = G[k * P + tx + 16 * y];
#pragma unroll
      for (int x = 0; x < MT; ++x)
#pragma unroll
        for (int y = 0; y < MT; ++y) cacc[x][y] = fmaf(a[x], r[y], cacc[x][y]);
    }
#pragma unroll
    for (int x = 0; x < MT; ++x)
#pragma unroll
      for (int y = 0; y < MT; ++y) outC[(ty + 16 * x) * D + tx + 16 * y] = cscale * cacc[x][y];
  }
}

// ---------------------------------------------------------------------------
// Gram/write + Cholesky solve.  text=true: the L text tokens of (b,h), output
// C/2 into half_text, no M.  Otherwise frame t = blockIdx.x of (b,h).
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_gram_solve(Dims dm, Inputs in, Work w, bool text) {
  constexpr int TT = 32;            // tokens per smem stage
  constexpr int RPT = 2 * D / 16;   // rows of [A;B] per thread
  constexpr int CPT = D / 16;       // cols per thread
  constexpr int P = D + 1;          // padded pitch of the solve matrices
  extern __shared__ float sm[];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int b = blockIdx.z, h = blockIdx.y, t = blockIdx.x;

  const T *kp, *vp;
  const float* bp;
  long long ntok;
  float* outM = nullptr;
  float* outC;
  float cscale = 1.0f;
  if (text) {
    kp = static_cast<const T*>(in.text_k) + ((long long)b * dm.L * dm.H + h) * D;
    vp = static_cast<const T*>(in.text_v) + ((long long)b * dm.L * dm.H + h) * D;
    bp = in.text_beta + (long long)b * dm.L * dm.H + h;
    ntok = dm.L;
    outC = w.half_text + ((long long)b * dm.H + h) * D * D;
    cscale = 0.5f;
  } else {
    if (is_anchor(dm, t)) return;
    long long tok0 = ((long long)b * dm.T + t) * dm.N;
    kp = static_cast<const T*>(in.k) + (tok0 * dm.H + h) * D;
    vp = static_cast<const T*>(in.v) + (tok0 * dm.H + h) * D;
    bp = in.beta + tok0 * dm.H + h;
    ntok = dm.N;
    long long fh = ((long long)b * dm.T + t) * dm.H + h;
    outM = w.M + fh * D * D;
    outC = w.Cm + fh * D * D;
  }
  const long long ts = (long long)dm.H * D;  // element stride between tokens

  // ---- phase 1: [A; B] = sum_i [beta_i k_i; beta_i v_i] k_i^T -------------
  float* Lf = sm;              // [TT][2D]
  float* Rf = sm + TT * 2 * D; // [TT][D]
  float acc[RPT][CPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[i][j] = 0.f;

  for (long long base = 0; base < ntok; base += TT) {
    for (int idx = tid; idx < TT * D; idx += kThreads) {
      int i = idx / D, c = idx % D;
      long long tok = base + i;
      float kk = 0.f, vv = 0.f, bb = 0.f;
      if (tok < ntok) {
        kk = ldf(kp + tok * ts + c);
        vv = ldf(vp + tok * ts + c);
        bb = __ldg(bp + tok * dm.H);
      }
      Lf[i * 2 * D + c] = bb * kk;
      Lf[i * 2 * D + D + c] = bb * vv;
      Rf[i * D + c] = kk;
    }
    __syncthreads();
#pragma unroll 4
    for (int i = 0; i < TT; ++i) {
      float a[RPT], r[CPT];
#pragma unroll
      for (int x = 0; x < RPT; ++x) a[x] = Lf[i * 2 * D + ty + 16 * x];
#pragma unroll
      for (int y = 0; y < CPT; ++y) r[y] = Rf[i * D + tx + 16 * y];
#pragma unroll
      for (int x = 0; x < RPT; ++x)
#pragma unroll
        for (int y = 0; y < CPT; ++y) acc[x][y] = fmaf(a[x], r[y], acc[x][y]);
    }
    __syncthreads();
  }

  // ---- phase 2: G = I + A (lower Cholesky in place), Bs = B ---------------
  float* G = sm;            // [D][P]
  float* Bs = sm + D * P;   // [D][P]

#pragma unroll
  for (int x = 0; x < RPT; ++x) {
    int r = ty + 16 * x;
#pragma unroll
    for (int y = 0; y < CPT; ++y) {
      int c = tx + 16 * y;
      if (r < D) G[r * P + c] = acc[x][y] + (r == c ? 1.0f : 0.0f);
      else Bs[(r - D) * P + c] = acc[x][y];
    }
  }
  __syncthreads();

  spd_solve<D>(sm, outM, outC, cscale);
}

__global__ void k_half_init(Dims dm, const float* __restrict__ init, float* __restrict__ half, long long n) {
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) half[i] = 0.5f * init[i];
}


// ---------------------------------------------------------------------------
// State scan.  grid (D/RB row blocks, 2 directions, B*H).  Rows of the state
// evolve independently (s_row <- alpha s_row M + c_row), so each CTA carries
// RB rows of one chain and reads the whole M_t.  Thread tile: 4 rows x CPT
// columns of the new state, from S^T (rows contiguous, one 16-byte load per
// k) and M (CPT contiguous columns per k).  The next frame's M, C rows and
// alpha are loaded into registers while the current frame computes.
// ---------------------------------------------------------------------------
template <int D, int RB>
__global__ void __launch_bounds__(kThreads)
k_scan(Dims dm, Inputs in, Work w) {
  constexpr int RG = RB / 4;               // row groups of 4
  constexpr int CG = kThreads / RG;        // column groups
  constexpr int CPT = D / CG;              // columns per thread
  constexpr int NV4 = D * D / 4 / kThreads;
  static_assert(CPT >= 1 && CG * CPT == D, "scan tiling");
  extern __shared__ float sm[];
  float* Ms = sm;          // [D][D]
  float* St = sm + D * D;  // [D][RB]  (S transposed)
  const int tid = threadIdx.x, cq = tid % CG, rq = tid / CG;
  const int c0 = cq * CPT, r0 = rq * 4;
  const int row0 = blockIdx.x * RB, dir = blockIdx.y, bh = blockIdx.z;
  const int b = bh / dm.H, h = bh % dm.H;
  const long long DD = (long long)D * D;
  // start state: half the text state, or the carried forward state
  const float* half = ((dir == 0 && in.fwd_init) ? in.fwd_init : w.half_text) + (long long)bh * DD;
  float* snap = (dir == 0 ? w.fsnap : w.bsnap) + (long long)bh * (dm.C + 1) * DD;
  auto frame = [&](int st) { return dir == 0 ? st : dm.T - 1 - st; };
  auto gidx = [&](int r, int c) { return (long long)(row0 + r0 + r) * D + c0 + c; };

  float cur[4][CPT];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      cur[r][c] = half[gidx(r, c)];
      snap[(dir == 0 ? 0 : (long long)dm.C * DD) + gidx(r, c)] = cur[r][c];
    }
#pragma unroll
  for (int c = 0; c < CPT; ++c)
    *reinterpret_cast<float4*>(St + (c0 + c) * RB + r0) = make_float4(cur[0][c], cur[1][c], cur[2][c], cur[3][c]);

  float4 mreg[NV4];
  float creg[4][CPT];
  float areg = 0.f;
  auto prefetch = [&](int st) {
    const int t = frame(st);
    const long long fh = ((long long)b * dm.T + t) * dm.H + h;
    const float4* Mg = reinterpret_cast<const float4*>(w.M + fh * DD);
#pragma unroll
    for (int v = 0; v < NV4; ++v) mreg[v] = __ldg(Mg + tid + v * kThreads);
    const float* Cg = w.Cm + fh * DD;
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < CPT; ++c) creg[r][c] = __ldg(Cg + gidx(r, c));
    areg = __ldg(in.alpha + fh);
  };
  auto next_write = [&](int st) {  // first step >= st whose frame is written
    while (st < dm.T && is_anchor(dm, frame(st))) ++st;
    return st;
  };
  int nxt = next_write(0);
  if (nxt < dm.T) prefetch(nxt);
  __syncthreads();

  for (int st = 0; st < dm.T; ++st) {
    const int t = frame(st);
    if (st == nxt) {
#pragma unroll
      for (int v = 0; v < NV4; ++v) reinterpret_cast<float4*>(Ms)[tid + v * kThreads] = mreg[v];
      const float a = areg;
      float cc[4][CPT];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < CPT; ++c) cc[r][c] = creg[r][c];
      __syncthreads();
      nxt = next_write(st + 1);
      if (nxt < dm.T) prefetch(nxt);  // in flight during this frame's arithmetic
      float acc[4][CPT];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[r][c] = 0.f;
#pragma unroll 8
      for (int i = 0; i < D; ++i) {
        const float4 sv = *reinterpret_cast<const float4*>(St + i * RB + r0);
        float mv[CPT];
        if (CPT == 2) {
          const float2 m2 = *reinterpret_cast<const float2*>(Ms + i * D + c0);
          mv[0] = m2.x;
          mv[CPT - 1] = m2.y;
        } else {
#pragma unroll
          for (int c = 0; c < CPT; ++c) mv[c] = Ms[i * D + c0 + c];
        }
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          acc[0][c] = fmaf(sv.x, mv[c], acc[0][c]);
          acc[1][c] = fmaf(sv.y, mv[c], acc[1][c]);
          acc[2][c] = fmaf(sv.z, mv[c], acc[2][c]);
          acc[3][c] = fmaf(sv.w, mv[c], acc[3][c]);
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < CPT; ++c) cur[r][c] = fmaf(a, acc[r][c], cc[r][c]);
      __syncthreads();
#pragma unroll
      for (int c = 0; c < CPT; ++c)
        *reinterpret_cast<float4*>(St + (c0 + c) * RB + r0) = make_float4(cur[0][c], cur[1][c], cur[2][c], cur[3][c]);
      // the next written frame's M store is followed by a barrier before S is read
    }
    int snap_idx = -1;
    if (dir == 0) {
      if ((t + 1) % dm.chunk == 0) snap_idx = (t + 1) / dm.chunk;
      else if (t + 1 == dm.T) snap_idx = dm.C;
    } else if (t % dm.chunk == 0) {
      snap_idx = t / dm.chunk;
    }
    if (snap_idx >= 0) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < CPT; ++c) snap[(long long)snap_idx * DD + gidx(r, c)] = cur[r][c];
    }
  }
}

// ---------------------------------------------------------------------------
// State read + RMSNorm + gate.  grid (tiles, groups, B*H).
// ---------------------------------------------------------------------------
template <typename T, typename To, int D>
__global__ void __launch_bounds__(kThreads)
k_read(Dims dm, Inputs in, Work w) {
  constexpr int TQ = 32;
  constexpr int GROUPS = kThreads / D;   // token groups
  constexpr int TPT = TQ / GROUPS;       // tokens per thread
  constexpr int P = D + 1;
  constexpr int NW = D / 32;             // warps per token group
  extern __shared__ float sm[];
  float* Rs = sm;              // [D][P]
  float* Qs = sm + D * P;      // [TQ][D]
  float* red = Qs + TQ * D;    // [TQ][NW]
  const int tid = threadIdx.x, i = tid % D, tg = tid / D;
  const int bh = blockIdx.z, b = bh / dm.H, h = bh % dm.H;
  int f0, f1, ridx;
  if (!query_group(dm, blockIdx.y, f0, f1, ridx)) return;
  const long long ntok = (long long)(f1 - f0) * dm.N;
  const long long tbase = (long long)blockIdx.x * TQ;
  if (tbase >= ntok) return;
  const long long DD = (long long)D * D;

  const float* fs = w.fsnap + ((long long)bh * (dm.C + 1) + (ridx < dm.C ? max(ridx - 1, 0) : 0)) * DD;
  const float* bs = w.bsnap + ((long long)bh * (dm.C + 1) + (ridx < dm.C ? min(ridx + 2, dm.C) : dm.C)) * DD;
  float* Rg = w.R + ((long long)bh * (dm.C + 1) + ridx) * DD;
  for (int idx = tid; idx < D * D; idx += kThreads) {
    float r = fs[idx] + bs[idx];
    Rs[(idx / D) * P + (idx % D)] = r;
    if (blockIdx.x == 0) Rg[idx] = r;
  }
  const T* q = static_cast<const T*>(in.q);
  for (int idx = tid; idx < TQ * D; idx += kThreads) {
    int tk = idx / D, c = idx % D;
    long long tok = tbase + tk;
    float v = 0.f;
    if (tok < ntok) {
      long long row = ((long long)b * dm.T + f0) * dm.N + tok;
      v = ldf(q + (row * dm.H + h) * D + c);
    }
    Qs[tk * D + c] = v;
  }
  __syncthreads();

  float o[TPT];
#pragma unroll
  for (int x = 0; x < TPT; ++x) o[x] = 0.f;
#pragma unroll 4
  for (int jj = 0; jj < D; ++jj) {
    const float r = Rs[i * P + jj];
#pragma unroll
    for (int x = 0; x < TPT; ++x) o[x] = fmaf(r, Qs[(tg * TPT + x) * D + jj], o[x]);
  }
  const int lane = tid & 31, wid = (tid % D) / 32;
#pragma unroll
  for (int x = 0; x < TPT; ++x) {
    float s = o[x] * o[x];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) red[(tg * TPT + x) * NW + wid] = s;
  }
  __syncthreads();
  const T* g = static_cast<const T*>(in.gate_lin);
  To* y = static_cast<To*>(in.y);
  const float wgt = in.rms_weight ? __ldg(in.rms_weight + (long long)h * D + i) : 1.0f;
#pragma unroll
  for (int x = 0; x < TPT; ++x) {
    const int tk = tg * TPT + x;
    const long long tok = tbase + tk;
    if (tok >= ntok) continue;
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < NW; ++u) ss += red[tk * NW + u];
    const float rs = rsqrtf(ss / D + dm.eps);
    const long long row = ((long long)b * dm.T + f0) * dm.N + tok;
    const long long gi = (row * dm.H + h) * D + i;
    const float val = sigm(ldf(g + gi)) * o[x] * rs * wgt;
    if (dm.out_mode == 0) {
      stf(y + ((row * dm.H + h) * 2 + 1) * D + i, val);
    } else {
      To* p = y + gi;
      stf(p, to_f(*p) + val);
    }
  }
}

// ---------------------------------------------------------------------------
// Windowed + anchor softmax, online (flash style).  grid (q tiles, groups, B*H).
// ---------------------------------------------------------------------------
template <typename T, typename To, int D>
__global__ void __launch_bounds__(kThreads)
k_softmax(Dims dm, Inputs in, Work w) {
  constexpr int TQ = 64, TK = 64;
  constexpr int QP = D + 4, KP = D + 1, PP = TK + 1;
  constexpr int DPL = D / 32;  // output dims per lane
  extern __shared__ float sm[];
  float* Qs = sm;                  // [TQ][QP]
  float* Ks = Qs + TQ * QP;        // [TK][KP]
  float* Vs = Ks + TK * KP;        // [TK][D]
  float* Ps = Vs + TK * D;         // [TQ][PP]
  float* mrow = Ps + TQ * PP;      // [TQ]
  float* lrow = mrow + TQ;         // [TQ]
  float* crow = lrow + TQ;         // [TQ]
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int lane = tid & 31, wid = tid >> 5;
  const int bh = blockIdx.z, b = bh / dm.H, h = bh % dm.H;
  int f0, f1, ridx;
  if (!query_group(dm, blockIdx.y, f0, f1, ridx)) return;
  const long long ntok = (long long)(f1 - f0) * dm.N;
  const long long tbase = (long long)blockIdx.x * TQ;
  if (tbase >= ntok) return;

  // key frame intervals
  int iv0[3], iv1[3], niv = 0;
  if (ridx == dm.C) {
    iv0[0] = 0; iv1[0] = dm.T; niv = 1;
  } else {
    const int lo = max(0, (ridx - 1) * dm.chunk), hi = min(dm.T, (ridx + 2) * dm.chunk);
    if (dm.anchors && lo > 0) { iv0[niv] = 0; iv1[niv] = 1; ++niv; }
    iv0[niv] = lo; iv1[niv] = hi; ++niv;
    if (dm.anchors && hi < dm.T) { iv0[niv] = dm.T - 1; iv1[niv] = dm.T; ++niv; }
  }

  const T* q = static_cast<const T*>(in.q);
  const T* kp = static_cast<const T*>(in.k);
  const T* vp = static_cast<const T*>(in.v);
  const float qs = dm.scale * 1.4426950408889634f;  // scores in log2 units
  const long long bq = (long long)b * dm.T * dm.N;   // first token of batch b
  for (int idx = tid; idx < TQ * D; idx += kThreads) {
    int r = idx / D, c = idx % D;
    long long tok = tbase + r;
    float v = 0.f;
    if (tok < ntok) v = qs * ldf(q + ((bq + (long long)f0 * dm.N + tok) * dm.H + h) * D + c);
    Qs[r * QP + c] = v;
  }
  if (tid < TQ) { mrow[tid] = -INFINITY; lrow[tid] = 0.f; crow[tid] = 0.f; }

  float oacc[8][DPL];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int u = 0; u < DPL; ++u) oacc[r][u] = 0.f;

  for (int v_ = 0; v_ < niv; ++v_) {
    const long long kstart = bq + (long long)iv0[v_] * dm.N;
    const long long klen = (long long)(iv1[v_] - iv0[v_]) * dm.N;
    for (long long kb = 0; kb < klen; kb += TK) {
      __syncthreads();  // previous tile fully consumed
      for (int idx = tid; idx < TK * D; idx += kThreads) {
        int r = idx / D, c = idx % D;
        float kv = 0.f, vv = 0.f;
        if (kb + r < klen) {
          long long off = ((kstart + kb + r) * dm.H + h) * D + c;
          kv = ldf(kp + off);
          vv = ldf(vp + off);
        }
        Ks[r * KP + c] = kv;
        Vs[r * D + c] = vv;
      }
      __syncthreads();
      // scores: rows ty*4+a, cols tx+16*c
      float s[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) s[a][c] = 0.f;
#pragma unroll 4
      for (int d = 0; d < D; ++d) {
        float qa[4], kc[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) qa[a] = Qs[(ty * 4 + a) * QP + d];
#pragma unroll
        for (int c = 0; c < 4; ++c) kc[c] = Ks[(tx + 16 * c) * KP + d];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) s[a][c] = fmaf(qa[a], kc[c], s[a][c]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int r = ty * 4 + a;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (kb + tx + 16 * c >= klen) s[a][c] = -INFINITY;
          mx = fmaxf(mx, s[a][c]);
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float mold = mrow[r];
        const float mnew = fmaxf(mold, mx);
        const float msub = (mnew == -INFINITY) ? 0.f : mnew;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float p = exp2f(s[a][c] - msub);
          Ps[r * PP + tx + 16 * c] = p;
          sum += p;
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        __syncwarp();
        if (tx == 0) {
          const float corr = exp2f(mold - msub);
          crow[r] = corr;
          lrow[r] = lrow[r] * corr + sum;
          mrow[r] = mnew;
        }
      }
      __syncthreads();
      // O = O * corr + P V ; warp wid owns rows wid*8..+8, lane owns dims lane+32u
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float corr = crow[wid * 8 + r];
#pragma unroll
        for (int u = 0; u < DPL; ++u) oacc[r][u] *= corr;
      }
#pragma unroll 4
      for (int c = 0; c < TK; ++c) {
        float vv[DPL];
#pragma unroll
        for (int u = 0; u < DPL; ++u) vv[u] = Vs[c * D + lane + 32 * u];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float p = Ps[(wid * 8 + r) * PP + c];
#pragma unroll
          for (int u = 0; u < DPL; ++u) oacc[r][u] = fmaf(p, vv[u], oacc[r][u]);
        }
      }
    }
  }
  __syncthreads();
  const T* g = static_cast<const T*>(in.gate_sm);
  To* y = static_cast<To*>(in.y);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int rr = wid * 8 + r;
    const long long tok = tbase + rr;
    if (tok >= ntok) continue;
    const float invl = 1.0f / lrow[rr];
    const long long row = bq + (long long)f0 * dm.N + tok;
    if (in.sm_lse != nullptr && lane == 0)  // natural log of the row's sum of exp(s q k)
      in.sm_lse[row * dm.H + h] = (mrow[rr] + log2f(lrow[rr])) * 0.6931471805599453f;
#pragma unroll
    for (int u = 0; u < DPL; ++u) {
      const int i = lane + 32 * u;
      const long long gi = (row * dm.H + h) * D + i;
      const float val = sigm(ldf(g + gi)) * oacc[r][u] * invl;
      if (dm.out_mode == 0) stf(y + ((row * dm.H + h) * 2) * D + i, val);
      else stf(y + gi, val);
    }
  }
}

// ------------------------------------------------------------- dispatch ----
template <typename T, int D>
cudaError_t solve_launch(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s, bool text) {
  constexpr int P = D + 1;
  const size_t smem = sizeof(float) * (size_t)max(3 * D * P, 32 * 3 * D);
  auto kern = k_gram_solve<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(text ? 1 : d.T, d.H, d.B);
  kern<<<grid, kThreads, smem, s>>>(d, in, w, text);
  return cudaGetLastError();
}

template <int D>
cudaError_t scan_launch(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  constexpr int RB = D >= 64 ? 16 : 32;
  const size_t smem = sizeof(float) * (size_t)(D * D + RB * D);
  auto kern = k_scan<D, RB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(D / RB, 2, d.B * d.H);
  kern<<<grid, kThreads, smem, s>>>(d, in, w);
  return cudaGetLastError();
}

int num_groups(const Dims& d) { return d.C + (d.anchors ? 2 : 0); }

template <typename T, typename To, int D>
cudaError_t read_launch(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  constexpr int TQ = 32;
  const size_t smem = sizeof(float) * (size_t)(D * (D + 1) + TQ * D + TQ * (D / 32));
  auto kern = k_read<T, To, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long maxtok = (long long)d.chunk * d.N;
  dim3 grid((unsigned)((maxtok + TQ - 1) / TQ), num_groups(d), d.B * d.H);
  kern<<<grid, kThreads, smem, s>>>(d, in, w);
  return cudaGetLastError();
}

template <typename T, typename To, int D>
cudaError_t softmax_launch(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  constexpr int TQ = 64, TK = 64;
  const size_t smem = sizeof(float) * (size_t)(TQ * (D + 4) + TK * (D + 1) + TK * D + TQ * (TK + 1) + 3 * TQ);
  auto kern = k_softmax<T, To, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long maxtok = (long long)d.chunk * d.N;
  dim3 grid((unsigned)((maxtok + TQ - 1) / TQ), num_groups(d), d.B * d.H);
  kern<<<grid, kThreads, smem, s>>>(d, in, w);
  return cudaGetLastError();
}

#define VDN_DISPATCH_D(FN, ...)                                                   \
  switch (d.dk) {                                                                 \
    case 32: return FN<32>(__VA_ARGS__);                                          \
    case 64: return FN<64>(__VA_ARGS__);                                          \
    case 128: return FN<128>(__VA_ARGS__);                                        \
    default: return cudaErrorInvalidValue;                                        \
  }

template <int D> cudaError_t solve_f(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s, bool text) {
  return d.bf16 ? solve_launch<__nv_bfloat16, D>(d, in, w, s, text) : solve_launch<float, D>(d, in, w, s, text);
}
using bf16 = __nv_bfloat16;
template <int D> cudaError_t read_f(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (d.bf16) return d.out_bf16 ? read_launch<bf16, bf16, D>(d, in, w, s) : read_launch<bf16, float, D>(d, in, w, s);
  return d.out_bf16 ? read_launch<float, bf16, D>(d, in, w, s) : read_launch<float, float, D>(d, in, w, s);
}
template <int D> cudaError_t softmax_f(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (d.bf16)
    return d.out_bf16 ? softmax_launch<bf16, bf16, D>(d, in, w, s) : softmax_launch<bf16, float, D>(d, in, w, s);
  return d.out_bf16 ? softmax_launch<float, bf16, D>(d, in, w, s) : softmax_launch<float, float, D>(d, in, w, s);
}

}  // namespace

cudaError_t launch_text(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  const long long n = (long long)d.B * d.H * d.dv * d.dk;
  if (d.L > 0) { VDN_DISPATCH_D(solve_f, d, in, w, s, true) }
  if (in.init_state) {
    k_half_init<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(d, in.init_state, w.half_text, n);
    return cudaGetLastError();
  }
  return cudaMemsetAsync(w.half_text, 0, sizeof(float) * n, s);
}

cudaError_t launch_solve_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  VDN_DISPATCH_D(solve_f, d, in, w, s, false)
}

cudaError_t launch_scan_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  VDN_DISPATCH_D(scan_launch, d, in, w, s)
}

cudaError_t launch_read_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  VDN_DISPATCH_D(read_f, d, in, w, s)
}

cudaError_t launch_softmax_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  VDN_DISPATCH_D(softmax_f, d, in, w, s)
}

}  // namespace vdn
