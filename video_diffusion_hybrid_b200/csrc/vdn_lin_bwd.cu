// Backward pass of the linear (Video Delta Attention) branch, SIMT fp32.
//
// The forward (PaperDaily digest, sections 三 and 四; deepmagic post, closed
// form of the frame write) per batch b and head h is
//   F_0 = forward start, F_{t+1} = (alpha_t F_t + B_t) M_t      (t written)
//   G_T = S_x / 2,       G_t     = (alpha_t G_{t+1} + B_t) M_t  (t written)
//   anchor frames: F_{t+1} = F_t, G_t = G_{t+1};   M_t = (I + A_t)^-1
//   R_t = F[lo(t)] + G[hi(t)],  o = R_t q,  y = sigmoid(g) * w * o / rms(o).
// Given dy (the gradient of the loss with respect to y's linear slot), these
// kernels form the gradients of q, k, v, beta, alpha, the gate logits, the
// RMSNorm weight and the forward start state; the text state is a constant.
//
//   k_bwd_states  : every F_j and G_j (the forward keeps chunk snapshots only)
//   k_bwd_read    : RMSNorm / gate backward, dq = R^T do, dR_t = sum do q^T,
//                   per query frame t; the RMS weight's per-frame partials
//                   (SIMT; for bf16 with d = 128 the tensor-core form in
//                   vdn_lin_bwd_read_tc.cu runs instead)
//   k_bwd_adjoint : lambda_j = dL/dF_j from j = T down, mu_j = dL/dG_j from
//                   j = 0 up; per written frame the products lambda_{t+1} M_t
//                   and mu_t M_t (dX of the frame's two writes)
//   k_bwd_frame   : dA_t = -(F_{t+1}^T dXf_t + G_t^T dXb_t) symmetrised,
//                   dB_t = dXf_t + dXb_t, dalpha_t
//   k_bwd_tokens  : dk = beta ((dA + dA^T) k + dB^T v), dv = beta dB k,
//                   dbeta = k^T dA k + v^T dB k (SIMT; for bf16 k, v with d = 64
//                   or 128 the tensor-core form in vdn_lin_bwd_tc.cu runs instead)
//   k_bwd_rms     : the RMS weight's gradient, summed over frames and batch
#include "vdn_internal.h"
#include "simt_common.cuh"

namespace vdn {
namespace {

constexpr int kBT = 256;  // threads per CTA
constexpr int kTok = 32;  // tokens per tile of the token kernels

struct BwdWork {
  float* Fst;  // [B,H,T+1,D,D]  F_j, the forward state over frames < j
  float* Gst;  // [B,H,T+1,D,D]  G_j, the backward state over frames >= j
  float* dRp;  // [B,T,H,D,D]    dL/dR summed over the tokens of query frame t
  float* dXf;  // [B,T,H,D,D]    lambda_{t+1} M_t, then the symmetrised dA_t
  float* dXb;  // [B,T,H,D,D]    mu_t M_t, then dB_t
  float* dwp;  // [B,T,H,D]      RMS weight gradient of frame t
};

struct Grads {
  const void* dy;
  float *dq, *dk, *dv, *dbeta, *dalpha, *dgate, *drms, *dfwd;
  uint32_t* status;
};

// The states a query of frame t reads: F[read_lo] + G[read_hi].
__host__ __device__ __forceinline__ int read_lo(const Dims& d, int t) {
  if (is_anchor(d, t)) return 0;
  return max(0, d.chunk * (t / d.chunk - 1));
}
__host__ __device__ __forceinline__ int read_hi(const Dims& d, int t) {
  if (is_anchor(d, t)) return d.T;
  return min(d.T, d.chunk * (t / d.chunk + 2));
}

__device__ __forceinline__ float4 ld4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float4 add4(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 axpy4(float a, float4 x, float4 y) {
  return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Row tiling of the two chain kernels: RB rows of a D x D state per CTA,
// each thread RPT rows x 4 columns (one float4 per row).
template <int D> struct Chain {
  static constexpr int RB = D == 32 ? 32 : 16;
  static constexpr int CG = D / 4, RG = kBT / CG, RPT = RB / RG, XP = D + 4, NV4 = D * D / 4 / kBT;
  static_assert(RG * RPT == RB && NV4 * 4 * kBT == D * D, "chain tiling");
  static constexpr size_t smem = sizeof(float) * (D * D + RB * XP);
};

// acc[p] = X[row p] M over the CTA's rows: Ms [D][D], Xs [RB][XP].
template <int D>
__device__ __forceinline__ void rows_times_m(const float* Ms, const float* Xs, int rl0, int c0,
                                             float4 (&acc)[Chain<D>::RPT]) {
  constexpr int RPT = Chain<D>::RPT, XP = Chain<D>::XP;
#pragma unroll
  for (int p = 0; p < RPT; ++p) acc[p] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    const float4 m = *reinterpret_cast<const float4*>(Ms + k * D + c0);
#pragma unroll
    for (int p = 0; p < RPT; ++p) acc[p] = axpy4(Xs[(rl0 + p) * XP + k], m, acc[p]);
  }
}

// ---------------------------------------------------------------------------
// Every state of both scans.  grid (D / RB, 2 directions, B*H).  The forward
// stored M_t and, in the slot of C_t, either C_t = B_t M_t (S' = alpha S M +
// C) or B_t itself (S' = (alpha S + B_t) M); w.bform says which.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBT) k_bwd_states(Dims dm, Inputs in, Work w, BwdWork bw) {
  using CH = Chain<D>;
  constexpr int RB = CH::RB, CG = CH::CG, RPT = CH::RPT, XP = CH::XP, NV4 = CH::NV4;
  extern __shared__ float4 sm4[];
  float* Ms = reinterpret_cast<float*>(sm4);
  float* Xs = Ms + D * D;
  const int tid = threadIdx.x, c0 = (tid % CG) * 4, rl0 = (tid / CG) * RPT;
  const int row0 = blockIdx.x * RB, dir = blockIdx.y, bh = blockIdx.z;
  const int b = bh / dm.H, h = bh % dm.H;
  const long long DD = (long long)D * D;
  const float* start = ((dir == 0 && in.fwd_init) ? in.fwd_init : w.half_text) + bh * DD;
  float* out = (dir == 0 ? bw.Fst : bw.Gst) + (long long)bh * (dm.T + 1) * DD;
  auto gi = [&](int p) { return (long long)(row0 + rl0 + p) * D + c0; };
  auto frame = [&](int s) { return dir == 0 ? s : dm.T - 1 - s; };

  float4 cur[RPT];
#pragma unroll
  for (int p = 0; p < RPT; ++p) {
    cur[p] = ld4(start + gi(p));
    st4(out + (dir == 0 ? 0 : dm.T) * DD + gi(p), cur[p]);
  }
  float4 mreg[NV4], creg[RPT];
  float areg = 0.f;
  auto prefetch = [&](int s) {
    if (s >= dm.T || is_anchor(dm, frame(s))) return;
    const long long fh = ((long long)b * dm.T + frame(s)) * dm.H + h;
    const float4* Mg = reinterpret_cast<const float4*>(w.M + fh * DD);
#pragma unroll
    for (int v = 0; v < NV4; ++v) mreg[v] = __ldg(Mg + tid + v * kBT);
#pragma unroll
    for (int p = 0; p < RPT; ++p) creg[p] = ld4(w.Cm + fh * DD + gi(p));
    areg = __ldg(in.alpha + fh);
  };
  prefetch(0);
  for (int s = 0; s < dm.T; ++s) {
    const int t = frame(s);
    float* dst = out + (long long)(dir == 0 ? t + 1 : t) * DD;
    if (is_anchor(dm, t)) {  // an identity step
#pragma unroll
      for (int p = 0; p < RPT; ++p) st4(dst + gi(p), cur[p]);
      prefetch(s + 1);
      continue;
    }
#pragma unroll
    for (int v = 0; v < NV4; ++v) reinterpret_cast<float4*>(Ms)[tid + v * kBT] = mreg[v];
    const float a = areg;
    float4 cm[RPT];
#pragma unroll
    for (int p = 0; p < RPT; ++p) {
      cm[p] = creg[p];
      const float4 x = w.bform ? axpy4(a, cur[p], cm[p]) : cur[p];
      st4(Xs + (rl0 + p) * XP + c0, x);
    }
    __syncthreads();
    prefetch(s + 1);
    float4 acc[RPT];
    rows_times_m<D>(Ms, Xs, rl0, c0, acc);
#pragma unroll
    for (int p = 0; p < RPT; ++p) {
      cur[p] = w.bform ? acc[p] : axpy4(a, acc[p], cm[p]);
      st4(dst + gi(p), cur[p]);
    }
    __syncthreads();  // Ms and Xs are rewritten by the next step
  }
}

// ---------------------------------------------------------------------------
// The adjoint scans.  grid (D / RB, 2, B*H).  Direction 0 runs the forward
// chain's adjoint lambda_j = dL/dF_j from j = T down to 0; direction 1 the
// backward chain's mu_j = dL/dG_j from j = 0 up to T.  At a written frame t
//   dXf_t = lambda_{t+1} M_t,  lambda_t = alpha_t dXf_t + direct_F(t)
//   dXb_t = mu_t M_t,          mu_{t+1} = alpha_t dXb_t + direct_G(t + 1)
// (M_t is symmetric), at an anchor the adjoint passes through.  direct_F(j)
// sums dR of the query frames that read F_j, direct_G(j) those that read G_j.
// lambda_0 goes to dfwd (when given).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBT) k_bwd_adjoint(Dims dm, Inputs in, Work w, BwdWork bw, float* dfwd) {
  using CH = Chain<D>;
  constexpr int RB = CH::RB, CG = CH::CG, RPT = CH::RPT, XP = CH::XP, NV4 = CH::NV4;
  extern __shared__ float4 sm4[];
  float* Ms = reinterpret_cast<float*>(sm4);
  float* Xs = Ms + D * D;
  const int tid = threadIdx.x, c0 = (tid % CG) * 4, rl0 = (tid / CG) * RPT;
  const int row0 = blockIdx.x * RB, dir = blockIdx.y, bh = blockIdx.z;
  const int b = bh / dm.H, h = bh % dm.H;
  const long long DD = (long long)D * D;
  const int T = dm.T, span = 2 * dm.chunk;
  auto gi = [&](int p) { return (long long)(row0 + rl0 + p) * D + c0; };
  auto frame = [&](int s) { return dir == 0 ? T - 1 - s : s; };
  // adds dR of every query frame that reads state j of this direction
  auto add_direct = [&](float4 (&v)[RPT], int j) {
    const int t0 = dir == 0 ? j : max(0, j - span), t1 = dir == 0 ? min(T, j + span) : j;
    auto add_frame = [&](int tq) {
      const float* src = bw.dRp + (((long long)b * T + tq) * dm.H + h) * DD;
#pragma unroll
      for (int p = 0; p < RPT; ++p) v[p] = add4(v[p], ld4(src + gi(p)));
    };
    for (int tq = t0; tq < t1; ++tq)
      if ((dir == 0 ? read_lo(dm, tq) : read_hi(dm, tq)) == j) add_frame(tq);
    // the anchor query frame outside that window (it reads F_0 and G_T)
    if (dm.anchors) {
      const int ta = dir == 0 ? T - 1 : 0;
      if (j == (dir == 0 ? 0 : T) && (ta < t0 || ta >= t1)) add_frame(ta);
    }
  };

  float4 cur[RPT];
#pragma unroll
  for (int p = 0; p < RPT; ++p) cur[p] = make_float4(0.f, 0.f, 0.f, 0.f);
  add_direct(cur, dir == 0 ? T : 0);
  float4 mreg[NV4];
  float areg = 0.f;
  auto prefetch = [&](int s) {
    if (s >= T || is_anchor(dm, frame(s))) return;
    const long long fh = ((long long)b * T + frame(s)) * dm.H + h;
    const float4* Mg = reinterpret_cast<const float4*>(w.M + fh * DD);
#pragma unroll
    for (int v = 0; v < NV4; ++v) mreg[v] = __ldg(Mg + tid + v * kBT);
    areg = __ldg(in.alpha + fh);
  };
  prefetch(0);
  for (int s = 0; s < T; ++s) {
    const int t = frame(s);
    const int j = dir == 0 ? t : t + 1;  // the state index this step reaches
    if (is_anchor(dm, t)) {
      add_direct(cur, j);
      prefetch(s + 1);
      continue;
    }
    const long long fh = ((long long)b * T + t) * dm.H + h;
#pragma unroll
    for (int v = 0; v < NV4; ++v) reinterpret_cast<float4*>(Ms)[tid + v * kBT] = mreg[v];
    const float a = areg;
#pragma unroll
    for (int p = 0; p < RPT; ++p) st4(Xs + (rl0 + p) * XP + c0, cur[p]);
    __syncthreads();
    prefetch(s + 1);
    float4 acc[RPT];
    rows_times_m<D>(Ms, Xs, rl0, c0, acc);
    float* dX = (dir == 0 ? bw.dXf : bw.dXb) + fh * DD;
#pragma unroll
    for (int p = 0; p < RPT; ++p) {
      st4(dX + gi(p), acc[p]);
      cur[p] = make_float4(a * acc[p].x, a * acc[p].y, a * acc[p].z, a * acc[p].w);
    }
    add_direct(cur, j);
    __syncthreads();
  }
  if (dir == 0 && dfwd != nullptr) {
#pragma unroll
    for (int p = 0; p < RPT; ++p) st4(dfwd + bh * DD + gi(p), cur[p]);
  }
}

// ---------------------------------------------------------------------------
// Read backward.  grid (T, H, B), one CTA per query frame and head, tiles of
// 32 tokens.  R = F[lo] + G[hi] stays in shared memory.
//   o = R q, r = (mean o^2 + eps)^-1/2, n = o r, y = sigmoid(g) w n
//   dg = dy w n s (1 - s),  dn = dy s w,  do = r (dn - n mean(dn n))
//   dq = R^T do,  dR += do q^T,  dw += dy s n
// ---------------------------------------------------------------------------
template <typename Ti, typename Ty, int D>
__global__ void __launch_bounds__(kBT, 1) k_bwd_read(Dims dm, Inputs in, Work w, BwdWork bw, Grads gr) {
  constexpr int RP = D + 1, QP = D + 4, MI = D / 32, RT = D / 16;
  extern __shared__ float4 sm4[];
  float* Rs = reinterpret_cast<float*>(sm4);  // [D][RP]
  float* Qs = Rs + D * RP;                    // [kTok][QP]
  float* Os = Qs + kTok * QP;                 // [kTok][QP]  do
  float* red = Os + kTok * QP;                // [8][D]
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int tx = tid & 15, ty = tid >> 4;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int T = dm.T, H = dm.H, N = dm.N;
  const long long DD = (long long)D * D, bh = (long long)b * H + h;
  const long long fh = ((long long)b * T + t) * H + h;
  {
    const float* F = bw.Fst + (bh * (T + 1) + read_lo(dm, t)) * DD;
    const float* G = bw.Gst + (bh * (T + 1) + read_hi(dm, t)) * DD;
    for (int e = tid * 4; e < D * D; e += kBT * 4) {
      const float4 v = add4(ld4(F + e), ld4(G + e));
      float* r = Rs + (e / D) * RP + (e % D);
      r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
    }
  }
  const Ti* q = static_cast<const Ti*>(in.q);
  const Ti* gl = static_cast<const Ti*>(in.gate_lin);
  const Ty* dy = static_cast<const Ty*>(gr.dy);
  const int yslots = dm.out_mode == 0 ? 2 : 1, yslot = dm.out_mode == 0 ? 1 : 0;
  float wv[MI];
#pragma unroll
  for (int m = 0; m < MI; ++m) wv[m] = in.rms_weight ? __ldg(in.rms_weight + h * D + lane + 32 * m) : 1.0f;
  float dR[RT][RT], dw[MI];
#pragma unroll
  for (int a = 0; a < RT; ++a)
#pragma unroll
    for (int c = 0; c < RT; ++c) dR[a][c] = 0.f;
#pragma unroll
  for (int m = 0; m < MI; ++m) dw[m] = 0.f;
  auto tok = [&](int n) { return ((long long)b * T + t) * N + n; };  // token row (without head)

  for (int n0 = 0; n0 < N; n0 += kTok) {
    for (int e = tid; e < kTok * D; e += kBT) {
      const int r = e / D, c = e % D, n = n0 + r;
      Qs[r * QP + c] = n < N ? to_f(q[(tok(n) * H + h) * D + c]) : 0.f;
    }
    __syncthreads();
    // ---- o = R q for the warp's four tokens
    float o[4][MI];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int m = 0; m < MI; ++m) o[p][m] = 0.f;
#pragma unroll 2
    for (int j = 0; j < D; j += 4) {
      float4 qv[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) qv[p] = *reinterpret_cast<const float4*>(Qs + (wp * 4 + p) * QP + j);
#pragma unroll
      for (int m = 0; m < MI; ++m) {
        const float* rr = Rs + (lane + 32 * m) * RP + j;
        const float r0 = rr[0], r1 = rr[1], r2 = rr[2], r3 = rr[3];
#pragma unroll
        for (int p = 0; p < 4; ++p)
          o[p][m] = fmaf(qv[p].x, r0, fmaf(qv[p].y, r1, fmaf(qv[p].z, r2, fmaf(qv[p].w, r3, o[p][m]))));
      }
    }
    // ---- RMSNorm and gate backward, row by row
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int r = wp * 4 + p, n = n0 + r;
      float* dor = Os + r * QP;
      if (n >= N) {  // warp-uniform
#pragma unroll
        for (int m = 0; m < MI; ++m) dor[lane + 32 * m] = 0.f;
        continue;
      }
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < MI; ++m) ss = fmaf(o[p][m], o[p][m], ss);
      ss = warp_sum(ss);
      const float rinv = rsqrtf(ss / D + dm.eps);
      const long long row = tok(n) * H + h;
      float dn[MI], nh[MI], dot = 0.f;
#pragma unroll
      for (int m = 0; m < MI; ++m) {
        const int i = lane + 32 * m;
        const float g = to_f(gl[row * D + i]);
        const float dyv = to_f(dy[(row * yslots + yslot) * D + i]);
        const float s = sigm(g);
        nh[m] = o[p][m] * rinv;
        gr.dgate[row * D + i] = dyv * nh[m] * wv[m] * s * (1.0f - s);
        dn[m] = dyv * s * wv[m];
        dw[m] = fmaf(dyv * s, nh[m], dw[m]);
        dot = fmaf(dn[m], nh[m], dot);
      }
      dot = warp_sum(dot) / D;
#pragma unroll
      for (int m = 0; m < MI; ++m) dor[lane + 32 * m] = rinv * (dn[m] - nh[m] * dot);
    }
    __syncthreads();
    // ---- dq = R^T do
    {
      float dq[4][MI];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int m = 0; m < MI; ++m) dq[p][m] = 0.f;
#pragma unroll 2
      for (int i = 0; i < D; i += 4) {
        float4 dv4[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) dv4[p] = *reinterpret_cast<const float4*>(Os + (wp * 4 + p) * QP + i);
#pragma unroll
        for (int m = 0; m < MI; ++m) {
          const int j = lane + 32 * m;
          const float r0 = Rs[i * RP + j], r1 = Rs[(i + 1) * RP + j], r2 = Rs[(i + 2) * RP + j],
                      r3 = Rs[(i + 3) * RP + j];
#pragma unroll
          for (int p = 0; p < 4; ++p)
            dq[p][m] = fmaf(dv4[p].x, r0, fmaf(dv4[p].y, r1, fmaf(dv4[p].z, r2, fmaf(dv4[p].w, r3, dq[p][m]))));
        }
      }
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int n = n0 + wp * 4 + p;
        if (n >= N) continue;
        float* dst = gr.dq + (tok(n) * H + h) * D;
#pragma unroll
        for (int m = 0; m < MI; ++m) dst[lane + 32 * m] = dm.grad_acc ? __fadd_rn(dst[lane + 32 * m], dq[p][m]) : dq[p][m];
      }
    }
    // ---- dR += do q^T over the tile's tokens
#pragma unroll 4
    for (int r = 0; r < kTok; ++r) {
      float dv[RT], qv[RT];
#pragma unroll
      for (int a = 0; a < RT; ++a) dv[a] = Os[r * QP + ty + 16 * a];
#pragma unroll
      for (int c = 0; c < RT; ++c) qv[c] = Qs[r * QP + tx + 16 * c];
#pragma unroll
      for (int a = 0; a < RT; ++a)
#pragma unroll
        for (int c = 0; c < RT; ++c) dR[a][c] = fmaf(dv[a], qv[c], dR[a][c]);
    }
    __syncthreads();  // Qs and Os are rewritten by the next tile
  }
  float* dst = bw.dRp + fh * DD;
#pragma unroll
  for (int a = 0; a < RT; ++a)
#pragma unroll
    for (int c = 0; c < RT; ++c) dst[(ty + 16 * a) * D + tx + 16 * c] = dR[a][c];
  if (bw.dwp != nullptr) {
#pragma unroll
    for (int m = 0; m < MI; ++m) red[wp * D + lane + 32 * m] = dw[m];
    __syncthreads();
    for (int i = tid; i < D; i += kBT) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) s += red[k * D + i];
      bw.dwp[fh * D + i] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// Per written frame: dA_t, dB_t, dalpha_t.  grid (T, H, B).
//   dA = -(F_{t+1}^T dXf + G_t^T dXb)  (M = (I + A)^-1: dA = -M dM M, and
//        M X^T = F_{t+1}^T for the forward write, G_t^T for the backward)
//   dB = dXf + dXb,  dalpha = <dXf, F_t> + <dXb, G_{t+1}>
// The symmetrised dA + dA^T replaces dXf and dB replaces dXb in place.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBT) k_bwd_frame(Dims dm, BwdWork bw, float* dalpha) {
  constexpr int RT = D / 16, KC = 16, SP = D + 1;
  extern __shared__ float4 sm4[];
  float* sm = reinterpret_cast<float*>(sm4);
  __shared__ float red[kBT / 32];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long fh = ((long long)b * dm.T + t) * dm.H + h;
  if (is_anchor(dm, t)) {
    if (tid == 0) dalpha[fh] = 0.f;
    return;
  }
  const long long DD = (long long)D * D, bh = (long long)b * dm.H + h;
  const float* F1 = bw.Fst + (bh * (dm.T + 1) + t + 1) * DD;
  const float* F0 = bw.Fst + (bh * (dm.T + 1) + t) * DD;
  const float* G0 = bw.Gst + (bh * (dm.T + 1) + t) * DD;
  const float* G1 = bw.Gst + (bh * (dm.T + 1) + t + 1) * DD;
  float* Xf = bw.dXf + fh * DD;
  float* Xb = bw.dXb + fh * DD;
  float acc[RT][RT];
#pragma unroll
  for (int a = 0; a < RT; ++a)
#pragma unroll
    for (int c = 0; c < RT; ++c) acc[a][c] = 0.f;
  float* sF = sm;               // [KC][D] rows r of F_{t+1}
  float* sX = sm + KC * D;      // dXf
  float* sG = sm + 2 * KC * D;  // G_t
  float* sY = sm + 3 * KC * D;  // dXb
  for (int r0 = 0; r0 < D; r0 += KC) {
    for (int e = tid * 4; e < KC * D; e += kBT * 4) {
      const long long ge = (long long)r0 * D + e;
      st4(sF + e, ld4(F1 + ge));
      st4(sX + e, ld4(Xf + ge));
      st4(sG + e, ld4(G0 + ge));
      st4(sY + e, ld4(Xb + ge));
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < KC; ++r) {
      float fi[RT], gi[RT], xj[RT], yj[RT];
#pragma unroll
      for (int a = 0; a < RT; ++a) {
        fi[a] = sF[r * D + ty + 16 * a];
        gi[a] = sG[r * D + ty + 16 * a];
      }
#pragma unroll
      for (int c = 0; c < RT; ++c) {
        xj[c] = sX[r * D + tx + 16 * c];
        yj[c] = sY[r * D + tx + 16 * c];
      }
#pragma unroll
      for (int a = 0; a < RT; ++a)
#pragma unroll
        for (int c = 0; c < RT; ++c) acc[a][c] = fmaf(fi[a], xj[c], fmaf(gi[a], yj[c], acc[a][c]));
    }
    __syncthreads();
  }
  // dalpha and dB (every read of dXf, dXb above is done)
  float da = 0.f;
  for (int e = tid * 4; e < D * D; e += kBT * 4) {
    const float4 x = ld4(Xf + e), y = ld4(Xb + e), f = ld4(F0 + e), g = ld4(G1 + e);
    da += x.x * f.x + x.y * f.y + x.z * f.z + x.w * f.w + y.x * g.x + y.y * g.y + y.z * g.z + y.w * g.w;
    st4(Xb + e, add4(x, y));
  }
  da = warp_sum(da);
  if ((tid & 31) == 0) red[tid >> 5] = da;
  float* S = sm;  // [D][SP] dA (staging no longer needed)
#pragma unroll
  for (int a = 0; a < RT; ++a)
#pragma unroll
    for (int c = 0; c < RT; ++c) S[(ty + 16 * a) * SP + tx + 16 * c] = -acc[a][c];
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kBT / 32; ++k) s += red[k];
    dalpha[fh] = s;
  }
  for (int e = tid; e < D * D; e += kBT) {
    const int i = e / D, j = e % D;
    Xf[e] = S[i * SP + j] + S[j * SP + i];
  }
}

// ---------------------------------------------------------------------------
// Per token: dk, dv, dbeta.  grid (T, H, B), tiles of 32 tokens; the frame's
// symmetrised dA and dB stay in shared memory.  Anchor frames are not
// written: their tokens get zero gradients.
// ---------------------------------------------------------------------------
template <typename Ti, int D>
__global__ void __launch_bounds__(kBT, 1) k_bwd_tokens(Dims dm, Inputs in, BwdWork bw, Grads gr) {
  constexpr int SP = D + 1, QP = D + 4, MI = D / 32;
  extern __shared__ float4 sm4[];
  float* As = reinterpret_cast<float*>(sm4);  // [D][SP]  dA + dA^T
  float* Bs = As + D * SP;                    // [D][SP]  dB
  float* Ks = Bs + D * SP;                    // [kTok][QP]
  float* Vs = Ks + kTok * QP;                 // [kTok][QP]
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int T = dm.T, H = dm.H, N = dm.N;
  const long long DD = (long long)D * D, fh = ((long long)b * T + t) * H + h;
  auto row_of = [&](int n) { return (((long long)b * T + t) * N + n) * H + h; };
  if (is_anchor(dm, t)) {
    // not written: zero dk, dv (left as they are when adding to the softmax branch's share)
    for (long long e = tid; !dm.grad_acc && e < (long long)N * D; e += kBT) {
      const long long row = row_of((int)(e / D));
      gr.dk[row * D + e % D] = 0.f;
      gr.dv[row * D + e % D] = 0.f;
    }
    for (int n = tid; n < N; n += kBT) gr.dbeta[row_of(n)] = 0.f;
    return;
  }
  for (int e = tid * 4; e < D * D; e += kBT * 4) {
    const float4 a = ld4(bw.dXf + fh * DD + e), c = ld4(bw.dXb + fh * DD + e);
    float* pa = As + (e / D) * SP + e % D;
    float* pb = Bs + (e / D) * SP + e % D;
    pa[0] = a.x; pa[1] = a.y; pa[2] = a.z; pa[3] = a.w;
    pb[0] = c.x; pb[1] = c.y; pb[2] = c.z; pb[3] = c.w;
  }
  const Ti* kp = static_cast<const Ti*>(in.k);
  const Ti* vp = static_cast<const Ti*>(in.v);
  for (int n0 = 0; n0 < N; n0 += kTok) {
    for (int e = tid; e < kTok * D; e += kBT) {
      const int r = e / D, c = e % D, n = n0 + r;
      const long long g = row_of(min(n, N - 1)) * D + c;
      Ks[r * QP + c] = n < N ? to_f(kp[g]) : 0.f;
      Vs[r * QP + c] = n < N ? to_f(vp[g]) : 0.f;
    }
    __syncthreads();
    float p1[4][MI], p2[4][MI], p3[4][MI];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int m = 0; m < MI; ++m) p1[p][m] = p2[p][m] = p3[p][m] = 0.f;
#pragma unroll 1
    for (int i = 0; i < D; i += 4) {
      float4 k4[4], v4[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        k4[p] = *reinterpret_cast<const float4*>(Ks + (wp * 4 + p) * QP + i);
        v4[p] = *reinterpret_cast<const float4*>(Vs + (wp * 4 + p) * QP + i);
      }
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
#pragma unroll
        for (int m = 0; m < MI; ++m) {
          const int j = lane + 32 * m;
          const float a = As[(i + ii) * SP + j], bb = Bs[(i + ii) * SP + j], bt = Bs[j * SP + i + ii];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float kk = ii == 0 ? k4[p].x : ii == 1 ? k4[p].y : ii == 2 ? k4[p].z : k4[p].w;
            const float vv = ii == 0 ? v4[p].x : ii == 1 ? v4[p].y : ii == 2 ? v4[p].z : v4[p].w;
            p1[p][m] = fmaf(kk, a, p1[p][m]);
            p2[p][m] = fmaf(vv, bb, p2[p][m]);
            p3[p][m] = fmaf(kk, bt, p3[p][m]);
          }
        }
      }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int r = wp * 4 + p, n = n0 + r;
      if (n >= N) continue;  // warp-uniform
      const long long row = row_of(n);
      const float be = __ldg(in.beta + row);
      float db = 0.f;
#pragma unroll
      for (int m = 0; m < MI; ++m) {
        const int j = lane + 32 * m;
        // the sum rounds the product first (no fused multiply-add), as adding
        // the two branches' separate outputs would
        const float gk = be * (p1[p][m] + p2[p][m]), gv = be * p3[p][m];
        gr.dk[row * D + j] = dm.grad_acc ? __fadd_rn(gr.dk[row * D + j], gk) : gk;
        gr.dv[row * D + j] = dm.grad_acc ? __fadd_rn(gr.dv[row * D + j], gv) : gv;
        db = fmaf(0.5f * Ks[r * QP + j], p1[p][m], fmaf(Vs[r * QP + j], p3[p][m], db));
      }
      db = warp_sum(db);
      if (lane == 0) gr.dbeta[row] = db;
    }
    __syncthreads();
  }
}

// drms[h, i] = sum over batch and frames of the per-frame partials.
template <int D>
__global__ void k_bwd_rms(Dims dm, const float* __restrict__ dwp, float* __restrict__ drms) {
  const int h = blockIdx.x;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float s = 0.f;
    for (int bt = 0; bt < dm.B * dm.T; ++bt) s += __ldg(dwp + ((long long)bt * dm.H + h) * D + i);
    drms[h * D + i] = s;
  }
}

template <int D> constexpr size_t read_smem() { return sizeof(float) * (D * (D + 1) + 2 * kTok * (D + 4) + 8 * D); }
template <int D> constexpr size_t frame_smem() {
  return sizeof(float) * (4 * 16 * D > D * (D + 1) ? 4 * 16 * D : D * (D + 1));
}
template <int D> constexpr size_t tokens_smem() { return sizeof(float) * (2 * D * (D + 1) + 2 * kTok * (D + 4)); }

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename Ti, typename Ty, int D>
cudaError_t launch_all(const Dims& d, const Inputs& in, const Work& w, const BwdWork& bw, const Grads& g,
                       cudaStream_t s) {
  cudaError_t e;
  const int BH = d.B * d.H;
  const dim3 chain(D / Chain<D>::RB, 2, BH), frames(d.T, d.H, d.B);
  if ((e = set_smem(k_bwd_states<D>, Chain<D>::smem)) != cudaSuccess) return e;
  k_bwd_states<D><<<chain, kBT, Chain<D>::smem, s>>>(d, in, w, bw);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (bwd_read_tc_supported(d)) {
    e = launch_bwd_read_tc(d, in, bw.Fst, bw.Gst, g.dy, g.dq, g.dgate, bw.dRp, bw.dwp, g.status, s);
    if (e != cudaSuccess) return e;
  } else {
    if ((e = set_smem(k_bwd_read<Ti, Ty, D>, read_smem<D>())) != cudaSuccess) return e;
    k_bwd_read<Ti, Ty, D><<<frames, kBT, read_smem<D>(), s>>>(d, in, w, bw, g);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = set_smem(k_bwd_adjoint<D>, Chain<D>::smem)) != cudaSuccess) return e;
  k_bwd_adjoint<D><<<chain, kBT, Chain<D>::smem, s>>>(d, in, w, bw, g.dfwd);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = set_smem(k_bwd_frame<D>, frame_smem<D>())) != cudaSuccess) return e;
  k_bwd_frame<D><<<frames, kBT, frame_smem<D>(), s>>>(d, bw, g.dalpha);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (bwd_tokens_tc_supported(d)) {
    e = launch_bwd_tokens_tc(d, in, bw.dXf, bw.dXb, g.dk, g.dv, g.dbeta, g.status, s);
    if (e != cudaSuccess) return e;
  } else {
    if ((e = set_smem(k_bwd_tokens<Ti, D>, tokens_smem<D>())) != cudaSuccess) return e;
    k_bwd_tokens<Ti, D><<<frames, kBT, tokens_smem<D>(), s>>>(d, in, bw, g);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (g.drms != nullptr) {
    k_bwd_rms<D><<<d.H, 128, 0, s>>>(d, bw.dwp, g.drms);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_d(const Dims& d, const Inputs& in, const Work& w, const BwdWork& bw, const Grads& g,
                     cudaStream_t s) {
  if (d.bf16)
    return d.out_bf16 ? launch_all<__nv_bfloat16, __nv_bfloat16, D>(d, in, w, bw, g, s)
                      : launch_all<__nv_bfloat16, float, D>(d, in, w, bw, g, s);
  return d.out_bf16 ? launch_all<float, __nv_bfloat16, D>(d, in, w, bw, g, s)
                    : launch_all<float, float, D>(d, in, w, bw, g, s);
}

}  // namespace

size_t lin_bwd_workspace(const Dims& d, size_t* off) {
  const size_t DDb = sizeof(float) * (size_t)d.dk * d.dk, bh = (size_t)d.B * d.H;
  const size_t fr = (size_t)d.B * d.T * d.H;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  size_t o = 0;
  const size_t sizes[6] = {bh * (d.T + 1) * DDb, bh * (d.T + 1) * DDb, fr * DDb, fr * DDb, fr * DDb,
                           fr * sizeof(float) * d.dk};
  for (int i = 0; i < 6; ++i) {
    if (off) off[i] = o;
    o += up(sizes[i]);
  }
  return o;
}

cudaError_t launch_lin_bwd(const Dims& d, const Inputs& in, const Work& w, const LinBwdArgs& a, cudaStream_t s) {
  size_t off[6];
  lin_bwd_workspace(d, off);
  char* base = static_cast<char*>(a.workspace);
  BwdWork bw;
  bw.Fst = reinterpret_cast<float*>(base + off[0]);
  bw.Gst = reinterpret_cast<float*>(base + off[1]);
  bw.dRp = reinterpret_cast<float*>(base + off[2]);
  bw.dXf = reinterpret_cast<float*>(base + off[3]);
  bw.dXb = reinterpret_cast<float*>(base + off[4]);
  bw.dwp = a.drms ? reinterpret_cast<float*>(base + off[5]) : nullptr;
  Grads g{a.dy, a.dq, a.dk, a.dv, a.dbeta, a.dalpha, a.dgate, a.drms, a.dfwd, a.status};
  switch (d.dk) {
    case 32: return launch_d<32>(d, in, w, bw, g, s);
    case 64: return launch_d<64>(d, in, w, bw, g, s);
    case 128: return launch_d<128>(d, in, w, bw, g, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vdn
