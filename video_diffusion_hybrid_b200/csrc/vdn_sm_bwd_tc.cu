// Backward of the windowed softmax branch on the tensor cores (tcgen05):
// fp16 operands, fp32 scores, statistics and accumulation.
//
// The forward (PaperDaily digest section 二; deepmagic post and aimodeling
// news, the windowed softmax with first/last-frame anchors) gives, per query
// row, y_sm = sigmoid(g) o with o = softmax(s q K^T) V over the keys its mask
// allows.  With dy the gradient of y's softmax slot:
//   dO = dy sigmoid(g),  Delta = <dO, o>,  dg = dy o sigmoid'(g)
//   P = exp(s q k^T - LSE),  dS = P (dO v^T - Delta)
//   dq = s dS K,  dk = s dS^T Q,  dv = P^T dO
// the plain derivative of the forward (the pages describe the forward only).
//
// Operand precision.  The products take fp16 operands (11 significant bits):
// q, k, v are converted exactly from bf16 (any |x| < 65504), and P, dS and dO
// are rounded to fp16, which keeps the gradients within about 2e-3 of their
// RMS where bf16 operands gave about 1.5e-2.  dO is scaled by one power of two
// per call (its largest magnitude to [0.5, 1)) so that small upstream
// gradients do not underflow; the scale is taken out in the epilogues.
//
//   k_sbwd_cvt   : fp16 copies of q, k, v
//   k_sbwd_amax  : max |dO| over the call, k_sbwd_do: the scaled fp16 dO
//   k_sbwd_q_tc  : 128 query rows of one frame-head, three passes over the
//                  key tiles: (A) S = Q K^T, the row max m; (B) P = 2^(s c - m c)
//                  as fp16 over S in TMEM, O += P V and the row sum l -> LSE and
//                  o = O / l, then dg and Delta in fp32 from o, dy and g; (C) S
//                  and dP = dO V^T, dS = P (dP - Delta) over S, dQ += dS K.
//                  Given the forward's log-sum-exp, pass A is skipped and pass
//                  B takes it as the reference in place of m (P stays <= 1; l
//                  and with it o and LSE are still formed here).
//   k_sbwd_kv_tc : 128 key rows of one frame-head, over every query tile that
//                  sees the key frame (the mask is symmetric): S^T = K Q^T,
//                  dP^T = V dO^T, P^T and dS^T over them, dV += P^T dO,
//                  dK += dS^T Q.
//
// Roles (384 threads): warp 0 producer (TMA; in the key kernel its lanes also
// stage LSE and Delta of each query tile), warp 1 TMEM allocator and MMA
// issuer (lane 0), warps 4..11 softmax and epilogues: two warps per TMEM lane
// quadrant (thread = TMEM lane = row), each with half of the columns.
// Every mbarrier wait is bounded; on expiry the CTA records VDN_ERR_TIMEOUT in
// the status words, stops issuing, drains and frees its TMEM.
#include <cuda_fp16.h>

#include "tc_common.cuh"

namespace vdn {
namespace {
using namespace tc;

constexpr int BR = 128;  // rows of a tile (queries or keys)
constexpr int kThr = 384;       // warps 0..3 roles, 4..11 softmax
constexpr int kSoftWarps = 8;   // two per TMEM lane quadrant, each with half the columns
constexpr int ST = 2;    // ring stages
constexpr float kLog2e = 1.4426950408889634f;

struct SmTcWork {
  __half *q16, *k16, *v16;  // [B*T*N, H, D]  fp16 copies of q, k, v
  __half* dO;               // [B*T*N, H, D]  dy sigmoid(g_sm) times the call's scale
  float* lse2;              // [B*T*N, H]     log2-sum-exp2 of the scores in log2 units
  float* delta;             // [B*T*N, H]     <dO, o> (unscaled)
  unsigned* amax;           // max |dO| as float bits (non-negative)
  uint32_t* status;         // bounded-wait status words
};

// Instruction descriptor, kind::f16 with fp16 A and B, fp32 D, dense (the
// same tcgen05.mma kind as bf16: mma_bf16 / mma_bf16_ts issue it, the types
// come from this descriptor).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// The power of two that brings max |dO| into [0.5, 1) (1 for an all-zero dO).
__device__ __forceinline__ float do_scale(const unsigned* amax) {
  const float a = __uint_as_float(*amax);
  if (!(a > 0.f) || !(a < 3.0e38f)) return 1.0f;
  return exp2f(-ceilf(log2f(a)));
}

static __device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Packed fp16 pairs of a 128-column score tile written back by two warps per
// row: the warp of half h reads columns [64 h, 64 h + 64) and writes its 32
// packed columns inside that range, chunk q (32 scores) at pk_col(q), so no
// write lands on columns the other warp has still to read.  The 16 keys of
// k-step k then sit at pk_k(k).
__host__ __device__ constexpr uint32_t pk_col(int q) { return 64u * (q >> 1) + 16u * (q & 1); }
__host__ __device__ constexpr uint32_t pk_k(int k) { return 8u * k + 32u * (k >> 2); }

// Named barrier of the eight softmax warps (barrier 0 is __syncthreads).
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ float sigmf(float x) { return 1.0f / (1.0f + __expf(-x)); }
__device__ __forceinline__ float tof(float x) { return x; }
__device__ __forceinline__ float tof(__nv_bfloat16 x) { return __bfloat162float(x); }

// Work item -> (frame, b, h, first row of the tile within the frame).  The
// anchor frames' items (whose row or key sets span every frame) come first.
__device__ __forceinline__ void decode(const Dims& d, long long item, int& f, int& b, int& h, int& n0) {
  const int per = (d.N + BR - 1) / BR;
  const long long BH = (long long)d.B * d.H;
  long long bh, rem;
  if (d.anchors) {
    const long long na = 2 * BH * per;
    if (item < na) {
      const long long a = item / (BH * per);
      rem = item % (BH * per);
      bh = rem / per;
      n0 = (int)(rem % per) * BR;
      f = a == 0 ? 0 : d.T - 1;
    } else {
      const long long it = item - na, per_bh = (long long)(d.T - 2) * per;
      bh = it / per_bh;
      rem = it % per_bh;
      f = 1 + (int)(rem / per);
      n0 = (int)(rem % per) * BR;
    }
  } else {
    const long long per_bh = (long long)d.T * per;
    bh = item / per_bh;
    rem = item % per_bh;
    f = (int)(rem / per);
    n0 = (int)(rem % per) * BR;
  }
  b = (int)(bh / d.H);
  h = (int)(bh % d.H);
}

// The token intervals (absolute token rows) of the frames a query of frame f
// attends to; by the symmetry of the mask also the query rows that see key
// frame f.  Three fixed slots, unused ones empty.
struct Iv {
  int beg[3], len[3];
};
__device__ __forceinline__ Iv intervals(const Dims& d, int f, int base) {
  Iv v;
  if (is_anchor(d, f)) {
    v.beg[0] = base; v.len[0] = d.T * d.N;
    v.beg[1] = base; v.len[1] = 0;
    v.beg[2] = base; v.len[2] = 0;
    return v;
  }
  const int c = f / d.chunk;
  const int lo = max(0, d.chunk * (c - 1)), hi = min(d.T, d.chunk * (c + 2));
  v.beg[0] = base; v.len[0] = (d.anchors && lo > 0) ? d.N : 0;
  v.beg[1] = base + lo * d.N; v.len[1] = (hi - lo) * d.N;
  v.beg[2] = base + (d.T - 1) * d.N; v.len[2] = (d.anchors && hi < d.T) ? d.N : 0;
  return v;
}
__device__ __forceinline__ int n_tiles(const Iv& v) {
  int n = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) n += (v.len[i] + BR - 1) / BR;
  return n;
}
__device__ __forceinline__ void tile_of(const Iv& v, int j, int& r0, int& valid) {
  r0 = 0;
  valid = 0;
  bool found = false;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int nt = (v.len[i] + BR - 1) / BR;
    if (!found) {
      if (j < nt) {
        r0 = v.beg[i] + j * BR;
        valid = min(BR, v.len[i] - j * BR);
        found = true;
      } else {
        j -= nt;
      }
    }
  }
}

// ----------------------------------------------------- elementwise (SIMT) --
__global__ void __launch_bounds__(256) k_sbwd_cvt(const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                                                  const __nv_bfloat16* __restrict__ c, __half* __restrict__ a16,
                                                  __half* __restrict__ b16, __half* __restrict__ c16, long long n8) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const __nv_bfloat16* src[3] = {a, b, c};
    __half* dst[3] = {a16, b16, c16};
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src[t]) + i);
      const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&raw);
      uint4 out;
      uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(x[e]);
        o[e] = pack_h2(f.x, f.y);
      }
      reinterpret_cast<uint4*>(dst[t])[i] = out;
    }
  }
}

// dO = dy sigmoid(g) over every (row, column); dy in y's layout (slot 0 of
// [.., 2, D], or the summed y).  MODE 0: max |dO| into ws.amax; MODE 1: the
// scaled fp16 dO.
template <typename Ty, int D, int MODE>
__global__ void __launch_bounds__(256) k_sbwd_do(Dims dm, Inputs in, const void* dyp, SmTcWork ws, long long rows) {
  const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(in.gate_sm);
  const Ty* dy = static_cast<const Ty*>(dyp);
  const int ys = dm.out_mode == 0 ? 2 : 1;
  const float sc = MODE == 1 ? do_scale(ws.amax) : 1.0f;
  float mx = 0.f;
  const long long n = rows * D;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / D;
    const int c = (int)(e % D);
    const float v = tof(dy[row * ys * D + c]) * sigmf(__bfloat162float(g[e]));
    if (MODE == 0) mx = fmaxf(mx, fabsf(v));
    else ws.dO[e] = __float2half_rn(v * sc);
  }
  if (MODE == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) atomicMax(ws.amax, __float_as_uint(mx));
  }
}

// ------------------------------------------------------------- dQ kernel --
// TMEM: S buffers 0 and 1 at columns 0 and 384, dP at 128, and at 256 the
// accumulator of the pass: O in pass B, dQ in pass C (O is read out before
// the first dQ product, which waits for the softmax of pass C's first tile).
// Every pass alternates the S buffers, so the product of tile s + 1 runs
// while the softmax works on tile s (in pass C, dP of tile s + 1 waits for
// the softmax of s, then the softmax of s + 1 overlaps dQ(s) and S(s + 2)).
template <int D, typename Ty>
__global__ void __launch_bounds__(kThr, 1)
k_sbwd_q_tc(Dims dm, Inputs in, const void* dyp, SmTcWork ws, float* dq, float* dgate, const float* lse_in,
            const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
            const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  constexpr int NB = D / 64;
  constexpr uint32_t TILE = BR * D * 2;
  constexpr uint32_t COL_P = 128, COL_ACC = 256;
  enum { B_QD = 0, B_FULL = 1, B_EMPTY = B_FULL + ST, B_SFULL = B_EMPTY + ST, B_SFULLC = B_SFULL + 2, B_SDONE,
         B_ODONE, B_DQ, B_DRAIN, NBARS };
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = sm;
  unsigned char* sDO = sQ + TILE;
  unsigned char* sK = sDO + TILE;       // ST stages
  unsigned char* sV = sK + ST * TILE;   // ST stages
  float* red = reinterpret_cast<float*>(sV + ST * TILE);  // [3][2][BR]: row max, sum, Delta of each half
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 6 * BR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*reinterpret_cast<volatile uint32_t*>(ws.status) != 0u) return;
  int f, b, h, n0;
  decode(dm, blockIdx.x, f, b, h, n0);
  const int base = b * dm.T * dm.N;
  const int q0 = base + f * dm.N + n0, qvalid = min(BR, dm.N - n0);
  const Iv iv = intervals(dm, f, base);
  // with the forward's log-sum-exp (lse_in) there is no pass A
  const int nt = n_tiles(iv), pa = lse_in != nullptr ? 0 : nt, nab = pa + nt, nsteps = pa + 2 * nt;
  const Ctl ctl{abort_flag, ws.status, (unsigned)TAG_SMBWD_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto sbuf = [](int s) { return (s & 1) ? 384u : 0u; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBARS; ++i) mbar_init(bar(i), i == B_SDONE ? kSoftWarps : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---- producer: Q and dO once; K for pass A, K and V for passes B and C
    if (lane == 0) {
      mbar_expect_tx(bar(B_QD), 2 * TILE);
      for (int c = 0; c < NB; ++c) {
        tma_load_3d(smem_u32(sQ + c * BR * 128), &tmq, bar(B_QD), c * 64, h, q0);
        tma_load_3d(smem_u32(sDO + c * BR * 128), &tmdo, bar(B_QD), c * 64, h, q0);
      }
      int issued = 0;
      for (int s = 0; s < nsteps; ++s) {
        const bool withv = s >= pa;
        int k0, kv;
        tile_of(iv, s < pa ? s : (s < nab ? s - pa : s - nab), k0, kv);
        const int st = s % ST;
        if (s >= ST && !mbar_wait(bar(B_EMPTY + st), (s / ST - 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_FULL + st), withv ? 2 * TILE : TILE);
        for (int c = 0; c < NB; ++c) {
          tma_load_3d(smem_u32(sK + st * TILE + c * BR * 128), &tmk, bar(B_FULL + st), c * 64, h, k0);
          if (withv) tma_load_3d(smem_u32(sV + st * TILE + c * BR * 128), &tmv, bar(B_FULL + st), c * 64, h, k0);
        }
        issued = s + 1;
      }
      mbar_drain(bar(B_QD), 0);
      for (int s = issued - ST < 0 ? 0 : issued - ST; s < issued; ++s)
        mbar_drain(bar(B_FULL + s % ST), (s / ST) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_f16(BR, BR, false);
      constexpr uint32_t ID_G = idesc_f16(BR, D, true);
      const uint64_t qd = sdesc(smem_u32(sQ), 16, 1024), dod = sdesc(smem_u32(sDO), 16, 1024);
      const uint64_t kd0 = sdesc(smem_u32(sK), 16, 1024), vd0 = sdesc(smem_u32(sV), 16, 1024);
      const uint64_t kmn0 = sdesc(smem_u32(sK), BR * 128, 1024);  // K as the MN-major B of dQ += dS K
      const uint64_t vmn0 = sdesc(smem_u32(sV), BR * 128, 1024);  // V as the MN-major B of O += P V
      // D(128 x 128) = A(128 x D) B(128 x D)^T, both K-major in 64-column blocks
      auto gemm_t = [&](uint32_t dst, uint64_t a, uint64_t bdsc) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * (BR * 128) + (k & 3) * 32;
          mma_bf16(dst, dadd(a, off), dadd(bdsc, off), ID_S, k > 0 ? 1u : 0u);
        }
      };
      // D(128 x D) += A(TMEM, 128 x 128 fp16 pairs) B(128 x D, MN-major)
      auto gemm_ts = [&](uint32_t dst, uint32_t a, uint64_t bmn, bool first) {
#pragma unroll
        for (int k = 0; k < BR / 16; ++k)
          mma_bf16_ts(dst, a + pk_k(k), dadd(bmn, k * 16 * 128), ID_G, (first && k == 0) ? 0u : 1u);
      };
      // S(s) of passes A and B into buffer s & 1; in pass A the stage is free
      // once S has read K
      auto issue_s = [&](int s) -> bool {
        const int st = s % ST;
        if (!mbar_wait(bar(B_FULL + st), (s / ST) & 1, ctl)) return false;
        tc_fence_after();
        gemm_t(tmem + sbuf(s), qd, dadd(kd0, st * TILE));
        mma_commit(bar(B_SFULL + (s & 1)));
        if (s < pa) mma_commit(bar(B_EMPTY + st));
        return true;
      };
      bool ok = mbar_wait(bar(B_QD), 0, ctl) && issue_s(0) && (nab < 2 || issue_s(1));
      for (int s = 0; ok && s < nab; ++s) {
        ok = mbar_wait(bar(B_SDONE), s & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        if (s >= pa) {
          gemm_ts(tmem + COL_ACC, tmem + sbuf(s), dadd(vmn0, (s % ST) * TILE), s == pa);  // O += P V
          mma_commit(bar(B_EMPTY + s % ST));
        }
        // buffer s & 1 again: P(s) is read by the P V above, issued first
        if (s + 2 < nab) ok = issue_s(s + 2);
      }
      if (ok) mma_commit(bar(B_ODONE));
      // pass C: S(s) into buffer s & 1 as soon as the buffer's dS was read by
      // dQ, dP(s + 1) right after the softmax of s, then dQ(s): the softmax of
      // s + 1 starts while dQ(s) and S(s + 2) run
      auto wait_full = [&](int s) {
        if (!mbar_wait(bar(B_FULL + s % ST), (s / ST) & 1, ctl)) return false;
        tc_fence_after();
        return true;
      };
      if (ok && nsteps > nab) {
        ok = wait_full(nab);
        if (ok) {
          gemm_t(tmem + sbuf(nab), qd, dadd(kd0, (nab % ST) * TILE));
          gemm_t(tmem + COL_P, dod, dadd(vd0, (nab % ST) * TILE));
          mma_commit(bar(B_SFULLC));
          if (nab + 1 < nsteps && (ok = wait_full(nab + 1)))
            gemm_t(tmem + sbuf(nab + 1), qd, dadd(kd0, ((nab + 1) % ST) * TILE));
        }
      }
      for (int s = nab; ok && s < nsteps; ++s) {
        ok = mbar_wait(bar(B_SDONE), s & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        if (s + 1 < nsteps) {  // its stage was waited for with S(s + 1)
          gemm_t(tmem + COL_P, dod, dadd(vd0, ((s + 1) % ST) * TILE));
          mma_commit(bar(B_SFULLC));
        }
        gemm_ts(tmem + COL_ACC, tmem + sbuf(s), dadd(kmn0, (s % ST) * TILE), s == nab);  // dQ += dS K
        mma_commit(bar(B_EMPTY + s % ST));
        if (s + 2 < nsteps && (ok = wait_full(s + 2)))
          gemm_t(tmem + sbuf(s + 2), qd, dadd(kd0, ((s + 2) % ST) * TILE));
      }
      mma_commit(bar(B_DQ));
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    // ---- softmax: two warps per TMEM lane quadrant, each with half the columns
    const int quad = warp & 3, half = (warp - 4) >> 2, row = quad * 32 + lane;
    const uint32_t la = tmem + ((uint32_t)(quad * 32) << 16);
    const float c = dm.scale * kLog2e;
    const bool valid = row < qvalid;
    const long long grow = (long long)(q0 + row) * dm.H + h;
    const float sc = do_scale(ws.amax);
    float m = -INFINITY;
    bool ok = true;
    // ---- pass A: this half's row max of the scores (no exponentials)
    for (int s = 0; ok && s < pa; ++s) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + (s & 1)), (s >> 1) & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      int k0, kv;
      tile_of(iv, s, k0, kv);
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * half + qq;
        float v[32];
        tmem_ld32(la + sbuf(s) + 32 * q, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmaxf(m, 32 * q + i < kv ? v[i] : -INFINITY);
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_SDONE));
    }
    // the exponent reference mc: the forward's log-sum-exp (in log2 units;
    // it bounds every scaled score, rows past the frame take the tile's first
    // row's), or the row max over both halves (every softmax warp reaches this
    // barrier; finite: the first key of every tile is valid)
    float mc;
    if (pa == 0) {
      mc = lse_in[(long long)(q0 + (valid ? row : 0)) * dm.H + h] * kLog2e;
    } else {
      red[half * BR + row] = m;
      softmax_bar();
      mc = fmaxf(m, red[(1 - half) * BR + row]) * c;
    }
    // ---- pass B: P = 2^(s c - mc) <= 1 (fp16) over S for O += P V; the row sum l
    float l = 0.f;
    for (int s = pa; ok && s < nab; ++s) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + (s & 1)), (s >> 1) & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      int k0, kv;
      tile_of(iv, s - pa, k0, kv);
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * half + qq;
        float v[32];
        tmem_ld32(la + sbuf(s) + 32 * q, v);
        tmem_wait_ld();
        uint32_t pk[16];
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int k = 32 * q + 2 * i;
          const float p0 = k < kv ? ex2(fmaf(v[2 * i], c, -mc)) : 0.f;
          const float p1 = k + 1 < kv ? ex2(fmaf(v[2 * i + 1], c, -mc)) : 0.f;
          ps0 += p0;
          ps1 += p1;
          pk[i] = pack_h2(p0, p1);
        }
        l += ps0 + ps1;
        tmem_st16(la + sbuf(s) + pk_col(q), pk);  // inside this half's columns, behind its reads
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(bar(B_SDONE));
    }
    red[2 * BR + half * BR + row] = l;
    softmax_bar();
    l += red[2 * BR + (1 - half) * BR + row];
    const float lse2 = mc + __log2f(l), inv_l = 1.0f / l;
    if (ok && valid && half == 0) ws.lse2[grow] = lse2;
    // ---- o: dg = dy o sigmoid'(g), Delta = <dy sigmoid(g), o>, this half's columns
    float del = 0.f;
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar(B_ODONE), 0, ctl))) {
      tc_fence_after();
      const int ys = dm.out_mode == 0 ? 2 : 1;
      const Ty* dy = static_cast<const Ty*>(dyp) + grow * ys * D;
      const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(in.gate_sm) + grow * D;
      float* dgr = dgate + grow * D;
#pragma unroll 1
      for (int q = half * (D / 64); q < (half + 1) * (D / 64); ++q) {
        float o[32];
        tmem_ld32(la + COL_ACC + 32 * q, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= inv_l;
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 dg4;
            float* dgp = reinterpret_cast<float*>(&dg4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int col = 32 * q + i + e;
              const float sg = sigmf(__bfloat162float(g[col]));
              const float dyv = tof(dy[col]);
              del = fmaf(dyv * sg, o[i + e], del);
              dgp[e] = dyv * o[i + e] * sg * (1.0f - sg);
            }
            *reinterpret_cast<float4*>(dgr + 32 * q + i) = dg4;
          }
        }
      }
    } else {
      ok = false;
    }
    red[4 * BR + half * BR + row] = del;
    softmax_bar();
    del += red[4 * BR + (1 - half) * BR + row];
    if (ok && valid && half == 0) ws.delta[grow] = del;
    const float dels = del * sc;  // in the units of the scaled dO
    // ---- pass C: dS = P (dP - Delta) (fp16) over S for dQ += dS K
    for (int s = nab; ok && s < nsteps; ++s) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SFULLC), (s - nab) & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      int k0, kv;
      tile_of(iv, s - nab, k0, kv);
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * half + qq;
        float vs[32], vp[32];
        tmem_ld32(la + sbuf(s) + 32 * q, vs);
        tmem_ld32(la + COL_P + 32 * q, vp);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int k = 32 * q + 2 * i;
          const float p0 = k < kv ? ex2(fmaf(vs[2 * i], c, -lse2)) : 0.f;
          const float p1 = k + 1 < kv ? ex2(fmaf(vs[2 * i + 1], c, -lse2)) : 0.f;
          pk[i] = pack_h2(p0 * (vp[2 * i] - dels), p1 * (vp[2 * i + 1] - dels));
        }
        tmem_st16(la + sbuf(s) + pk_col(q), pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(bar(B_SDONE));
    }
    // ---- epilogue: dq = s dQ / scale of dO, this half's columns
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar(B_DQ), 0, ctl))) {
      tc_fence_after();
      const float fq = dm.scale / sc;
      float* dst = dq + grow * D;
#pragma unroll
      for (int q = half * (D / 64); q < (half + 1) * (D / 64); ++q) {
        float v[32];
        tmem_ld32(la + COL_ACC + 32 * q, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + 32 * q + i) =
                make_float4(v[i] * fq, v[i + 1] * fq, v[i + 2] * fq, v[i + 3] * fq);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, 512);
}

// ---------------------------------------------------------- dK, dV kernel --
template <int D>
__global__ void __launch_bounds__(kThr, 1)
k_sbwd_kv_tc(Dims dm, SmTcWork ws, float* dk, float* dv, const __grid_constant__ CUtensorMap tmq,
             const __grid_constant__ CUtensorMap tmdo, const __grid_constant__ CUtensorMap tmk,
             const __grid_constant__ CUtensorMap tmv) {
  constexpr int NB = D / 64;
  constexpr uint32_t TILE = BR * D * 2;
  constexpr uint32_t COL_S = 0, COL_P = 128, COL_V = 256, COL_K = 256 + D;
  enum { B_KV = 0, B_FULL = 1, B_EMPTY = B_FULL + ST, B_SFULL = B_EMPTY + ST, B_SDONE, B_DONE, B_DRAIN, NBARS };
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sK = sm;
  unsigned char* sV = sK + TILE;
  unsigned char* sQ = sV + TILE;        // ST stages
  unsigned char* sDO = sQ + ST * TILE;  // ST stages
  float* sL = reinterpret_cast<float*>(sDO + ST * TILE);  // [ST][BR] LSE (log2 units) of the tile's queries
  float* sD = sL + ST * BR;                               // [ST][BR] Delta
  uint64_t* bars = reinterpret_cast<uint64_t*>(sD + ST * BR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*reinterpret_cast<volatile uint32_t*>(ws.status) != 0u) return;
  int f, b, h, n0;
  decode(dm, blockIdx.x, f, b, h, n0);
  const int base = b * dm.T * dm.N;
  const int k0 = base + f * dm.N + n0, kvalid = min(BR, dm.N - n0);
  const Iv iv = intervals(dm, f, base);
  const int nt = n_tiles(iv);
  const Ctl ctl{abort_flag, ws.status, (unsigned)TAG_SMBWD_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const float sc = do_scale(ws.amax);

  if (threadIdx.x == 0) {
    // FULL: the TMA transaction arrival plus the producer warp's arrival after
    // it staged LSE and Delta; SDONE: one arrival per softmax warp
    for (int i = 0; i < NBARS; ++i)
      mbar_init(bar(i), i == B_SDONE ? kSoftWarps : (i == B_FULL || i == B_FULL + 1) ? 2 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---- producer: K, V once; per query tile Q and dO by TMA, LSE and Delta by the lanes
    if (lane == 0) {
      mbar_expect_tx(bar(B_KV), 2 * TILE);
      for (int c = 0; c < NB; ++c) {
        tma_load_3d(smem_u32(sK + c * BR * 128), &tmk, bar(B_KV), c * 64, h, k0);
        tma_load_3d(smem_u32(sV + c * BR * 128), &tmv, bar(B_KV), c * 64, h, k0);
      }
    }
    int issued = 0;
    for (int j = 0; j < nt; ++j) {
      int r0, rv;
      tile_of(iv, j, r0, rv);
      const int st = j % ST;
      if (j >= ST && !__all_sync(0xffffffffu, mbar_wait(bar(B_EMPTY + st), (j / ST - 1) & 1, ctl))) break;
      if (lane == 0) {
        mbar_expect_tx(bar(B_FULL + st), 2 * TILE);
        for (int c = 0; c < NB; ++c) {
          tma_load_3d(smem_u32(sQ + st * TILE + c * BR * 128), &tmq, bar(B_FULL + st), c * 64, h, r0);
          tma_load_3d(smem_u32(sDO + st * TILE + c * BR * 128), &tmdo, bar(B_FULL + st), c * 64, h, r0);
        }
      }
      for (int r = lane; r < BR; r += 32) {
        const bool v = r < rv;
        const long long gi = (long long)(r0 + r) * dm.H + h;
        sL[st * BR + r] = v ? ws.lse2[gi] : INFINITY;  // 2^(s c - inf) = 0: no weight
        sD[st * BR + r] = v ? ws.delta[gi] * sc : 0.f;  // in the units of the scaled dO
      }
      mbar_arrive_warp(bar(B_FULL + st));
      issued = j + 1;
    }
    if (lane == 0) {
      mbar_drain(bar(B_KV), 0);
      for (int j = issued - ST < 0 ? 0 : issued - ST; j < issued; ++j)
        mbar_drain(bar(B_FULL + j % ST), (j / ST) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_f16(BR, BR, false);
      constexpr uint32_t ID_G = idesc_f16(BR, D, true);
      const uint64_t kd = sdesc(smem_u32(sK), 16, 1024), vd = sdesc(smem_u32(sV), 16, 1024);
      const uint64_t qd0 = sdesc(smem_u32(sQ), 16, 1024), dod0 = sdesc(smem_u32(sDO), 16, 1024);
      const uint64_t qmn0 = sdesc(smem_u32(sQ), BR * 128, 1024), domn0 = sdesc(smem_u32(sDO), BR * 128, 1024);
      auto gemm_t = [&](uint32_t dst, uint64_t a, uint64_t bdsc) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * (BR * 128) + (k & 3) * 32;
          mma_bf16(dst, dadd(a, off), dadd(bdsc, off), ID_S, k > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar(B_KV), 0, ctl);
      for (int j = 0; ok && j < nt; ++j) {
        const int st = j % ST;
        ok = mbar_wait(bar(B_FULL + st), (j / ST) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        gemm_t(tmem + COL_S, kd, dadd(qd0, st * TILE));   // S^T = K Q^T
        gemm_t(tmem + COL_P, vd, dadd(dod0, st * TILE));  // dP^T = V dO^T
        mma_commit(bar(B_SFULL));
        ok = mbar_wait(bar(B_SDONE), j & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        const uint64_t qmn = dadd(qmn0, st * TILE), domn = dadd(domn0, st * TILE);
#pragma unroll
        for (int k = 0; k < BR / 16; ++k) {
          const uint32_t acc = (j > 0 || k > 0) ? 1u : 0u;
          mma_bf16_ts(tmem + COL_V, tmem + COL_S + pk_k(k), dadd(domn, k * 16 * 128), ID_G, acc);  // dV += P^T dO
          mma_bf16_ts(tmem + COL_K, tmem + COL_P + pk_k(k), dadd(qmn, k * 16 * 128), ID_G, acc);   // dK += dS^T Q
        }
        mma_commit(bar(B_EMPTY + st));
      }
      mma_commit(bar(B_DONE));
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    // ---- softmax: two warps per TMEM lane quadrant, each with half the query columns
    const int quad = warp & 3, half = (warp - 4) >> 2, row = quad * 32 + lane;
    const uint32_t la = tmem + ((uint32_t)(quad * 32) << 16);
    const float c = dm.scale * kLog2e;
    bool ok = true;
    for (int j = 0; ok && j < nt; ++j) {
      const int st = j % ST;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SFULL), j & 1, ctl) &&
                                       mbar_wait(bar(B_FULL + st), (j / ST) & 1, ctl))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* L = sL + st * BR;
      const float* Dl = sD + st * BR;
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * half + qq;
        float vs[32], vp[32];
        tmem_ld32(la + COL_S + 32 * q, vs);
        tmem_ld32(la + COL_P + 32 * q, vp);
        tmem_wait_ld();
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int qc = 32 * q + 2 * i;
          const float p0 = ex2(fmaf(vs[2 * i], c, -L[qc]));
          const float p1 = ex2(fmaf(vs[2 * i + 1], c, -L[qc + 1]));
          pp[i] = pack_h2(p0, p1);
          pd[i] = pack_h2(p0 * (vp[2 * i] - Dl[qc]), p1 * (vp[2 * i + 1] - Dl[qc + 1]));
        }
        tmem_st16(la + COL_S + pk_col(q), pp);
        tmem_st16(la + COL_P + pk_col(q), pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(bar(B_SDONE));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0, ctl))) {
      tc_fence_after();
      const bool valid = row < kvalid;
      const long long gi = ((long long)(k0 + row) * dm.H + h) * D;
      const float fv = 1.0f / sc, fk = dm.scale / sc;  // the scale of dO taken out
#pragma unroll
      for (int q = half * (D / 64); q < (half + 1) * (D / 64); ++q) {
        float a[32], g[32];
        tmem_ld32(la + COL_V + 32 * q, a);
        tmem_ld32(la + COL_K + 32 * q, g);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            *reinterpret_cast<float4*>(dv + gi + 32 * q + i) =
                make_float4(a[i] * fv, a[i + 1] * fv, a[i + 2] * fv, a[i + 3] * fv);
            *reinterpret_cast<float4*>(dk + gi + 32 * q + i) =
                make_float4(g[i] * fk, g[i + 1] * fk, g[i + 2] * fk, g[i + 3] * fk);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, 512);
}

template <int D> constexpr size_t q_smem() {
  return 1024 + (2 + 2 * ST) * (size_t)BR * D * 2 + 6 * BR * 4 + 16 * 8 + 16;
}
template <int D> constexpr size_t kv_smem() {
  return 1024 + (2 + 2 * ST) * (size_t)BR * D * 2 + 2 * ST * BR * 4 + 16 * 8 + 16;
}

unsigned grid_for(long long n) {
  const long long b = (n + 255) / 256;
  return (unsigned)(b < 148LL * 16 ? (b > 0 ? b : 1) : 148LL * 16);
}

template <int D, typename Ty>
cudaError_t launch_d(const Dims& d, const Inputs& in, const SmTcArgs& a, cudaStream_t s) {
  const long long tokens = (long long)d.B * d.T * d.N, rows = tokens * d.H;
  SmTcWork ws{static_cast<__half*>(a.q16), static_cast<__half*>(a.k16), static_cast<__half*>(a.v16),
              static_cast<__half*>(a.dO16), a.lse2, a.delta, a.amax, a.status};
  cudaError_t e;
  const long long n8 = rows * D / 8;
  k_sbwd_cvt<<<grid_for(n8), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(in.q), static_cast<const __nv_bfloat16*>(in.k),
                                          static_cast<const __nv_bfloat16*>(in.v), ws.q16, ws.k16, ws.v16, n8);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_sbwd_do<Ty, D, 0><<<grid_for(rows * D), 256, 0, s>>>(d, in, a.dy, ws, rows);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_sbwd_do<Ty, D, 1><<<grid_for(rows * D), 256, 0, s>>>(d, in, a.dy, ws, rows);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap mq, mdo, mk, mv;
  if (!make_token_map(&mq, ws.q16, tokens, d.H, D, BR) || !make_token_map(&mdo, ws.dO, tokens, d.H, D, BR) ||
      !make_token_map(&mk, ws.k16, tokens, d.H, D, BR) || !make_token_map(&mv, ws.v16, tokens, d.H, D, BR))
    return cudaErrorInvalidValue;
  const long long items = (long long)d.B * d.H * d.T * ((d.N + BR - 1) / BR);
  auto kq = k_sbwd_q_tc<D, Ty>;
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)q_smem<D>())) != cudaSuccess)
    return e;
  kq<<<(unsigned)items, kThr, q_smem<D>(), s>>>(d, in, a.dy, ws, a.dq, a.dgate, a.lse_in, mq, mdo, mk, mv);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_sbwd_kv_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kv_smem<D>())) !=
      cudaSuccess)
    return e;
  k_sbwd_kv_tc<D><<<(unsigned)items, kThr, kv_smem<D>(), s>>>(d, ws, a.dk, a.dv, mq, mdo, mk, mv);
  return cudaGetLastError();
}

}  // namespace

bool sm_bwd_tc_supported(const Dims& d) {
  if (!d.bf16 || d.dk != d.dv || (d.dk != 64 && d.dk != 128)) return false;
  if ((long long)d.B * d.T * d.N + BR >= (1LL << 31)) return false;  // int32 TMA row coordinates
  if ((long long)d.B * d.H * d.T * ((d.N + BR - 1) / BR) > 0x7FFFFFFFLL) return false;
  return encode_fn() != nullptr;
}

// [status 256 B][q16][k16][v16][dO16][lse2][delta][amax 256 B], 256-byte aligned regions
size_t sm_bwd_tc_workspace(const Dims& d, size_t* off) {
  const size_t rows = (size_t)d.B * d.T * d.N * d.H;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t sizes[8] = {256, rows * d.dk * 2, rows * d.dk * 2, rows * d.dv * 2, rows * d.dv * 2, rows * 4, rows * 4, 256};
  size_t o = 0;
  for (int i = 0; i < 8; ++i) {
    if (off) off[i] = o;
    o += up(sizes[i]);
  }
  return o;
}

cudaError_t launch_sm_bwd_tc(const Dims& d, const Inputs& in, const SmTcArgs& a, cudaStream_t s) {
  if (d.dk == 128) return d.out_bf16 ? launch_d<128, __nv_bfloat16>(d, in, a, s) : launch_d<128, float>(d, in, a, s);
  if (d.dk == 64) return d.out_bf16 ? launch_d<64, __nv_bfloat16>(d, in, a, s) : launch_d<64, float>(d, in, a, s);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
