// Video Delta Attention at d = 256 (fp32 arithmetic; bf16 or fp32 q, gates):
// the SPD solve by 128 x 128 blocks, the state scans with M_t streamed through
// shared memory in row chunks, and the state read with R streamed the same
// way.  At d = 256 one state, one M_t and one R are 256 KB each in fp32, more
// than a CTA's shared memory, so none is held whole on chip.  The per-frame
// Gram of this size runs on the tensor cores (block mode of the Gram kernel).
//
// What is computed is the same as at smaller d (deepmagic post
// "用兩條分支取代一條", the closed form S_t = (alpha_t S_{t-1} + B_t)(I + A_t)^-1;
// PaperDaily digest sections 三 and 四, the two scans, the half-text start
// states and the read):
//   M_t = (I + A_t)^-1,
//   S <- (alpha_t S + B_t) M_t forward and backward (anchors: identity),
//   o = R q with R = forward + backward chunk-boundary states, RMSNorm, gate.
#include "vdn_internal.h"
#include "simt_common.cuh"
#include "sweep.cuh"

namespace vdn {
namespace {

constexpr int DB = 256;       // d
constexpr int TB = 128;       // block edge of the solve
constexpr int PB = TB + 4;    // shared pitch of a 128 x 128 tile (16-byte rows)
constexpr int kThreadsB = 256;

// ------------------------------------------------------ 128 x 128 tiles --
// Thread (ty, tx) of a 16 x 16 grid owns the 8 x 8 block at rows 8 ty, columns
// 8 tx (the layout of the register sweep).

__device__ __forceinline__ void tile_ld(float (&g)[8][8], const float* src, int ld) {
  const int r0 = (threadIdx.x >> 4) * 8, c0 = (threadIdx.x & 15) * 8;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const float4 x = *reinterpret_cast<const float4*>(src + (long long)(r0 + a) * ld + c0);
    const float4 y = *reinterpret_cast<const float4*>(src + (long long)(r0 + a) * ld + c0 + 4);
    g[a][0] = x.x; g[a][1] = x.y; g[a][2] = x.z; g[a][3] = x.w;
    g[a][4] = y.x; g[a][5] = y.y; g[a][6] = y.z; g[a][7] = y.w;
  }
}

__device__ __forceinline__ void tile_st(float* dst, int ld, const float (&g)[8][8], float sgn) {
  const int r0 = (threadIdx.x >> 4) * 8, c0 = (threadIdx.x & 15) * 8;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    *reinterpret_cast<float4*>(dst + (long long)(r0 + a) * ld + c0) =
        make_float4(sgn * g[a][0], sgn * g[a][1], sgn * g[a][2], sgn * g[a][3]);
    *reinterpret_cast<float4*>(dst + (long long)(r0 + a) * ld + c0 + 4) =
        make_float4(sgn * g[a][4], sgn * g[a][5], sgn * g[a][6], sgn * g[a][7]);
  }
}

// the transpose of the block: element (r, c) goes to dst[c * ld + r]
__device__ __forceinline__ void tile_st_t(float* dst, int ld, const float (&g)[8][8]) {
  const int r0 = (threadIdx.x >> 4) * 8, c0 = (threadIdx.x & 15) * 8;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    *reinterpret_cast<float4*>(dst + (long long)(c0 + c) * ld + r0) = make_float4(g[0][c], g[1][c], g[2][c], g[3][c]);
    *reinterpret_cast<float4*>(dst + (long long)(c0 + c) * ld + r0 + 4) =
        make_float4(g[4][c], g[5][c], g[6][c], g[7][c]);
  }
}

// acc (+/-)= op(A) op(B) over 128 x 128 tiles in shared memory (pitch PB);
// op = transpose when TA / TBT.
template <bool TA, bool TBT, bool NEG>
__device__ __forceinline__ void mm128(float (&acc)[8][8], const float* A, const float* B) {
  const int r0 = (threadIdx.x >> 4) * 8, c0 = (threadIdx.x & 15) * 8;
#pragma unroll 1
  for (int k = 0; k < TB; k += 4) {
    float av[8][4], bv[4][8];
    if (!TA) {
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float4 x = *reinterpret_cast<const float4*>(A + (r0 + a) * PB + k);
        av[a][0] = x.x; av[a][1] = x.y; av[a][2] = x.z; av[a][3] = x.w;
      }
    } else {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const float4 x = *reinterpret_cast<const float4*>(A + (k + kk) * PB + r0);
        const float4 y = *reinterpret_cast<const float4*>(A + (k + kk) * PB + r0 + 4);
        av[0][kk] = x.x; av[1][kk] = x.y; av[2][kk] = x.z; av[3][kk] = x.w;
        av[4][kk] = y.x; av[5][kk] = y.y; av[6][kk] = y.z; av[7][kk] = y.w;
      }
    }
    if (!TBT) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const float4 x = *reinterpret_cast<const float4*>(B + (k + kk) * PB + c0);
        const float4 y = *reinterpret_cast<const float4*>(B + (k + kk) * PB + c0 + 4);
        bv[kk][0] = x.x; bv[kk][1] = x.y; bv[kk][2] = x.z; bv[kk][3] = x.w;
        bv[kk][4] = y.x; bv[kk][5] = y.y; bv[kk][6] = y.z; bv[kk][7] = y.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(B + (c0 + c) * PB + k);
        bv[0][c] = x.x; bv[1][c] = x.y; bv[2][c] = x.z; bv[3][c] = x.w;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float x = NEG ? -av[a][kk] : av[a][kk];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(x, bv[kk][c], acc[a][c]);
      }
  }
}

__device__ __forceinline__ void zero(float (&g)[8][8]) {
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) g[a][c] = 0.f;
}

__device__ __forceinline__ void add_identity(float (&g)[8][8]) {
  if ((threadIdx.x >> 4) == (threadIdx.x & 15)) {
#pragma unroll
    for (int a = 0; a < 8; ++a) g[a][a] += 1.0f;
  }
}

// ------------------------------------------------------------ block solve --
// M = G^-1 for G = I + A = [[G11, G12], [G12^T, G22]] (blocks of 128) by the
// block form of the sweep:
//   X = G11^-1,  W = X G12,  Y = (G22 - G12^T W)^-1 (inverse of the Schur
//   complement),  M22 = Y,  M12 = -W Y,  M21 = M12^T,  M11 = X - M12 W^T,
// the two block inverses by the register sweep (panels of 8 pivots).  Then C = B M by blocks.
// One CTA per frame-head; A_t (from the Gram) is overwritten by M_t in place,
// each block only after it has been read.  TEXT: A_x, B_x of the text; writes
// S_x / 2 = B_x M_x / 2 to the half-text state (the A_x slot is scratch).
template <bool TEXT>
__global__ void __launch_bounds__(kThreadsB, 1)
k_solve_block(Dims dm, Work w) {
  extern __shared__ __align__(16) float smb[];
  float* T0 = smb;              // [128][PB] each
  float* T1 = T0 + TB * PB;
  float* T2 = T1 + TB * PB;
  float* rowbuf = T2 + TB * PB;  // the panel sweep's rows, Z and V
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (!TEXT && is_anchor(dm, t)) return;
  const long long DD = (long long)DB * DB;
  const long long fh = ((long long)b * dm.T + t) * dm.H + h, bh = (long long)b * dm.H + h;
  float* gM = TEXT ? w.text_gram + bh * 2 * DD : w.M + fh * DD;  // A on entry, M on exit
  const float* gB = TEXT ? gM + DD : w.Cm + fh * DD;
  float* outC = TEXT ? w.half_text + bh * DD : w.Cm + fh * DD;
  const float cscale = TEXT ? 0.5f : 1.0f;
  auto blk = [&](float* base, int i, int j) { return base + (long long)(i * TB) * DB + j * TB; };

  float g[8][8], acc[8][8];
  // X = G11^-1: kept in T0 and (as scratch until M11 replaces it) in M's block (0, 0)
  tile_ld(g, blk(gM, 0, 0), DB);
  add_identity(g);
  sweep_panels<TB>(g, rowbuf);  // g = -X
  tile_st(T0, PB, g, -1.f);
  tile_st(blk(gM, 0, 0), DB, g, -1.f);
  tile_ld(acc, blk(gM, 0, 1), DB);  // G12
  tile_st(T1, PB, acc, 1.f);
  __syncthreads();
  // W = X G12 -> T2
  zero(acc);
  mm128<false, false, false>(acc, T0, T1);
  tile_st(T2, PB, acc, 1.f);
  __syncthreads();
  // Y = (G22 - G12^T W)^-1
  tile_ld(g, blk(gM, 1, 1), DB);
  add_identity(g);
  mm128<true, false, true>(g, T1, T2);
  sweep_panels<TB>(g, rowbuf);  // g = -Y
  __syncthreads();            // every read of T1 (G12) done
  tile_st(T1, PB, g, -1.f);
  tile_st(blk(gM, 1, 1), DB, g, -1.f);  // M22
  __syncthreads();
  // M12 = -W Y -> T0 (X is no longer needed in shared memory), M12 and M21 to global
  zero(acc);
  mm128<false, false, true>(acc, T2, T1);
  tile_st(T0, PB, acc, 1.f);
  tile_st(blk(gM, 0, 1), DB, acc, 1.f);
  tile_st_t(blk(gM, 1, 0), DB, acc);
  __syncthreads();
  // M11 = X - M12 W^T (this thread's block of X from global, written by itself)
  tile_ld(g, blk(gM, 0, 0), DB);
  mm128<false, true, true>(g, T0, T2);
  tile_st(blk(gM, 0, 0), DB, g, 1.f);
  __syncthreads();  // M complete in global memory
  if (!TEXT && w.M16 != nullptr) {
    // operand of the tensor-core scan: M's bf16 [hi | lo] rows, 8 entries a thread per pass
    __nv_bfloat16* mh = static_cast<__nv_bfloat16*>(w.M16) + fh * 2 * DD;
    for (int e = threadIdx.x * 8; e < DD; e += kThreadsB * 8) {
      const float4 x0 = *reinterpret_cast<const float4*>(gM + e), x1 = *reinterpret_cast<const float4*>(gM + e + 4);
      const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      uint32_t hv[4], lv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat16 a = __float2bfloat16_rn(x[2 * j]), c = __float2bfloat16_rn(x[2 * j + 1]);
        const __nv_bfloat16 ra = __float2bfloat16_rn(x[2 * j] - __bfloat162float(a));
        const __nv_bfloat16 rc = __float2bfloat16_rn(x[2 * j + 1] - __bfloat162float(c));
        hv[j] = (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(c) << 16);
        lv[j] = (uint32_t)__bfloat16_as_ushort(ra) | ((uint32_t)__bfloat16_as_ushort(rc) << 16);
      }
      *reinterpret_cast<uint4*>(mh + e) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      *reinterpret_cast<uint4*>(mh + DD + e) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
    }
  }
  // frames: the scan steps S <- (alpha S + B_t) M_t itself, B_t stays in the C_t slot
  if (!TEXT && w.bform) return;

  // C = B M by blocks: C(rb, cb) = B(rb, 0) M(0, cb) + B(rb, 1) M(1, cb).  B's row
  // block is in shared memory before C overwrites it (in place for frames).
  for (int rb = 0; rb < 2; ++rb) {
    tile_ld(g, blk(const_cast<float*>(gB), rb, 0), DB);
    tile_st(T0, PB, g, 1.f);
    tile_ld(g, blk(const_cast<float*>(gB), rb, 1), DB);
    tile_st(T1, PB, g, 1.f);
    for (int cb = 0; cb < 2; ++cb) {
      zero(acc);
      tile_ld(g, blk(gM, 0, cb), DB);
      tile_st(T2, PB, g, 1.f);
      __syncthreads();
      mm128<false, false, false>(acc, T0, T2);
      __syncthreads();
      tile_ld(g, blk(gM, 1, cb), DB);
      tile_st(T2, PB, g, 1.f);
      __syncthreads();
      mm128<false, false, false>(acc, T1, T2);
      tile_st(blk(outC, rb, cb), DB, acc, cscale);
      __syncthreads();
    }
  }
}

// ------------------------------------------------------------------ scan --
// grid (DB / RB row blocks, 2 directions, B * H).  Rows of the state evolve
// independently (s_row <- (alpha s_row + b_row) M), so a CTA carries RB rows of
// one chain: thread (rq, cq) holds rows 8 rq .. 8 rq + 7 and columns 4 cq ..
// 4 cq + 3 of its block, and the block's transpose sits in shared memory for
// the products.  M_t streams through a double buffer in shared memory, KC
// rows at a time, the next chunk's asynchronous copy in flight while the
// current one computes.  Three CTAs per SM keep every chain of a launch
// resident at once (each CTA runs all the frames, so a second wave would
// double the time).
constexpr int RB = 32, KC = 16;

__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ int snap_slot_big(const Dims& d, int dir, int t) {
  if (dir == 0) {
    if ((t + 1) % d.chunk == 0) return (t + 1) / d.chunk;
    return (t + 1 == d.T) ? d.C : -1;
  }
  return (t % d.chunk == 0) ? t / d.chunk : -1;
}

__global__ void __launch_bounds__(kThreadsB, 3)
k_scan_big(Dims dm, Inputs in, Work w) {
  extern __shared__ __align__(16) float smb[];
  float* St = smb;            // [DB][RB]     this CTA's rows of S, transposed
  float* Mc = St + DB * RB;   // [2][KC][DB]  chunks of M_t's rows
  const int tid = threadIdx.x, cq = tid & 63, rq = tid >> 6;
  const int r0 = rq * 8, c0 = cq * 4;
  const int row0 = blockIdx.x * RB, dir = blockIdx.y, bh = blockIdx.z;
  const int b = bh / dm.H, h = bh % dm.H;
  const long long DD = (long long)DB * DB;
  // start state: half the text state, or the carried forward state
  const float* half = ((dir == 0 && in.fwd_init) ? in.fwd_init : w.half_text) + (long long)bh * DD;
  float* snap = (dir == 0 ? w.fsnap : w.bsnap) + (long long)bh * (dm.C + 1) * DD;
  auto gidx = [&](int r, int c) { return (long long)(row0 + r0 + r) * DB + c0 + c; };

  // the state lives in St (transposed); a thread's 8 x 4 block is in registers
  // only while it is formed
  auto put_state = [&](const float (&v)[8][4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      *reinterpret_cast<float4*>(St + (c0 + c) * RB + r0) = make_float4(v[0][c], v[1][c], v[2][c], v[3][c]);
      *reinterpret_cast<float4*>(St + (c0 + c) * RB + r0 + 4) = make_float4(v[4][c], v[5][c], v[6][c], v[7][c]);
    }
  };
  auto snapshot = [&](int slot, const float (&v)[8][4]) {
#pragma unroll
    for (int r = 0; r < 8; ++r)
      *reinterpret_cast<float4*>(snap + (long long)slot * DD + gidx(r, 0)) = make_float4(v[r][0], v[r][1], v[r][2], v[r][3]);
  };
  {
    float v[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float4 x = *reinterpret_cast<const float4*>(half + gidx(r, 0));
      v[r][0] = x.x; v[r][1] = x.y; v[r][2] = x.z; v[r][3] = x.w;
    }
    snapshot(dir == 0 ? 0 : dm.C, v);
    put_state(v);
  }

  bool x_ready = false;  // St holds X = alpha S + B of the next written frame
  for (int st = 0; st < dm.T; ++st) {
    const int t = dir == 0 ? st : dm.T - 1 - st;
    const int slot = snap_slot_big(dm, dir, t);
    if (!is_anchor(dm, t)) {
      const long long fh = ((long long)b * dm.T + t) * dm.H + h;
      const float* Mg = w.M + fh * DD;
      const float* Bg = w.Cm + fh * DD;  // B_t (the solve leaves it in the C_t slot)
      const float alpha = __ldg(in.alpha + fh);
      // X = alpha S + B_t in place of this CTA's rows (the closed form
      // S_t = (alpha S + B_t) M_t).  After a written frame the previous
      // step already left X in St; here only before the first one.
      if (!x_ready) {
        float bv[8][4];  // this thread's 8 x 4 block of B_t, one 16-byte load per row
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(Bg + gidx(r, 0)));
          bv[r][0] = v.x; bv[r][1] = v.y; bv[r][2] = v.z; bv[r][3] = v.w;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float4 x = *reinterpret_cast<const float4*>(St + (c0 + c) * RB + r0);
          float4 y = *reinterpret_cast<const float4*>(St + (c0 + c) * RB + r0 + 4);
          x.x = fmaf(alpha, x.x, bv[0][c]);
          x.y = fmaf(alpha, x.y, bv[1][c]);
          x.z = fmaf(alpha, x.z, bv[2][c]);
          x.w = fmaf(alpha, x.w, bv[3][c]);
          y.x = fmaf(alpha, y.x, bv[4][c]);
          y.y = fmaf(alpha, y.y, bv[5][c]);
          y.z = fmaf(alpha, y.z, bv[6][c]);
          y.w = fmaf(alpha, y.w, bv[7][c]);
          *reinterpret_cast<float4*>(St + (c0 + c) * RB + r0) = x;
          *reinterpret_cast<float4*>(St + (c0 + c) * RB + r0 + 4) = y;
        }
      }
      float acc[8][4];
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
      auto fetch = [&](int kc) {  // rows [KC kc, KC kc + KC) of M_t into buffer kc & 1
        float* dst = Mc + (kc & 1) * KC * DB;
#pragma unroll
        for (int v = 0; v < KC * DB / 4 / kThreadsB; ++v) {
          const int e = (tid + v * kThreadsB) * 4;
          cp_async16(dst + e, Mg + (long long)kc * KC * DB + e);
        }
        cp_async_commit();
      };
      fetch(0);
      for (int kc = 0; kc < DB / KC; ++kc) {
        if (kc + 1 < DB / KC) {
          fetch(kc + 1);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        __syncthreads();  // chunk kc (and the state) visible to every thread
        const float* mc = Mc + (kc & 1) * KC * DB;
        const int k0 = kc * KC;
#pragma unroll 4
        for (int k = 0; k < KC; ++k) {
          const float4 s0 = *reinterpret_cast<const float4*>(St + (k0 + k) * RB + r0);
          const float4 s1 = *reinterpret_cast<const float4*>(St + (k0 + k) * RB + r0 + 4);
          const float4 m = *reinterpret_cast<const float4*>(mc + k * DB + c0);
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
          const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
          for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(sv[r], mv[c], acc[r][c]);
        }
        __syncthreads();  // chunk kc read by every thread before its buffer is refilled
      }
      if (slot >= 0) snapshot(slot, acc);
      // the next written frame's X = alpha' S + B' straight from the new state
      // in registers (anchors lie only before the first and after the last
      // written frame, so nothing reads S from St in between); every read of
      // this step's X finished at its last barrier
      int tn = -1;
      for (int sn = st + 1; sn < dm.T && tn < 0; ++sn) {
        const int tt = dir == 0 ? sn : dm.T - 1 - sn;
        if (!is_anchor(dm, tt)) tn = tt;
      }
      if (tn >= 0) {
        const long long fn = ((long long)b * dm.T + tn) * dm.H + h;
        const float* Bn = w.Cm + fn * DD;
        const float an = __ldg(in.alpha + fn);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(Bn + gidx(r, 0)));
          acc[r][0] = fmaf(an, acc[r][0], v.x);
          acc[r][1] = fmaf(an, acc[r][1], v.y);
          acc[r][2] = fmaf(an, acc[r][2], v.z);
          acc[r][3] = fmaf(an, acc[r][3], v.w);
        }
        x_ready = true;
      } else {
        x_ready = false;
      }
      put_state(acc);  // X for the next written frame, or the final state
    } else if (slot >= 0) {
      float v[8][4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(St + (c0 + c) * RB + r0);
        const float4 y = *reinterpret_cast<const float4*>(St + (c0 + c) * RB + r0 + 4);
        v[0][c] = x.x; v[1][c] = x.y; v[2][c] = x.z; v[3][c] = x.w;
        v[4][c] = y.x; v[5][c] = y.y; v[6][c] = y.z; v[7][c] = y.w;
      }
      snapshot(slot, v);
    }
  }
}

// ------------------------------------------------------------------ read --
// grid (token tiles, query groups, B * H).  A CTA takes TQ tokens of one query
// group, all reading the same R = forward + backward snapshot; R is formed and
// streamed RC rows at a time.  Thread (warp wp, lane) computes, for tokens
// lane and lane + 32, outputs 4 wp .. 4 wp + 3 of every chunk; the RMSNorm
// sums are combined across the warps in shared memory.
constexpr int TQR = 64, RC = 32, RP = DB + 4, QP = TQR + 1;

template <typename T, typename To>
__global__ void __launch_bounds__(kThreadsB)
k_read_big(Dims dm, Inputs in, Work w) {
  extern __shared__ __align__(16) float smb[];
  float* qT = smb;               // [DB][QP]  the query tile, transposed
  float* Rc = qT + DB * QP;      // [RC][RP]  a chunk of R's rows
  float* red = Rc + RC * RP;     // [8][TQR]  partial sums of squares
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int bh = blockIdx.z, b = bh / dm.H, h = bh % dm.H;
  int f0, f1, ridx;
  if (!query_group(dm, blockIdx.y, f0, f1, ridx)) return;
  const long long ntok = (long long)(f1 - f0) * dm.N;
  const long long tbase = (long long)blockIdx.x * TQR;
  if (tbase >= ntok) return;
  const long long DD = (long long)DB * DB;
  const float* fs = w.fsnap + ((long long)bh * (dm.C + 1) + (ridx < dm.C ? max(ridx - 1, 0) : 0)) * DD;
  const float* bs = w.bsnap + ((long long)bh * (dm.C + 1) + (ridx < dm.C ? min(ridx + 2, dm.C) : dm.C)) * DD;
  float* Rg = w.R + ((long long)bh * (dm.C + 1) + ridx) * DD;
  const long long row_first = ((long long)b * dm.T + f0) * dm.N + tbase;  // token row of tile row 0

  const T* q = static_cast<const T*>(in.q);
  for (int idx = tid; idx < TQR * DB; idx += kThreadsB) {
    const int j = idx / DB, k = idx % DB;
    qT[k * QP + j] = (tbase + j < ntok) ? ldf(q + ((row_first + j) * dm.H + h) * DB + k) : 0.f;
  }

  float o[2][DB / RC][4];
#pragma unroll
  for (int rc = 0; rc < DB / RC; ++rc) {
    __syncthreads();  // the previous chunk fully read (and the query tile written)
    for (int e = tid * 4; e < RC * DB; e += kThreadsB * 4) {
      const int r = e / DB, k = e % DB;
      const long long gi = (long long)(rc * RC + r) * DB + k;
      const float4 a = *reinterpret_cast<const float4*>(fs + gi);
      const float4 c = *reinterpret_cast<const float4*>(bs + gi);
      const float4 s = make_float4(a.x + c.x, a.y + c.y, a.z + c.z, a.w + c.w);
      *reinterpret_cast<float4*>(Rc + r * RP + k) = s;
      if (blockIdx.x == 0) *reinterpret_cast<float4*>(Rg + gi) = s;
    }
    __syncthreads();
    float acc[2][4];
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[x][i] = 0.f;
#pragma unroll 2
    for (int k = 0; k < DB; k += 4) {
      float rv[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = *reinterpret_cast<const float4*>(Rc + (wp * 4 + i) * RP + k);
        rv[i][0] = x.x; rv[i][1] = x.y; rv[i][2] = x.z; rv[i][3] = x.w;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const float q0 = qT[(k + kk) * QP + lane], q1 = qT[(k + kk) * QP + lane + 32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[0][i] = fmaf(rv[i][kk], q0, acc[0][i]);
          acc[1][i] = fmaf(rv[i][kk], q1, acc[1][i]);
        }
      }
    }
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[x][rc][i] = acc[x][i];
  }
  // RMSNorm over the d outputs of each token
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    float ss = 0.f;
#pragma unroll
    for (int rc = 0; rc < DB / RC; ++rc)
#pragma unroll
      for (int i = 0; i < 4; ++i) ss = fmaf(o[x][rc][i], o[x][rc][i], ss);
    red[wp * TQR + lane + 32 * x] = ss;
  }
  __syncthreads();
  const T* g = static_cast<const T*>(in.gate_lin);
  To* y = static_cast<To*>(in.y);
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int j = lane + 32 * x;
    if (tbase + j >= ntok) continue;
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) ss += red[u * TQR + j];
    const float rs = rsqrtf(ss / DB + dm.eps);
    const long long row = row_first + j;
#pragma unroll
    for (int rc = 0; rc < DB / RC; ++rc)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = rc * RC + wp * 4 + i;
        const long long gi = (row * dm.H + h) * DB + col;
        const float wgt = in.rms_weight ? __ldg(in.rms_weight + (long long)h * DB + col) : 1.0f;
        const float val = sigm(ldf(g + gi)) * o[x][rc][i] * rs * wgt;
        if (dm.out_mode == 0) {
          stf(y + ((row * dm.H + h) * 2 + 1) * DB + col, val);
        } else {
          To* p = y + gi;
          stf(p, to_f(*p) + val);
        }
      }
  }
}

}  // namespace

bool big_d(const Dims& d) { return d.dk == DB && d.dv == DB; }

cudaError_t launch_solve_big(const Dims& d, const Work& w, cudaStream_t s, bool text) {
  if (!big_d(d)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * (size_t)(3 * TB * PB + sweep_panel_floats<TB>());
  auto kern = text ? k_solve_block<true> : k_solve_block<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(text ? 1 : d.T, d.H, d.B), kThreadsB, smem, s>>>(d, w);
  return cudaGetLastError();
}

cudaError_t launch_scan_big(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (!big_d(d)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * (size_t)(DB * RB + 2 * KC * DB);
  cudaError_t e = cudaFuncSetAttribute(k_scan_big, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_scan_big<<<dim3(DB / RB, 2, d.B * d.H), kThreadsB, smem, s>>>(d, in, w);
  return cudaGetLastError();
}

template <typename T, typename To>
static cudaError_t read_big(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)(DB * QP + RC * RP + 8 * TQR);
  auto kern = k_read_big<T, To>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long max_tok = (long long)d.chunk * d.N;
  const long long tiles = (max_tok + TQR - 1) / TQR;
  if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<dim3((unsigned)tiles, d.C + (d.anchors ? 2 : 0), d.B * d.H), kThreadsB, smem, s>>>(d, in, w);
  return cudaGetLastError();
}

cudaError_t launch_read_big(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (!big_d(d)) return cudaErrorInvalidValue;
  using bf16 = __nv_bfloat16;
  if (d.bf16) return d.out_bf16 ? read_big<bf16, bf16>(d, in, w, s) : read_big<bf16, float>(d, in, w, s);
  return d.out_bf16 ? read_big<float, bf16>(d, in, w, s) : read_big<float, float>(d, in, w, s);
}

}  // namespace vdn
