// Chunk composition of the frame maps on the tensor cores (bf16 inputs, d = 128).
//
// What it computes: every written frame acts on a scan state as the affine
// map S -> alpha_t S M_t + C_t (deepmagic post "用兩條分支取代一條", the
// frame-wise closed form S_t = (alpha_t S_{t-1} + B_t)(I + A_t)^{-1}, with
// M_t = (I + A_t)^{-1} and C_t = B_t M_t), so the written frames
// f_1 < ... < f_n of a chunk (anchor frames are identity maps) compose into
// one map of the same form:
//   forward  S -> Lam S P + Cf,    P = M_{f_1} ... M_{f_n},  Lam = prod alpha_f,
//                                  Cf <- alpha_f Cf M_f + C_f  (f increasing, from 0)
//   backward S -> Lam S P^T + Cb,  Cb <- alpha_f Cb M_f + C_f  (f decreasing, from 0)
// (the reversed product of the symmetric M_f is P^T).  Both chains are the
// scan's own step X <- alpha X M + C over the chunk's frames: the P chain
// from X = I with alpha = 1 and no C, the two Horner chains from X = 0, run
// as X <- (alpha X + B_f) M_f since C_f = B_f M_f (the solve leaves B_f).
// The chunk-stepped scan then takes 1 / chunk of the frame scan's steps.
//
// One CTA per (chunk, batch-head) and direction (384 threads): the forward
// CTA carries P and Cf (two 128 x 128 accumulators sharing the B operand
// M_f), the backward CTA carries Cb.
//   warp 0      TMA producer: M_f's bf16 split (written by the solve), once
//               the previous products are done.
//   warp 1      TMEM allocator; lane 0 issues X M_f ~ X_hi M_hi + X_hi M_lo +
//               X_lo M_hi (24 MMAs per chain, M_f rows as the K-major B
//               operand since M_f is symmetric).
//   warps 4..11 epilogue, one row per thread and half of the columns per
//               warp: the new X in fp32, split back into the A operand, and
//               after the last frame the outputs: P as its bf16 split
//               (row-major, the layout of M's split), Cf / Cb in fp32, Lam.
#include "tc_common.cuh"

namespace vdn {
namespace {
using namespace tc;

constexpr int D = 128;
constexpr int kThreadsCmp = 384;
constexpr int kMaxChunk = 5;             // the chunk length (checked at the boundary)
constexpr uint32_t CHUNK = D * 128;      // 64 K-columns of a 128-row bf16 operand (SW128): 16 KB
constexpr uint32_t OPBYTES = 2 * CHUNK;  // one 128 x 128 bf16 operand
constexpr uint32_t SPLIT = 2 * OPBYTES;  // hi then lo: 64 KB
enum { B_BFULL = 0, B_AREADY = 1, B_MDONE = 2, B_DRAIN = 3, NBARS = 4 };

// The written frames of chunk c in the direction's order.
struct ChunkFrames {
  int f[kMaxChunk];
  int n;
};
__device__ __forceinline__ ChunkFrames frames_of(const Dims& d, int c, int dir) {
  ChunkFrames r;
  r.n = 0;
  const int f0 = c * d.chunk, f1 = min(f0 + d.chunk, d.T);
#pragma unroll
  for (int i = 0; i < kMaxChunk; ++i) {
    const int t = dir == 0 ? f0 + i : f1 - 1 - i;
    if (t >= f0 && t < f1 && !is_anchor(d, t)) r.f[r.n++] = t;
  }
  return r;
}

__device__ __forceinline__ void st_global_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// 32 values of `row` (columns 32q..32q+31) split into bf16 hi / lo: into the
// K-major A operand in shared memory, or as row-major rows in global memory.
__device__ __forceinline__ void split_to_smem(int q, int row, unsigned char* sA, const float (&s)[32]) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int k0 = q * 32 + 8 * e;
    const uint32_t off = (k0 >> 6) * CHUNK + row * 128 + (((((k0 & 63) >> 3) ^ (row & 7))) << 4);
    uint32_t h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x0 = s[8 * e + 2 * j], x1 = s[8 * e + 2 * j + 1];
      h[j] = pack_bf16(x0, x1);
      l[j] = pack_bf16(x0 - __uint_as_float(h[j] << 16), x1 - __uint_as_float(h[j] & 0xFFFF0000u));
    }
    *reinterpret_cast<uint4*>(sA + off) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(sA + OPBYTES + off) = make_uint4(l[0], l[1], l[2], l[3]);
  }
}
__device__ __forceinline__ void split_to_global(__nv_bfloat16* hi_row, __nv_bfloat16* lo_row, int q,
                                                const float (&s)[32]) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x0 = s[8 * e + 2 * j], x1 = s[8 * e + 2 * j + 1];
      h[j] = pack_bf16(x0, x1);
      l[j] = pack_bf16(x0 - __uint_as_float(h[j] << 16), x1 - __uint_as_float(h[j] & 0xFFFF0000u));
    }
    st_global_v4(hi_row + q * 32 + 8 * e, make_uint4(h[0], h[1], h[2], h[3]));
    st_global_v4(lo_row + q * 32 + 8 * e, make_uint4(l[0], l[1], l[2], l[3]));
  }
}
__device__ __forceinline__ void store_f32(float* dst, const float (&s)[32]) {
#pragma unroll
  for (int u = 0; u < 8; ++u) *reinterpret_cast<float4*>(dst + 4 * u) = make_float4(s[4 * u], s[4 * u + 1], s[4 * u + 2], s[4 * u + 3]);
}

__global__ void __launch_bounds__(kThreadsCmp, 1)
k_compose_tc(Dims dm, Inputs in, Work w, const __grid_constant__ CUtensorMap tmm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA0 = sm;            // P (forward) or Cb (backward), hi | lo, K-major SW128
  unsigned char* sA1 = sA0 + SPLIT;   // Cf (forward), hi | lo
  unsigned char* sB = sA1 + SPLIT;    // M_f hi | lo
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + SPLIT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*reinterpret_cast<volatile uint32_t*>(w.status) != 0u) return;
  const int c = blockIdx.x, bh = blockIdx.y, dir = blockIdx.z;
  const int b = bh / dm.H, h = bh % dm.H;
  const bool fwd = dir == 0;
  const ChunkFrames fr = frames_of(dm, c, dir);
  const int n = fr.n;
  const long long bch = ((long long)b * dm.C + c) * dm.H + h;  // chunk-map index
  const Ctl ctl{abort_flag, w.status, (unsigned)TAG_COMPOSE_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto fh_of = [&](int t) { return ((long long)b * dm.T + t) * dm.H + h; };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_BFULL), 1);
    mbar_init(bar(B_AREADY), 8);  // one arrival per epilogue warp
    mbar_init(bar(B_MDONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Phases: BFULL and MDONE complete once per frame step i; AREADY once for
  // the start operands and once after each step but the last, so step i's
  // MMAs wait for AREADY phase i.
  if (warp == 0) {
    if (lane == 0) {
      int nb = 0;
      for (int i = 0; i < n; ++i) {
        const long long fh = fh_of(fr.f[i]);
        if (i > 0 && !mbar_wait(bar(B_MDONE), (i - 1) & 1, ctl)) break;  // B free
        mbar_expect_tx(bar(B_BFULL), SPLIT);
        for (int part = 0; part < 2; ++part)
          for (int cc = 0; cc < 2; ++cc)
            tma_load_2d(smem_u32(sB + part * OPBYTES + cc * CHUNK), &tmm, bar(B_BFULL), cc * 64,
                        (int)((fh * 2 + part) * D));
        ++nb;
      }
      if (nb > 0) mbar_drain(bar(B_BFULL), (nb - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID = idesc_bf16(128, D, false);
      const uint64_t a0 = sdesc(smem_u32(sA0), 16, 1024), a1 = sdesc(smem_u32(sA1), 16, 1024),
                     b0 = sdesc(smem_u32(sB), 16, 1024);
      for (int i = 0; i < n; ++i) {
        if (!mbar_wait(bar(B_AREADY), i & 1, ctl)) break;
        if (!mbar_wait(bar(B_BFULL), i & 1, ctl)) break;
        tc_fence_after();
#pragma unroll
        for (int chain = 0; chain < 2; ++chain) {
          if (chain == 1 && !fwd) break;
          const uint64_t ad = chain == 0 ? a0 : a1;
#pragma unroll
          for (int pass = 0; pass < 3; ++pass) {  // hi hi, hi lo, lo hi
            const uint32_t ao = pass == 2 ? OPBYTES : 0u, bo = pass == 1 ? OPBYTES : 0u;
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
              mma_bf16(tmem + 128 * chain, dadd(ad, ao + (k >> 2) * CHUNK + (k & 3) * 32),
                       dadd(b0, bo + (k >> 2) * CHUNK + (k & 3) * 32), ID, (pass | k) ? 1u : 0u);
          }
        }
        mma_commit(bar(B_MDONE));
      }
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3, half = (warp - 4) >> 2, row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + half * 64;
    const long long DD = (long long)D * D;
    __nv_bfloat16* p_hi = static_cast<__nv_bfloat16*>(w.P16) + (bch * 2 * D + row) * D;
    __nv_bfloat16* p_lo = p_hi + DD;
    float* cf_row = w.Cf + bch * DD + (long long)row * D;
    float* cb_row = w.Cb + bch * DD + (long long)row * D;
    // The Horner chains in the B form (the solve left B_f in the C_f slot):
    // X <- alpha_f X M_f + B_f M_f = (alpha_f X + B_f) M_f, so step i multiplies
    // alpha_{f_i} X_{i-1} + B_{f_i} (formed here) by M_{f_i}.  Start operands:
    // P = I (forward) and the first frame's B (X_0 = 0).
    auto brow = [&](int i) { return w.Cm + fh_of(fr.f[i]) * DD + (long long)row * D; };
#pragma unroll 1
    for (int q = 2 * half; q < 2 * half + 2; ++q) {
      float s0[32], z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s0[i] = (fwd && q * 32 + i == row) ? 1.f : 0.f;
        z[i] = 0.f;
      }
      if (n == 0) {  // no written frame: the identity map
        if (fwd) {
          split_to_global(p_hi, p_lo, q, s0);
          store_f32(cf_row + q * 32, z);
        } else {
          store_f32(cb_row + q * 32, z);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 b4 = __ldg(reinterpret_cast<const float4*>(brow(0) + q * 32) + u);
          z[4 * u] = b4.x; z[4 * u + 1] = b4.y; z[4 * u + 2] = b4.z; z[4 * u + 3] = b4.w;
        }
        if (fwd) {
          split_to_smem(q, row, sA0, s0);
          split_to_smem(q, row, sA1, z);
        } else {
          split_to_smem(q, row, sA0, z);
        }
      }
    }
    if (n > 0) {
      fence_proxy_async_smem();
      mbar_arrive_warp(bar(B_AREADY));
    }
    float lam = 1.f;
    for (int i = 0; i < n; ++i) {
      lam *= __ldg(in.alpha + fh_of(fr.f[i]));
      const bool last = i == n - 1;
      // the next frame's alpha and B rows (the next step's operand)
      const float anext = last ? 0.f : __ldg(in.alpha + fh_of(fr.f[i + 1]));
      const float* bnext = last ? nullptr : brow(i + 1);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_MDONE), i & 1, ctl))) break;
      tc_fence_after();
#pragma unroll 1
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * half + qq;
        float x[32], y[32];
        tmem_ld32(lane_addr + qq * 32, x);
        if (fwd) tmem_ld32(lane_addr + 128 + qq * 32, y);
        tmem_wait_ld();
        float* acc = fwd ? y : x;  // the Horner chain's new value
        if (last) {
          if (fwd) {
            split_to_global(p_hi, p_lo, q, x);
            store_f32(cf_row + q * 32, y);
          } else {
            store_f32(cb_row + q * 32, x);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {  // the next operand: alpha_next X + B_next
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(bnext + q * 32) + u);
            acc[4 * u] = fmaf(anext, acc[4 * u], b4.x);
            acc[4 * u + 1] = fmaf(anext, acc[4 * u + 1], b4.y);
            acc[4 * u + 2] = fmaf(anext, acc[4 * u + 2], b4.z);
            acc[4 * u + 3] = fmaf(anext, acc[4 * u + 3], b4.w);
          }
          split_to_smem(q, row, sA0, x);
          if (fwd) split_to_smem(q, row, sA1, y);
        }
      }
      tc_fence_before();  // TMEM reads done before the next products
      if (!last) {
        fence_proxy_async_smem();
        mbar_arrive_warp(bar(B_AREADY));
      }
    }
    if (fwd && threadIdx.x == 128) w.lam[bch] = lam;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, 256);
}

}  // namespace

cudaError_t launch_compose_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (d.dk != D || d.dv != D || w.M16 == nullptr || w.P16 == nullptr || d.chunk > kMaxChunk)
    return cudaErrorInvalidValue;
  CUtensorMap mm;
  const long long fh = (long long)d.B * d.T * d.H;
  if (!make_matrix_map(&mm, w.M16, fh * 2 * D, D, 128)) return cudaErrorInvalidValue;
  const size_t smem = 1024 + 3 * (size_t)SPLIT + NBARS * 8 + 16;
  cudaError_t e = cudaFuncSetAttribute(k_compose_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_compose_tc<<<dim3(d.C, d.B * d.H, 2), kThreadsCmp, smem, s>>>(d, in, w, mm);
  return cudaGetLastError();
}

}  // namespace vdn
