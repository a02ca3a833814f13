// State read of the linear branch on the tensor cores, with the RMSNorm and
// sigmoid-gate epilogue fused (bf16 q / gates, fp32 accumulation).
//
// What it computes (PaperDaily digest section 三: the query reads the forward
// state before its window and the backward state after it and adds the two;
// the linear branch is RMS-normalised and then gated):
//   R_c = S^f(frames < 5(c-1)) + S^b(frames >= 5(c+2))      per chunk c
//   R_anchor = S_init_f + S_init_b                           anchor query frames
//   o = R q,  y_lin = sigmoid(g_lin) * o / sqrt(mean(o^2) + eps) [* w]
//
// k_read_table builds every R once per (batch, head, chunk): fp32 for
// inspection and, for the MMA, two bf16 terms R_hi = bf16(R) and
// R_lo = bf16(R - R_hi).  q is exact in bf16 and products accumulate in fp32,
// so o = Q R_hi^T + Q R_lo^T carries R to about 16 significant bits (a single
// bf16 R loses too much: o can be small next to |R| |q|, and the RMSNorm then
// scales the rounding up).  k_read_tc then runs, per CTA, a run of up to kTilesPerCta
// tiles of 128 query tokens of one (batch, head, query group); runs are
// launched with the heads varying fastest:
//   warp 0      TMA producer: R once (resident), then Q tiles into a
//               three-stage ring that the products alone release.
//   warp 3      TMA producer of the gate tiles (two-stage ring).
//   warp 1      TMEM allocator; lane 0 issues O_t = Q_t R_hi^T + Q_t R_lo^T
//               (M=128 tokens, N=d_v, K=d_k, both operands K-major in SMEM)
//               into one of two TMEM accumulators.
//   warps 4..11 epilogue, one token per thread (= TMEM lane) and half of d_v
//               per warp (warps w and w + 4 share the TMEM lanes of one
//               32-token quarter): sum of squares over all of d_v, rsqrt,
//               gate from the SMEM tile.  bf16 y with both branch slots: a
//               full tile's outputs overwrite its gates in shared memory (same
//               swizzled layout) and
//   warp 2      stores them with TMA, then returns the gate stage; other
//               tiles and outputs go out as one 32-byte store per 8 outputs.
#include "tc_common.cuh"

namespace vdn {

// Wait limit, in clock cycles, of the epilogue warps' waits in k_read_tc (the
// roles that wait for the tensor cores' products); 0 = the default of every
// bounded wait (about one second).  vdn_debug_set_read_wait_limit sets it, so
// that a test can make those waits run out and check the timeout path.
__device__ long long g_read_epilogue_limit = 0;

namespace {
using namespace tc;

constexpr int TQ = 128;          // tokens per tile
constexpr int kTilesPerCta = 32; // tiles of one query group handled by a CTA (amortises its R load)
constexpr int kThreadsR = 384;
constexpr int kQStages = 3;      // Q ring of k_read_tc (the gate ring has two)
constexpr int kReadBars = 1 + 2 * kQStages + 2 * 2 + 2 * 2 + 2 + 1;

// ------------------------------------------------------------ read table --
__global__ void k_read_table(Dims dm, Work w, __nv_bfloat16* __restrict__ r16) {
  const int c = blockIdx.x, bh = blockIdx.y;
  const long long DD = (long long)dm.dv * dm.dk;
  const float* fs = w.fsnap + ((long long)bh * (dm.C + 1) + (c < dm.C ? max(c - 1, 0) : 0)) * DD;
  const float* bs = w.bsnap + ((long long)bh * (dm.C + 1) + (c < dm.C ? min(c + 2, dm.C) : dm.C)) * DD;
  float* R = w.R + ((long long)bh * (dm.C + 1) + c) * DD;
  __nv_bfloat16* R16 = r16 + ((long long)bh * (dm.C + 1) + c) * 2 * DD;  // [hi | lo]
  for (long long i = threadIdx.x; i < DD; i += blockDim.x) {
    const float r = fs[i] + bs[i];
    R[i] = r;
    const __nv_bfloat16 hi = __float2bfloat16_rn(r);
    R16[i] = hi;
    R16[DD + i] = __float2bfloat16_rn(r - __bfloat162float(hi));
  }
}

// ------------------------------------------------------------ work items --
struct Run {
  int b, h, ridx;
  long long tok0;  // absolute first token of the run
  int ntiles;      // tiles in this run
  int rows_left;   // valid rows from tok0 to the end of the group
};

__device__ __forceinline__ void group_of(const Dims& d, int g, int& f0, int& f1, int& ridx) {
  if (g < d.C) {
    f0 = g * d.chunk;
    f1 = min(d.T, f0 + d.chunk);
    if (d.anchors) {
      if (f0 == 0) f0 = 1;
      if (f1 == d.T) f1 = d.T - 1;
    }
    ridx = g;
  } else {
    f0 = (g == d.C) ? 0 : d.T - 1;
    f1 = f0 + 1;
    ridx = d.C;
  }
}

__host__ __device__ inline int runs_of_rows(long long rows) {
  const long long tiles = (rows + TQ - 1) / TQ;
  return (int)((tiles + kTilesPerCta - 1) / kTilesPerCta);
}

__device__ bool decode_run(const Dims& d, long long item, Run& r) {
  const int ngroups = d.C + (d.anchors ? 2 : 0);
  long long per_bh = 0;
  for (int g = 0; g < ngroups; ++g) {
    int f0, f1, ri;
    group_of(d, g, f0, f1, ri);
    if (f1 > f0) per_bh += runs_of_rows((long long)(f1 - f0) * d.N);
  }
  if (per_bh == 0) return false;
  // heads vary fastest: CTAs running at the same time read the same token rows
  // (every head's q and gate of a token are one contiguous row)
  const long long nbh = (long long)d.B * d.H;
  const long long bh = item % nbh;
  long long rem = item / nbh;
  if (rem >= per_bh) return false;
  for (int g = 0; g < ngroups; ++g) {
    int f0, f1, ri;
    group_of(d, g, f0, f1, ri);
    if (f1 <= f0) continue;
    const long long rows = (long long)(f1 - f0) * d.N;
    const int nr = runs_of_rows(rows);
    if (rem < nr) {
      r.b = (int)(bh / d.H);
      r.h = (int)(bh % d.H);
      r.ridx = ri;
      const long long first_tile = rem * kTilesPerCta;
      const long long tiles = (rows + TQ - 1) / TQ;
      r.ntiles = (int)min((long long)kTilesPerCta, tiles - first_tile);
      r.tok0 = (long long)r.b * d.T * d.N + (long long)f0 * d.N + first_tile * TQ;
      r.rows_left = (int)(rows - first_tile * TQ);
      return true;
    }
    rem -= nr;
  }
  return false;
}

// y[0..8) (+)= v: fp32 rows go out as one 256-bit store (32-byte aligned),
// bf16 rows as one 128-bit store.
template <typename To> __device__ __forceinline__ void put8(To* p, float (&v)[8], bool add);
template <> __device__ __forceinline__ void put8<float>(float* p, float (&v)[8], bool add) {
  if (add) {
    float o[8];
    asm volatile("ld.global.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(o[0]), "=f"(o[1]), "=f"(o[2]), "=f"(o[3]), "=f"(o[4]), "=f"(o[5]), "=f"(o[6]), "=f"(o[7])
                 : "l"(p));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += o[i];
  }
  asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
               "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}
template <> __device__ __forceinline__ void put8<__nv_bfloat16>(__nv_bfloat16* p, float (&v)[8], bool add) {
  if (add) {
    const uint4 o = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] += __uint_as_float(u[e] << 16);
      v[2 * e + 1] += __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
  *reinterpret_cast<uint4*>(p) =
      make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}

// y[0..16) (+)= v as whole 32-byte sectors: bf16 rows as one 256-bit store,
// fp32 rows as two (dst 32-byte aligned).
template <typename To> __device__ __forceinline__ void put16(To* p, float (&v)[16], bool add);
template <> __device__ __forceinline__ void put16<float>(float* p, float (&v)[16], bool add) {
  put8<float>(p, *reinterpret_cast<float(*)[8]>(v), add);
  put8<float>(p + 8, *reinterpret_cast<float(*)[8]>(v + 8), add);
}
template <> __device__ __forceinline__ void put16<__nv_bfloat16>(__nv_bfloat16* p, float (&v)[16], bool add) {
  if (add) {
    uint32_t o[8];
    asm volatile("ld.global.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]), "=r"(o[7])
                 : "l"(p));
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      v[2 * e] += __uint_as_float(o[e] << 16);
      v[2 * e + 1] += __uint_as_float(o[e] & 0xFFFF0000u);
    }
  }
  uint32_t u[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) u[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(u[0]), "r"(u[1]), "r"(u[2]),
               "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
               : "memory");
}

// TMA loads with an L2 eviction-priority policy (createpolicy): R's split,
// re-read by every tile of a run, is kept (evict_last); the streaming Q tiles
// go first (evict_first)
__device__ __forceinline__ uint64_t l2_policy_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma_load_2d_pol(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pol(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                int z, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "l"(pol)
      : "memory");
}

// L2 prefetch of a tensor-map box (no shared memory, no barrier)
__device__ __forceinline__ void prefetch_box_3d(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// sigmoid from the exponential and an approximate reciprocal (both a few ulp;
// exp(-g) overflowing to inf gives 0, the limit)
__device__ __forceinline__ float sigmoid_fast(float g) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + __expf(-g)));
  return r;
}

// ------------------------------------------------------------------ kernel --
// TMA store of a tile from shared memory (bulk group of the issuing thread)
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}

// TY: y is bf16 with the two branch slots side by side (out_mode 0): full
// tiles go out through the gate tile's shared memory and TMA stores (tmy),
// partial tiles (and every other y) through per-thread stores.
template <int D, typename To>
__global__ void __launch_bounds__(kThreadsR, 1)
k_read_tc(Dims dm, Inputs in, Work w, const __grid_constant__ CUtensorMap tmq,
          const __grid_constant__ CUtensorMap tmg, const __grid_constant__ CUtensorMap tmr,
          const __grid_constant__ CUtensorMap tmy) {
  constexpr int NB = D / 64;
  constexpr uint32_t RBYTES = 2 * D * D * 2;  // hi and lo terms
  constexpr uint32_t TBYTES = TQ * D * 2;  // one Q or gate tile
  constexpr int QS = kQStages, GS = 2;
  constexpr uint32_t kCols = 2 * D <= 128 ? 128 : 256;
  constexpr int HD = D / 2;  // columns per epilogue warp
  enum { B_R = 0, B_QFULL = 1, B_QEMPTY = B_QFULL + QS, B_GFULL = B_QEMPTY + QS, B_GEMPTY = B_GFULL + GS,
         B_AFULL = B_GEMPTY + GS, B_AEMPTY = B_AFULL + 2, B_YREADY = B_AEMPTY + 2, B_DRAIN = B_YREADY + GS,
         NBARS = B_DRAIN + 1 };
  static_assert(NBARS == kReadBars, "barrier count");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sR = sm;
  unsigned char* sQ = sR + RBYTES;
  unsigned char* sG = sQ + QS * TBYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sG + GS * TBYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sW = reinterpret_cast<float*>(tmem_slot + 4);  // [D] RMSNorm weight (ones if none)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*reinterpret_cast<volatile uint32_t*>(w.status) != 0u) return;
  Run run;
  if (!decode_run(dm, blockIdx.x, run)) return;
  const Ctl ctl{abort_flag, w.status, (unsigned)TAG_READ_TC};
  // the epilogue warps' waits: the settable limit (the producers, the MMA
  // issuer and the store issuer keep the default, and drain what they issued
  // whatever happens)
  const Ctl ectl{abort_flag, w.status, (unsigned)TAG_READ_TC, g_read_epilogue_limit};
  auto bar = [&](int i) { return smem_u32(bars + i); };
  constexpr bool TY = sizeof(To) == 2;
  const bool ty = TY && dm.out_mode == 0;
  auto full_tile = [&](int t) { return run.rows_left - t * TQ >= TQ; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBARS; ++i)
      mbar_init(bar(i), (i == B_AEMPTY || i == B_AEMPTY + 1 || i == B_YREADY || i == B_YREADY + 1)
                            ? 8    // one arrival per epilogue warp
                            : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kCols);
  for (int i = threadIdx.x; i < D; i += blockDim.x)
    sW[i] = in.rms_weight ? in.rms_weight[(long long)run.h * D + i] : 1.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // R once, then the Q ring (released by the products alone, so the
    // products run up to QS tiles ahead of the epilogue)
    if (lane == 0) {
      const int rrow = ((run.b * dm.H + run.h) * (dm.C + 1) + run.ridx) * 2 * D;
      mbar_expect_tx(bar(B_R), RBYTES);
      for (int part = 0; part < 2; ++part)
        for (int c = 0; c < NB; ++c)
          tma_load_2d(smem_u32(sR + part * D * D * 2 + c * D * 128), &tmr, bar(B_R), c * 64, rrow + part * D);
      int last[QS];
      for (int s = 0; s < QS; ++s) last[s] = -1;
      for (int t = 0; t < run.ntiles; ++t) {
        const int s = t % QS;
        const int tok = (int)(run.tok0 + (long long)t * TQ);
        if (t >= QS && !mbar_wait(bar(B_QEMPTY + s), (t / QS - 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_QFULL + s), TBYTES);
        for (int c = 0; c < NB; ++c)
          tma_load_3d(smem_u32(sQ + s * TBYTES + c * TQ * 128), &tmq, bar(B_QFULL + s), c * 64, run.h, tok);
        last[s] = t;
      }
      mbar_drain(bar(B_R), 0);
      for (int s = 0; s < QS; ++s)
        if (last[s] >= 0) mbar_drain(bar(B_QFULL + s), (last[s] / QS) & 1);
    }
  } else if (warp == 3) {
    // the gate ring (released once a tile's outputs have left its stage)
    if (lane == 0) {
      int last[GS] = {-1, -1};
      for (int t = 0; t < run.ntiles; ++t) {
        const int s = t % GS;
        const int tok = (int)(run.tok0 + (long long)t * TQ);
        if (t >= GS && !mbar_wait(bar(B_GEMPTY + s), (t / GS - 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_GFULL + s), TBYTES);
        for (int c = 0; c < NB; ++c)
          tma_load_3d(smem_u32(sG + s * TBYTES + c * TQ * 128), &tmg, bar(B_GFULL + s), c * 64, run.h, tok);
        last[s] = t;
      }
      for (int s = 0; s < GS; ++s)
        if (last[s] >= 0) mbar_drain(bar(B_GFULL + s), (last[s] / GS) & 1);
    }
  } else if (warp == 2) {
    // stores of full bf16 tiles from the gate stage the epilogue overwrote,
    // then the stage goes back to the gate producer
    if (lane == 0) {
      for (int t = 0; t < run.ntiles; ++t) {
        const int s = t % GS;
        if (!mbar_wait(bar(B_YREADY + s), (t / GS) & 1, ctl)) break;
        if (ty && full_tile(t)) {
          const int tok = (int)(run.tok0 + (long long)t * TQ);
          for (int c = 0; c < NB; ++c) tma_store_3d(&tmy, smem_u32(sG + s * TBYTES + c * TQ * 128), D + c * 64, run.h, tok);
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
        mbar_arrive(bar(B_GEMPTY + s));
      }
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID = idesc_bf16(TQ, D, false);
      const uint64_t rdesc = sdesc(smem_u32(sR), 16, 1024), qdesc0 = sdesc(smem_u32(sQ), 16, 1024);
      bool ok = mbar_wait(bar(B_R), 0, ctl);
      for (int t = 0; ok && t < run.ntiles; ++t) {
        const int s = t % QS, a = t & 1;
        if (!mbar_wait(bar(B_QFULL + s), (t / QS) & 1, ctl)) break;
        if (t >= 2 && !mbar_wait(bar(B_AEMPTY + a), (t / 2 - 1) & 1, ctl)) break;
        tc_fence_after();
        const uint64_t qd = dadd(qdesc0, s * TBYTES);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma_bf16(tmem + a * D, dadd(qd, (k >> 2) * (TQ * 128) + (k & 3) * 32),
                     dadd(rdesc, part * D * D * 2 + (k >> 2) * (D * 128) + (k & 3) * 32), ID, (part | k) ? 1u : 0u);
        }
        mma_commit(bar(B_AFULL + a));
        mma_commit(bar(B_QEMPTY + s));
      }
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const bool add = dm.out_mode != 0;
    for (int t = 0; t < run.ntiles; ++t) {
      const int s = t % GS, a = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_AFULL + a), (t / 2) & 1, ectl))) break;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_GFULL + s), (t / GS) & 1, ectl))) break;
      tc_fence_after();
      // own half of the row into o, the other half only for the sum of squares
      float o[HD];
      float ss[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ss[u] = 0.f;
#pragma unroll
      for (int q = 0; q < HD / 32; ++q) tmem_ld32(lane_addr + a * D + half * HD + q * 32, *reinterpret_cast<float(*)[32]>(o + q * 32));
#pragma unroll
      for (int q = 0; q < HD / 32; ++q) {
        float v[32];
        tmem_ld32(lane_addr + a * D + (1 - half) * HD + q * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ss[i & 7] = fmaf(v[i], v[i], ss[i & 7]);
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_AEMPTY + a));  // accumulator free for tile t + 2
#pragma unroll
      for (int i = 0; i < HD; ++i) ss[i & 7] = fmaf(o[i], o[i], ss[i & 7]);
      const float rs =
          rsqrtf((((ss[0] + ss[1]) + (ss[2] + ss[3])) + ((ss[4] + ss[5]) + (ss[6] + ss[7]))) / D + dm.eps);
      const int rows_valid = min(TQ, run.rows_left - t * TQ);
      const bool valid = row < rows_valid;
      const bool via_smem = ty && rows_valid == TQ;  // uniform over the CTA
      const long long tok = run.tok0 + (long long)t * TQ + row;
      const long long gi = (tok * dm.H + run.h) * D;
      To* y = static_cast<To*>(in.y) + (dm.out_mode == 0 ? 2 * gi + D : gi) + half * HD;
      unsigned char* grow = sG + s * TBYTES + row * 128;
#pragma unroll
      for (int ch = 0; ch < HD / 8; ++ch) {
        const int col0 = half * HD + ch * 8;
        // 8 gate values of this row from the 128B-swizzled tile (64 columns per slab)
        uint4* gp = reinterpret_cast<uint4*>(grow + (col0 >> 6) * (TQ * 128) + ((((col0 & 63) >> 3) ^ (row & 7)) << 4));
        const uint4 raw = *gp;
        const float4 w0 = *reinterpret_cast<const float4*>(sW + col0);
        const float4 w1 = *reinterpret_cast<const float4*>(sW + col0 + 4);
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
        float yv[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float g0 = __uint_as_float(u[e] << 16), g1 = __uint_as_float(u[e] & 0xFFFF0000u);
          yv[2 * e] = o[ch * 8 + 2 * e] * rs * wv[2 * e] * sigmoid_fast(g0);
          yv[2 * e + 1] = o[ch * 8 + 2 * e + 1] * rs * wv[2 * e + 1] * sigmoid_fast(g1);
        }
        if (via_smem) {
          // the outputs take the place of the gates they used (same layout as y's tile)
          *gp = make_uint4(pack_bf16(yv[0], yv[1]), pack_bf16(yv[2], yv[3]), pack_bf16(yv[4], yv[5]),
                           pack_bf16(yv[6], yv[7]));
        } else if (valid) {
          put8<To>(y + ch * 8, yv, add);
        }
      }
      fence_proxy_async_smem();  // the outputs visible to the TMA store
      mbar_arrive_warp(bar(B_YREADY + s));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, kCols);
}

// ------------------------------------------------------------ d = 256 --
// The same read at d = 256.  R's split (256 KB) does not fit beside a query
// tile, so it streams through shared memory in K-chunks of 64 (hi and lo of
// all 256 rows, 64 KB per chunk, two-stage ring) once per 128-token tile; the
// chunks stay in L2 across the CTAs of a query group.  Per tile, 32 MMAs of
// M = 128, N = 256, K = 16 accumulate O = Q R_hi^T + Q R_lo^T into one of two
// 256-column TMEM accumulators.  Epilogue: eight warps, each owning 128 of the
// 256 columns of its 32 rows; a first pass over all 256 TMEM columns forms the
// sum of squares, a second pass its own outputs (gates read from global after
// the producer prefetched the tile's gate boxes into L2 with its Q tile; y
// written in whole 32-byte sectors).
constexpr int D2 = 256;

template <typename To>
__global__ void __launch_bounds__(kThreadsR, 1)
k_read256_tc(Dims dm, Inputs in, Work w, const __grid_constant__ CUtensorMap tmq,
             const __grid_constant__ CUtensorMap tmr, const __grid_constant__ CUtensorMap tmg) {
  constexpr uint32_t QCH = TQ * 128;        // one 64-column chunk of the Q tile: 16 KB
  constexpr uint32_t QBYTES = 4 * QCH;      // the Q tile
  constexpr uint32_t RHALF = D2 * 128;      // 64 columns of all 256 rows of R_hi (or R_lo): 32 KB
  constexpr uint32_t RST = 2 * RHALF;       // one ring stage: hi then lo
  enum { B_QFULL = 0, B_QEMPTY = 1, B_RFULL = 2, B_REMPTY = 4, B_AFULL = 6, B_AEMPTY = 8, B_DRAIN = 10, NBARS = 11 };
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = sm;
  unsigned char* sR = sQ + QBYTES;          // 2 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + 2 * RST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sW = reinterpret_cast<float*>(tmem_slot + 4);  // [256] RMSNorm weight (ones if none)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*reinterpret_cast<volatile uint32_t*>(w.status) != 0u) return;
  Run run;
  if (!decode_run(dm, blockIdx.x, run)) return;
  const Ctl ctl{abort_flag, w.status, (unsigned)TAG_READ_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBARS; ++i) mbar_init(bar(i), (i == B_AEMPTY || i == B_AEMPTY + 1) ? 8 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  for (int i = threadIdx.x; i < D2; i += blockDim.x)
    sW[i] = in.rms_weight ? in.rms_weight[(long long)run.h * D2 + i] : 1.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const int rrow = ((run.b * dm.H + run.h) * (dm.C + 1) + run.ridx) * 2 * D2;
      const uint64_t pol_last = l2_policy_last(), pol_first = l2_policy_first();
      int nq = 0, nr = 0;
      // the gates of a tile go to L2 with its Q tile: the epilogue reads them
      // with plain loads one product later
      auto prefetch_gates = [&](int j) {
        if (j >= run.ntiles) return;
        const int tok = (int)(run.tok0 + (long long)j * TQ);
        for (int c = 0; c < 4; ++c) prefetch_box_3d(&tmg, c * 64, run.h, tok);
      };
      prefetch_gates(0);
      for (int j = 0; j < run.ntiles; ++j) {
        const int tok = (int)(run.tok0 + (long long)j * TQ);
        if (j > 0 && !mbar_wait(bar(B_QEMPTY), (j - 1) & 1, ctl)) break;
        prefetch_gates(j + 1);
        mbar_expect_tx(bar(B_QFULL), QBYTES);
        for (int c = 0; c < 4; ++c)
          tma_load_3d_pol(smem_u32(sQ + c * QCH), &tmq, bar(B_QFULL), c * 64, run.h, tok, pol_first);
        ++nq;
        bool ok = true;
        for (int kc = 0; kc < 4; ++kc) {
          const int u = j * 4 + kc, s = u & 1;
          if (u >= 2 && !mbar_wait(bar(B_REMPTY + s), ((u >> 1) - 1) & 1, ctl)) { ok = false; break; }
          mbar_expect_tx(bar(B_RFULL + s), RST);
          tma_load_2d_pol(smem_u32(sR + s * RST), &tmr, bar(B_RFULL + s), kc * 64, rrow, pol_last);
          tma_load_2d_pol(smem_u32(sR + s * RST + RHALF), &tmr, bar(B_RFULL + s), kc * 64, rrow + D2, pol_last);
          ++nr;
        }
        if (!ok) break;
      }
      // the last copies land before the CTA can exit (bounded, whatever the other roles do)
      if (nq > 0) mbar_drain(bar(B_QFULL), (nq - 1) & 1);
      for (int u = nr - 2 < 0 ? 0 : nr - 2; u < nr; ++u) mbar_drain(bar(B_RFULL + (u & 1)), (u >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID = idesc_bf16(TQ, D2, false);
      const uint64_t qdesc = sdesc(smem_u32(sQ), 16, 1024), rdesc = sdesc(smem_u32(sR), 16, 1024);
      bool ok = true;
      for (int j = 0; ok && j < run.ntiles; ++j) {
        const int acc = j & 1;
        if (j >= 2 && !mbar_wait(bar(B_AEMPTY + acc), ((j >> 1) - 1) & 1, ctl)) break;
        if (!mbar_wait(bar(B_QFULL), j & 1, ctl)) break;
        for (int kc = 0; kc < 4; ++kc) {
          const int u = j * 4 + kc, s = u & 1;
          if (!mbar_wait(bar(B_RFULL + s), (u >> 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16(tmem + acc * D2, dadd(qdesc, kc * QCH + ks * 32), dadd(rdesc, s * RST + part * RHALF + ks * 32),
                       ID, (kc | part | ks) ? 1u : 0u);
          mma_commit(bar(B_REMPTY + s));
        }
        if (!ok) break;
        mma_commit(bar(B_AFULL + acc));
        mma_commit(bar(B_QEMPTY));
      }
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const bool add = dm.out_mode != 0;
    for (int j = 0; j < run.ntiles; ++j) {
      const int acc = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_AFULL + acc), (j >> 1) & 1, ctl))) break;
      tc_fence_after();
      float ss[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) ss[u] = 0.f;
#pragma unroll 1
      for (int q = 0; q < D2 / 32; ++q) {
        float v[32];
        tmem_ld32(lane_addr + acc * D2 + q * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ss[i & 7] = fmaf(v[i], v[i], ss[i & 7]);
      }
      const float rs =
          rsqrtf((((ss[0] + ss[1]) + (ss[2] + ss[3])) + ((ss[4] + ss[5]) + (ss[6] + ss[7]))) / D2 + dm.eps);
      const int rows_valid = min(TQ, run.rows_left - j * TQ);
      const bool valid = row < rows_valid;
      const long long tok = run.tok0 + (long long)j * TQ + row;
      const long long gi = (tok * dm.H + run.h) * D2;
      To* y = static_cast<To*>(in.y) + (dm.out_mode == 0 ? 2 * gi + D2 : gi);
      const __nv_bfloat16* grow = static_cast<const __nv_bfloat16*>(in.gate_lin) + gi;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        const int col0 = half * 128 + q * 32;
        float v[32];
        tmem_ld32(lane_addr + acc * D2 + col0, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const uint4 r0 = __ldg(reinterpret_cast<const uint4*>(grow + col0 + ch * 16));
            const uint4 r1 = __ldg(reinterpret_cast<const uint4*>(grow + col0 + ch * 16 + 8));
            const uint32_t gu[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            float yv[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int i0 = ch * 16 + 2 * e;
              yv[2 * e] = v[i0] * rs * sW[col0 + i0] * sigmoid_fast(__uint_as_float(gu[e] << 16));
              yv[2 * e + 1] = v[i0 + 1] * rs * sW[col0 + i0 + 1] * sigmoid_fast(__uint_as_float(gu[e] & 0xFFFF0000u));
            }
            put16<To>(y + col0 + ch * 16, yv, add);
          }
        }
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_AEMPTY + acc));  // accumulator free for tile j + 2
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, 512);
}

long long num_runs(const Dims& d) {
  const int ngroups = d.C + (d.anchors ? 2 : 0);
  long long per_bh = 0;
  for (int g = 0; g < ngroups; ++g) {
    int f0, f1;
    if (g < d.C) {
      f0 = g * d.chunk;
      f1 = std::min(d.T, f0 + d.chunk);
      if (d.anchors) {
        if (f0 == 0) f0 = 1;
        if (f1 == d.T) f1 = d.T - 1;
      }
    } else {
      f0 = (g == d.C) ? 0 : d.T - 1;
      f1 = f0 + 1;
    }
    if (f1 > f0) per_bh += runs_of_rows((long long)(f1 - f0) * d.N);
  }
  return per_bh * d.B * d.H;
}

template <int D, typename To>
cudaError_t launch(const Dims& d, const Inputs& in, const Work& w, __nv_bfloat16* r16, cudaStream_t s) {
  k_read_table<<<dim3(d.C + 1, d.B * d.H), 256, 0, s>>>(d, w, r16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mg, mr, my;
  const long long tokens = (long long)d.B * d.T * d.N;
  if (!make_token_map(&mq, in.q, tokens, d.H, D, TQ) || !make_token_map(&mg, in.gate_lin, tokens, d.H, D, TQ) ||
      !make_matrix_map(&mr, r16, (long long)d.B * d.H * (d.C + 1) * 2 * D, D, D))
    return cudaErrorInvalidValue;
  // bf16 y with both slots: the store map over [tokens, H, 2 D] (slot 1 = columns D..2D-1);
  // otherwise unused (a copy of the gate map keeps the argument valid)
  if (sizeof(To) == 2 && d.out_mode == 0) {
    if (!make_token_map(&my, in.y, tokens, d.H, 2 * D, TQ)) return cudaErrorInvalidValue;
  } else {
    my = mg;
  }
  const size_t smem = 1024 + 2 * (size_t)D * D * 2 + (kQStages + 2) * (size_t)TQ * D * 2 + kReadBars * 8 + 16 + D * 4;
  auto kern = k_read_tc<D, To>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long items = num_runs(d);
  if (items <= 0 || items > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)items, kThreadsR, smem, s>>>(d, in, w, mq, mg, mr, my);
  return cudaGetLastError();
}

template <typename To>
cudaError_t launch256(const Dims& d, const Inputs& in, const Work& w, __nv_bfloat16* r16, cudaStream_t s) {
  k_read_table<<<dim3(d.C + 1, d.B * d.H), 256, 0, s>>>(d, w, r16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mr, mg;
  const long long tokens = (long long)d.B * d.T * d.N;
  if (!make_token_map(&mq, in.q, tokens, d.H, D2, TQ) || !make_token_map(&mg, in.gate_lin, tokens, d.H, D2, TQ) ||
      !make_matrix_map(&mr, r16, (long long)d.B * d.H * (d.C + 1) * 2 * D2, D2, D2))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + 4 * (size_t)TQ * 128 + 2 * 2 * (size_t)D2 * 128 + 11 * 8 + 16 + D2 * 4;
  auto kern = k_read256_tc<To>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long items = num_runs(d);
  if (items <= 0 || items > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)items, kThreadsR, smem, s>>>(d, in, w, mq, mr, mg);
  return cudaGetLastError();
}

}  // namespace

bool read_tc_supported(const Dims& d) {
  if (!d.bf16 || d.dk != d.dv || (d.dk != 64 && d.dk != 128 && d.dk != 256)) return false;
  if ((long long)d.B * d.T * d.N >= (1LL << 31)) return false;
  if ((long long)d.B * d.H * (d.C + 1) * 2 * d.dk >= (1LL << 31)) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_read_tc(const Dims& d, const Inputs& in, const Work& w, void* r16, cudaStream_t s) {
  __nv_bfloat16* r = static_cast<__nv_bfloat16*>(r16);
  if (d.dk == 256) return d.out_bf16 ? launch256<__nv_bfloat16>(d, in, w, r, s) : launch256<float>(d, in, w, r, s);
  if (d.dk == 128) return d.out_bf16 ? launch<128, __nv_bfloat16>(d, in, w, r, s) : launch<128, float>(d, in, w, r, s);
  if (d.dk == 64) return d.out_bf16 ? launch<64, __nv_bfloat16>(d, in, w, r, s) : launch<64, float>(d, in, w, r, s);
  return cudaErrorInvalidValue;
}

}  // namespace vdn

extern "C" vdn_status vdn_debug_set_read_wait_limit(unsigned long long cycles) {
  if (cycles > (unsigned long long)vdn::tc::kWaitCycles) return VDN_ERR_INVALID_ARG;
  const long long v = (long long)cycles;
  return cudaMemcpyToSymbol(vdn::g_read_epilogue_limit, &v, sizeof(v)) == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}
