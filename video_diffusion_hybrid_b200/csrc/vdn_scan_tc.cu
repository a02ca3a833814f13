// Forward and backward state scan on the tensor cores (bf16 inputs, d = 128).
//
// What it computes (deepmagic post "用兩條分支取代一條", the frame-wise closed
// form; PaperDaily digest section 三, the two directions and the half-text
// start states): per (batch, head) and direction, from S = S_x / 2,
//   S <- alpha_t S M_t + C_t        for every written (non-anchor) frame t,
// frames in increasing order forward and decreasing order backward, anchor
// frames leaving S unchanged, with the state saved at every chunk boundary:
//   forward  slot j : frames < min(5j, T)      (slot 0 = start state)
//   backward slot j : frames >= min(5j, T)     (slot C = start state)
//
// Rows of S evolve independently (each row is its own affine recurrence), so
// a chain is carried by a pair of CTAs on neighbouring SMs (a cluster of
// two), each holding 64 of the 128 state rows.  Each step is one
// tcgen05.mma.cta_group::2 product S M_t with M = 128 (64 rows per CTA) and
// N = 128 (each CTA holds 64 of M_t's rows as its half of B, so M_t crosses
// from memory once per pair).  fp32 accuracy comes from the bf16 hi/lo split
// of both factors (x = hi + lo with hi = bf16(x), lo = bf16(x - hi)):
//   S M ~ S_hi M_hi + S_hi M_lo + S_lo M_hi
// which keeps about 16 significant bits per step; M_t's split is written by
// the solve, S's by this kernel's epilogue.  M_t is symmetric (the inverse
// of an SPD matrix), so its rows serve as the K-major B operand.  Two SMs per
// chain double the SMs a batch of chains occupies and halve each SM's
// product and epilogue per step.
//
// Roles (384 threads per CTA; the two directions of a head read the same
// M_t, C_t, in opposite orders):
//   warp 0      TMA producer (both CTAs): this CTA's half of M_t's split once
//               the previous product is done (bytes counted on the leader's
//               barrier), its 64 rows of C_t once its epilogue has read them.
//   warp 1      TMEM allocator (both CTAs); lane 0 of the leader (rank 0)
//               issues the 24 MMAs of S M_t for the pair.
//   warps 4..11 epilogue (both CTAs): accumulator layout of a 64-row CTA
//               share, TMEM lane l = row (l mod 64), column half (l / 64);
//               warps w and w + 4 take 32 columns each.  S = alpha_t (S M_t)
//               + C_t in fp32, chunk-boundary snapshots to global memory, and
//               the new S split back into the A operand.
// M_t and C_t are double-buffered, so the copies for step i + 1 overlap step
// i; S is single-buffered (each step depends on the one before).
#include "tc_common.cuh"

namespace vdn {
namespace {
using namespace tc;

constexpr int D = 128;
constexpr int R = 64;                    // state rows per CTA
constexpr int kThreadsScan = 384;
constexpr uint32_t CHUNK = R * 128;      // 64 K-columns of a 64-row bf16 operand (SW128): 8 KB
constexpr uint32_t OPBYTES = 2 * CHUNK;  // one 64 x 128 bf16 operand
constexpr uint32_t SPLIT = 2 * OPBYTES;  // hi then lo: 32 KB
constexpr uint32_t CBOX = R * 128;       // 32 fp32 columns x 64 rows (SW128): 8 KB
constexpr uint32_t CBYTES = 4 * CBOX;    // this CTA's rows of C_t: 32 KB
constexpr uint32_t kTmemScan = 64;       // accumulator columns (64 rows x 128 as 128 lanes x 64)
// M_t and C_t are double-buffered (slot = step & 1).  SREADY lives on the
// leader (one arrival per epilogue warp of both CTAs); BEMPTY is committed by
// the leader's MMAs to both CTAs; CEMPTY takes this CTA's eight warps.
enum { B_BFULL = 0, B_CFULL = 2, B_BEMPTY = 4, B_CEMPTY = 6, B_SREADY = 8, B_MDONE = 9, B_DRAIN = 10, NBARS = 11 };

__device__ __forceinline__ int frame_at(const Dims& d, int dir, int st) { return dir == 0 ? st : d.T - 1 - st; }

// first scan position >= st whose frame is written (T if none)
__device__ __forceinline__ int next_written(const Dims& d, int dir, int st) {
  while (st < d.T && is_anchor(d, frame_at(d, dir, st))) ++st;
  return st;
}

// snapshot slot taken after the frame at scan position st, or -1
__device__ __forceinline__ int snap_slot(const Dims& d, int dir, int st) {
  const int t = frame_at(d, dir, st);
  if (dir == 0) {
    if ((t + 1) % d.chunk == 0) return (t + 1) / d.chunk;
    return (t + 1 == d.T) ? d.C : -1;
  }
  return (t % d.chunk == 0) ? t / d.chunk : -1;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void st_global_v8(float* p, const float* v) {
  asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
               "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}

// Snapshot slots taken after the frames at scan positions [p0, p1) (the
// state is the same across them): at most two with anchors at both ends; a
// longer run (never produced by the anchor rule) falls back to the loop.
struct Slots {
  int a, b, p0, p1;
};
__device__ __forceinline__ Slots slots_of(const Dims& dm, int dir, int p0, int p1) {
  Slots r{-1, -1, p0, p1};
  if (p1 - p0 <= 2) {
    if (p0 < p1) r.a = snap_slot(dm, dir, p0);
    if (p0 + 1 < p1) r.b = snap_slot(dm, dir, p0 + 1);
    r.p0 = r.p1 = 0;
  }
  return r;
}

__device__ __forceinline__ void store_row32(float* dst, const float* s) {
#pragma unroll
  for (int u = 0; u < 4; ++u) st_global_v8(dst + 8 * u, s + 8 * u);
}

// 32 consecutive state values (columns 32q..32q+31) of the row at `row` of
// this CTA's 64-row share, split into the A operand.
__device__ __forceinline__ void split_chunk(int q, int row, unsigned char* sA, const float (&s)[32]) {
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

// ... and into the snapshot slots the scan positions it stands for take.
__device__ __forceinline__ void snap_chunk(const Dims& dm, int dir, const Slots& sl, float* snap_row, int q,
                                           const float (&s)[32]) {
  const long long DD = (long long)D * D;
  if (sl.a >= 0) store_row32(snap_row + sl.a * DD + q * 32, s);
  if (sl.b >= 0) store_row32(snap_row + sl.b * DD + q * 32, s);
  for (int p = sl.p0; p < sl.p1; ++p) {
    const int k = snap_slot(dm, dir, p);
    if (k >= 0) store_row32(snap_row + k * DD + q * 32, s);
  }
}

// CH = false: one step per written frame, S <- alpha_t S M_t + C_t (tmm over
// M's split, tmc over C_t).  CH = true: one step per chunk with the composed
// maps, S <- Lam_c S P_c + Cf_c forward and S <- Lam_c S P_c^T + Cb_c
// backward (tmm over P_c's split, tmc over [Cf; Cb]); every step ends on a
// chunk boundary, so every step is a snapshot.
template <bool CH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsScan, 1)
k_scan_tc(Dims dm, Inputs in, Work w, const __grid_constant__ CUtensorMap tmm, const __grid_constant__ CUtensorMap tmc) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = sm;            // this CTA's rows of S, hi | lo, K-major SW128
  unsigned char* sB = sA + SPLIT;    // 2 slots: this CTA's half of M_t (64 rows), hi | lo, K-major SW128
  unsigned char* sC = sB + 2 * SPLIT;  // 2 slots: this CTA's rows of C_t, fp32, 4 boxes of 32 columns, SW128
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + 2 * CBYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // no early exit: both CTAs of the pair must reach the cluster barriers
  const uint32_t rank = cta_rank();
  const bool lead = rank == 0;
  const int chain = blockIdx.x >> 1;
  const int dir = chain & 1, bh = chain >> 1;
  const int b = bh / dm.H, h = bh % dm.H;
  const int row0 = R * (int)rank;  // first state row of this CTA
  const Ctl ctl{abort_flag, w.status, (unsigned)TAG_SCAN_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto lbar = [&](int i) { return map_rank(smem_u32(bars + i), 0); };
  auto fh_of = [&](int t) { return ((long long)b * dm.T + t) * dm.H + h; };
  int nw = 0;  // steps: written frames, or chunks
  if (CH) nw = dm.C;
  else
    for (int t = 0; t < dm.T; ++t) nw += is_anchor(dm, t) ? 0 : 1;
  // chunk mode: the chunk of step i, its chunk-map index, and the rows of its
  // C constant (Cb after all Cf) in the [Cf; Cb] array
  const long long nbch = (long long)dm.B * dm.C * dm.H;
  auto chunk_of = [&](int i) { return dir == 0 ? i : dm.C - 1 - i; };
  auto bch_of = [&](int c) { return ((long long)b * dm.C + c) * dm.H + h; };
  // forward chunk steps multiply by P_c (not symmetric): B is P_c read
  // N-contiguous (MN-major); every other step reads rows of a symmetric M_t
  // or of P_c for P_c^T (K-major)
  const bool mn = CH && dir == 0;

  if (threadIdx.x == 0) {
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar(B_BFULL + k), 1);
      mbar_init(bar(B_CFULL + k), 1);
      mbar_init(bar(B_BEMPTY + k), 1);
      mbar_init(bar(B_CEMPTY + k), 8);  // one arrival per epilogue warp of this CTA
    }
    mbar_init(bar(B_SREADY), 16);  // one arrival per epilogue warp of the pair
    mbar_init(bar(B_MDONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc2(smem_u32(tmem_slot), kTmemScan);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Phases: MDONE completes once per written step i, SREADY once for the
  // start state and once per step (step i's MMA waits for phase i); a slot's
  // FULL and EMPTY barriers once per use of the slot (step i uses slot i & 1,
  // its (i >> 1)-th use).  No role can run two phases ahead of a waiter.
  if (warp == 0) {
    if (lane == 0) {
      int nb = 0, nc = 0;
      // this CTA's halves of M_t, C_t of the step two ahead are pulled into
      // L2 early, so that the single-buffered loads below (issued only when
      // their buffer frees) run at L2 rather than HBM latency
      auto prefetch_step = [&](int pst) {
        if (CH) {
          if (pst >= nw) return;
          const long long pb = bch_of(chunk_of(pst));
          prefetch_l2(static_cast<const __nv_bfloat16*>(w.P16) + pb * 2 * D * D, SPLIT * 2);
          prefetch_l2(w.Cf + ((dir == 0 ? 0 : nbch) + pb) * D * D + (long long)row0 * D, CBYTES);
          return;
        }
        if (pst >= dm.T) return;
        const long long pfh = fh_of(frame_at(dm, dir, pst));
        const __nv_bfloat16* m16 = static_cast<const __nv_bfloat16*>(w.M16);
        prefetch_l2(m16 + ((pfh * 2) * D + row0) * D, OPBYTES);
        prefetch_l2(m16 + ((pfh * 2 + 1) * D + row0) * D, OPBYTES);
        prefetch_l2(w.Cm + (pfh * D + row0) * D, CBYTES);
      };
      auto next_pos = [&](int p) { return CH ? p + 1 : next_written(dm, dir, p + 1); };
      int st = CH ? 0 : next_written(dm, dir, 0);
      int pst = st;
      prefetch_step(pst);
      pst = next_pos(pst);
      prefetch_step(pst);
      for (int i = 0; i < nw; ++i, st = next_pos(st)) {
        // B rows (of M's or P_c's split) and C rows of this step
        const long long mrow = CH ? bch_of(chunk_of(i)) : fh_of(frame_at(dm, dir, st));
        const long long crow = CH ? (dir == 0 ? 0 : nbch) + mrow : mrow;
        pst = next_pos(pst);
        prefetch_step(pst);
        const int slot = i & 1;
        // slot free: the product (B) and this CTA's epilogue (C) of step i - 2 are done
        if (i >= 2 && !mbar_wait_cl(bar(B_BEMPTY + slot), ((i - 2) >> 1) & 1, ctl)) break;
        if (lead) mbar_expect_tx(bar(B_BFULL + slot), 2 * SPLIT);
        for (int part = 0; part < 2; ++part)
          for (int c = 0; c < 2; ++c) {
            // K-major: rows row0.. of the matrix, K chunk c; MN-major: its
            // columns row0.. (this CTA's half of N), K rows 64c..
            const int x = mn ? row0 : c * 64;
            const int y = (int)((mrow * 2 + part) * D + (mn ? 64 * c : row0));
            tma_load_2d_pair(smem_u32(sB + slot * SPLIT + part * OPBYTES + c * CHUNK), &tmm, lbar(B_BFULL + slot),
                             x, y);
          }
        ++nb;
        if (i >= 2 && !mbar_wait_cl(bar(B_CEMPTY + slot), ((i - 2) >> 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_CFULL + slot), CBYTES);
        for (int c = 0; c < 4; ++c)
          tma_load_2d(smem_u32(sC + slot * CBYTES + c * CBOX), &tmc, bar(B_CFULL + slot), c * 32,
                      (int)(crow * D + row0));
        ++nc;
      }
      // the last copies land before the pair can exit (the leader's B
      // barriers count both CTAs' bytes)
      for (int n = nb - 2 < 0 ? 0 : nb - 2; lead && n < nb; ++n) mbar_drain(bar(B_BFULL + (n & 1)), (n >> 1) & 1);
      for (int n = nc - 2 < 0 ? 0 : nc - 2; n < nc; ++n) mbar_drain(bar(B_CFULL + (n & 1)), (n >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      // M = 128 over the pair, N = 128; B K-major, or MN-major (forward chunk steps)
      const uint32_t ID = mn ? idesc_bf16(2 * R, D, true) : idesc_bf16(2 * R, D, false);
      const uint64_t a0 = sdesc(smem_u32(sA), 16, 1024), b0 = sdesc(smem_u32(sB), 16, 1024);
      for (int i = 0; i < nw; ++i) {
        const int slot = i & 1;
        if (!mbar_wait_cl(bar(B_SREADY), i & 1, ctl)) break;
        if (!mbar_wait_cl(bar(B_BFULL + slot), (i >> 1) & 1, ctl)) break;
        tc_fence_after();
        const uint64_t bs = dadd(b0, slot * SPLIT);
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {  // hi hi, hi lo, lo hi
          const uint32_t ao = pass == 2 ? OPBYTES : 0u, bo = pass == 1 ? OPBYTES : 0u;
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            mma2_bf16(tmem, dadd(a0, ao + (k >> 2) * CHUNK + (k & 3) * 32),
                      dadd(bs, bo + (mn ? k * 16 * 128 : (k >> 2) * CHUNK + (k & 3) * 32)), ID, (pass | k) ? 1u : 0u);
        }
        commit2(bar(B_MDONE));
        commit2(map_rank(bar(B_MDONE), 1));
        commit2(bar(B_BEMPTY + slot));
        commit2(map_rank(bar(B_BEMPTY + slot), 1));
      }
      commit2(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const int tl = quad * 32 + lane;             // TMEM lane
    const int srow = tl & (R - 1), ch = tl >> 6;  // row of this CTA's share, column half
    const int q = 2 * ch + half;                  // this thread's 32 columns: 32q .. 32q + 31
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + half * 32;
    const long long DD = (long long)D * D;
    const int row = row0 + srow;  // state row
    float* snap_row = (dir == 0 ? w.fsnap : w.bsnap) + (long long)bh * (dm.C + 1) * DD + (long long)row * D;
    // C-slot item k (one per step, slot k & 1): this CTA's 32 columns of its
    // row, into registers; the slot goes back to the producer at once
    auto read_c = [&](int k, float (&cv)[32]) -> bool {
      const int slot = k & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_cl(bar(B_CFULL + slot), (k >> 1) & 1, ctl))) return false;
      const unsigned char* crow = sC + slot * CBYTES + q * CBOX + srow * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 c4 = *reinterpret_cast<const float4*>(crow + ((u ^ (srow & 7)) << 4));
        cv[4 * u] = c4.x; cv[4 * u + 1] = c4.y; cv[4 * u + 2] = c4.z; cv[4 * u + 3] = c4.w;
      }
      mbar_arrive_warp(bar(B_CEMPTY + slot));
      return true;
    };
    // x <- a x + c (both 32 values, paired fp32 FMAs)
    auto axpy = [&](float a, float (&x)[32], const float (&c)[32], float (&out)[32]) {
      const float2 a2 = make_float2(a, a);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float2 r = fma2(a2, make_float2(x[2 * u], x[2 * u + 1]), make_float2(c[2 * u], c[2 * u + 1]));
        out[2 * u] = r.x;
        out[2 * u + 1] = r.y;
      }
    };
    // Frame steps (B form): step i's product is X_i M_t with X_i = alpha_t S + B_t
    // (the solve left B_t in the C_t slot), so the product is the new state and
    // the epilogue of step i forms X_{i+1} from the next frame's alpha and B.
    // Chunk steps (C form): the product is S P (or S P^T), the epilogue adds
    // Lam and the chunk constant.
    int st = CH ? 0 : next_written(dm, dir, 0);
    bool ok = true;
    {
      // start state: its own slot, then (frame steps) the slots of leading
      // unwritten frames
      const float* start = (dir == 0 && in.fwd_init) ? in.fwd_init : w.half_text;
      const float* src = start + (long long)bh * DD + (long long)row * D;
      const int start_slot = dir == 0 ? 0 : dm.C;
      float s[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src + q * 32) + u);
        s[4 * u] = v.x; s[4 * u + 1] = v.y; s[4 * u + 2] = v.z; s[4 * u + 3] = v.w;
      }
      if (CH) {
        split_chunk(q, srow, sA, s);
      } else if (nw > 0) {
        float x[32];
        ok = read_c(0, x);
        if (ok) {
          axpy(__ldg(in.alpha + fh_of(frame_at(dm, dir, st))), s, x, x);
          split_chunk(q, srow, sA, x);
        }
      }
      if (ok) {
        fence_proxy_async_smem();
        arrive_cluster_warp(lbar(B_SREADY));
      }
      store_row32(snap_row + start_slot * DD + q * 32, s);
      if (!CH) snap_chunk(dm, dir, slots_of(dm, dir, 0, st), snap_row, q, s);
    }
    for (int i = 0; ok && i < nw; ++i) {
      const int st_next = CH ? st + 1 : next_written(dm, dir, st + 1);
      const int cst = chunk_of(i);  // chunk steps: the chunk, and the boundary slot it ends on
      const Slots sl = CH ? Slots{dir == 0 ? cst + 1 : cst, -1, 0, 0} : slots_of(dm, dir, st, st_next);
      const bool more = i + 1 < nw;
      // the C-slot values this epilogue adds (they do not depend on the
      // product): chunk steps this step's constant, frame steps the next B
      float cv[32];
      if (CH || more) {
        if (!read_c(CH ? i : i + 1, cv)) break;
      }
      const float alpha = CH ? w.lam[bch_of(cst)]
                             : (more ? __ldg(in.alpha + fh_of(frame_at(dm, dir, st_next))) : 0.f);
      if (!__all_sync(0xffffffffu, mbar_wait_cl(bar(B_MDONE), i & 1, ctl))) break;
      tc_fence_after();
      float v[32];
      tmem_ld32(lane_addr, v);
      tmem_wait_ld();
      tc_fence_before();  // TMEM reads done before the next product
      if (CH) {
        axpy(alpha, v, cv, v);  // S = Lam (S P) + Cf
        split_chunk(q, srow, sA, v);
      } else if (more) {
        axpy(alpha, v, cv, cv);  // X = alpha_next S + B_next; v is the new state
        split_chunk(q, srow, sA, cv);
      }
      if (CH || more) {
        fence_proxy_async_smem();  // new A operand visible to the tensor cores
        arrive_cluster_warp(lbar(B_SREADY));
      }
      // snapshots after the hand-off: the next product does not wait for them
      snap_chunk(dm, dir, sl, snap_row, q, v);
      st = st_next;
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory or barriers
  tc_fence_after();
  if (warp == 1) tmem_free2(tmem, kTmemScan);
}

// ----------------------------------------------------------- d = 256 --
// The same frame scan at d = 256, S <- (alpha_t S + B_t) M_t.  The state
// rows split over a CTA pair again, now 128 rows per CTA, and each step is
// one tcgen05.mma.cta_group::2 product with M = 256 (the pair) and N = 256
// (each CTA holds the 128 rows of M_t's split that are its half of B), K =
// 256, over the same three bf16 hi/lo terms.  The A operand, this CTA's rows
// of X = alpha S + B_t as hi | lo, lives in TMEM (columns 256..383 and
// 384..511, two bf16 a column: the TS form), next to the accumulator
// (columns 0..255: lane = row of this CTA's share, column = state column).
// Shared memory holds a ring of three stages of M_t's split, each one
// 64-wide K-chunk of both terms (32 KB; the product of a chunk's three terms
// releases its stage), and the next frame's B_t rows as eight boxes of 32
// columns (fp32, 16 KB each), loaded by TMA while the product runs.
// Epilogue warps 4..11: warp w takes TMEM lanes 32 (w mod 4) .. + 31 and the
// columns 128 ((w - 4) / 4) .. + 127 (boxes 4 ((w - 4) / 4) .. + 3), in four
// groups of 32.
namespace s256 {
constexpr int D = 256;
constexpr int R = 128;                   // state rows per CTA
constexpr int kThreads = 384;
constexpr uint32_t CHUNK = R * 128;      // 64 K-columns of a 128-row bf16 operand (SW128): 16 KB
constexpr uint32_t STAGE = 2 * CHUNK;    // hi | lo of one K-chunk of this CTA's half of M_t: 32 KB
constexpr int ST = 3;                    // ring stages
constexpr int KCH = D / 64;              // K-chunks per step
constexpr uint32_t CBOX = R * 128;       // 32 fp32 columns x 128 rows (SW128): 16 KB
constexpr uint32_t kTmem = 512;
constexpr uint32_t COL_AHI = 256, COL_ALO = 384;
// FULL lives on the leader (both CTAs' bytes), EMPTY is committed by the
// leader's MMAs to both CTAs, SREADY takes one arrival per epilogue warp of
// the pair; CFULL / CEMPTY (one per column half) guard this CTA's B_t boxes.
enum { B_FULL = 0, B_EMPTY = ST, B_CFULL = 2 * ST, B_CEMPTY = 2 * ST + 2, B_SREADY = 2 * ST + 4, B_MDONE, B_DRAIN,
       NBARS };

__host__ __device__ constexpr size_t smem_bytes() { return 1024 + ST * (size_t)STAGE + 8 * (size_t)CBOX + NBARS * 8 + 16; }

// A operand from TMEM for the pair (bf16 pairs packed in 32-bit columns, lane = row)
__device__ __forceinline__ void mma2_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 32 values of X (K-columns col .. col + 31 of this lane's row) into the A
// operand's hi and lo columns
__device__ __forceinline__ void split_to_tmem(uint32_t lane_addr, int col, const float (&x)[32]) {
  uint32_t hv[16], lv[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float x0 = x[2 * j], x1 = x[2 * j + 1];
    hv[j] = pack_bf16(x0, x1);
    lv[j] = pack_bf16(x0 - __uint_as_float(hv[j] << 16), x1 - __uint_as_float(hv[j] & 0xFFFF0000u));
  }
  tmem_st16(lane_addr + COL_AHI + col / 2, hv);
  tmem_st16(lane_addr + COL_ALO + col / 2, lv);
}

// this lane's 32 values of box `box` (its row of the CTA's share)
__device__ __forceinline__ void box32(const unsigned char* sC, int box, int srow, float (&v)[32]) {
  const unsigned char* p = sC + box * CBOX + srow * 128;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float4 a = *reinterpret_cast<const float4*>(p + ((u ^ (srow & 7)) << 4));
    v[4 * u] = a.x; v[4 * u + 1] = a.y; v[4 * u + 2] = a.z; v[4 * u + 3] = a.w;
  }
}

__device__ __forceinline__ void ld32(const float* src, float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(src) + u);
    v[4 * u] = a.x; v[4 * u + 1] = a.y; v[4 * u + 2] = a.z; v[4 * u + 3] = a.w;
  }
}

__device__ __forceinline__ void snap32(const Dims& dm, int dir, const Slots& sl, float* snap_row, int col,
                                       const float (&v)[32]) {
  const long long DD = (long long)D * D;
  if (sl.a >= 0) store_row32(snap_row + sl.a * DD + col, v);
  if (sl.b >= 0) store_row32(snap_row + sl.b * DD + col, v);
  for (int p = sl.p0; p < sl.p1; ++p) {
    const int k = snap_slot(dm, dir, p);
    if (k >= 0) store_row32(snap_row + k * DD + col, v);
  }
}
}  // namespace s256

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(s256::kThreads, 1)
k_scan256_tc(Dims dm, Inputs in, Work w, const __grid_constant__ CUtensorMap tmm,
             const __grid_constant__ CUtensorMap tmc) {
  constexpr int D = s256::D, R = s256::R, ST = s256::ST, KCH = s256::KCH;
  constexpr uint32_t CHUNK = s256::CHUNK, STAGE = s256::STAGE, CBOX = s256::CBOX;
  constexpr int B_FULL = s256::B_FULL, B_EMPTY = s256::B_EMPTY, B_CFULL = s256::B_CFULL, B_CEMPTY = s256::B_CEMPTY,
                B_SREADY = s256::B_SREADY, B_MDONE = s256::B_MDONE, B_DRAIN = s256::B_DRAIN, NBARS = s256::NBARS;
  using s256::box32;
  using s256::ld32;
  using s256::snap32;
  using s256::split_to_tmem;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sB = sm;                // ST stages: a K-chunk of this CTA's half of M_t, hi | lo, K-major SW128
  unsigned char* sC = sB + ST * STAGE;   // 8 boxes: this CTA's rows of the next B_t, fp32 SW128
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + 8 * CBOX);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // no early exit: both CTAs of the pair must reach the cluster barriers
  const uint32_t rank = cta_rank();
  const bool lead = rank == 0;
  const int chain = blockIdx.x >> 1;
  const int dir = chain & 1, bh = chain >> 1;
  const int b = bh / dm.H, h = bh % dm.H;
  const int row0 = R * (int)rank;
  const Ctl ctl{abort_flag, w.status, (unsigned)TAG_SCAN_TC};
  const long long DD = (long long)D * D;
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto lbar = [&](int i) { return map_rank(smem_u32(bars + i), 0); };
  auto fh_of = [&](int t) { return ((long long)b * dm.T + t) * dm.H + h; };
  int nw = 0;
  for (int t = 0; t < dm.T; ++t) nw += is_anchor(dm, t) ? 0 : 1;

  if (threadIdx.x == 0) {
    for (int k = 0; k < ST; ++k) {
      mbar_init(bar(B_FULL + k), 1);
      mbar_init(bar(B_EMPTY + k), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar(B_CFULL + k), 1);
      mbar_init(bar(B_CEMPTY + k), 4);  // the four epilogue warps of that column half
    }
    mbar_init(bar(B_SREADY), 16);
    mbar_init(bar(B_MDONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc2(smem_u32(tmem_slot), s256::kTmem);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Load g = i KCH + c (step i, K-chunk c) uses stage g mod ST, its
  // (g / ST)-th use; FULL and EMPTY of a stage complete once per use.  B_t
  // item k (the k-th written frame's rows, read by the epilogue that forms
  // X_k) fills the boxes; CFULL / CEMPTY complete once per item.
  if (warp == 0) {
    if (lane == 0) {
      // (no L2 prefetch of later steps: the ring and the B_t boxes are
      // loaded a step ahead already, and a prefetch two steps ahead measured
      // slower: 0.61 vs 0.57 ms)
      bool ok = true;
      int nc[2] = {0, 0};  // items loaded, per column half
      auto load_item = [&](int k, int kst) -> bool {
        const long long crow = fh_of(frame_at(dm, dir, kst)) * D + row0;
        for (int hf = 0; hf < 2; ++hf) {
          if (k >= 1 && !mbar_wait_cl(bar(B_CEMPTY + hf), (k - 1) & 1, ctl)) return false;
          mbar_expect_tx(bar(B_CFULL + hf), 4 * CBOX);
          for (int x = 0; x < 4; ++x)
            tma_load_2d(smem_u32(sC + (4 * hf + x) * CBOX), &tmc, bar(B_CFULL + hf), (4 * hf + x) * 32, (int)crow);
          ++nc[hf];
        }
        return true;
      };
      int st = next_written(dm, dir, 0);
      if (nw > 0) ok = load_item(0, st);
      int nl = 0;
      for (int i = 0; ok && i < nw; ++i) {
        const long long mrow = fh_of(frame_at(dm, dir, st));
        const int st_next = next_written(dm, dir, st + 1);
        for (int c = 0; c < KCH; ++c) {
          const int g = i * KCH + c, s = g % ST, u = g / ST;
          if (u >= 1 && !mbar_wait_cl(bar(B_EMPTY + s), (u - 1) & 1, ctl)) { ok = false; break; }
          if (lead) mbar_expect_tx(bar(B_FULL + s), 2 * STAGE);
          for (int part = 0; part < 2; ++part)
            tma_load_2d_pair(smem_u32(sB + s * STAGE + part * CHUNK), &tmm, lbar(B_FULL + s), c * 64,
                             (int)((mrow * 2 + part) * D + row0));
          ++nl;
        }
        // the next frame's B_t, once the epilogue has formed X_i from item i
        if (ok && i + 1 < nw) ok = load_item(i + 1, st_next);
        st = st_next;
      }
      // the last copies land before the pair can exit (the leader's FULL
      // barriers count both CTAs' bytes); each is its stage's last use
      for (int n = nl - ST < 0 ? 0 : nl - ST; lead && n < nl; ++n) mbar_drain(bar(B_FULL + n % ST), (n / ST) & 1);
      for (int hf = 0; hf < 2; ++hf)
        if (nc[hf] > 0) mbar_drain(bar(B_CFULL + hf), (nc[hf] - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      const uint32_t ID = idesc_bf16(2 * R, D, false);
      const uint64_t b0 = sdesc(smem_u32(sB), 16, 1024);
      bool ok = true;
      for (int i = 0; ok && i < nw; ++i) {
        if (!mbar_wait_cl(bar(B_SREADY), i & 1, ctl)) break;
        tc_fence_after();
        for (int c = 0; c < KCH; ++c) {
          const int g = i * KCH + c, s = g % ST, u = g / ST;
          if (!mbar_wait_cl(bar(B_FULL + s), u & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bs = dadd(b0, s * STAGE);
#pragma unroll
          for (int pass = 0; pass < 3; ++pass) {  // hi hi, hi lo, lo hi
            const uint32_t acol = (pass == 2 ? s256::COL_ALO : s256::COL_AHI) + c * 32;
            const uint32_t bo = pass == 1 ? CHUNK : 0u;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              s256::mma2_bf16_ts(tmem, tmem + acol + kk * 8, dadd(bs, bo + kk * 32), ID, (c | pass | kk) ? 1u : 0u);
          }
          commit2(bar(B_EMPTY + s));
          commit2(map_rank(bar(B_EMPTY + s), 1));
        }
        if (!ok) break;
        commit2(bar(B_MDONE));
        commit2(map_rank(bar(B_MDONE), 1));
      }
      commit2(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const int srow = quad * 32 + lane;  // TMEM lane = row of this CTA's share
    const int row = row0 + srow;        // state row
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    float* snap_row = (dir == 0 ? w.fsnap : w.bsnap) + (long long)bh * (dm.C + 1) * DD + (long long)row * D;
    // item k's boxes of this column half, into X = a s + B_t and the A operand
    // (s: four groups of 32 from `get`), then the half's boxes are released
    int st = next_written(dm, dir, 0);
    bool ok = true;
    {
      // start state: its own slot and those of leading unwritten frames; X_0
      const float* start = (dir == 0 && in.fwd_init) ? in.fwd_init : w.half_text;
      const float* src = start + (long long)bh * DD + (long long)row * D;
      const int start_slot = dir == 0 ? 0 : dm.C;
      const Slots sl = slots_of(dm, dir, 0, st);
      const float a = nw > 0 ? __ldg(in.alpha + fh_of(frame_at(dm, dir, st))) : 0.f;
      if (nw > 0) ok = __all_sync(0xffffffffu, mbar_wait_cl(bar(B_CFULL + half), 0, ctl));
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int col = 128 * half + 32 * j;
        float sv[32];
        ld32(src + col, sv);
        store_row32(snap_row + start_slot * DD + col, sv);
        snap32(dm, dir, sl, snap_row, col, sv);
        if (nw > 0 && ok) {
          float cv[32];
          box32(sC, 4 * half + j, srow, cv);
#pragma unroll
          for (int u = 0; u < 32; ++u) cv[u] = fmaf(a, sv[u], cv[u]);
          split_to_tmem(lane_addr, col, cv);
        }
      }
      if (nw > 0 && ok) {
        mbar_arrive_warp(bar(B_CEMPTY + half));
        tmem_wait_st();
        tc_fence_before();
        arrive_cluster_warp(lbar(B_SREADY));
      }
    }
    for (int i = 0; ok && i < nw; ++i) {
      const int st_next = next_written(dm, dir, st + 1);
      const Slots sl = slots_of(dm, dir, st, st_next);
      const bool more = i + 1 < nw;
      const float a = more ? __ldg(in.alpha + fh_of(frame_at(dm, dir, st_next))) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait_cl(bar(B_MDONE), i & 1, ctl))) { ok = false; break; }
      // item i + 1: the next frame's B_t
      if (more && !__all_sync(0xffffffffu, mbar_wait_cl(bar(B_CFULL + half), (i + 1) & 1, ctl))) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int col = 128 * half + 32 * j;
        float v[32];
        tmem_ld32(lane_addr + col, v);
        tmem_wait_ld();
        if (more) {
          float cv[32];
          box32(sC, 4 * half + j, srow, cv);
#pragma unroll
          for (int u = 0; u < 32; ++u) cv[u] = fmaf(a, v[u], cv[u]);  // X = alpha_next S + B_next
          split_to_tmem(lane_addr, col, cv);
        }
        snap32(dm, dir, sl, snap_row, col, v);
      }
      if (more) {
        mbar_arrive_warp(bar(B_CEMPTY + half));
        tmem_wait_st();
      }
      tc_fence_before();  // TMEM reads and writes done before the next product
      if (more) arrive_cluster_warp(lbar(B_SREADY));
      st = st_next;
    }
  }

  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_free2(tmem, s256::kTmem);
}

}  // namespace

bool scan_tc_supported(const Dims& d) {
  // the tensor-core scan steps the joint solve's B form only
  if (d.update != 0) return false;
  if (!scan_tc_layout(d.bf16 != 0, d.dk, d.dv) || !gram_tc_supported(d)) return false;
  if ((long long)d.B * d.T * d.H * 2 * d.dk >= (1LL << 31)) return false;  // TMA row coordinates
  if ((long long)d.B * d.H * 4 > 0x7FFFFFFFLL) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_scan_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s, bool chunks) {
  if (d.dk != D || w.M16 == nullptr || (chunks && w.P16 == nullptr)) return cudaErrorInvalidValue;
  CUtensorMap mm, mc;
  if (chunks) {
    const long long nbch = (long long)d.B * d.C * d.H;
    if (!make_matrix_map(&mm, w.P16, nbch * 2 * D, D, R) || !make_matrix_map_f32(&mc, w.Cf, 2 * nbch * D, D, R))
      return cudaErrorInvalidValue;
  } else {
    const long long fh = (long long)d.B * d.T * d.H;
    if (!make_matrix_map(&mm, w.M16, fh * 2 * D, D, R) || !make_matrix_map_f32(&mc, w.Cm, fh * D, D, R))
      return cudaErrorInvalidValue;
  }
  // one CTA per SM (the two CTAs of a pair sit on two SMs): at least 120 KB
  const size_t need = 1024 + 3 * (size_t)SPLIT + 2 * (size_t)CBYTES + NBARS * 8 + 16;
  const size_t smem = need < 120 * 1024 ? 120 * 1024 : need;
  auto kern = chunks ? k_scan_tc<true> : k_scan_tc<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(2 * d.B * d.H * 2), kThreadsScan, smem, s>>>(d, in, w, mm, mc);  // a CTA pair per chain
  return cudaGetLastError();
}

bool scan256_tc_supported(const Dims& d) {
  if (d.update != 0 || !d.bf16 || d.dk != s256::D || d.dv != s256::D) return false;
  if ((long long)d.B * d.T * d.H * 2 * s256::D >= (1LL << 31)) return false;  // TMA row coordinates
  if ((long long)d.B * d.H * 4 > 0x7FFFFFFFLL) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_scan256_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (!scan256_tc_supported(d) || w.M16 == nullptr) return cudaErrorInvalidValue;
  CUtensorMap mm, mc;
  const long long fh = (long long)d.B * d.T * d.H;
  if (!make_matrix_map(&mm, w.M16, fh * 2 * s256::D, s256::D, s256::R) ||
      !make_matrix_map_f32(&mc, w.Cm, fh * s256::D, s256::D, s256::R))
    return cudaErrorInvalidValue;
  const size_t smem = s256::smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(k_scan256_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_scan256_tc<<<(unsigned)(2 * d.B * d.H * 2), s256::kThreads, smem, s>>>(d, in, w, mm, mc);  // a CTA pair per chain
  return cudaGetLastError();
}

}  // namespace vdn
