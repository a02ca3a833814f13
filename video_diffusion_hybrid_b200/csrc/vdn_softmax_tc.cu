// Windowed + anchor softmax on the 5th-generation tensor cores (tcgen05),
// bf16 q/k/v, fp32 scores, softmax and accumulation.
//
// What it computes (PaperDaily digest section 二; deepmagic post
// "用兩條分支取代一條"; aimodeling news "The VDN split"): for a query in chunk
// c the keys of chunks c-1..c+1 (clipped) plus the two anchor frames; anchor
// query frames attend to every frame; y_sm = sigmoid(g_sm) * softmax(s q K^T) V.
//
// One CTA = two tiles of 128 query rows (256 rows) of one (batch, head, query
// group); a query group is the non-anchor frames of one chunk, or one anchor
// frame, so every row has the same key set: at most three contiguous token
// intervals (anchor frame 0, the window, anchor frame T-1).  Both query tiles
// share every K / V tile.
//
// Roles (384 threads):
//   warp 0      TMA producer of Q (both tiles, once) and of the K ring (three
//               stages, freed after both S_0 and S_1 of that tile).
//   warp 2      TMA producer of the V ring (two stages, freed after both PVs).
//   warp 1      TMEM allocator; lane 0 issues every tcgen05.mma.  Per key tile
//               j the tensor pipe runs, in this order,
//                 O_0 += P_0(j) V_j,  S_0 = Q_0 K_{j+1}^T,  O_1 += P_1(j) V_j,  S_1 = Q_1 K_{j+1}^T
//               where each P V is issued as two 64-key halves, the first as
//               soon as the softmax has stored that half of P (it then runs
//               while the softmax computes the second half)
//               so that while one softmax warpgroup works on its tile the pipe
//               computes the other tile's product (ping-pong).  S: M=128, N=128,
//               K=d, both operands from SMEM; PV: A = P from TMEM (TS form).
//   warps 4..7  softmax of query tile 0, warps 8..11 of query tile 1: thread r
//               owns row r (= TMEM lane r), a key tile in two halves of 64
//               keys.  A full half after the first key tile takes one pass:
//               P = 2^(s c - m c) with the running max m, kept when the half's
//               sum of P is at most 2^8 (then no weight exceeds 2^8).
//               Otherwise, and in the first and partial tiles, two passes over
//               the half: its max, then P.  O is rescaled only when a row max
//               grew by more than 8 in exp2 units (exact: p <= 2^8 then, and O
//               and the row sum share the same stale max).  The row sum adds
//               the bf16-rounded P (mixed bf16 + fp32 adds), so every output
//               row is an exact convex combination of V rows.  Epilogue:
//               O / l, gate, store.
//
// TMEM (512 columns): O_0 [0,128), O_1 [128,256), S_0 [256,384), S_1 [384,512);
// P_t lives in the first 64 columns of S_t (keys 0..63 in the first 32).  A
// tile's next S is issued after its PV by the same thread, and tcgen05.mma operations of one thread run in
// issue order, so P_t(j) is consumed before S_t(j+1) overwrites it.
//
// Every mbarrier wait is bounded (about one second of clock cycles); on
// expiry the CTA records VDN_ERR_TIMEOUT in the workspace status words, stops
// issuing, drains its own copies and MMAs and frees its TMEM.
#include "tc_common.cuh"

namespace vdn {
namespace {
using namespace tc;

constexpr int BM = 128;           // query rows per tile
constexpr int NQ = 2;             // query tiles per CTA
constexpr int BN = 128;           // keys per tile
constexpr int kThreadsTC = 384;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

__host__ __device__ constexpr uint32_t col_o(int t) { return 128u * t; }
__host__ __device__ constexpr uint32_t col_s(int t) { return 256u + 128u * t; }

// ------------------------------------------------------ work decomposition --
struct Tile {
  int b, h, q0, qrows;      // absolute first query token, valid rows (of 256)
  int niv;                  // key interval slots (always 3; unused ones empty)
  int kbeg[3], klen[3];     // absolute first key token, length
};

__host__ __device__ inline void group_frames(const Dims& d, int g, int& f0, int& f1, int& ridx) {
  if (g < d.C) {
    f0 = g * d.chunk;
    f1 = f0 + d.chunk < d.T ? f0 + d.chunk : d.T;
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

__host__ __device__ inline long long pairs_of_rows(long long rows) { return (rows + NQ * BM - 1) / (NQ * BM); }

// Text cross-attention: item -> 256 query rows of one (b, h) over all T*N
// video tokens; one key interval, the L text tokens of batch b.
__device__ bool decode_item_cross(const Dims& d, long long item, Tile& t) {
  const long long rows = (long long)d.T * d.N;
  const long long per_bh = pairs_of_rows(rows);
  const long long bh = item / per_bh, qp = item % per_bh;
  if (bh >= (long long)d.B * d.H) return false;
  t.b = (int)(bh / d.H);
  t.h = (int)(bh % d.H);
  t.q0 = (int)((long long)t.b * rows + qp * NQ * BM);
  t.qrows = (int)min((long long)NQ * BM, rows - qp * NQ * BM);
  t.niv = 3;
  t.kbeg[0] = t.b * d.L; t.klen[0] = d.L;
  t.kbeg[1] = 0; t.klen[1] = 0;
  t.kbeg[2] = 0; t.klen[2] = 0;
  return true;
}

// Item order: all anchor-row pairs first (longest), then per (b, h) the
// regular groups in chunk order, so concurrent CTAs share K/V windows in L2.
__device__ bool decode_item(const Dims& d, long long item, Tile& t) {
  const int n_anc = d.anchors ? 2 : 0;
  const long long pairs_a = pairs_of_rows(d.N);
  const long long anc_items = (long long)d.B * d.H * n_anc * pairs_a;
  int g;
  long long bh, qp;
  if (item < anc_items) {
    bh = item / (n_anc * pairs_a);
    const long long r = item % (n_anc * pairs_a);
    g = d.C + (int)(r / pairs_a);
    qp = r % pairs_a;
  } else {
    const long long it = item - anc_items;
    long long per_bh = 0;
    for (int gg = 0; gg < d.C; ++gg) {
      int f0, f1, ri;
      group_frames(d, gg, f0, f1, ri);
      if (f1 > f0) per_bh += pairs_of_rows((long long)(f1 - f0) * d.N);
    }
    if (per_bh == 0) return false;
    bh = it / per_bh;
    long long rem = it % per_bh;
    g = -1;
    qp = 0;
    for (int gg = 0; gg < d.C; ++gg) {
      int f0, f1, ri;
      group_frames(d, gg, f0, f1, ri);
      if (f1 <= f0) continue;
      const long long np = pairs_of_rows((long long)(f1 - f0) * d.N);
      if (rem < np) { g = gg; qp = rem; break; }
      rem -= np;
    }
    if (g < 0) return false;
  }
  if (bh >= (long long)d.B * d.H) return false;
  t.b = (int)(bh / d.H);
  t.h = (int)(bh % d.H);
  int f0, f1, ridx;
  group_frames(d, g, f0, f1, ridx);
  if (f1 <= f0) return false;
  const int base = t.b * d.T * d.N;
  const int rows = (f1 - f0) * d.N;
  t.q0 = base + f0 * d.N + (int)qp * NQ * BM;
  t.qrows = min(NQ * BM, rows - (int)qp * NQ * BM);
  // three fixed interval slots (static indices keep the tile in registers);
  // an unused slot has length 0 and holds no key tile
  t.niv = 3;
  if (ridx == d.C) {
    t.kbeg[0] = base; t.klen[0] = d.T * d.N;
    t.kbeg[1] = base; t.klen[1] = 0;
    t.kbeg[2] = base; t.klen[2] = 0;
  } else {
    const int lo = max(0, (ridx - 1) * d.chunk), hi = min(d.T, (ridx + 2) * d.chunk);
    t.kbeg[0] = base; t.klen[0] = (d.anchors && lo > 0) ? d.N : 0;
    t.kbeg[1] = base + lo * d.N; t.klen[1] = (hi - lo) * d.N;
    t.kbeg[2] = base + (d.T - 1) * d.N; t.klen[2] = (d.anchors && hi < d.T) ? d.N : 0;
  }
  return true;
}

__device__ __forceinline__ int num_key_tiles(const Tile& t) {
  int n = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) n += (t.klen[i] + BN - 1) / BN;
  return n;
}

// Key tile j -> (first key token, valid keys).
__device__ __forceinline__ void key_tile(const Tile& t, int j, int& k0, int& kvalid) {
  // fixed trip count and static indices: the tile stays in registers
  k0 = 0;
  kvalid = 0;
  bool found = false;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int nt = (t.klen[i] + BN - 1) / BN;
    if (!found) {
      if (j < nt) {
        k0 = t.kbeg[i] + j * BN;
        kvalid = min(BN, t.klen[i] - j * BN);
        found = true;
      } else {
        j -= nt;
      }
    }
  }
}

// sigmoid from the exponential and an approximate reciprocal (a few ulp;
// exp(-x) overflowing to inf gives 0, the limit)
__device__ __forceinline__ float sigm(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + __expf(-x)));
  return r;
}

template <typename To> __device__ __forceinline__ void store4(To* p, float a, float b, float c, float d);
template <> __device__ __forceinline__ void store4<float>(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float a, float b, float c,
                                                                   float d) {
  uint2 u;
  u.x = pack_bf16(a, b);
  u.y = pack_bf16(c, d);
  *reinterpret_cast<uint2*>(p) = u;
}

// lo and hi halves of a packed bf16 pair added exactly into two fp32 sums
__device__ __forceinline__ void add_bf16x2_f32(float& s_lo, float& s_hi, uint32_t u) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tadd.rn.f32.bf16 %0, lo, %0;\n\t"
      "add.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(s_lo), "+f"(s_hi)
      : "r"(u));
}

// ------------------------------------------------------------------ kernel --
// X: the text cross-attention (keys and values from the text tokens, every
// query sees all of its batch's L text tokens, no gate, y[B,T,N,H,d_v]).
template <int D, typename To, bool X>
__global__ void __launch_bounds__(kThreadsTC, 1)
k_softmax_tc(Dims dm, Inputs in, Work w, const __grid_constant__ CUtensorMap tmq,
             const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  constexpr int NB = D / 64;                 // 64-wide column blocks of a row
  constexpr uint32_t QTILE = BM * D * 2;
  constexpr uint32_t KVBYTES = BN * D * 2;
  constexpr int KST = 3, VST = 2;            // K and V ring depths
  // P_t of a key tile is handed over in two 64-key halves: B_PFULL (keys
  // 0..63) and B_PFULL2 (64..127); B_OHALF marks O += P_t(j)[:, :64] V_j done
  enum { B_Q = 0, B_KFULL = 1, B_KEMPTY = 4, B_VFULL = 7, B_VEMPTY = 9, B_SFULL = 11, B_PFULL = 13, B_ODONE = 15,
         B_DRAIN = 17, B_PFULL2 = 18, B_OHALF = 20, NBARS = 22 };
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = sm;                    // NQ tiles
  unsigned char* sK = sQ + NQ * QTILE;       // KST stages
  unsigned char* sV = sK + KST * KVBYTES;    // VST stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VST * KVBYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a CTA of this launch already gave up on a wait: fail fast, touch nothing
  if (*reinterpret_cast<volatile uint32_t*>(w.status) != 0u) return;
  Tile tile;
  if (!(X ? decode_item_cross(dm, blockIdx.x, tile) : decode_item(dm, blockIdx.x, tile))) return;  // uniform
  const int ntiles = num_key_tiles(tile);
  const Ctl ctl{abort_flag, w.status, (unsigned)TAG_SOFTMAX_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };

  if (threadIdx.x == 0) {
    // P_FULL: one arrival per softmax warp
    for (int i = 0; i < NBARS; ++i)
      mbar_init(bar(i), (i == B_PFULL || i == B_PFULL + 1 || i == B_PFULL2 || i == B_PFULL2 + 1) ? 4 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ Q and K producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmq)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
      mbar_expect_tx(bar(B_Q), NQ * QTILE);
      for (int t = 0; t < NQ; ++t)
        for (int c = 0; c < NB; ++c)
          tma_load_3d(smem_u32(sQ + t * QTILE + c * BM * 128), &tmq, bar(B_Q), c * 64, tile.h, tile.q0 + t * BM);
      int nk = 0;  // K tiles issued
      for (int j = 0; j < ntiles; ++j) {
        int k0, kv;
        key_tile(tile, j, k0, kv);
        const int sk = j % KST;
        if (j >= KST && !mbar_wait(bar(B_KEMPTY + sk), (j / KST - 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_KFULL + sk), KVBYTES);
        for (int c = 0; c < NB; ++c)
          tma_load_3d(smem_u32(sK + sk * KVBYTES + c * BN * 128), &tmk, bar(B_KFULL + sk), c * 64, tile.h, k0);
        nk = j + 1;
      }
      // drain: every copy issued into this CTA's shared memory has landed
      // (the last tile issued into each stage is one of the last KST)
      mbar_drain(bar(B_Q), 0);
      for (int jj = nk - KST < 0 ? 0 : nk - KST; jj < nk; ++jj)
        mbar_drain(bar(B_KFULL + jj % KST), (jj / KST) & 1);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
      int nv = 0;  // V tiles issued
      for (int j = 0; j < ntiles; ++j) {
        int k0, kv;
        key_tile(tile, j, k0, kv);
        const int sv = j % VST;
        if (j >= VST && !mbar_wait(bar(B_VEMPTY + sv), (j / VST - 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_VFULL + sv), KVBYTES);
        for (int c = 0; c < NB; ++c)
          tma_load_3d(smem_u32(sV + sv * KVBYTES + c * BN * 128), &tmv, bar(B_VFULL + sv), c * 64, tile.h, k0);
        nv = j + 1;
      }
      for (int jj = nv - VST < 0 ? 0 : nv - VST; jj < nv; ++jj)
        mbar_drain(bar(B_VFULL + jj % VST), (jj / VST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(BM, BN, false);
      constexpr uint32_t ID_O = idesc_bf16(BM, D, true);
      // descriptors built once; each k-step adds a compile-time offset
      const uint64_t qdesc[NQ] = {sdesc(smem_u32(sQ), 16, 1024), sdesc(smem_u32(sQ + QTILE), 16, 1024)};
      const uint64_t kdesc0 = sdesc(smem_u32(sK), 16, 1024);
      const uint64_t vdesc0 = sdesc(smem_u32(sV), BN * 128, 1024);
      // S_t = Q_t K_j^T and O_t += P_t(j) V_j, issued once the barriers they
      // need have been cleared (waits first, then the MMAs back to back).
      auto mma_s = [&](int t, int j) {
        const int sk = j % KST;
        const uint64_t qd = t == 0 ? qdesc[0] : qdesc[1], kd = dadd(kdesc0, sk * KVBYTES);
        const uint32_t dst = tmem + col_s(t);
        mma_bf16(dst, qd, kd, ID_S, 0u);
#pragma unroll
        for (int k = 1; k < D / 16; ++k)
          mma_bf16(dst, dadd(qd, (k >> 2) * (BM * 128) + (k & 3) * 32), dadd(kd, (k >> 2) * (BN * 128) + (k & 3) * 32),
                   ID_S, 1u);
        mma_commit(bar(B_SFULL + t));
        if (t == NQ - 1) mma_commit(bar(B_KEMPTY + sk));  // K_j read by both tiles
      };
      // O_t += P_t(j)[:, 64 h : 64 h + 64] V_j[64 h : 64 h + 64, :]
      auto mma_pv = [&](int t, int j, int h) {
        const int sv = j % VST;
        const uint64_t vd = dadd(vdesc0, sv * KVBYTES);
        const uint32_t dst = tmem + col_o(t), pa = tmem + col_s(t);
#pragma unroll
        for (int k = 4 * h; k < 4 * h + 4; ++k)
          mma_bf16_ts(dst, pa + 8 * k, dadd(vd, k * 16 * 128), ID_O, (j > 0 || k > 0) ? 1u : 0u);
        if (h == 0) {
          mma_commit(bar(B_OHALF + t));
        } else {
          mma_commit(bar(B_ODONE + t));
          if (t == NQ - 1) mma_commit(bar(B_VEMPTY + sv));  // V_j read by both tiles
        }
      };
      bool ok = mbar_wait(bar(B_Q), 0, ctl) && mbar_wait(bar(B_KFULL), 0, ctl);
      if (ok) {
        tc_fence_after();
        mma_s(0, 0);
        mma_s(1, 0);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const bool more = j + 1 < ntiles;
        for (int t = 0; ok && t < NQ; ++t) {
          ok = mbar_wait(bar(B_PFULL + t), j & 1, ctl) &&
               (t > 0 || mbar_wait(bar(B_VFULL + j % VST), (j / VST) & 1, ctl));
          if (!ok) break;
          tc_fence_after();
          mma_pv(t, j, 0);
          ok = mbar_wait(bar(B_PFULL2 + t), j & 1, ctl) &&
               (t > 0 || !more || mbar_wait(bar(B_KFULL + (j + 1) % KST), ((j + 1) / KST) & 1, ctl));
          if (!ok) break;
          tc_fence_after();
          mma_pv(t, j, 1);
          if (more) mma_s(t, j + 1);
        }
      }
      // drain: completion of every MMA issued by this thread
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;          // query tile of this warpgroup
    const int quad = warp & 3;              // TMEM lane quadrant
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t scol = lane_addr + col_s(t), ocol = lane_addr + col_o(t);
    const float c = dm.scale * 1.4426950408889634f;  // log2 units
    const float thresh = kRescaleLog2 / c;            // raw-score units
    float m_used = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < ntiles; ++j) {
      // every TMEM access below is warp-collective: keep control flow warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + t), j & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      int k0, kvalid;
      key_tile(tile, j, k0, kvalid);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t sh = scol + 64 * h;  // scores of keys [64 h, 64 h + 64)
        const int kvh = kvalid - 64 * h;    // valid keys of this half (may be <= 0)
        bool done = false;
        // Fast path (a full half after the first key tile): one pass with the
        // running max, kept when the half's sum of P is at most 2^8 (a rounded
        // sum of non-negative terms bounds each term, so no weight exceeds 2^8).
        if (j > 0 && kvh >= 64) {
          const float2 c2 = make_float2(c, c), nmc2 = make_float2(-m_used * c, -m_used * c);
          float ps[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) ps[u] = 0.f;
          float pk[32];
          auto chunk = [&](const float (&v)[32], int o) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 x = fma2(make_float2(v[2 * i], v[2 * i + 1]), c2, nmc2);
              const uint32_t u = pack_bf16(ex2(x.x), ex2(x.y));
              add_bf16x2_f32(ps[2 * (i & 3)], ps[2 * (i & 3) + 1], u);
              pk[o + i] = __uint_as_float(u);
            }
          };
          float va[32], vb[32];
          tmem_ld32(sh, va);
          tmem_wait_ld();
          tmem_ld32(sh + 32, vb);
          chunk(va, 0);
          tmem_wait_ld();
          chunk(vb, 16);
          const float psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
          if (!__any_sync(0xffffffffu, !(psum <= 256.0f))) {
            tmem_st32(scol + 32 * h, pk);  // P columns [32 h, 32 h + 32): keys of this half
            l_sum += psum;
            done = true;
          }
        }
        if (!done) {
          // Exact path on the half: its max, O rescaled if the row max grew by
          // more than 8 (exp2 units), then P.
          float v0[32], v1[32];
          tmem_ld32(sh, v0);
          tmem_ld32(sh + 32, v1);
          tmem_wait_ld();
          float pm[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            pm[i & 7] = fmaxf(pm[i & 7], i < kvh ? v0[i] : -INFINITY);
            pm[i & 7] = fmaxf(pm[i & 7], 32 + i < kvh ? v1[i] : -INFINITY);
          }
          const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                 fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
          const bool need = mx > m_used + thresh;
          float f = 1.0f;
          if (need) {
            f = (m_used == -INFINITY) ? 0.f : ex2((m_used - mx) * c);
            l_sum *= f;
            m_used = mx;
          }
          // O holds products already issued: those of key tile j - 1 (h = 0) or
          // the first half of tile j (h = 1); rescale once they are complete
          if ((j > 0 || h == 1) && __any_sync(0xffffffffu, need)) {
            const bool st = h == 0 ? mbar_wait(bar(B_ODONE + t), (j - 1) & 1, ctl)
                                   : mbar_wait(bar(B_OHALF + t), j & 1, ctl);
            if (!__all_sync(0xffffffffu, st)) { ok = false; break; }
            tc_fence_after();
            float v[32];
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
              tmem_ld32(ocol + q * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= f;
              tmem_st32(ocol + q * 32, v);
            }
            tmem_wait_st();
          }
          const float mc = m_used * c;
          float ps[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) ps[u] = 0.f;
          float pk[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = 2 * i < kvh ? ex2(fmaf(v0[2 * i], c, -mc)) : 0.f;
            const float p1 = 2 * i + 1 < kvh ? ex2(fmaf(v0[2 * i + 1], c, -mc)) : 0.f;
            const uint32_t u = pack_bf16(p0, p1);
            add_bf16x2_f32(ps[2 * (i & 3)], ps[2 * (i & 3) + 1], u);
            pk[i] = __uint_as_float(u);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = 32 + 2 * i < kvh ? ex2(fmaf(v1[2 * i], c, -mc)) : 0.f;
            const float p1 = 32 + 2 * i + 1 < kvh ? ex2(fmaf(v1[2 * i + 1], c, -mc)) : 0.f;
            const uint32_t u = pack_bf16(p0, p1);
            add_bf16x2_f32(ps[2 * (i & 3)], ps[2 * (i & 3) + 1], u);
            pk[16 + i] = __uint_as_float(u);
          }
          tmem_st32(scol + 32 * h, pk);
          l_sum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(bar(h == 0 ? B_PFULL + t : B_PFULL2 + t));
      }
    }
    // ---- epilogue: O / l, gate, store
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar(B_ODONE + t), (ntiles - 1) & 1, ctl))) {
      tc_fence_after();
      const float inv = 1.0f / l_sum;
      const int trow = t * BM + row;
      const bool valid = trow < tile.qrows;
      const long long tok = (long long)tile.q0 + trow;
      const long long gi = (tok * dm.H + tile.h) * D;
      // the row's log-sum-exp, natural log (l_sum counts the row max at
      // weight 2^(m - m_used) >= 1, so this bounds every scaled score)
      if (!X && in.sm_lse != nullptr && valid)
        in.sm_lse[tok * dm.H + tile.h] = (m_used * c + __log2f(l_sum)) * 0.6931471805599453f;
      To* y = static_cast<To*>(in.y) + ((!X && dm.out_mode == 0) ? 2 * gi : gi);
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        float v[32];
        tmem_ld32(ocol + q * 32, v);
        tmem_wait_ld();
        if (valid && X) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            store4<To>(y + q * 32 + i, v[i] * inv, v[i + 1] * inv, v[i + 2] * inv, v[i + 3] * inv);
        } else if (valid) {
          float g[32];
          if (dm.bf16) {
            const uint4* gp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(in.gate_sm) + gi + q * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 raw = __ldg(gp + u);
              const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float2 f2 = __bfloat1622float2(h2[e]);
                g[u * 8 + 2 * e] = f2.x;
                g[u * 8 + 2 * e + 1] = f2.y;
              }
            }
          } else {
            const float4* gp = reinterpret_cast<const float4*>(static_cast<const float*>(in.gate_sm) + gi + q * 32);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              float4 f4 = __ldg(gp + u);
              g[4 * u] = f4.x; g[4 * u + 1] = f4.y; g[4 * u + 2] = f4.z; g[4 * u + 3] = f4.w;
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            store4<To>(y + q * 32 + i, sigm(g[i]) * v[i] * inv, sigm(g[i + 1]) * v[i + 1] * inv,
                       sigm(g[i + 2]) * v[i + 2] * inv, sigm(g[i + 3]) * v[i + 3] * inv);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, kTmemCols);
}

// ------------------------------------------------------------------- host --
long long num_items(const Dims& d) {
  const int n_anc = d.anchors ? 2 : 0;
  long long per_bh = 0;
  for (int g = 0; g < d.C; ++g) {
    int f0, f1, ri;
    group_frames(d, g, f0, f1, ri);
    if (f1 > f0) per_bh += pairs_of_rows((long long)(f1 - f0) * d.N);
  }
  return (long long)d.B * d.H * (per_bh + n_anc * pairs_of_rows(d.N));
}

template <int D, typename To, bool X>
cudaError_t launch_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const long long tokens = (long long)d.B * d.T * d.N;
  const long long ktok = X ? (long long)d.B * d.L : tokens;  // key / value tokens
  if (!make_token_map(&mq, in.q, tokens, d.H, D, BM) ||
      !make_token_map(&mk, X ? in.text_k : in.k, ktok, d.H, D, BN) ||
      !make_token_map(&mv, X ? in.text_v : in.v, ktok, d.H, D, BN))
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + (size_t)NQ * BM * D * 2 + 5 * (size_t)BN * D * 2 + 22 * 8 + 16;
  auto kern = k_softmax_tc<D, To, X>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long items = X ? (long long)d.B * d.H * pairs_of_rows((long long)d.T * d.N) : num_items(d);
  if (items <= 0 || items > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)items, kThreadsTC, smem, s>>>(d, in, w, mq, mk, mv);
  return cudaGetLastError();
}

}  // namespace

bool softmax_tc_supported(const Dims& d) {
  if (!d.bf16 || d.dk != d.dv) return false;
  if (d.dk != 64 && d.dk != 128) return false;
  // token indices of the TMA coordinates are int32 (plus one tile of overhang)
  if ((long long)d.B * d.T * d.N + NQ * BM >= (1LL << 31)) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_softmax_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (d.dk == 128)
    return d.out_bf16 ? launch_tc<128, __nv_bfloat16, false>(d, in, w, s) : launch_tc<128, float, false>(d, in, w, s);
  if (d.dk == 64)
    return d.out_bf16 ? launch_tc<64, __nv_bfloat16, false>(d, in, w, s) : launch_tc<64, float, false>(d, in, w, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_text_xattn_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (d.L <= 0 || (long long)d.B * d.L + NQ * BM >= (1LL << 31)) return cudaErrorInvalidValue;
  if (d.dk == 128)
    return d.out_bf16 ? launch_tc<128, __nv_bfloat16, true>(d, in, w, s) : launch_tc<128, float, true>(d, in, w, s);
  if (d.dk == 64)
    return d.out_bf16 ? launch_tc<64, __nv_bfloat16, true>(d, in, w, s) : launch_tc<64, float, true>(d, in, w, s);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
