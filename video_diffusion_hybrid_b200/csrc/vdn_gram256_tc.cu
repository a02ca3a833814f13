// Per-frame Gram and write matrices of Video Delta Attention at d = 256 on the
// tensor cores, one CTA pair per frame-head (bf16 k / v, fp32 beta and
// accumulation).
//
// What it computes (PaperDaily digest section 四: all tokens of a frame are
// written jointly; deepmagic post "用兩條分支取代一條": A is the weighted key
// Gram matrix and B the value-key write matrix of the closed form):
//   A_t = K^T (beta K),   B_t = V^T (beta K)
// over the frame's N tokens (TEXT: A_x, B_x over batch b's L text tokens),
// into the M_t / C_t slots (the text_gram region) where the solve replaces them.
//
// The pair splits the 256 columns of k and v: CTA r streams columns
// 128 r .. 128 r + 127 of K and V (64-token tiles, two-stage ring) and forms
// its half of beta K as two bf16 terms (hi = bf16(beta k), lo = bf16(beta k -
// hi)), double-buffered so that scaling and products overlap.  The leader
// issues, per 16 tokens, the pair products
//   A += K^T (beta K)_hi + K^T (beta K)_lo,   B += V^T (beta K)_hi + V^T (beta K)_lo
// with M = 256 (each CTA's half of K^T or V^T: its 128 rows of A or B) and N =
// 256 (each CTA's half of beta K), both operands MN-major straight from the
// token-major tiles.  So every k and v element crosses from memory once, and
// each CTA ends with its 128 rows of A_t (TMEM columns 0..255) and of B_t
// (256..511), which its four scaling warps then write out.
//
// Roles (256 threads per CTA):
//   warp 0      TMA producer of this CTA's K and V halves (own barriers).
//   warp 1      TMEM allocator (both CTAs); lane 0 of the leader issues the MMAs.
//   warps 4..7  two threads per token row: this CTA's half of beta K, then the
//               arrival (one per warp) on the leader's barrier, which tells the
//               leader that both the tile and its scaled copy are in place;
//               afterwards the epilogue, TMEM -> rows of A_t and B_t.
#include "tc_common.cuh"

namespace vdn {
namespace {
using namespace tc;

constexpr int D = 256;                // head dim
constexpr int HALF = 128;             // columns of k, v per CTA
constexpr int TT = 64;                // tokens per tile
constexpr int NB = HALF / 64;         // 64-column chunks of a half
constexpr uint32_t TB = TT * HALF * 2;  // one K or V half-tile (bytes)
constexpr uint32_t STAGE = 2 * TB;      // K then V
constexpr int ST = 2;
constexpr int kThreads = 256;
constexpr uint32_t kCols = 512;       // A (0..255) and B (256..511)
// beta K is double-buffered too (slot j & 1 for tile j), so the scaling of
// tile j + 1 runs while the pair's products of tile j do
enum { B_KVFULL = 0, B_KVEMPTY = 2, B_KBFULL = 4, B_KBEMPTY = 6, B_ACC = 8, B_DRAIN = 9, NBARS = 10 };

__device__ __forceinline__ void st_v8(float* p, const float* v) {
  asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
               "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}

template <bool TEXT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_gram256_tc(Dims dm, Inputs in, Work w, const __grid_constant__ CUtensorMap tmk,
             const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sKV = sm;                // ST stages of [K half | V half]
  unsigned char* sKB = sKV + ST * STAGE;  // 2 slots of this CTA's half of beta K: high term, low term
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKB + 2 * 2 * TB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool lead = rank == 0;
  // pair p: heads vary fastest, then frames (TEXT: the batch)
  const long long p = blockIdx.x >> 1;
  const int h = (int)(p % dm.H);
  const int t = TEXT ? 0 : (int)((p / dm.H) % dm.T);
  const int b = TEXT ? (int)(p / dm.H) : (int)(p / ((long long)dm.H * dm.T));
  // both CTAs of a pair take the same decision, before any cluster barrier
  if (!TEXT && is_anchor(dm, t)) return;
  const int col0 = HALF * (int)rank;  // this CTA's columns of k and v, and rows of A and B
  const int ntok = TEXT ? dm.L : dm.N;
  const int ntiles = (ntok + TT - 1) / TT;
  const long long tok0 = TEXT ? (long long)b * dm.L : ((long long)b * dm.T + t) * dm.N;
  const float* betap = TEXT ? in.text_beta : in.beta;
  const long long DD = (long long)D * D;
  float* outA = TEXT ? w.text_gram + ((long long)b * dm.H + h) * 2 * DD : w.M + (((long long)b * dm.T + t) * dm.H + h) * DD;
  float* outB = TEXT ? outA + DD : w.Cm + (((long long)b * dm.T + t) * dm.H + h) * DD;
  const Ctl ctl{abort_flag, w.status, (unsigned)TAG_GRAM_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto lbar = [&](int i) { return map_rank(smem_u32(bars + i), 0); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBARS; ++i)
      mbar_init(bar(i), (i == B_KBFULL || i == B_KBFULL + 1) ? 8 : 1);  // KBFULL: 4 warps x 2 CTAs
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc2(smem_u32(tmem_slot), kCols);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int last[ST] = {-1, -1};
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % ST;
        // stage free: the pair's products of tile j - ST are done (the leader commits to both CTAs)
        if (j >= ST && !mbar_wait_cl(bar(B_KVEMPTY + s), (j / ST - 1) & 1, ctl)) break;
        const int tok = (int)(tok0 + (long long)j * TT);
        mbar_expect_tx(bar(B_KVFULL + s), STAGE);
        for (int c = 0; c < NB; ++c) {
          tma_load_3d(smem_u32(sKV + s * STAGE + c * TT * 128), &tmk, bar(B_KVFULL + s), col0 + c * 64, h, tok);
          tma_load_3d(smem_u32(sKV + s * STAGE + TB + c * TT * 128), &tmv, bar(B_KVFULL + s), col0 + c * 64, h, tok);
        }
        last[s] = j;
      }
      for (int s = 0; s < ST; ++s)
        if (last[s] >= 0) mbar_drain(bar(B_KVFULL + s), (last[s] / ST) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      // MN-major operands: M (or N) = this CTA's 128 columns in 64-wide
      // chunks TT*128 bytes apart, 8-token groups 1024 bytes apart, 16 tokens
      // (2048 bytes) per K-step; M = N = 256 over the pair
      constexpr uint32_t ID = idesc_bf16(2 * HALF, D, true) | (1u << 15);
      const uint64_t kbdesc0 = sdesc(smem_u32(sKB), TT * 128, 1024);
      const uint64_t kvdesc0 = sdesc(smem_u32(sKV), TT * 128, 1024);
      bool ok = true;
      for (int j = 0; ok && j < ntiles; ++j) {
        const int s = j % ST;
        // both CTAs' tiles landed and their halves of beta K written
        const int kb = j & 1;
        if (!mbar_wait_cl(bar(B_KBFULL + kb), (j >> 1) & 1, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t kd = dadd(kvdesc0, s * STAGE), vd = dadd(kd, TB);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint64_t bd = dadd(kbdesc0, (2 * kb + part) * TB);
#pragma unroll
          for (int k = 0; k < TT / 16; ++k) {
            const uint32_t acc = (j | part | k) ? 1u : 0u;
            mma2_bf16(tmem, dadd(kd, k * 2048), dadd(bd, k * 2048), ID, acc);
            mma2_bf16(tmem + D, dadd(vd, k * 2048), dadd(bd, k * 2048), ID, acc);
          }
        }
        commit2(bar(B_KVEMPTY + s));
        commit2(map_rank(bar(B_KVEMPTY + s), 1));
        commit2(bar(B_KBEMPTY + kb));
        commit2(map_rank(bar(B_KBEMPTY + kb), 1));
      }
      if (ok) {
        commit2(bar(B_ACC));
        commit2(map_rank(bar(B_ACC), 1));
      }
      commit2(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int quad = warp - 4;
    const int row = quad * 32 + lane;  // TMEM lane = row of this CTA's share of A and B
    bool ok = true;
    // token row of the tile for the beta K split: two threads per row, each
    // taking half of the row's 16-byte units
    const int srow = row % TT, shalf = row / TT;
    auto beta_of = [&](int j) {
      const int tk = j * TT + srow;
      return tk < ntok ? __ldg(betap + (tok0 + tk) * dm.H + h) : 0.f;
    };
    float beta_next = beta_of(0);
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % ST;
      const float beta = beta_next;
      if (j + 1 < ntiles) beta_next = beta_of(j + 1);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_KVFULL + s), (j / ST) & 1, ctl))) { ok = false; break; }
      // slot j & 1 of the scaled copy: the pair's products of tile j - 2 are done with it
      const int kb = j & 1;
      unsigned char* sHi = sKB + 2 * kb * TB;
      unsigned char* sLo = sHi + TB;
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait_cl(bar(B_KBEMPTY + kb), ((j >> 1) - 1) & 1, ctl))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int uu = 0; uu < NB * 4; ++uu) {
        const int unit = shalf * NB * 4 + uu, c = unit >> 3, q = unit & 7;
        const uint32_t off = c * TT * 128 + srow * 128 + ((q ^ (srow & 7)) << 4);
        const uint4 raw = *reinterpret_cast<const uint4*>(sKV + s * STAGE + off);
        const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t hv[4], lv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = __uint_as_float(u[e] << 16) * beta;
          const float x1 = __uint_as_float(u[e] & 0xFFFF0000u) * beta;
          hv[e] = pack_bf16(x0, x1);
          lv[e] = pack_bf16(x0 - __uint_as_float(hv[e] << 16), x1 - __uint_as_float(hv[e] & 0xFFFF0000u));
        }
        *reinterpret_cast<uint4*>(sHi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(sLo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
      }
      fence_proxy_async_smem();
      arrive_cluster_warp(lbar(B_KBFULL + kb));
    }
    // ---- epilogue: this CTA's rows of A_t and B_t (fp32, row-major)
    if (__all_sync(0xffffffffu, ok && mbar_wait_cl(bar(B_ACC), 0, ctl))) {
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
      float* Ag = outA + (long long)(col0 + row) * D;
      float* Bg = outB + (long long)(col0 + row) * D;
#pragma unroll 1
      for (int q = 0; q < 2 * D / 32; ++q) {
        float v[32];
        tmem_ld32(lane_addr + q * 32, v);
        tmem_wait_ld();
        float* dst = q < D / 32 ? Ag + q * 32 : Bg + (q - D / 32) * 32;
#pragma unroll
        for (int i = 0; i < 32; i += 8) st_v8(dst + i, v + i);
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory or barriers
  tc_fence_after();
  if (warp == 1) tmem_free2(tmem, kCols);
}

template <bool TEXT>
cudaError_t launch(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  CUtensorMap mk, mv;
  const long long tokens = TEXT ? (long long)d.B * d.L : (long long)d.B * d.T * d.N;
  if (!make_token_map(&mk, TEXT ? in.text_k : in.k, tokens, d.H, D, TT) ||
      !make_token_map(&mv, TEXT ? in.text_v : in.v, tokens, d.H, D, TT))
    return cudaErrorInvalidValue;
  // one CTA per SM (the 512 TMEM columns; the two CTAs of a pair on two SMs)
  const size_t need = 1024 + ST * (size_t)STAGE + 4 * (size_t)TB + NBARS * 8 + 16;
  const size_t smem = need < 120 * 1024 ? 120 * 1024 : need;
  auto kern = k_gram256_tc<TEXT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long pairs = (long long)d.B * d.H * (TEXT ? 1 : d.T);
  if (pairs <= 0 || 2 * pairs > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)(2 * pairs), kThreads, smem, s>>>(d, in, w, mk, mv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gram256_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s, bool text) {
  if (d.dk != D || d.dv != D) return cudaErrorInvalidValue;
  if (text && (d.L <= 0 || (long long)d.B * d.L >= (1LL << 31))) return cudaErrorInvalidValue;
  return text ? launch<true>(d, in, w, s) : launch<false>(d, in, w, s);
}

}  // namespace vdn
