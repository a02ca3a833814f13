// Per-token gradients of the frame write on the tensor cores (tcgen05), the
// last step of the linear branch's backward for bf16 k and v.
//
// The frame write (PaperDaily digest section 四; deepmagic post, closed form)
// forms A_t = sum_i beta_i k_i k_i^T and B_t = sum_i beta_i v_i k_i^T; given
// their gradients, dA_t (taken symmetrised, dA + dA^T) and dB_t, each token
// of the frame gets
//   dk = beta ((dA + dA^T) k + dB^T v),  dv = beta dB k,
//   dbeta = k^T dA k + v^T dB k = 1/2 <k, (dA + dA^T) k> + <v, dB k>.
// Over a 128-token tile with K, V [128 x d] (rows = tokens):
//   P1 = K (dA + dA^T),  P2 = V dB,  P3 = K dB^T
//   dk = beta (P1 + P2),  dv = beta P3,  dbeta = sum_j (1/2 K P1 + V P3).
//
// One CTA per (frame, head, 64 output columns); the frame's tokens in tiles
// of 128 through a two-stage TMA ring.  The fp32 matrices enter as bf16 hi +
// lo pairs (about 16 significant bits; k and v are exact in bf16), so each
// product is two MMAs with fp32 accumulation.  The B operands, written once by
// the epilogue warps in the 128-byte swizzled layout:
//   (dA + dA^T) rows j of the CTA's columns, K-major (the matrix is symmetric);
//   dB rows j, K-major, for P3 = K dB^T;
//   dB columns j over all rows, MN-major, for P2 = V dB.
// Roles (256 threads): warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer, warps 4..7 the B operands and then the epilogue (thread = token row
// = TMEM lane), with the accumulators double-buffered across tiles.  dbeta
// collects one partial per column block by atomic adds (two terms for d = 128:
// the sum does not depend on their order).  Every mbarrier wait is bounded.
#include "tc_common.cuh"

namespace vdn {
namespace {
using namespace tc;

constexpr int TT = 128;  // tokens per tile
constexpr int CW = 64;   // output columns per CTA
constexpr int kThrT = 256;
constexpr int STT = 2;   // K / V ring stages

// byte offset of element (r, c) in a 128-byte swizzled tile whose rows are
// `rows` long blocks of 64 bf16 columns
__device__ __forceinline__ uint32_t swz(int r, int c, int rows) {
  return (uint32_t)((c >> 6) * rows * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}

template <int D>
__global__ void __launch_bounds__(kThrT, 1)
k_bwd_tokens_tc(Dims dm, Inputs in, const float* __restrict__ dAs, const float* __restrict__ dB, float* dk, float* dv,
                float* dbeta, uint32_t* status, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv) {
  constexpr int NB = D / 64;
  constexpr uint32_t TILE = TT * D * 2;  // one K or V tile
  constexpr uint32_t BOP = CW * D * 2;   // one B operand (64 x d, either major)
  enum { B_FULL = 0, B_EMPTY = STT, B_BREADY = 2 * STT, B_ACC = 2 * STT + 1, B_TFREE = B_ACC + 2, B_DRAIN = B_TFREE + 2,
         NBARS };
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sKV = sm;                   // STT stages of [K | V]
  unsigned char* sB = sKV + STT * 2 * TILE;  // [dAs hi, lo][dB (K-major) hi, lo][dB (MN-major) hi, lo]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + 6 * BOP);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = blockIdx.x % (D / CW), t = blockIdx.x / (D / CW), h = blockIdx.y, b = blockIdx.z;
  const int N = dm.N, H = dm.H;
  const long long fh = ((long long)b * dm.T + t) * H + h, tok0 = ((long long)b * dm.T + t) * N;
  if (is_anchor(dm, t)) {  // not written: zero dk, dv (dbeta is cleared by the launcher);
                           // left as they are when adding to the softmax branch's share
    for (long long e = threadIdx.x; !dm.grad_acc && e < (long long)N * (CW / 4); e += kThrT) {
      const long long g = ((tok0 + e / (CW / 4)) * H + h) * D + cb * CW + (e % (CW / 4)) * 4;
      *reinterpret_cast<float4*>(dk + g) = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(dv + g) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  if (*reinterpret_cast<volatile uint32_t*>(status) != 0u) return;
  const int ntiles = (N + TT - 1) / TT;
  const Ctl ctl{abort_flag, status, (unsigned)TAG_LINBWD_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };

  if (threadIdx.x == 0) {
    // EMPTY: the MMA commit plus the epilogue warps (they read K and V too)
    for (int i = 0; i < NBARS; ++i)
      mbar_init(bar(i), (i == B_EMPTY || i == B_EMPTY + 1) ? 5 : (i == B_BREADY || i == B_TFREE || i == B_TFREE + 1) ? 4 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % STT;
        if (j >= STT && !mbar_wait(bar(B_EMPTY + st), (j / STT - 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_FULL + st), 2 * TILE);
        const int row = (int)(tok0 + (long long)j * TT);
        for (int c = 0; c < NB; ++c) {
          tma_load_3d(smem_u32(sKV + st * 2 * TILE + c * TT * 128), &tmk, bar(B_FULL + st), c * 64, h, row);
          tma_load_3d(smem_u32(sKV + st * 2 * TILE + TILE + c * TT * 128), &tmv, bar(B_FULL + st), c * 64, h, row);
        }
        issued = j + 1;
      }
      for (int j = issued - STT < 0 ? 0 : issued - STT; j < issued; ++j)
        mbar_drain(bar(B_FULL + j % STT), (j / STT) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID_K = idesc_bf16(TT, CW, false), ID_M = idesc_bf16(TT, CW, true);
      const uint64_t kv0 = sdesc(smem_u32(sKV), 16, 1024);
      uint64_t bk[4], bm[2];
      for (int p = 0; p < 4; ++p) bk[p] = sdesc(smem_u32(sB + p * BOP), 16, 1024);       // dAs hi, lo, dB hi, lo
      for (int p = 0; p < 2; ++p) bm[p] = sdesc(smem_u32(sB + (4 + p) * BOP), CW * 128, 1024);
      bool ok = mbar_wait(bar(B_BREADY), 0, ctl);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % STT, buf = j & 1;
        ok = mbar_wait(bar(B_FULL + st), (j / STT) & 1, ctl) &&
             (j < 2 || mbar_wait(bar(B_TFREE + buf), ((j >> 1) - 1) & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc0 = tmem + 256u * buf;  // P1, P2, P3 at +0, +64, +128
        const uint64_t kd = dadd(kv0, st * 2 * TILE), vd = dadd(kd, TILE);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t aoff = (k >> 2) * (TT * 128) + (k & 3) * 32;
            const uint32_t boff = (k >> 2) * (CW * 128) + (k & 3) * 32;
            const uint32_t acc = (part | k) ? 1u : 0u;
            mma_bf16(acc0, dadd(kd, aoff), dadd(bk[part], boff), ID_K, acc);                // K (dA + dA^T)
            mma_bf16(acc0 + 64, dadd(vd, aoff), dadd(bm[part], k * 2048), ID_M, acc);     // V dB
            mma_bf16(acc0 + 128, dadd(kd, aoff), dadd(bk[2 + part], boff), ID_K, acc);    // K dB^T
          }
        }
        mma_commit(bar(B_ACC + buf));
        mma_commit(bar(B_EMPTY + st));
      }
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int tid = threadIdx.x - 128, quad = warp - 4, row = quad * 32 + lane;
    // ---- B operands: fp32 -> bf16 hi + lo, 128-byte swizzled, one 16-byte unit
    // (8 elements) at a time
    const float* A = dAs + fh * D * D;
    const float* Bm = dB + fh * D * D;
    for (int u = tid; u < CW * D / 8; u += 128) {
      const int r = u / (D / 8), c = (u % (D / 8)) * 8;  // K-major: row r = output column j, columns c..c+7 = i
      const int j = cb * CW + r;
      const float* srcs[2] = {A + (long long)j * D + c, Bm + (long long)j * D + c};
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const float4 x0 = __ldg(reinterpret_cast<const float4*>(srcs[m]));
        const float4 x1 = __ldg(reinterpret_cast<const float4*>(srcs[m]) + 1);
        const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        uint32_t hv[4], lv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hv[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
          lv[e] = pack_bf16(x[2 * e] - __uint_as_float(hv[e] << 16), x[2 * e + 1] - __uint_as_float(hv[e] & 0xFFFF0000u));
        }
        const uint32_t off = swz(r, c, CW);
        *reinterpret_cast<uint4*>(sB + (2 * m) * BOP + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(sB + (2 * m + 1) * BOP + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
      }
    }
    for (int u = tid; u < D * CW / 8; u += 128) {
      const int i = u / (CW / 8), c = (u % (CW / 8)) * 8;  // MN-major: row i of dB, columns j = cb * CW + c..c+7
      const float* src = Bm + (long long)i * D + cb * CW + c;
      const float4 x0 = __ldg(reinterpret_cast<const float4*>(src));
      const float4 x1 = __ldg(reinterpret_cast<const float4*>(src) + 1);
      const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      uint32_t hv[4], lv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hv[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        lv[e] = pack_bf16(x[2 * e] - __uint_as_float(hv[e] << 16), x[2 * e + 1] - __uint_as_float(hv[e] & 0xFFFF0000u));
      }
      const uint32_t off = swz(i, c, D);
      *reinterpret_cast<uint4*>(sB + 4 * BOP + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      *reinterpret_cast<uint4*>(sB + 5 * BOP + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
    }
    fence_proxy_async_smem();
    mbar_arrive_warp(bar(B_BREADY));
    // ---- epilogue per tile: dk, dv and the dbeta partial of this CTA's columns
    const uint32_t la = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = true;
    for (int j = 0; ok && j < ntiles; ++j) {
      const int st = j % STT, buf = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_ACC + buf), (j >> 1) & 1, ctl) &&
                                       mbar_wait(bar(B_FULL + st), (j / STT) & 1, ctl))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int tok = j * TT + row;
      const bool valid = tok < N;
      const long long grow = (tok0 + tok) * H + h;
      const float be = valid ? __ldg(in.beta + grow) : 0.f;
      const unsigned char* sK = sKV + st * 2 * TILE;
      const unsigned char* sV = sK + TILE;
      float dbp = 0.f;
#pragma unroll
      for (int q = 0; q < CW / 32; ++q) {
        float p1[32], p2[32], p3[32];
        const uint32_t a = la + 256u * buf + 32 * q;
        tmem_ld32(a, p1);
        tmem_ld32(a + 64, p2);
        tmem_ld32(a + 128, p3);
        tmem_wait_ld();
        const int c0 = cb * CW + 32 * q;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint4 kr = *reinterpret_cast<const uint4*>(sK + swz(row, c0 + 8 * u, TT));
          const uint4 vr = *reinterpret_cast<const uint4*>(sV + swz(row, c0 + 8 * u, TT));
          const uint32_t ku[4] = {kr.x, kr.y, kr.z, kr.w}, vu[4] = {vr.x, vr.y, vr.z, vr.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i0 = 8 * u + 2 * e;
            dbp = fmaf(0.5f * __uint_as_float(ku[e] << 16), p1[i0], dbp);
            dbp = fmaf(0.5f * __uint_as_float(ku[e] & 0xFFFF0000u), p1[i0 + 1], dbp);
            dbp = fmaf(__uint_as_float(vu[e] << 16), p3[i0], dbp);
            dbp = fmaf(__uint_as_float(vu[e] & 0xFFFF0000u), p3[i0 + 1], dbp);
          }
        }
        if (valid) {
          float* dkr = dk + grow * D + c0;
          float* dvr = dv + grow * D + c0;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 gk = make_float4(be * (p1[i] + p2[i]), be * (p1[i + 1] + p2[i + 1]), be * (p1[i + 2] + p2[i + 2]),
                                    be * (p1[i + 3] + p2[i + 3]));
            float4 gv = make_float4(be * p3[i], be * p3[i + 1], be * p3[i + 2], be * p3[i + 3]);
            if (dm.grad_acc) {  // products rounded first (no fused multiply-add)
              const float4 pk = *reinterpret_cast<const float4*>(dkr + i), pv = *reinterpret_cast<const float4*>(dvr + i);
              gk = make_float4(__fadd_rn(pk.x, gk.x), __fadd_rn(pk.y, gk.y), __fadd_rn(pk.z, gk.z), __fadd_rn(pk.w, gk.w));
              gv = make_float4(__fadd_rn(pv.x, gv.x), __fadd_rn(pv.y, gv.y), __fadd_rn(pv.z, gv.z), __fadd_rn(pv.w, gv.w));
            }
            *reinterpret_cast<float4*>(dkr + i) = gk;
            *reinterpret_cast<float4*>(dvr + i) = gv;
          }
        }
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_TFREE + buf));
      mbar_arrive_warp(bar(B_EMPTY + st));
      if (valid) atomicAdd(dbeta + grow, dbp);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, 512);
}

template <int D> constexpr size_t tokens_tc_smem() {
  return 1024 + STT * 2 * (size_t)TT * D * 2 + 6 * (size_t)CW * D * 2 + 16 * 8 + 16;
}

template <int D>
cudaError_t launch_d(const Dims& d, const Inputs& in, const float* dAs, const float* dB, float* dk, float* dv,
                     float* dbeta, uint32_t* status, cudaStream_t s) {
  CUtensorMap mk, mv;
  const long long tokens = (long long)d.B * d.T * d.N;
  if (!make_token_map(&mk, in.k, tokens, d.H, D, TT) || !make_token_map(&mv, in.v, tokens, d.H, D, TT))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(dbeta, 0, sizeof(float) * tokens * d.H, s);
  if (e != cudaSuccess) return e;
  auto kern = k_bwd_tokens_tc<D>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tokens_tc_smem<D>())) !=
      cudaSuccess)
    return e;
  kern<<<dim3(d.T * (D / CW), d.H, d.B), kThrT, tokens_tc_smem<D>(), s>>>(d, in, dAs, dB, dk, dv, dbeta, status, mk, mv);
  return cudaGetLastError();
}

}  // namespace

bool bwd_tokens_tc_supported(const Dims& d) {
  if (!d.bf16 || d.dk != d.dv || (d.dk != 64 && d.dk != 128)) return false;
  if ((long long)d.B * d.T * d.N + TT >= (1LL << 31)) return false;
  if ((long long)d.T * 2 > 65535) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_bwd_tokens_tc(const Dims& d, const Inputs& in, const float* dAs, const float* dB, float* dk,
                                 float* dv, float* dbeta, uint32_t* status, cudaStream_t s) {
  if (d.dk == 128) return launch_d<128>(d, in, dAs, dB, dk, dv, dbeta, status, s);
  if (d.dk == 64) return launch_d<64>(d, in, dAs, dB, dk, dv, dbeta, status, s);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
