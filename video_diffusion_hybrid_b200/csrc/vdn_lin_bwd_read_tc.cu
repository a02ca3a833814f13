// Read backward of the linear branch on the tensor cores (tcgen05): d = 128,
// bf16 q and gates.
//
// The read (PaperDaily digest section 三: queries read the forward state
// before their window plus the backward state after it; the read is RMS-
// normalised and gated) is, per token of query frame t,
//   o = R q (R = F[lo(t)] + G[hi(t)]),  r = (mean o^2 + eps)^-1/2,  n = o r,
//   y = sigmoid(g) w n.
// Its derivative, with dy the gradient of y's linear slot:
//   dg = dy w n s (1 - s),  dn = dy s w,  do = r (dn - n mean(dn n)),
//   dq = R^T do,  dR = sum over the frame's tokens of do q^T,  dw = sum dy s n.
// Over a 128-token tile Q (rows = tokens):
//   O = Q R^T,  dQ = dO R,  dR += dO^T Q.
//
// One CTA per (frame, head), the frame's tokens in tiles of 128 (TMA ring of
// two).  R enters as bf16 hi + lo (about 16 significant bits) in one 128-byte
// swizzled [i][j] layout that serves as the K-major B of O = Q R^T and as the
// MN-major B of dQ = dO R; dO, formed per row by the epilogue warps, enters
// as hi + lo in one [token][i] layout that serves as the K-major A of dQ and
// as the MN-major A of dR = dO^T Q (q itself is the MN-major B there).  dR
// accumulates in TMEM over the frame's tiles.
// Roles (256 threads): warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer, warps 4..7 R's split, then per tile the RMSNorm / gate backward
// (thread = token row = TMEM lane; the gate and dy rows arrive through a
// per-warp transpose buffer, loaded with lane = column so that the loads are
// coalesced) and the dq store; at the end dR (thread = row i) and the RMS
// weight partials, whose column sums over the tile's rows are taken by a
// transpose-reduce within each warp.  Every mbarrier wait is bounded.
#include "tc_common.cuh"

namespace vdn {
namespace {
using namespace tc;

constexpr int D = 128;
constexpr int TT = 128;  // tokens per tile
constexpr int kThrR = 256;
constexpr int STR = 2;   // Q ring stages
constexpr uint32_t TILE = TT * D * 2;

__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((c >> 6) * 128 * 128 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}
__device__ __forceinline__ int rd_lo(const Dims& d, int t) {
  return is_anchor(d, t) ? 0 : max(0, d.chunk * (t / d.chunk - 1));
}
__device__ __forceinline__ int rd_hi(const Dims& d, int t) {
  return is_anchor(d, t) ? d.T : min(d.T, d.chunk * (t / d.chunk + 2));
}
__device__ __forceinline__ float sigm_f(float x) { return 1.0f / (1.0f + __expf(-x)); }
__device__ __forceinline__ float tofr(float x) { return x; }
__device__ __forceinline__ float tofr(__nv_bfloat16 x) { return __bfloat162float(x); }

// 8 fp32 values as bf16 hi + lo at byte offset `off` of the two tiles
__device__ __forceinline__ void put_split8(unsigned char* hi, unsigned char* lo, uint32_t off, const float (&x)[8]) {
  uint32_t hv[4], lv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    hv[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
    lv[e] = pack_bf16(x[2 * e] - __uint_as_float(hv[e] << 16), x[2 * e + 1] - __uint_as_float(hv[e] & 0xFFFF0000u));
  }
  *reinterpret_cast<uint4*>(hi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  *reinterpret_cast<uint4*>(lo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
}

template <typename Ty>
__global__ void __launch_bounds__(kThrR, 1)
k_bwd_read_tc(Dims dm, Inputs in, const float* __restrict__ Fst, const float* __restrict__ Gst, const void* dyp,
              float* dq, float* dgate, float* dRp, float* dwp, uint32_t* status,
              const __grid_constant__ CUtensorMap tmq) {
  enum { B_FULL = 0, B_EMPTY = STR, B_RREADY = 2 * STR, B_OFULL, B_OFREE, B_DOREADY, B_DOFREE, B_DQFULL, B_DQFREE,
         B_DRDONE, B_DRAIN, NBARS };
  constexpr uint32_t COL_O = 0, COL_DQ = 128, COL_DR = 256;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sR = sm;                 // hi, lo
  unsigned char* sQ = sR + 2 * TILE;      // STR stages
  unsigned char* sDO = sQ + STR * TILE;   // hi, lo
  // per epilogue warp a 32 x 33 transpose buffer for the gate and dy rows;
  // after the last tile the same space collects the RMS weight partials [4][D]
  float* tbuf = reinterpret_cast<float*>(sDO + 2 * TILE);
  float* red = tbuf;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tbuf + 4 * 32 * 33);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = dm.N, H = dm.H, T = dm.T;
  const long long fh = ((long long)b * T + t) * H + h, bh = (long long)b * H + h, tok0 = ((long long)b * T + t) * N;
  if (*reinterpret_cast<volatile uint32_t*>(status) != 0u) return;
  const int ntiles = (N + TT - 1) / TT;
  const Ctl ctl{abort_flag, status, (unsigned)TAG_LINBWD_TC};
  auto bar = [&](int i) { return smem_u32(bars + i); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBARS; ++i)
      mbar_init(bar(i), (i == B_RREADY || i == B_OFREE || i == B_DOREADY || i == B_DQFREE) ? 4 : 1);
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
        const int st = j % STR;
        if (j >= STR && !mbar_wait(bar(B_EMPTY + st), (j / STR - 1) & 1, ctl)) break;
        mbar_expect_tx(bar(B_FULL + st), TILE);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem_u32(sQ + st * TILE + c * TT * 128), &tmq, bar(B_FULL + st), c * 64, h,
                      (int)(tok0 + (long long)j * TT));
        issued = j + 1;
      }
      for (int j = issued - STR < 0 ? 0 : issued - STR; j < issued; ++j)
        mbar_drain(bar(B_FULL + j % STR), (j / STR) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID_O = idesc_bf16(TT, D, false);                 // K-major A and B
      constexpr uint32_t ID_Q = idesc_bf16(TT, D, true);                  // B MN-major
      constexpr uint32_t ID_R = idesc_bf16(D, D, true) | (1u << 15);      // A and B MN-major
      const uint64_t rk[2] = {sdesc(smem_u32(sR), 16, 1024), sdesc(smem_u32(sR + TILE), 16, 1024)};
      const uint64_t rm[2] = {sdesc(smem_u32(sR), TT * 128, 1024), sdesc(smem_u32(sR + TILE), TT * 128, 1024)};
      const uint64_t dk_[2] = {sdesc(smem_u32(sDO), 16, 1024), sdesc(smem_u32(sDO + TILE), 16, 1024)};
      const uint64_t dm_[2] = {sdesc(smem_u32(sDO), TT * 128, 1024), sdesc(smem_u32(sDO + TILE), TT * 128, 1024)};
      const uint64_t qk0 = sdesc(smem_u32(sQ), 16, 1024), qm0 = sdesc(smem_u32(sQ), TT * 128, 1024);
      bool ok = mbar_wait(bar(B_RREADY), 0, ctl);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % STR;
        ok = mbar_wait(bar(B_FULL + st), (j / STR) & 1, ctl) && (j == 0 || mbar_wait(bar(B_OFREE), (j - 1) & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        // O = Q R^T
        const uint64_t qk = dadd(qk0, st * TILE), qm = dadd(qm0, st * TILE);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * (TT * 128) + (k & 3) * 32;
            mma_bf16(tmem + COL_O, dadd(qk, off), dadd(rk[part], off), ID_O, (part | k) ? 1u : 0u);
          }
        mma_commit(bar(B_OFULL));
        ok = mbar_wait(bar(B_DOREADY), j & 1, ctl) && (j == 0 || mbar_wait(bar(B_DQFREE), (j - 1) & 1, ctl));
        if (!ok) break;
        tc_fence_after();
        // dQ = dO R: dO_hi R_hi + dO_hi R_lo + dO_lo R_hi (K = i)
#pragma unroll
        for (int term = 0; term < 3; ++term) {
          const int pa = term == 2 ? 1 : 0, pb = term == 1 ? 1 : 0;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t aoff = (k >> 2) * (TT * 128) + (k & 3) * 32;
            mma_bf16(tmem + COL_DQ, dadd(dk_[pa], aoff), dadd(rm[pb], k * 2048), ID_Q, (term | k) ? 1u : 0u);
          }
        }
        mma_commit(bar(B_DQFULL));
        // dR += dO^T Q (K = the tile's tokens)
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int k = 0; k < TT / 16; ++k)
            mma_bf16(tmem + COL_DR, dadd(dm_[part], k * 2048), dadd(qm, k * 2048), ID_R, (j | part | k) ? 1u : 0u);
        mma_commit(bar(B_DOFREE));
        mma_commit(bar(B_EMPTY + st));
      }
      if (ok) mma_commit(bar(B_DRDONE));
      mma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    const int tid = threadIdx.x - 128, quad = warp - 4, row = quad * 32 + lane;
    const uint32_t la = tmem + ((uint32_t)(quad * 32) << 16);
    // ---- R = F[lo] + G[hi] as bf16 hi + lo
    {
      const float* F = Fst + (bh * (T + 1) + rd_lo(dm, t)) * D * D;
      const float* G = Gst + (bh * (T + 1) + rd_hi(dm, t)) * D * D;
      for (int u = tid; u < D * D / 8; u += 128) {
        const int i = u / (D / 8), c = (u % (D / 8)) * 8;
        const float4* f4 = reinterpret_cast<const float4*>(F + i * D + c);
        const float4* g4 = reinterpret_cast<const float4*>(G + i * D + c);
        const float4 a0 = __ldg(f4), a1 = __ldg(f4 + 1), b0 = __ldg(g4), b1 = __ldg(g4 + 1);
        const float x[8] = {a0.x + b0.x, a0.y + b0.y, a0.z + b0.z, a0.w + b0.w,
                            a1.x + b1.x, a1.y + b1.y, a1.z + b1.z, a1.w + b1.w};
        put_split8(sR, sR + TILE, swz(i, c), x);
      }
      fence_proxy_async_smem();
      mbar_arrive_warp(bar(B_RREADY));
    }
    const __nv_bfloat16* gl = static_cast<const __nv_bfloat16*>(in.gate_lin);
    const Ty* dy = static_cast<const Ty*>(dyp);
    const int ys = dm.out_mode == 0 ? 2 : 1, yslot = dm.out_mode == 0 ? 1 : 0;
    const bool want_dw = dwp != nullptr;
    float dwacc[D / 32];
#pragma unroll
    for (int q = 0; q < D / 32; ++q) dwacc[q] = 0.f;
    float* tb = tbuf + quad * 32 * 33;
    // columns [32 q, 32 q + 32) of the gate and dy rows of the warp's 32 tokens:
    // loaded with lane = column (coalesced), handed to lane = row through tb
    auto rows_gdy = [&](int j, int q, float (&g)[32], float (&dyv)[32]) {
      float tg[32], td[32];  // all 64 loads in flight at once
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        const long long gr = (tok0 + min(j * TT + quad * 32 + r, N - 1)) * H + h;
        tg[r] = __bfloat162float(gl[gr * D + 32 * q + lane]);
        td[r] = tofr(dy[(gr * ys + yslot) * D + 32 * q + lane]);
      }
#pragma unroll
      for (int r = 0; r < 32; ++r) tb[r * 33 + lane] = tg[r];
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = tb[lane * 33 + i];
      __syncwarp();
#pragma unroll
      for (int r = 0; r < 32; ++r) tb[r * 33 + lane] = td[r];
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) dyv[i] = tb[lane * 33 + i];
      __syncwarp();
    };
    bool ok = true;
    for (int j = 0; ok && j < ntiles; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_OFULL), j & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      const int tok = j * TT + row;
      const bool valid = tok < N;
      const long long grow = (tok0 + (valid ? tok : 0)) * H + h;
      // pass 1: the row's RMS
      float ss = 0.f;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        float o[32];
        tmem_ld32(la + COL_O + 32 * q, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(o[i], o[i], ss);
      }
      const float rinv = rsqrtf(ss / D + dm.eps);
      // pass 2: dg, the RMS weight partials and mean(dn n)
      float dot = 0.f;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        float o[32], g[32], dyv[32];
        rows_gdy(j, q, g, dyv);
        tmem_ld32(la + COL_O + 32 * q, o);
        tmem_wait_ld();
        float dwv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c = 32 * q + i;
          const float w = in.rms_weight ? __ldg(in.rms_weight + h * D + c) : 1.0f;
          const float dv_ = valid ? dyv[i] : 0.f;
          const float sg = sigm_f(g[i]), nh = o[i] * rinv;
          dwv[i] = dv_ * sg * nh;
          o[i] = dv_ * nh * w * sg * (1.0f - sg);  // dg, in place
          dot = fmaf(dv_ * sg * w, nh, dot);
        }
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dgate + grow * D + 32 * q + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
        }
        if (want_dw) {
          // column sums over the warp's 32 rows: lane l ends with column 32 q + l
#pragma unroll
          for (int sft = 16; sft >= 1; sft >>= 1) {
            const bool up = (lane & sft) != 0;
#pragma unroll
            for (int i = 0; i < sft; ++i) {
              const float send = up ? dwv[i] : dwv[i + sft];
              const float keep = up ? dwv[i + sft] : dwv[i];
              dwv[i] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
            }
          }
          dwacc[q] += dwv[0];
        }
      }
      dot /= D;
      // pass 3: dO = r (dn - n mean(dn n)) as bf16 hi + lo, once the products
      // of the previous tile have read the last one
      if (!__all_sync(0xffffffffu, j == 0 || mbar_wait(bar(B_DOFREE), (j - 1) & 1, ctl))) { ok = false; break; }
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        float o[32], g[32], dyv[32];
        rows_gdy(j, q, g, dyv);
        tmem_ld32(la + COL_O + 32 * q, o);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = 8 * u + e, c = 32 * q + i;
            const float w = in.rms_weight ? __ldg(in.rms_weight + h * D + c) : 1.0f;
            x[e] = valid ? rinv * (dyv[i] * sigm_f(g[i]) * w - o[i] * rinv * dot) : 0.f;
          }
          put_split8(sDO, sDO + TILE, swz(row, 32 * q + 8 * u), x);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(bar(B_OFREE));
      mbar_arrive_warp(bar(B_DOREADY));
      // dq
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_DQFULL), j & 1, ctl))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        float v[32];
        tmem_ld32(la + COL_DQ + 32 * q, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4* p = reinterpret_cast<float4*>(dq + grow * D + 32 * q + i);
            float4 x = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            if (dm.grad_acc) {
              const float4 o = *p;
              x = make_float4(__fadd_rn(o.x, x.x), __fadd_rn(o.y, x.y), __fadd_rn(o.z, x.z), __fadd_rn(o.w, x.w));
            }
            *p = x;
          }
        }
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_DQFREE));
    }
    // ---- dR of the frame (thread = row i) and the RMS weight partials
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar(B_DRDONE), 0, ctl))) {
      tc_fence_after();
      float* dst = dRp + fh * D * D + (long long)row * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        float v[32];
        tmem_ld32(la + COL_DR + 32 * q, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(dst + 32 * q + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    }
    if (want_dw) {
      asm volatile("bar.sync 1, 128;" ::: "memory");  // every warp is done with its transpose buffer
#pragma unroll
      for (int q = 0; q < D / 32; ++q) red[quad * D + 32 * q + lane] = dwacc[q];
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
      dwp[fh * D + tid] = red[tid] + red[D + tid] + red[2 * D + tid] + red[3 * D + tid];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_free(tmem, 512);
}

constexpr size_t read_tc_smem() { return 1024 + 6 * (size_t)TILE + 4 * 32 * 33 * 4 + 16 * 8 + 16; }

template <typename Ty>
cudaError_t launch_t(const Dims& d, const Inputs& in, const float* Fst, const float* Gst, const void* dy, float* dq,
                     float* dgate, float* dRp, float* dwp, uint32_t* status, cudaStream_t s) {
  CUtensorMap mq;
  if (!make_token_map(&mq, in.q, (long long)d.B * d.T * d.N, d.H, D, TT)) return cudaErrorInvalidValue;
  auto kern = k_bwd_read_tc<Ty>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)read_tc_smem());
  if (e != cudaSuccess) return e;
  kern<<<dim3(d.T, d.H, d.B), kThrR, read_tc_smem(), s>>>(d, in, Fst, Gst, dy, dq, dgate, dRp, dwp, status, mq);
  return cudaGetLastError();
}

}  // namespace

bool bwd_read_tc_supported(const Dims& d) {
  if (!d.bf16 || d.dk != 128 || d.dv != 128) return false;
  if ((long long)d.B * d.T * d.N + TT >= (1LL << 31)) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_bwd_read_tc(const Dims& d, const Inputs& in, const float* Fst, const float* Gst, const void* dy,
                               float* dq, float* dgate, float* dRp, float* dwp, uint32_t* status, cudaStream_t s) {
  return d.out_bf16 ? launch_t<__nv_bfloat16>(d, in, Fst, Gst, dy, dq, dgate, dRp, dwp, status, s)
                    : launch_t<float>(d, in, Fst, Gst, dy, dq, dgate, dRp, dwp, status, s);
}

}  // namespace vdn
