// Output projection of the hybrid attention layer on the tensor cores.
//
// What it computes (PaperDaily digest section 三: each branch is gated and
// projected back to the model width; the core's two outputs sit on a size-2
// axis, so one product with the stacked weight [W_o^sm; W_o^lin] equals the
// sum of the two separate projections):
//   out[m, n] = sum_k Y[m, k] W[k, n],   Y = y viewed as [B*T*N, H*2*d_v].
// bf16 operands with fp32 accumulation; and the FP8 linear layer of the
// deepmagic post ("生成比播放還快", section 實測數據: the per-block latency
// reaches its lowest figure with FP8 linear layers): e4m3 operands, the weight
// given transposed ([n, K]), out = (s_y s_w) * sum_k q_y[m, k] q_w[n, k].
//
// Persistent kernel on CTA pairs (clusters of two CTAs on neighbouring SMs):
// each pair computes 256 x 256 output tiles with tcgen05.mma.cta_group::2,
// M = 256 (128 rows in each CTA), N = 256 (each CTA holds 128 of the B
// columns), so every operand byte in shared memory feeds twice the products
// of a one-CTA tile.  Per CTA (256 threads):
//   warp 0      TMA producer: this CTA's A rows and B half, six stages of
//               128 bytes of K per row (64 bf16 or 128 e4m3), the bytes of
//               both CTAs counted on the leader's FULL barrier;
//   warp 1      TMEM allocation (512 columns: two 256-column accumulators)
//               and, in the leader, the MMA issuer: four products per stage,
//               then one commit to both CTAs' EMPTY barriers; the last stage
//               of a tile commits its accumulator to both CTAs' AFULL;
//   warps 4..7  epilogue: a thread per accumulator row (TMEM lane), 32-column
//               loads, the FP8 scale, the cast to the output type and 16-byte
//               stores of its row; then one arrival per warp on the leader's
//               AEMPTY, so that the next-but-one tile can reuse the columns.
// The two accumulators let one tile's epilogue run under the next tile's
// products.  Tiles go to the pairs round robin, columns fastest, so the pairs
// running at one time share A row blocks and the whole weight in L2.
// Every load lands in the issuing CTA alone: each CTA loads its own half.
//
// Every wait is bounded; on expiry the CTA records VDN_ERR_TIMEOUT and
// VDN_TAG_PROJ in the projection's status words (a library-owned device array,
// read by vdn_proj_device_status), stops issuing, drains what it issued and
// leaves through the pair's final cluster barrier.
#include <cuda_fp8.h>

#include "tc_common.cuh"

namespace vdn {

// Status words of the projection's bounded waits (no caller workspace).
__device__ uint32_t g_proj_status[2];

namespace {
using namespace tc;

constexpr int kThreadsG = 256;
constexpr int TM = 128;                        // rows per CTA (256 per pair)
constexpr int TN = 256;                        // columns per tile (128 per CTA in B)
constexpr int KBYTES = 128;                    // bytes of K per row and stage
constexpr int ST = 6;                          // stages
constexpr uint32_t ABYTES = TM * KBYTES;       // 16 KB
constexpr uint32_t BBYTES = (TN / 2) * KBYTES;  // 16 KB
constexpr uint32_t STAGE = ABYTES + BBYTES;
constexpr uint32_t kCols = 2 * TN;

// e4m3 A and B, fp32 D, both K-major (kind::f8f6f4 instruction descriptor:
// D format at bit 4, A and B formats at bits 7 and 10 (0 = E4M3), N / 8 at
// bit 17, M / 16 at bit 24)
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma2_e4m3(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct GemmArgs {
  int M, N, K;
  int tiles_n, tiles;  // column tiles, all tiles
  int nkb;             // K blocks of KBYTES per row
  void* out;
  const float* scales;  // FP8: {s_y, s_w}; null for bf16
};

// 32 accumulator values of one row to out (16-byte stores; `cols` valid)
__device__ __forceinline__ void store_row(float* dst, const float (&v)[32], int cols) {
#pragma unroll
  for (int i = 0; i < 32; i += 4)
    if (i < cols) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}
__device__ __forceinline__ void store_row(__nv_bfloat16* dst, const float (&v)[32], int cols) {
#pragma unroll
  for (int i = 0; i < 32; i += 8)
    if (i < cols)
      *reinterpret_cast<uint4*>(dst + i) = make_uint4(pack_bf16(v[i], v[i + 1]), pack_bf16(v[i + 2], v[i + 3]),
                                                      pack_bf16(v[i + 4], v[i + 5]), pack_bf16(v[i + 6], v[i + 7]));
}

// FP8 = false: A bf16 [M, K] (K-major), B = W bf16 [K, N] (N contiguous: MN-major).
// FP8 = true:  A e4m3 [M, K], B = W^T e4m3 [N, K] (both K-major).
template <bool FP8, typename To>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsG, 1)
k_gemm_tc(GemmArgs g, const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb) {
  enum { B_FULL = 0, B_EMPTY = ST, B_AFULL = 2 * ST, B_AEMPTY = 2 * ST + 2, B_DRAIN = 2 * ST + 4, NBARS };
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + ST * STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // no early exit: both CTAs of the pair must reach the cluster barriers
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool lead = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const Ctl ctl{abort_flag, g_proj_status, (unsigned)VDN_TAG_PROJ};
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto lbar = [&](int i) { return map_rank(smem_u32(bars + i), 0); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(B_AFULL + a), 1);
      mbar_init(bar(B_AEMPTY + a), 8);  // one arrival per epilogue warp of the pair
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc2(smem_u32(tmem_slot), kCols);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tma)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmb)) : "memory");
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < g.tiles; tile += npairs) {
        const int m0 = (tile / g.tiles_n) * 2 * TM + (int)rank * TM;
        const int n0 = (tile % g.tiles_n) * TN + (int)rank * (TN / 2);
        for (int kb = 0; kb < g.nkb; ++kb, ++it) {
          const int s = it % ST;
          if (it >= ST && !mbar_wait_cl(bar(B_EMPTY + s), (it / ST - 1) & 1, ctl)) { ok = false; break; }
          if (lead) mbar_expect_tx(bar(B_FULL + s), 2 * STAGE);
          const uint32_t sa = smem_u32(sm + s * STAGE), sb = sa + ABYTES;
          if (FP8) {
            tma_load_2d_pair(sa, &tma, lbar(B_FULL + s), kb * KBYTES, m0);
            tma_load_2d_pair(sb, &tmb, lbar(B_FULL + s), kb * KBYTES, n0);
          } else {
            tma_load_2d_pair(sa, &tma, lbar(B_FULL + s), kb * 64, m0);
            // W rows kb*64 .. +63, this CTA's 128 columns as two 64-column boxes
            tma_load_2d_pair(sb, &tmb, lbar(B_FULL + s), n0, kb * 64);
            tma_load_2d_pair(sb + 64 * 128, &tmb, lbar(B_FULL + s), n0 + 64, kb * 64);
          }
        }
      }
      // the leader's FULL barriers count both CTAs' bytes: once the last
      // phases it armed complete, every copy of the pair has landed
      if (lead)
        for (int j = it - ST < 0 ? 0 : it - ST; j < it; ++j) mbar_drain(bar(B_FULL + j % ST), (j / ST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && lead) {
      const uint32_t ID = FP8 ? idesc_e4m3(2 * TM, TN) : idesc_bf16(2 * TM, TN, true);
      const uint64_t a0 = sdesc(smem_u32(sm), 16, 1024);
      // B: K-major (FP8), or MN-major with the two 64-column chunks 8 KB apart
      const uint64_t b0 = FP8 ? sdesc(smem_u32(sm + ABYTES), 16, 1024) : sdesc(smem_u32(sm + ABYTES), 64 * 128, 1024);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < g.tiles; tile += npairs, ++tc) {
        const int a = tc & 1;
        if (tc >= 2 && !mbar_wait_cl(bar(B_AEMPTY + a), ((tc >> 1) - 1) & 1, ctl)) break;
        tc_fence_after();
        const uint32_t d = tmem + a * TN;
        for (int kb = 0; kb < g.nkb; ++kb, ++it) {
          const int s = it % ST;
          if (!mbar_wait_cl(bar(B_FULL + s), (it / ST) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t as = dadd(a0, s * STAGE), bs = dadd(b0, s * STAGE);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // A: 32 bytes of K per step inside the 128-byte swizzle row; B:
            // the same (K-major) or 16 rows of 128 bytes (MN-major)
            const uint64_t ak = dadd(as, k * 32), bk = dadd(bs, FP8 ? k * 32 : k * 16 * 128);
            if (FP8)
              mma2_e4m3(d, ak, bk, ID, (kb | k) ? 1u : 0u);
            else
              mma2_bf16(d, ak, bk, ID, (kb | k) ? 1u : 0u);
          }
          commit2(bar(B_EMPTY + s));
          commit2(map_rank(bar(B_EMPTY + s), 1));
        }
        if (!ok) break;
        commit2(bar(B_AFULL + a));
        commit2(map_rank(bar(B_AFULL + a), 1));
      }
      commit2(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int trow = quad * 32 + lane;  // TMEM lane = row of this CTA's half
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const float sc = FP8 ? __ldg(g.scales) * __ldg(g.scales + 1) : 1.0f;
    To* out = static_cast<To*>(g.out);
    int tc = 0;
    for (int tile = pair; tile < g.tiles; tile += npairs, ++tc) {
      const int a = tc & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_cl(bar(B_AFULL + a), (tc >> 1) & 1, ctl))) break;
      tc_fence_after();
      const long long row = (long long)(tile / g.tiles_n) * 2 * TM + (long long)rank * TM + trow;
      const int n0 = (tile % g.tiles_n) * TN;
      const bool valid = row < g.M;
#pragma unroll 1
      for (int c = 0; c < TN / 32; ++c) {
        float v[32];
        tmem_ld32(lane_addr + a * TN + 32 * c, v);
        tmem_wait_ld();
        if (FP8) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= sc;
        }
        const int cols = g.N - (n0 + 32 * c);
        if (valid && cols > 0) store_row(out + row * g.N + n0 + 32 * c, v, cols);
      }
      tc_fence_before();
      arrive_cluster_warp(lbar(B_AEMPTY + a));  // this accumulator is free again
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory or barriers
  tc_fence_after();
  if (warp == 1) tmem_free2(tmem, kCols);
}

constexpr size_t gemm_smem() { return 1024 + (size_t)ST * STAGE + 32 * 8 + 16; }

template <bool FP8, typename To>
vdn_status launch(int M, int K, int N, const void* y, const void* w, const float* scales, void* out, cudaStream_t s) {
  CUtensorMap ma, mb;
  if (FP8) {
    if (!make_matrix_map_u8(&ma, y, M, K, TM) || !make_matrix_map_u8(&mb, w, N, K, TN / 2)) return VDN_ERR_CUDA;
  } else {
    if (!make_matrix_map(&ma, y, M, K, TM) || !make_matrix_map(&mb, w, K, N, 64)) return VDN_ERR_CUDA;
  }
  GemmArgs g;
  g.M = M; g.N = N; g.K = K;
  g.tiles_n = (N + TN - 1) / TN;
  const long long tiles = (long long)((M + 2 * TM - 1) / (2 * TM)) * g.tiles_n;
  if (tiles > 0x3FFFFFFFLL) return VDN_ERR_UNSUPPORTED;
  g.tiles = (int)tiles;
  g.nkb = (int)(((long long)K * (FP8 ? 1 : 2) + KBYTES - 1) / KBYTES);
  g.out = out;
  g.scales = scales;
  auto kern = k_gemm_tc<FP8, To>;
  const size_t smem = gemm_smem();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return VDN_ERR_CUDA;
  // as many pairs as can be resident at once (a persistent grid), at most one per tile
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return VDN_ERR_CUDA;
  int pairs = sms / 2;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * pairs);
  lc.blockDim = dim3(kThreadsG);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  int active = 0;
  if (cudaOccupancyMaxActiveClusters(&active, reinterpret_cast<const void*>(kern), &lc) == cudaSuccess && active > 0)
    pairs = active < pairs ? active : pairs;
  else
    cudaGetLastError();
  if (pairs > g.tiles) pairs = g.tiles;
  kern<<<2 * pairs, kThreadsG, smem, s>>>(g, ma, mb);
  return cudaGetLastError() == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

}  // namespace

vdn_status out_proj(int M, int K, int N, int out_dtype, const void* y, const void* w, void* out, cudaStream_t s,
                    const float* scales) {
  if (!encode_fn()) return VDN_ERR_CUDA;
  uint32_t* st = status_of_proj();
  if (!st || cudaMemsetAsync(st, 0, sizeof(uint32_t) * 2, s) != cudaSuccess) return VDN_ERR_CUDA;
  if (scales)
    return out_dtype == VDN_BF16 ? launch<true, __nv_bfloat16>(M, K, N, y, w, scales, out, s)
                                 : launch<true, float>(M, K, N, y, w, scales, out, s);
  return out_dtype == VDN_BF16 ? launch<false, __nv_bfloat16>(M, K, N, y, w, nullptr, out, s)
                               : launch<false, float>(M, K, N, y, w, nullptr, out, s);
}

uint32_t* status_of_proj() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_proj_status) != cudaSuccess) return nullptr;
  return static_cast<uint32_t*>(p);
}

}  // namespace vdn
