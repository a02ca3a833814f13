// Ablation variants of the per-frame write, for comparison with the joint
// solve on the same scans, read and softmax.
//
// The Video DeltaNet pages set the joint frame write (every token of a frame
// solved together, S_t = (S_bar + B)(I + A)^-1) against two older rules
// (deepmagic post, its Video Delta Attention paragraph; aimodeling news, "The
// VDN split": no frame-size rescaling, unlike SANA-WM; PaperDaily digest,
// section 四, the token-level delta rule as the one-token case):
//   * frame-level independent writes (SANA-WM): every token of the frame
//     writes against the same frozen inherited state, and the sum is rescaled
//     by the frame size N:
//       S_t = S_bar + (1/N) sum_i beta_i (v_i - S_bar k_i) k_i^T
//           = S_bar (I - A/N) + B/N;
//   * the token-wise delta rule: the tokens write one after another in token
//     order, each against the state the previous one left:
//       S <- S + beta_i (v_i - S k_i) k_i^T = S (I - beta_i k_i k_i^T) + beta_i v_i k_i^T.
// Both are affine maps S -> S M'_t + C'_t of the inherited state S_bar =
// alpha_t S, so the scans take them exactly like the joint solve's (M_t, C_t):
// this kernel writes M'_t and C'_t into the same slots and the C-form scan
// steps S <- alpha_t S M'_t + C'_t.  M'_t of the token rule is not symmetric,
// so the backward scan uses the same M'_t (the frames are written in reverse
// order; the tokens of each frame keep their order).
//
// One CTA per (frame, batch, head), the stacked [M'; C'] (2D x D) held in
// registers in 4 x 16 tiles: row r of M' starts as e_r, row r of C' as 0,
// and token i updates row r by coef * k_i with
//   token rule: coef = beta_i (target_r - row_r . k_i),
//   frame rule: coef = beta_i (target_r - e_r . k_i) / N   (the frozen state),
// target_r = 0 for rows of M' and v_i[r - D] for rows of C'.  Rows never
// interact; tokens are staged in shared memory 16 at a time in their stored
// type by asynchronous copies, double-buffered, the next block in flight
// while the current one is applied.  With bf16 inputs (d = 64, 128) the frame rule
// instead takes A_t and B_t from the tensor-core Gram kernel and rescales
// them in place: M'_t = I - A_t / N, C'_t = B_t / N.
#include <cuda_bf16.h>

#include "vdn_internal.h"

namespace vdn {
namespace {

constexpr int kTB = 16;  // tokens per staged block

// Thread tile: RT = 4 rows x CT = 16 columns of the stacked map.  The CG =
// D / 16 threads of a row group are adjacent lanes, so a row's dot product
// with the key is their partial sums reduced by log2(CG) xor shuffles.  Keys
// stay in shared memory in their stored type (VW = 16 / sizeof(T) to a
// 16-byte load); lane cg of a group holds the columns VW cg + VW CG m +
// (0 .. VW - 1), so the group's 16-byte loads fall on distinct banks.  Per
// token a thread loads its 16 key columns and the 4 targets, and does 64
// (+ 64 for the dot) multiply-adds.
constexpr int RT = 4, CT = 16;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
// asynchronous copies into shared memory; an invalid source fills zeros
// (no bytes are read, src stays a valid address)
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// 16 bytes of shared memory as floats
__device__ __forceinline__ void ld_vec(const float* p, float* out) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
__device__ __forceinline__ void ld_vec(const __nv_bfloat16* p, float* out) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(u[i] << 16);
    out[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}
// 4 consecutive entries as floats
__device__ __forceinline__ void ld4(const float* p, float* out) { ld_vec(p, out); }
__device__ __forceinline__ void ld4(const __nv_bfloat16* p, float* out) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  out[0] = __uint_as_float(v.x << 16);
  out[1] = __uint_as_float(v.x & 0xFFFF0000u);
  out[2] = __uint_as_float(v.y << 16);
  out[3] = __uint_as_float(v.y & 0xFFFF0000u);
}

template <typename T, int D, int VAR>
__global__ void __launch_bounds__(2 * D / RT * (D / CT)) k_variant_map(Dims dm, Inputs in, Work w) {
  constexpr int R = 2 * D;            // rows of [M'; C']
  constexpr int CG = D / CT;          // threads per row group
  constexpr int NT = R / RT * CG;     // threads
  constexpr int VW = 16 / (int)sizeof(T);  // entries in 16 bytes
  constexpr int CPR = R / VW;         // 16-byte chunks of a token's [k; v] row
  static_assert(CT % VW == 0 && 32 % CG == 0, "variant tiling");
  __shared__ __align__(16) T sk[2][kTB][R];  // token j: k at [0, D), v at [D, 2D)
  __shared__ __align__(16) float sb[2][kTB];
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (is_anchor(dm, t)) return;  // anchor frames are not written
  const int tid = threadIdx.x, r0 = (tid / CG) * RT, cg = tid % CG;
  // column of this thread's entry c (0 .. CT - 1)
  auto col = [&](int c) { return VW * cg + (c / VW) * (VW * CG) + (c % VW); };
  const long long fh = ((long long)b * dm.T + t) * dm.H + h;
  const T* kp = static_cast<const T*>(in.k);
  const T* vp = static_cast<const T*>(in.v);
  const long long tok0 = ((long long)b * dm.T + t) * dm.N;  // first token of the frame
  // stage tokens n0 .. n0 + kTB - 1 into buffer buf (zeros past the frame)
  auto stage = [&](int buf, int n0) {
    for (int q = tid; q < kTB * CPR; q += NT) {
      const int j = q / CPR, u = (q % CPR) * VW, n = n0 + j;
      const bool ok = n < dm.N;
      const long long row = (tok0 + (ok ? n : 0)) * dm.H + h;
      const T* src = u < D ? kp + row * D + u : vp + row * D + (u - D);
      cp_async16(&sk[buf][j][u], src, ok);
    }
    if (tid < kTB) {
      const int n = n0 + tid;
      const bool ok = n < dm.N;
      cp_async4(&sb[buf][tid], in.beta + (tok0 + (ok ? n : 0)) * dm.H + h, ok);
    }
    cp_async_commit();
  };

  float z[RT][CT];
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int c = 0; c < CT; ++c) z[i][c] = (r0 + i == col(c)) ? 1.f : 0.f;  // e_r on rows of M'
  const float inv_n = 1.0f / (float)dm.N;
  const int nblk = (dm.N + kTB - 1) / kTB;

  stage(0, 0);
  cp_async_wait_all();
  __syncthreads();

  for (int blk = 0; blk < nblk; ++blk) {
    const int cur = blk & 1;
    const bool more = blk + 1 < nblk;
    // the other buffer was last read before the previous barrier
    if (more) stage(cur ^ 1, (blk + 1) * kTB);
#pragma unroll 1
    for (int j = 0; j < kTB; ++j) {
      const T* kv = sk[cur][j];
      const float beta = sb[cur][j];
      float k[CT];
#pragma unroll
      for (int c = 0; c < CT; c += VW) ld_vec(kv + col(c), k + c);
      // entries r0 .. r0 + 3 of [k; v]: the rows' k entries (rows of M') or
      // their value targets (rows of C')
      float ent[RT];
      ld4(kv + r0, ent);
      const bool mrow = r0 < D;
      float coef[RT];
      if (VAR == 2) {
        float dot[RT];
#pragma unroll
        for (int i = 0; i < RT; ++i) {
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int c = 0; c < CT; c += 2) {
            a0 = fmaf(z[i][c], k[c], a0);
            a1 = fmaf(z[i][c + 1], k[c + 1], a1);
          }
          dot[i] = a0 + a1;
        }
#pragma unroll
        for (int o = CG / 2; o > 0; o >>= 1)
#pragma unroll
          for (int i = 0; i < RT; ++i) dot[i] += __shfl_xor_sync(0xffffffffu, dot[i], o);
#pragma unroll
        for (int i = 0; i < RT; ++i) coef[i] = beta * ((mrow ? 0.f : ent[i]) - dot[i]);
      } else {
        // against the frozen state: the row's dot with the key is k[r] on rows of M', 0 on rows of C'
#pragma unroll
        for (int i = 0; i < RT; ++i) coef[i] = beta * inv_n * (mrow ? -ent[i] : ent[i]);
      }
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int c = 0; c < CT; ++c) z[i][c] = fmaf(coef[i], k[c], z[i][c]);
    }
    cp_async_wait_all();
    __syncthreads();
  }

  const long long DD = (long long)D * D;
#pragma unroll
  for (int i = 0; i < RT; ++i) {
    const int r = r0 + i;
    float* dst = r < D ? w.M + fh * DD + (long long)r * D : w.Cm + fh * DD + (long long)(r - D) * D;
#pragma unroll
    for (int c = 0; c < CT; c += 4)
      *reinterpret_cast<float4*>(dst + col(c)) = make_float4(z[i][c], z[i][c + 1], z[i][c + 2], z[i][c + 3]);
  }
}

// Frame-level writes from the tensor-core Gram: the M_t / C_t slots hold A_t
// and B_t, turned in place into M'_t = I - A_t / N and C'_t = B_t / N.
template <int D>
__global__ void k_frame_rescale(Dims dm, Work w) {
  const long long DD = (long long)D * D;
  const long long frames = (long long)dm.B * dm.T * dm.H;
  const float inv_n = 1.0f / (float)dm.N;
  const long long total = frames * (DD / 4);
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < total;
       q += (long long)gridDim.x * blockDim.x) {
    const long long fh = q / (DD / 4);
    const int t = (int)((fh / dm.H) % dm.T);
    if (is_anchor(dm, t)) continue;
    const int e = (int)(q % (DD / 4)) * 4, row = e / D, col = e % D;
    float4* m = reinterpret_cast<float4*>(w.M + fh * DD + e);
    float4* c = reinterpret_cast<float4*>(w.Cm + fh * DD + e);
    float4 a = *m, bb = *c;
    a.x = (row == col ? 1.f : 0.f) - a.x * inv_n;
    a.y = (row == col + 1 ? 1.f : 0.f) - a.y * inv_n;
    a.z = (row == col + 2 ? 1.f : 0.f) - a.z * inv_n;
    a.w = (row == col + 3 ? 1.f : 0.f) - a.w * inv_n;
    bb.x *= inv_n; bb.y *= inv_n; bb.z *= inv_n; bb.w *= inv_n;
    *m = a;
    *c = bb;
  }
}

template <typename T, int D>
cudaError_t variant_launch(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  constexpr int NT = 2 * D / RT * (D / CT);
  dim3 grid(d.T, d.H, d.B);
  if (d.update == 1)
    k_variant_map<T, D, 1><<<grid, NT, 0, s>>>(d, in, w);
  else
    k_variant_map<T, D, 2><<<grid, NT, 0, s>>>(d, in, w);
  return cudaGetLastError();
}

template <int D>
cudaError_t variant_f(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  return d.bf16 ? variant_launch<__nv_bfloat16, D>(d, in, w, s) : variant_launch<float, D>(d, in, w, s);
}

}  // namespace

cudaError_t launch_variant_maps(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s) {
  if (d.update != 1 && d.update != 2) return cudaErrorInvalidValue;
  if (d.update == 1 && gram_tc_supported(d) && d.dk <= 128) {
    // A_t, B_t on the tensor cores, then the 1/N rescale in place
    cudaError_t e = launch_gram_tc(d, in, w, s);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    if (d.dk == 128)
      k_frame_rescale<128><<<sms * 8, 256, 0, s>>>(d, w);
    else
      k_frame_rescale<64><<<sms * 8, 256, 0, s>>>(d, w);
    return cudaGetLastError();
  }
  switch (d.dk) {
    case 32: return variant_f<32>(d, in, w, s);
    case 64: return variant_f<64>(d, in, w, s);
    case 128: return variant_f<128>(d, in, w, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vdn
