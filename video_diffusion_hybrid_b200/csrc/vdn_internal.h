// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/vdn_hybrid.h"

namespace vdn {

// Problem description handed to every kernel (by value).
struct Dims {
  int B, T, N, H, dk, dv, L, chunk, anchors, C;
  float scale, eps;
  int out_mode;
  int bf16;      // inputs stored as bf16
  int out_bf16;  // y stored as bf16
  int scan_mode;  // 0 auto, 1 frame steps, 2 chunk steps (tensor-core scan)
  int update;     // 0 joint solve, 1 frame-level independent writes (1/N), 2 token-wise delta rule
  int grad_acc;   // linear-branch backward: add its dq, dk, dv into the outputs (the whole-core
                  // backward, after the softmax branch wrote its share) instead of overwriting
};

// Device-side status words at the head of the workspace; the tags are the
// header's VDN_TAG_* values.
enum : unsigned { TAG_NONE = VDN_TAG_NONE, TAG_SOFTMAX_TC = VDN_TAG_SOFTMAX, TAG_GRAM_TC = VDN_TAG_GRAM,
                  TAG_READ_TC = VDN_TAG_READ, TAG_SCAN_TC = VDN_TAG_SCAN, TAG_COMPOSE_TC = VDN_TAG_COMPOSE,
                  TAG_SMBWD_TC = VDN_TAG_SOFTMAX_BWD, TAG_LINBWD_TC = VDN_TAG_LINEAR_BWD };

struct Work {
  uint32_t* status;
  float* half_text;  // [B,H,dv,dk]
  float* M;          // [B,T,H,dk,dk]
  float* Cm;         // [B,T,H,dv,dk]
  float* fsnap;      // [B,H,C+1,dv,dk]
  float* bsnap;      // [B,H,C+1,dv,dk]
  float* R;          // [B,H,C+1,dv,dk]
  void* R16;         // [B,H,C+1,2,dv,dk] bf16 (hi, lo)
  float* text_gram;  // [B,H,2,dk,dk] A_x, B_x
  void* M16;         // [B,T,H,2,dk,dk] bf16 (hi, lo) of M; nullptr off the tensor-core scans
  // chunk maps (tensor-core scan only): P_c split, [Cf; Cb], Lam
  void* P16;         // [B,C,H,2,dk,dk] bf16 (hi, lo) of P_c
  float* Cf;         // [B,C,H,dv,dk]; Cb follows at Cf + B*C*H*dv*dk
  float* Cb;         // [B,C,H,dv,dk]
  float* lam;        // [B,C,H]
  // 1 when the tensor-core scan runs: it forms (alpha S + B_t) M_t itself, so
  // the solve leaves B_t in the C_t slot and skips the product C_t = B_t M_t
  int bform;
};

struct Inputs {
  const void *q, *k, *v;
  const float *beta, *alpha;
  const void *gate_sm, *gate_lin;
  const void *text_k, *text_v;
  const float *text_beta, *init_state, *rms_weight;
  void* y;
  const float* fwd_init;  // forward start state, or null (half the text state)
  float* sm_lse;          // softmax log-sum-exp per query row [B*T*N, H] (natural log), or null
};

__host__ __device__ inline bool is_anchor(const Dims& d, int t) {
  return d.anchors != 0 && (t == 0 || t == d.T - 1);
}

// Launchers (return cudaGetLastError after the launch).
cudaError_t launch_text(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
cudaError_t launch_solve_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
cudaError_t launch_solve_inplace(const Dims& d, const Work& w, cudaStream_t s);
cudaError_t launch_text_solve_sweep(const Dims& d, const Work& w, cudaStream_t s);
cudaError_t launch_text_gram_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
bool gram_tc_supported(const Dims& d);
cudaError_t launch_gram_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
// d = 256: a CTA pair per frame-head (text = true: per batch-head, over the text tokens)
cudaError_t launch_gram256_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s, bool text);
cudaError_t launch_scan_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
// the ablation variants' per-frame maps (M'_t, C'_t) into the M_t, C_t slots
cudaError_t launch_variant_maps(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
cudaError_t launch_read_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
cudaError_t launch_softmax_simt(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
bool softmax_tc_supported(const Dims& d);
cudaError_t launch_softmax_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
// text cross-attention: every query over the L text tokens of its batch, y[B,T,N,H,d_v]
cudaError_t launch_text_xattn_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
bool read_tc_supported(const Dims& d);
// the workspace holds the bf16 split of M (and the solve writes it) exactly when this holds
__host__ __device__ inline bool scan_tc_layout(bool bf16, int dk, int dv) { return bf16 && dk == 128 && dv == 128; }
bool scan_tc_supported(const Dims& d);
// d = 256: block solve, chunked scan and chunked read (SIMT), Gram in block mode
bool big_d(const Dims& d);
cudaError_t launch_solve_big(const Dims& d, const Work& w, cudaStream_t s, bool text);
cudaError_t launch_scan_big(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
cudaError_t launch_read_big(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
// chunks = false: the frame-stepped scan; true: stepped by the chunk maps of launch_compose_tc
cudaError_t launch_scan_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s, bool chunks);
cudaError_t launch_compose_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
// d = 256, bf16: the frame scan on the tensor cores (a CTA pair per chain), from
// the bf16 hi/lo split of M_t that the block solve writes
__host__ __device__ inline bool scan256_layout(bool bf16, int dk, int dv) { return bf16 && dk == 256 && dv == 256; }
bool scan256_tc_supported(const Dims& d);
cudaError_t launch_scan256_tc(const Dims& d, const Inputs& in, const Work& w, cudaStream_t s);
// out[M, N] = y[M, K] w[K, N] (bf16 operands, fp32 accumulation), tensor cores (vdn_gemm_tc.cu);
// scales != nullptr: e4m3 y [M, K] and w [N, K], dequantisation scales {s_y, s_w} in device memory
vdn_status out_proj(int M, int K, int N, int out_dtype, const void* y, const void* w, void* out, cudaStream_t s,
                    const float* scales = nullptr);
// device address of the projection's status words (library-owned), or null
uint32_t* status_of_proj();
vdn_status quantize_fp8(const void* x, int dtype, long long n, void* q, float* scale, cudaStream_t s);
// The chunk-composed scan where it helps: the compositions (one CTA per
// chunk, batch-head and direction) take about one wave of the SMs, and then
// the sequential chain is 5x shorter; with more chains than that the frame
// scan already fills the GPU and the composition is extra work.
inline bool use_chunk_scan(const Dims& d, int sms) {
  if (d.scan_mode != 0) return d.scan_mode == 2;
  return d.C >= 4 && 2LL * d.B * d.C * d.H <= sms;
}
cudaError_t launch_read_tc(const Dims& d, const Inputs& in, const Work& w, void* r16, cudaStream_t s);

// Backward of the linear branch (vdn_lin_bwd.cu): outputs and scratch
struct LinBwdArgs {
  const void* dy;  // gradient of y, y's layout and dtype (the linear slot is read)
  float *dq, *dk, *dv, *dbeta, *dalpha, *dgate, *drms, *dfwd;  // drms, dfwd may be null
  void* workspace;
  uint32_t* status;  // bounded-wait status words of the tensor-core kernels (cleared by the caller)
};
// bytes of the backward's scratch; off[0..5] (if not null) get the offsets of
// the all-frame states F, G, the per-frame dR, dXf, dXb and the RMS partials
size_t lin_bwd_workspace(const Dims& d, size_t* off);
cudaError_t launch_lin_bwd(const Dims& d, const Inputs& in, const Work& w, const LinBwdArgs& a, cudaStream_t s);
// its per-token step on the tensor cores (vdn_lin_bwd_tc.cu): bf16 k, v, d = 64 or 128;
// dAs = dA + dA^T and dB per frame-head [B,T,H,d,d]; clears and fills dbeta
bool bwd_tokens_tc_supported(const Dims& d);
// its read step on the tensor cores (vdn_lin_bwd_read_tc.cu): bf16, d = 128;
// Fst/Gst every state [B,H,T+1,d,d]; writes dq, dgate, dRp [B,T,H,d,d] and
// (if dwp) the RMS weight partials [B,T,H,d]
bool bwd_read_tc_supported(const Dims& d);
cudaError_t launch_bwd_read_tc(const Dims& d, const Inputs& in, const float* Fst, const float* Gst, const void* dy,
                               float* dq, float* dgate, float* dRp, float* dwp, uint32_t* status, cudaStream_t s);
cudaError_t launch_bwd_tokens_tc(const Dims& d, const Inputs& in, const float* dAs, const float* dB, float* dk,
                                 float* dv, float* dbeta, uint32_t* status, cudaStream_t s);

// Backward of the windowed softmax branch (vdn_sm_bwd.cu)
struct SmBwdArgs {
  const void* dy;  // gradient of y, y's layout and dtype (the softmax slot is read)
  float *dq, *dk, *dv, *dgate;
  void* workspace;
};
// bytes of its scratch (dO, LSE, Delta per query row); off[0..2] the offsets
size_t sm_bwd_workspace(const Dims& d, size_t* off);
cudaError_t launch_sm_bwd(const Dims& d, const Inputs& in, const SmBwdArgs& a, cudaStream_t s);
// its tensor-core form (vdn_sm_bwd_tc.cu): bf16 inputs, d = 64 or 128; fp16
// operands (exact copies of q, k, v; P, dS and a power-of-two scaled dO rounded)
struct SmTcArgs {
  const void* dy;
  float *dq, *dk, *dv, *dgate;
  void *q16, *k16, *v16, *dO16;  // [B*T*N, H, D] fp16 scratch
  float *lse2, *delta;           // [B*T*N, H] scratch
  unsigned* amax;                // max |dO| (cleared by the caller)
  uint32_t* status;              // bounded-wait status words (cleared by the caller)
  const float* lse_in;           // the forward's softmax log-sum-exp [B*T*N, H], or null
};
bool sm_bwd_tc_supported(const Dims& d);
// bytes of its scratch; off[0..7] (if not null): status, q16, k16, v16, dO16, lse2, delta, amax
size_t sm_bwd_tc_workspace(const Dims& d, size_t* off);
cudaError_t launch_sm_bwd_tc(const Dims& d, const Inputs& in, const SmTcArgs& a, cudaStream_t s);

}  // namespace vdn
