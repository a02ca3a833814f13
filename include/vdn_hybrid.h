/*
 * vdn_hybrid.h -- C ABI of the Video DeltaNet hybrid attention core on one
 * NVIDIA B200 (sm_100a).
 *
 * What it computes (sources: the PaperDaily digest "伯克利与Impossible视频生成:
 * 14.3秒视频6.70秒去噪", sections 二, 三 and 四; the deepmagic.app post
 * "生成比播放還快", section "用兩條分支取代一條"; the aimodeling.com news
 * "video-deltanet-h3-hybrid-attention", section "The VDN split"):
 *
 *   Video Delta Attention (linear branch).  For every non-anchor frame t and
 *   head, over the N tokens of the frame,
 *       A_t = sum_i beta_i k_i k_i^T,   B_t = sum_i beta_i v_i k_i^T,
 *       S_t = (alpha_t S_{t-1} + B_t) (I + A_t)^{-1},
 *   run forward (frames 0..T-1) and backward (T-1..0), both started from half
 *   of the text state S_x = B_x (I + A_x)^{-1} (one joint solve over the L text
 *   tokens).  The first and last frame (the anchors) are not written.  A query
 *   in chunk c = floor(t / 5) reads the forward state over frames < 5(c-1) plus
 *   the backward state over frames >= 5(c+2): o_lin = R q.  Anchor query frames
 *   read the two initial states (S_x).  Then
 *       y_lin = sigmoid(g_lin) * o_lin / sqrt(mean(o_lin^2) + eps) [* w].
 *
 *   Windowed softmax.  A query in chunk c attends to the keys of chunks
 *   c-1, c, c+1 (clipped at the ends), every query sees the anchor frames and
 *   anchor queries see every frame:  y_sm = sigmoid(g_sm) * softmax(s q K^T) V.
 *
 *   The backward of both branches (vdn_hybrid_lin_bwd, vdn_hybrid_sm_bwd, and
 *   the two together, summed, in vdn_hybrid_bwd) is the exact derivative of
 *   the forward above; the pages describe the forward only.
 *
 * Conventions for every entry point:
 *   - Ownership: the library allocates nothing.  The caller owns every input,
 *     the output and the workspace; all data pointers are DEVICE pointers on the
 *     current CUDA device, all struct pointers are HOST pointers read during the
 *     call only.
 *   - Asynchrony: work is enqueued on `stream` (NULL = legacy default stream)
 *     and the call returns without synchronising.  A forward call that runs the
 *     text and frame-write stages together on a large problem (B*T*H >= 1024,
 *     text tokens present, `stream` not capturing) runs the text stage on a
 *     stream it creates for that call, which first waits for `stream` and which
 *     `stream` waits for before the scans: the work stays ordered on `stream`.
 *   - Errors: arguments are validated before any launch; a status other than
 *     VDN_OK from validation means nothing was enqueued.  A launch failure is
 *     VDN_ERR_CUDA (the CUDA error is left for cudaGetLastError).
 *   - Aliasing: inputs are read-only; `y` and `workspace` must not overlap any
 *     input or each other.
 *   - Layouts are dense, row-major, innermost dimension last, no padding.
 */
#ifndef VDN_HYBRID_H
#define VDN_HYBRID_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so that the header needs no CUDA headers. */
typedef struct CUstream_st *vdn_stream_t;

typedef enum {
  VDN_OK = 0,
  VDN_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad enum, misaligned pointer */
  VDN_ERR_UNSUPPORTED = 2, /* a valid configuration this build does not implement (d, chunk) */
  VDN_ERR_WORKSPACE = 3,   /* workspace missing or smaller than vdn_hybrid_attn_workspace_size */
  VDN_ERR_CUDA = 4,        /* a CUDA call or launch failed */
  VDN_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (see vdn_hybrid_device_status) */
} vdn_status;

typedef enum {
  VDN_F32 = 0,  /* q, k, v, gates, text k/v in float32; exact mode (SIMT fp32 arithmetic) */
  VDN_BF16 = 1  /* the same tensors in bfloat16; fp32 accumulation and fp32 state */
} vdn_dtype;

typedef struct {
  int B;        /* batch (independent problems)                                   >= 1 */
  int T;        /* latent frames                                                  >= 2 */
  int N;        /* spatial tokens per frame                                       >= 1 */
  int H;        /* heads                                                          >= 1 */
  int d_k;      /* key/query head dim: 32, 64, 128 or 256.  256 needs dtype VDN_BF16
                   and runs the Video Delta Attention stages only (TEXT, SOLVE, SCAN,
                   READ); a call that includes VDN_STAGE_SOFTMAX returns
                   VDN_ERR_UNSUPPORTED without launching                            */
  int d_v;      /* value head dim; must equal d_k in this build                        */
  int L;        /* text tokens; 0 = no text (states start from init_state or zero)     */
  int chunk;    /* latent frames per chunk; must be 5                                  */
  int anchors;  /* 0 = no anchors, 4 = 4-way first/last-frame anchors                   */
  int dtype;    /* vdn_dtype                                                           */
  float softmax_scale; /* <= 0 selects 1/sqrt(d_k)                                    */
  float rms_eps;       /* <= 0 selects 1e-6                                            */
  int out_mode;        /* 0: y[B,T,N,H,2,d_v], slot 0 = softmax, slot 1 = linear;
                          1: y[B,T,N,H,d_v] = sum of the two gated branches           */
  int y_dtype;         /* vdn_dtype of y: VDN_F32 (default, also in bf16 mode) or
                          VDN_BF16 (rounded to nearest even on store)                  */
  int scan_mode;       /* how the tensor-core scan (VDN_BF16, d = 128) steps: 0 = auto,
                          1 = by frames, 2 = by chunks with composed chunk maps (the
                          frames of a chunk composed first, then one step per chunk).
                          Auto takes chunks when there are at least 4 and the 2*B*C*H
                          compositions fit one wave of the GPU's SMs (few chains, long
                          sequences), frames otherwise.  Other configurations step by
                          frames whatever the mode.                                    */
  int update;          /* the per-frame write of the linear branch: 0 = the joint
                          solve S_t = (alpha S + B_t)(I + A_t)^-1 (Video DeltaNet);
                          ablation baselines the pages compare it with (deepmagic
                          post, its Video Delta Attention paragraph; aimodeling
                          news, "The VDN split"): 1 = frame-level independent writes
                          against the frozen inherited state, rescaled by the frame
                          size (SANA-WM): S_t = S_bar (I - A_t/N) + B_t/N; 2 = the
                          token-wise delta rule, tokens written one after another
                          in token order.  The text state is the joint solve's in
                          every mode.  Modes 1 and 2 run the SIMT scan and need
                          d_k <= 128 (VDN_ERR_UNSUPPORTED otherwise)                 */
} vdn_hybrid_cfg;

typedef struct {
  const void *q, *k, *v;           /* [B,T,N,H,d_k] ([..,d_v] for v), dtype              */
  const float *beta;               /* [B,T,N,H]   write strengths (> 0)                  */
  const float *alpha;              /* [B,T,H]     decay gates in [0, 1]                  */
  const void *gate_sm, *gate_lin;  /* [B,T,N,H,d_v] gate logits, dtype                   */
  const void *text_k, *text_v;     /* [B,L,H,d_k] / [B,L,H,d_v], dtype; NULL iff L == 0   */
  const float *text_beta;          /* [B,L,H];  NULL iff L == 0                           */
  const float *init_state;         /* [B,H,d_v,d_k] full text state S_x used instead of a
                                      text solve (each direction starts from S_x / 2);
                                      only allowed with L == 0; NULL = zero state          */
  const float *rms_weight;         /* [H,d_v] RMSNorm weight, NULL = ones                 */
  void *y;                         /* output, cfg.y_dtype, shape per cfg.out_mode; every
                                      array pointer is 16-byte aligned, and a 32-byte
                                      aligned y lets the state read use its tensor-core
                                      kernel (same results either way)                    */
  void *workspace;                 /* device scratch, 256-byte aligned                   */
  size_t workspace_bytes;
  const float *fwd_init;           /* [B,H,d_v,d_k] streaming: the forward scan's start
                                      state (the forward state the previous segment ended
                                      with, slot C of its fwd_snap), carried across
                                      appended chunks of a live stream (Video DeltaNet,
                                      the livestream setting of the abstract).  NULL =
                                      half the text state, as the backward scan always
                                      starts.  Anchor query frames then read
                                      fwd_init + S_x / 2.  16-byte aligned, outside the
                                      workspace.                                           */
  float *sm_lse;                   /* [B,T,N,H] optional output of the forward's softmax
                                      stage: ln sum_j exp(s q k_j) over each query row's
                                      allowed keys, float32, 4-byte aligned; NULL = not
                                      written.  vdn_hybrid_sm_bwd takes it (grads->sm_lse)
                                      to skip recomputing the row statistics.              */
} vdn_hybrid_args;

/* Pipeline stages; vdn_hybrid_attn_fwd runs VDN_STAGE_ALL in this order. */
enum {
  VDN_STAGE_TEXT = 1u,   /* text solve (or init_state copy) -> half text state       */
  VDN_STAGE_SOLVE = 2u,  /* per-frame Gram/write + SPD solve -> M_t, C_t              */
  VDN_STAGE_SCAN = 4u,   /* forward/backward state scans -> chunk-boundary states     */
  VDN_STAGE_SOFTMAX = 8u,/* windowed softmax + gate -> y slot 0 (or y)                */
  VDN_STAGE_READ = 16u,  /* state read + RMSNorm + gate -> y slot 1 (or y += )        */
  VDN_STAGE_ALL = 31u,
  VDN_STAGE_SOFTMAX_BWD = 32u /* not a forward stage: vdn_hybrid_stage_impl's key for the
                                 softmax branch's backward (vdn_hybrid_sm_bwd)            */
};

/* Byte offsets of the intermediate values inside the workspace (float32
 * unless noted, dense).  C = ceil(T / chunk).  Stable across calls with the same cfg, so that
 * a caller can inspect the stages.
 *   status     : uint32 device status words (VDN_ERR_TIMEOUT flags)
 *   half_text  : [B,H,d_v,d_k]        S_x / 2, the start state of both scans
 *   frame_M    : [B,T,H,d_k,d_k]      (I + A_t)^{-1}        (anchor frames unset)
 *   frame_C    : [B,T,H,d_v,d_k]      C_t = B_t (I + A_t)^{-1}  (anchor frames unset); with the
 *                                     tensor-core scan (bf16, d = 128) and at d = 256 the write
 *                                     matrix B_t itself, since those scans step
 *                                     S <- (alpha_t S + B_t) M_t
 *   fwd_snap   : [B,H,C+1,d_v,d_k]    forward state over frames < min(5j, T)
 *   bwd_snap   : [B,H,C+1,d_v,d_k]    backward state over frames >= min(5j, T)
 *   read_table : [B,H,C+1,d_v,d_k]    R[c] = fwd_snap[max(c-1,0)] + bwd_snap[min(c+2,C)],
 *                                     R[C] = half_text * 2 (anchor query frames)
 *   read_table_bf16 : [B,H,C+1,2,d_v,d_k] bfloat16 hi/lo split of read_table,
 *                                     R_hi = bf16(R), R_lo = bf16(R - R_hi) (operand of
 *                                     the tensor-core read; written only on that path)
 *   text_gram  : [B,H,2,d,d]          A_x, B_x of the text tokens (tensor-core text
 *                                     path only)
 *   frame_M16  : [B,T,H,2,d,d]        bfloat16 hi/lo split of frame_M, the operand of the
 *                                     tensor-core scans (bf16 inputs with d = 128 or 256;
 *                                     an empty region otherwise)
 *   chunk_P16  : [B,C,H,2,d,d]        chunk maps (bf16, d = 128 only): bfloat16 hi/lo split of
 *                                     P_c = M_f1 ... M_fn over the chunk's written frames
 *   chunk_C    : [2,B,C,H,d_v,d_k]    the forward and backward constants Cf_c, Cb_c: the
 *                                     frames of chunk c map a state S to Lam_c S P_c + Cf_c
 *                                     (increasing order), Lam_c S P_c^T + Cb_c (decreasing)
 *   chunk_lam  : [B,C,H]              Lam_c, the product of the chunk's alpha_t
 *   The chunk maps are written when the scan steps by chunks (C >= 4), and left
 *   unset otherwise.                                                                     */
typedef struct {
  size_t status, half_text, frame_M, frame_C, fwd_snap, bwd_snap, read_table, read_table_bf16, text_gram, frame_M16,
      chunk_P16, chunk_C, chunk_lam, total;
} vdn_workspace_layout;

/* Bytes of workspace the configuration needs; 0 if cfg is invalid. */
size_t vdn_hybrid_attn_workspace_size(const vdn_hybrid_cfg *cfg);

/* Fill *out with the workspace layout of cfg.  Errors: VDN_ERR_INVALID_ARG,
 * VDN_ERR_UNSUPPORTED. */
vdn_status vdn_hybrid_workspace_layout(const vdn_hybrid_cfg *cfg, vdn_workspace_layout *out);

/* The whole hybrid attention core: all stages, in order, on `stream`. */
vdn_status vdn_hybrid_attn_fwd(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args,
                               vdn_stream_t stream);

/* A subset of the stages (bitwise OR of VDN_STAGE_*), in pipeline order.
 * Each stage reads what the earlier stages left in the workspace; running a
 * stage whose inputs were never produced gives unspecified (but in-bounds)
 * results.  Used to time and check the stages one by one. */
vdn_status vdn_hybrid_attn_fwd_stages(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args,
                                      unsigned stages, vdn_stream_t stream);

/* The whole core without a caller workspace, for callers that cannot
 * allocate device memory where they run it: runtimes that forbid allocation
 * after start-up, and plug-ins of another framework that are handed only their
 * input and output buffers.  The pages have no counterpart of this entry
 * point; it is a deployment convenience of this library.
 * Scratch: a library-owned device array of VDN_NOALLOC_SCRATCH_BYTES (static
 * storage on every GPU that loads the library, held until the process exits).
 * Those 16 MiB are reserved on each device where the library's module is
 * loaded, whether or not this entry point is ever called; CUDA_MODULE_LOADING
 * decides when that happens (at context creation when eager, at the library's
 * first kernel launch or symbol lookup on that device when lazy).
 * Arguments are those of vdn_hybrid_attn_fwd, except that args->workspace must
 * be NULL and args->workspace_bytes 0 (else VDN_ERR_INVALID_ARG).  A cfg whose
 * workspace (vdn_hybrid_attn_workspace_size) exceeds VDN_NOALLOC_SCRATCH_BYTES
 * returns VDN_ERR_WORKSPACE and launches nothing.
 * Set-up: every call looks up the array's device address in the current
 * device's context (so the address stays right after a device reset, which
 * may move the array); the first call on a device may load the module, so
 * make that first call before any stream capture.
 * Sharing: every call uses the same array, which keeps the last call's
 * contents (each call clears what must start at zero); calls whose work
 * overlaps on the GPU race on it and must be serialised by the caller.  The
 * device status words of the last call on the current device are read by
 * vdn_hybrid_noalloc_device_status. */
#define VDN_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
vdn_status vdn_hybrid_attn_fwd_noalloc(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args,
                                       vdn_stream_t stream);

/* Device status of the last vdn_hybrid_attn_fwd_noalloc call on the current
 * device (the first words of the library-owned array): VDN_OK, or
 * VDN_ERR_TIMEOUT if a bounded wait of one of its kernels gave up (its output
 * is then incomplete), with the kernel's VDN_TAG_* in *where (if not NULL).
 * Synchronises `stream` (give the stream of that call); VDN_ERR_CUDA if the
 * read fails. */
vdn_status vdn_hybrid_noalloc_device_status(vdn_stream_t stream, unsigned *where);

/* Kernel tags: which kernel's bounded wait gave up (vdn_hybrid_device_status). */
enum {
  VDN_TAG_NONE = 0,
  VDN_TAG_SOFTMAX = 1,      /* windowed softmax (and the text cross-attention)  */
  VDN_TAG_GRAM = 2,         /* per-frame and text Gram / write                  */
  VDN_TAG_READ = 3,         /* state read + RMSNorm + gate                      */
  VDN_TAG_SCAN = 4,         /* state scans                                      */
  VDN_TAG_COMPOSE = 5,      /* chunk composition                                */
  VDN_TAG_SOFTMAX_BWD = 6,  /* softmax branch backward                          */
  VDN_TAG_LINEAR_BWD = 7,   /* linear branch backward                           */
  VDN_TAG_PROJ = 8          /* output projection (vdn_proj_device_status)       */
};

/* Reads the device status words left by the most recent call on this
 * workspace (every fwd / fwd_stages call clears them first; synchronises `stream`).
 * Returns VDN_OK or VDN_ERR_TIMEOUT; *where (if not NULL) gets the VDN_TAG_* of
 * the kernel that gave up. */
vdn_status vdn_hybrid_device_status(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args,
                                    vdn_stream_t stream, unsigned *where);

/* Failure-path test hook (no counterpart on the pages).  Sets, on the current
 * device, the wait limit in SM clock cycles of the state read's epilogue warps
 * (the tensor-core read kernel at d = 64 or 128: the warps that wait for the
 * tensor cores' products); 0 restores the default of every bounded wait
 * (about one second).  With a limit shorter than the products take, those
 * waits run out: the kernel records VDN_ERR_TIMEOUT and VDN_TAG_READ in the
 * workspace status words, its producer and MMA roles stop issuing and drain
 * what they issued, and the CTAs exit with their rows of y's linear slot
 * unwritten (vdn_hybrid_device_status then reports the timeout; the context
 * stays usable).  Synchronous and not stream-ordered: call it with no work of
 * this library in flight on the device.  Errors: VDN_ERR_INVALID_ARG (cycles
 * above the default limit), VDN_ERR_CUDA. */
vdn_status vdn_debug_set_read_wait_limit(unsigned long long cycles);

/* Which implementation a stage uses for cfg: 0 = SIMT fp32, 1 = tcgen05 tensor
 * cores (TMA + TMEM), 2 = the ablation variants' per-frame map kernel (SOLVE
 * with cfg.update != 0), -1 = stage not supported for cfg.  Also answers for
 * VDN_STAGE_SOFTMAX_BWD, the softmax branch's backward. */
int vdn_hybrid_stage_impl(const vdn_hybrid_cfg *cfg, unsigned stage);

/* Static description of a status code. */
const char *vdn_status_string(vdn_status s);

/* ------------------------------------------------ backward of the linear branch
 * Gradients of a loss through the Video Delta Attention branch (its forward as
 * defined at the top of this header: PaperDaily digest sections 三 and 四,
 * deepmagic post closed form S_t = (alpha_t S + B_t)(I + A_t)^-1, RMSNorm and
 * gate of section 三).  The pages describe the forward only; the gradient is
 * that forward's exact derivative.  Given dy = dL/dy for the core's output,
 * the call writes dL/dq, dL/dk, dL/dv, dL/dbeta, dL/dalpha and dL/dgate_lin as
 * far as they flow through y's LINEAR slot (out_mode 0: slot 1 of dy is read;
 * out_mode 1: dy itself), plus dL/drms_weight and dL/dfwd_init if asked.  The
 * text state (text_k / text_v / text_beta, init_state) is a constant here.
 * The softmax branch's share of dq, dk, dv is not included.
 *
 * Precondition: args->workspace holds what vdn_hybrid_attn_fwd (or at least its
 * TEXT and SOLVE stages) wrote for the same cfg and the same inputs: M_t, the
 * write matrices and S_x / 2 are taken from there, not recomputed.
 * Reads cfg (update must be 0, d_k 32, 64 or 128 and T at most 65535, else
 * VDN_ERR_UNSUPPORTED)
 * and args q, k, v, beta, alpha, gate_lin, rms_weight, fwd_init, workspace
 * (y, gate_sm and the text pointers are ignored).  Computes in fp32: SIMT
 * kernels, except the per-token products, which run on the tensor cores for
 * VDN_BF16 inputs (the fp32 d x d factors and dO as bf16 hi + lo pairs): the
 * frame write's gradient (dk, dv, dbeta) at d_k 64 or 128, and the read's
 * (o again, dq, the per-frame dR) at d_k 128.  The call clears
 * and uses the status words at the head of args->workspace
 * (vdn_hybrid_device_status reads them). */
typedef struct {
  const void *dy;      /* dL/dy in y's shape (per cfg.out_mode) and cfg.y_dtype; 16-byte aligned */
  float *dq, *dk, *dv; /* [B,T,N,H,d] float32, overwritten; anchor frames' dk, dv are zero    */
  float *dbeta;        /* [B,T,N,H]   float32, overwritten                                   */
  float *dalpha;       /* [B,T,H]     float32, overwritten (zero at anchor frames)            */
  float *dgate_lin;    /* [B,T,N,H,d_v] float32, overwritten                                 */
  float *drms_weight;  /* [H,d_v] float32 or NULL; also when args->rms_weight is NULL (the
                          gradient at weight = ones)                                         */
  float *dfwd_init;    /* [B,H,d_v,d_k] float32 or NULL: dL/d(forward start state), i.e.
                          of args->fwd_init, or of S_x / 2 when that is NULL                  */
  void *workspace;     /* backward scratch, 256-byte aligned, no overlap with anything else  */
  size_t workspace_bytes; /* >= vdn_hybrid_lin_bwd_workspace_size(cfg)                       */
} vdn_lin_grads;

/* Bytes of backward scratch for cfg: every state of both scans and four
 * d x d matrices per frame-head (0.7 GB at B=1, T=90, H=24, d=128); 0 if cfg
 * is invalid or not supported by the backward. */
size_t vdn_hybrid_lin_bwd_workspace_size(const vdn_hybrid_cfg *cfg);

/* Enqueue the backward on `stream` (no synchronisation, no allocation).
 * Errors (nothing enqueued): VDN_ERR_INVALID_ARG (a NULL or misaligned pointer:
 * 16 bytes for q, k, v, gate_lin, dy, dq, dk, dv, dgate_lin, fwd_init,
 * dfwd_init; 4 for the others), VDN_ERR_UNSUPPORTED, VDN_ERR_WORKSPACE (either
 * workspace missing, misaligned or too small); VDN_ERR_CUDA for a launch
 * failure. */
vdn_status vdn_hybrid_lin_bwd(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args, const vdn_lin_grads *grads,
                              vdn_stream_t stream);

/* ----------------------------------------------- backward of the softmax branch
 * Gradients through the windowed softmax branch (defined at the top of this
 * header: PaperDaily digest section 二, the anchors of the deepmagic post and
 * the aimodeling news): given dy = dL/dy, the call writes dL/dq, dL/dk, dL/dv
 * and dL/dgate_sm as far as they flow through y's SOFTMAX slot (out_mode 0:
 * slot 0 of dy; out_mode 1: dy itself).  With vdn_hybrid_lin_bwd the two
 * branches' shares of dq, dk and dv add up to the whole core's gradient.
 * The exact derivative of the forward (the pages describe the forward only).
 * Reads cfg (update 0, d_k 32, 64 or 128 and T at most 65535, else
 * VDN_ERR_UNSUPPORTED) and
 * args q, k, v, gate_sm (the other pointers, the forward's workspace and its
 * output are not read: the softmax statistics and o are recomputed).  Two
 * implementations, chosen by cfg (vdn_hybrid_stage_impl(cfg,
 * VDN_STAGE_SOFTMAX_BWD) says which):
 *   - tensor cores (tcgen05) when dtype is VDN_BF16 and d_k is 64 or 128: the
 *     products take fp16 operands with fp32 accumulation.  q, k, v are copied
 *     to fp16 exactly (their magnitudes must stay below 65504); P, dS and dO
 *     are rounded to fp16, dO after scaling by one power of two per call (so
 *     that small upstream gradients keep their precision).  The status words of
 *     its bounded waits sit in the first 256 bytes of grads->workspace: read
 *     them with vdn_hybrid_device_status called with args->workspace set to
 *     grads->workspace;
 *   - otherwise SIMT fp32. */
typedef struct {
  const void *dy;      /* dL/dy in y's shape (per cfg.out_mode) and cfg.y_dtype; 16-byte aligned */
  float *dq, *dk, *dv; /* [B,T,N,H,d] float32, overwritten                                     */
  float *dgate_sm;     /* [B,T,N,H,d_v] float32, overwritten                                   */
  void *workspace;     /* scratch (status words, operand copies, dO, log-sum-exp and <dO, o> per
                          query row); 256-byte aligned                                        */
  size_t workspace_bytes; /* >= vdn_hybrid_sm_bwd_workspace_size(cfg)                           */
  const float *sm_lse; /* [B,T,N,H] or NULL: the forward's args->sm_lse for these inputs.  On the
                          tensor-core path it replaces the pass that recomputes each row's
                          maximum score (the log-sum-exp bounds every score, so it serves as the
                          exponent reference; the row sums are still formed here); the SIMT
                          path does not read it.  4-byte aligned                               */
} vdn_sm_grads;

/* Bytes of scratch for cfg (the larger of its two layouts: four fp16 rows of d and two
 * floats per query row and head, plus 512 bytes, for the tensor cores; each
 * region 256-byte aligned); 0 if cfg is invalid or
 * not supported. */
size_t vdn_hybrid_sm_bwd_workspace_size(const vdn_hybrid_cfg *cfg);

/* Enqueue the softmax branch's backward on `stream`.  Errors (nothing
 * enqueued): VDN_ERR_INVALID_ARG (a NULL or a not 16-byte aligned pointer),
 * VDN_ERR_UNSUPPORTED, VDN_ERR_WORKSPACE (grads->workspace missing,
 * misaligned or too small); VDN_ERR_CUDA for a launch failure. */
vdn_status vdn_hybrid_sm_bwd(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args, const vdn_sm_grads *grads,
                             vdn_stream_t stream);

/* ------------------------------------------------------ backward of the core
 * The whole core's gradient in one call: the exact derivative of the forward
 * at the top of this header (both branches; the pages describe the forward
 * only).  Given dy = dL/dy in y's shape and dtype, it writes dL/dq, dL/dk and
 * dL/dv with the two branches' shares summed on the device, and the
 * branch-specific gradients: dbeta, dalpha and dgate_lin (linear branch),
 * dgate_sm (softmax branch), and drms_weight and dfwd_init where asked.
 * Equivalent to vdn_hybrid_sm_bwd followed by vdn_hybrid_lin_bwd and a sum,
 * without the extra buffers: the softmax branch runs first and writes dq, dk,
 * dv; the linear branch then adds its share into them.
 *
 * Precondition, arguments and computation as for those two entry points (the
 * forward's workspace in args->workspace for the linear branch; the forward's
 * log-sum-exp in sm_lse, optional, for the softmax branch's tensor-core path).
 * Scratch: one region of vdn_hybrid_bwd_workspace_size(cfg) bytes shared by the
 * two branches in turn.  Status words of the bounded device waits: the
 * softmax branch's in the first 256 bytes of grads->workspace, the linear
 * branch's at the head of args->workspace; vdn_hybrid_device_status reads
 * either (args->workspace set to the region in question).
 * Errors (nothing enqueued): any error either branch's entry point reports
 * for the same arguments, checked for both before the first launch;
 * VDN_ERR_WORKSPACE for a missing, misaligned (256 bytes) or too small
 * grads->workspace; VDN_ERR_CUDA for a launch failure. */
typedef struct {
  const void *dy;      /* dL/dy in y's shape (per cfg.out_mode) and cfg.y_dtype; 16-byte aligned      */
  float *dq, *dk, *dv; /* [B,T,N,H,d] float32, overwritten with both branches' shares summed           */
  float *dbeta;        /* [B,T,N,H] float32, overwritten                                             */
  float *dalpha;       /* [B,T,H] float32, overwritten (zero at anchor frames)                        */
  float *dgate_lin;    /* [B,T,N,H,d_v] float32, overwritten                                         */
  float *dgate_sm;     /* [B,T,N,H,d_v] float32, overwritten                                         */
  float *drms_weight;  /* [H,d_v] float32 or NULL (as in vdn_lin_grads)                               */
  float *dfwd_init;    /* [B,H,d_v,d_k] float32 or NULL (as in vdn_lin_grads)                         */
  void *workspace;     /* scratch shared by the two branches, 256-byte aligned, no overlap with anything
                          else                                                                        */
  size_t workspace_bytes; /* >= vdn_hybrid_bwd_workspace_size(cfg)                                     */
  const float *sm_lse; /* [B,T,N,H] or NULL: the forward's args->sm_lse (as in vdn_sm_grads)           */
} vdn_hybrid_grads;

/* Bytes of scratch for vdn_hybrid_bwd: the larger of the softmax branch's scratch
 * and 256 bytes plus the linear branch's; 0 if cfg is invalid or not
 * supported by the backward. */
size_t vdn_hybrid_bwd_workspace_size(const vdn_hybrid_cfg *cfg);

/* Enqueue the whole core's backward on `stream` (no synchronisation, no
 * allocation). */
vdn_status vdn_hybrid_bwd(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args, const vdn_hybrid_grads *grads,
                          vdn_stream_t stream);

/* ------------------------------------------------------- text cross-attention
 * The DiT block's softmax cross-attention from the video tokens to the text
 * tokens (PaperDaily digest section 三: text enters the block both through the
 * states' initialisation and through cross-attention): for every video query
 * of batch b and head h, o = softmax(s q K_b^T) V_b over that batch's L text
 * tokens (no mask, no gate), s = cfg.softmax_scale (<= 0: 1/sqrt(d_k)).
 * Reads cfg B, T, N, H, d_k = d_v (64 or 128), L >= 1, dtype (VDN_BF16 only),
 * softmax_scale, y_dtype; args q [B,T,N,H,d_k], text_k [B,L,H,d_k],
 * text_v [B,L,H,d_v], y = the output o [B,T,N,H,d_v] in y_dtype, and the first
 * 256 bytes of workspace (status words, read by vdn_hybrid_device_status);
 * the other pointers are ignored.  On the tensor cores (the windowed softmax's
 * kernel with one key interval).  Errors: VDN_ERR_INVALID_ARG (L = 0, a NULL or
 * misaligned pointer), VDN_ERR_WORKSPACE (workspace NULL, misaligned or under
 * 256 bytes), VDN_ERR_UNSUPPORTED (fp32 inputs, d not 64 or 128). */
vdn_status vdn_text_cross_attn(const vdn_hybrid_cfg *cfg, const vdn_hybrid_args *args, vdn_stream_t stream);

/* ------------------------------------------------ the layer's output projection
 * PaperDaily digest section 三: each branch is gated, then projected back to
 * the model width.  With the core's output in out_mode 0 (y[B,T,N,H,2,d_v],
 * slot 0 softmax, slot 1 linear), one GEMM with the stacked weight equals the
 * sum of the two separate projections:
 *   out[m, n] = sum_k y[m, k] w[k, n],   y viewed as [M = B*T*N, K = H*2*d_v]
 * with row k = (h * 2 + slot) * d_v + i of w the weight of that output element. */
typedef struct {
  int M;          /* rows (tokens)                                                    >= 1 */
  int K;          /* the per-token output block, H*2*d_v; a multiple of 8           >= 8 */
  int N;          /* output width; a multiple of 8                                     >= 8 */
  int out_dtype;  /* vdn_dtype of out: VDN_F32 or VDN_BF16 (rounded to nearest even)       */
} vdn_proj_cfg;

/* out = y w on `stream`: y bfloat16 [M, K] row-major (the core's output with
 * y_dtype VDN_BF16), w bfloat16 [K, N] row-major, out [M, N] row-major in
 * out_dtype; fp32 accumulation.  Device pointers, 16-byte aligned, no overlap
 * of out with y or w.  On the tensor cores (tcgen05, pairs of CTAs on 256 x 256
 * output tiles); no workspace, nothing allocated.  The bounded waits of its
 * kernel record a timeout in library-owned status words (vdn_proj_device_status).
 * Calls that overlap on the GPU share those words.  Errors: VDN_ERR_INVALID_ARG
 * (a NULL or misaligned pointer, sizes), VDN_ERR_UNSUPPORTED (more than 2^30
 * output tiles), VDN_ERR_CUDA. */
vdn_status vdn_out_proj(const vdn_proj_cfg *cfg, const void *y, const void *w, void *out, vdn_stream_t stream);

/* ------------------------------------------------------------ FP8 linear layers
 * deepmagic post "生成比播放還快", section 實測數據: the per-block latency reaches
 * its lowest figure once optimized kernels and FP8 linear layers are added.  Tensors go to
 * FP8 E4M3 with one scale per tensor, s = amax|x| / 448 (the largest finite
 * e4m3; 1 for an all-zero tensor), q = e4m3(x * (1 / s)) rounded to nearest
 * even and saturated, so that x ~ q * s. */

/* q[i] = e4m3(x[i] / s) for the n elements of x (x_dtype VDN_F32 or VDN_BF16),
 * and s into *scale, all on `stream` (device pointers; x and q 16-byte aligned).
 * Errors: VDN_ERR_INVALID_ARG (NULL or misaligned pointers, n = 0, a dtype),
 * VDN_ERR_CUDA. */
vdn_status vdn_quantize_fp8(const void *x, int x_dtype, size_t n, void *q, float *scale, vdn_stream_t stream);

/* The output projection with e4m3 operands: out[M, N] = (s_y y)(s_w w) with y
 * e4m3 [M, K] row-major, the weight given TRANSPOSED as w_t e4m3 [N, K]
 * row-major (FP8 tensor-core GEMMs take both operands K-contiguous), scales =
 * {s_y, s_w} (two floats in device memory, e.g. as written by
 * vdn_quantize_fp8), out in cfg->out_dtype; fp32 accumulation on the tensor
 * cores (tcgen05 kind::f8f6f4, the scales applied in the epilogue), no
 * workspace.  K and N multiples of 16.  Errors as vdn_out_proj. */
vdn_status vdn_out_proj_fp8(const vdn_proj_cfg *cfg, const void *y, const void *w_t, const float *scales, void *out,
                            vdn_stream_t stream);

/* Status of the last vdn_out_proj / vdn_out_proj_fp8 on the current device
 * (synchronises `stream`): VDN_OK, or VDN_ERR_TIMEOUT when a bounded wait of its
 * kernel gave up (the output is then incomplete); *where (if not NULL) gets
 * VDN_TAG_PROJ or VDN_TAG_NONE.  Errors: VDN_ERR_CUDA. */
vdn_status vdn_proj_device_status(vdn_stream_t stream, unsigned *where);

#ifdef __cplusplus
}
#endif
#endif /* VDN_HYBRID_H */
