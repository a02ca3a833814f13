// C ABI entry points: argument validation, workspace layout, stage dispatch.
#include <cstdint>
#include <cstring>

#include "vdn_internal.h"

namespace vdn {

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

vdn_status check_cfg(const vdn_hybrid_cfg* c) {
  if (!c) return VDN_ERR_INVALID_ARG;
  if (c->B < 1 || c->T < 2 || c->N < 1 || c->H < 1 || c->L < 0) return VDN_ERR_INVALID_ARG;
  if (c->d_k < 1 || c->d_v < 1 || c->chunk < 1) return VDN_ERR_INVALID_ARG;
  if (c->anchors != 0 && c->anchors != 4) return VDN_ERR_INVALID_ARG;
  if (c->dtype != VDN_F32 && c->dtype != VDN_BF16) return VDN_ERR_INVALID_ARG;
  if (c->out_mode != 0 && c->out_mode != 1) return VDN_ERR_INVALID_ARG;
  if (c->y_dtype != VDN_F32 && c->y_dtype != VDN_BF16) return VDN_ERR_INVALID_ARG;
  if (c->scan_mode < 0 || c->scan_mode > 2) return VDN_ERR_INVALID_ARG;
  if (c->update < 0 || c->update > 2) return VDN_ERR_INVALID_ARG;
  if (!(c->softmax_scale == c->softmax_scale) || !(c->rms_eps == c->rms_eps)) return VDN_ERR_INVALID_ARG;
  if (c->d_k != 32 && c->d_k != 64 && c->d_k != 128 && c->d_k != 256) return VDN_ERR_UNSUPPORTED;
  if (c->d_v != c->d_k) return VDN_ERR_UNSUPPORTED;
  // d = 256: the per-frame Gram runs on the tensor cores only (bf16 inputs)
  if (c->d_k == 256 && c->dtype != VDN_BF16) return VDN_ERR_UNSUPPORTED;
  // the ablation variants run the SIMT (C-form) scan, built for d <= 128
  if (c->update != 0 && c->d_k > 128) return VDN_ERR_UNSUPPORTED;
  if (c->chunk != 5) return VDN_ERR_UNSUPPORTED;
  // grid limits of the launches (gridDim.y / gridDim.z <= 65535)
  if ((long long)c->B * c->H > 65535) return VDN_ERR_UNSUPPORTED;
  if (c->T / c->chunk + 3 > 65535) return VDN_ERR_UNSUPPORTED;
  // element counts must fit comfortably in int64 index arithmetic
  const double tokens = (double)c->B * c->T * c->N * c->H * (double)c->d_k;
  if (tokens * 2.0 > 9.0e18) return VDN_ERR_UNSUPPORTED;
  return VDN_OK;
}

Dims make_dims(const vdn_hybrid_cfg* c) {
  Dims d;
  d.B = c->B; d.T = c->T; d.N = c->N; d.H = c->H; d.dk = c->d_k; d.dv = c->d_v; d.L = c->L;
  d.chunk = c->chunk; d.anchors = c->anchors; d.C = (c->T + c->chunk - 1) / c->chunk;
  d.scale = c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / sqrtf((float)c->d_k);
  d.eps = c->rms_eps > 0.f ? c->rms_eps : 1e-6f;
  d.out_mode = c->out_mode;
  d.bf16 = c->dtype == VDN_BF16;
  d.out_bf16 = c->y_dtype == VDN_BF16;
  d.scan_mode = c->scan_mode;
  d.update = c->update;
  d.grad_acc = 0;
  return d;
}

void layout_of(const vdn_hybrid_cfg* c, vdn_workspace_layout* L) {
  const size_t C = (size_t)((c->T + c->chunk - 1) / c->chunk);
  const size_t dd = (size_t)c->d_v * c->d_k * sizeof(float);
  const size_t bh = (size_t)c->B * c->H;
  size_t off = 0;
  L->status = off;     off += up(kAlign);
  L->half_text = off;  off += up(bh * dd);
  L->frame_M = off;    off += up(bh * (size_t)c->T * (size_t)c->d_k * c->d_k * sizeof(float));
  L->frame_C = off;    off += up(bh * (size_t)c->T * dd);
  L->fwd_snap = off;   off += up(bh * (C + 1) * dd);
  L->bwd_snap = off;   off += up(bh * (C + 1) * dd);
  L->read_table = off; off += up(bh * (C + 1) * dd);
  L->read_table_bf16 = off; off += up(bh * (C + 1) * dd);  // hi and lo bf16 terms
  L->text_gram = off;  off += up(bh * 2 * dd);
  const bool tc_scan = scan_tc_layout(c->dtype == VDN_BF16, c->d_k, c->d_v);
  const size_t kk2 = 2 * (size_t)c->d_k * c->d_k * sizeof(__nv_bfloat16);  // one hi/lo split
  const bool m16 = tc_scan || scan256_layout(c->dtype == VDN_BF16, c->d_k, c->d_v);
  L->frame_M16 = off;
  if (m16) off += up(bh * (size_t)c->T * kk2);
  L->chunk_P16 = off;
  if (tc_scan) off += up(bh * C * kk2);
  L->chunk_C = off;
  if (tc_scan) off += up(2 * bh * C * dd);
  L->chunk_lam = off;
  if (tc_scan) off += up(bh * C * sizeof(float));
  L->total = off;
}

vdn_status check_args(const vdn_hybrid_cfg* c, const vdn_hybrid_args* a, unsigned stages) {
  if (!a) return VDN_ERR_INVALID_ARG;
  if ((stages & ~(unsigned)VDN_STAGE_ALL) != 0 || stages == 0) return VDN_ERR_INVALID_ARG;
  const void* req[] = {a->q, a->k, a->v, a->beta, a->alpha, a->gate_sm, a->gate_lin, a->y};
  for (const void* p : req)
    if (!p || !aligned(p, 16)) return VDN_ERR_INVALID_ARG;
  if (c->L > 0) {
    if (!a->text_k || !a->text_v || !a->text_beta || a->init_state) return VDN_ERR_INVALID_ARG;
    if (!aligned(a->text_k, 16) || !aligned(a->text_v, 16) || !aligned(a->text_beta, 4))
      return VDN_ERR_INVALID_ARG;
  } else if (a->text_k || a->text_v || a->text_beta) {
    return VDN_ERR_INVALID_ARG;
  }
  if (a->init_state && !aligned(a->init_state, 16)) return VDN_ERR_INVALID_ARG;
  if (a->rms_weight && !aligned(a->rms_weight, 4)) return VDN_ERR_INVALID_ARG;
  if (a->sm_lse && !aligned(a->sm_lse, 4)) return VDN_ERR_INVALID_ARG;
  vdn_workspace_layout L;
  layout_of(c, &L);
  if (!a->workspace || !aligned(a->workspace, kAlign) || a->workspace_bytes < L.total) return VDN_ERR_WORKSPACE;
  if (a->fwd_init) {
    // the scans overwrite the snapshot slots while they read the start state
    const char* f = static_cast<const char*>(static_cast<const void*>(a->fwd_init));
    const char* ws = static_cast<const char*>(a->workspace);
    const size_t fb = sizeof(float) * (size_t)c->B * c->H * c->d_v * c->d_k;
    if (!aligned(a->fwd_init, 16) || (f < ws + a->workspace_bytes && ws < f + fb)) return VDN_ERR_INVALID_ARG;
  }
  return VDN_OK;
}

Work work_of(const vdn_hybrid_cfg* c, const vdn_hybrid_args* a) {
  vdn_workspace_layout L;
  layout_of(c, &L);
  char* base = static_cast<char*>(a->workspace);
  Work w{};
  w.status = reinterpret_cast<uint32_t*>(base + L.status);
  w.half_text = reinterpret_cast<float*>(base + L.half_text);
  w.M = reinterpret_cast<float*>(base + L.frame_M);
  w.Cm = reinterpret_cast<float*>(base + L.frame_C);
  w.fsnap = reinterpret_cast<float*>(base + L.fwd_snap);
  w.bsnap = reinterpret_cast<float*>(base + L.bwd_snap);
  w.R = reinterpret_cast<float*>(base + L.read_table);
  w.R16 = base + L.read_table_bf16;
  w.text_gram = reinterpret_cast<float*>(base + L.text_gram);
  // the chunk maps exist for the d = 128 tensor-core scan only, M's split for both
  const bool tc_scan = scan_tc_layout(c->dtype == VDN_BF16, c->d_k, c->d_v);
  w.M16 = L.chunk_P16 > L.frame_M16 ? base + L.frame_M16 : nullptr;
  w.P16 = tc_scan ? base + L.chunk_P16 : nullptr;
  w.Cf = tc_scan ? reinterpret_cast<float*>(base + L.chunk_C) : nullptr;
  w.Cb = tc_scan ? w.Cf + (size_t)c->B * c->H * ((c->T + c->chunk - 1) / c->chunk) * c->d_v * c->d_k
                 : nullptr;
  w.lam = tc_scan ? reinterpret_cast<float*>(base + L.chunk_lam) : nullptr;
  return w;
}

// The text stage beside the frame write.  With text tokens, the text Gram
// and solve are a few dozen CTAs that the frame Gram and solve do not depend
// on (nor the reverse), so when one call runs both they go on a side stream
// (created for the call, highest priority) that waits for `s` first and that
// `s` waits for when the guard ends: the stage stays ordered on `s` like any
// other.  Not under stream capture, and not for problems too small to fill the
// GPU with the frame write.
struct TextFork {
  cudaStream_t side = nullptr;
  cudaEvent_t ev[2] = {nullptr, nullptr};
  cudaStream_t main = nullptr;
  bool forked = false;
  cudaError_t err = cudaSuccess;
  bool open(const Dims& d, cudaStream_t s) {
    if (d.L <= 0 || (long long)d.B * d.T * d.H < 1024) return false;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
      (void)cudaGetLastError();
      return false;
    }
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess ||
        cudaStreamCreateWithPriority(&side, cudaStreamNonBlocking, hi) != cudaSuccess ||
        cudaEventCreateWithFlags(&ev[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ev[1], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventRecord(ev[0], s) != cudaSuccess || cudaStreamWaitEvent(side, ev[0], 0) != cudaSuccess) {
      (void)cudaGetLastError();
      return false;  // the destructor releases what was created; nothing was enqueued on the side
    }
    main = s;
    forked = true;
    return true;
  }
  // `s` waits for everything enqueued on the side stream
  cudaError_t join() {
    if (!forked) return err;
    forked = false;
    if (err == cudaSuccess) err = cudaEventRecord(ev[1], side);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(main, ev[1], 0);
    return err;
  }
  ~TextFork() {
    join();
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);  // released once complete
    if (side) cudaStreamDestroy(side);  // likewise
  }
};

Inputs inputs_of(const vdn_hybrid_args* a) {
  Inputs in;
  in.q = a->q; in.k = a->k; in.v = a->v; in.beta = a->beta; in.alpha = a->alpha;
  in.gate_sm = a->gate_sm; in.gate_lin = a->gate_lin;
  in.text_k = a->text_k; in.text_v = a->text_v; in.text_beta = a->text_beta;
  in.init_state = a->init_state; in.rms_weight = a->rms_weight; in.y = a->y;
  in.fwd_init = a->fwd_init;
  in.sm_lse = a->sm_lse;
  return in;
}

// the backward covers the joint solve's write at d <= 128
vdn_status check_bwd_cfg(const vdn_hybrid_cfg* c) {
  vdn_status st = check_cfg(c);
  if (st != VDN_OK) return st;
  if (c->update != 0 || c->d_k > 128) return VDN_ERR_UNSUPPORTED;
  if (c->T > 65535) return VDN_ERR_UNSUPPORTED;  // frames index a grid axis of the backward kernels
  return VDN_OK;
}

}  // namespace
}  // namespace vdn

using namespace vdn;

extern "C" {

size_t vdn_hybrid_attn_workspace_size(const vdn_hybrid_cfg* cfg) {
  if (check_cfg(cfg) != VDN_OK) return 0;
  vdn_workspace_layout L;
  layout_of(cfg, &L);
  return L.total;
}

vdn_status vdn_hybrid_workspace_layout(const vdn_hybrid_cfg* cfg, vdn_workspace_layout* out) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!out) return VDN_ERR_INVALID_ARG;
  layout_of(cfg, out);
  return VDN_OK;
}

int vdn_hybrid_stage_impl(const vdn_hybrid_cfg* cfg, unsigned stage) {
  if (check_cfg(cfg) != VDN_OK) return -1;
  Dims d = make_dims(cfg);
  switch (stage) {
    case VDN_STAGE_SCAN:
      return (scan_tc_supported(d) || scan256_tc_supported(d)) ? 1 : 0;
    case VDN_STAGE_SOLVE:
      if (d.update != 0) return 2;  // the variant-map kernel
      return gram_tc_supported(d) ? 1 : 0;
    case VDN_STAGE_TEXT:
      return gram_tc_supported(d) ? 1 : 0;
    case VDN_STAGE_READ:
      return read_tc_supported(d) ? 1 : 0;
    case VDN_STAGE_SOFTMAX:
      if (big_d(d)) return -1;
      return softmax_tc_supported(d) ? 1 : 0;
    case VDN_STAGE_SOFTMAX_BWD:
      if (check_bwd_cfg(cfg) != VDN_OK) return -1;
      return sm_bwd_tc_supported(d) ? 1 : 0;
    default:
      return -1;
  }
}

vdn_status vdn_hybrid_attn_fwd_stages(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, unsigned stages,
                                      vdn_stream_t stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  st = check_args(cfg, args, stages);
  if (st != VDN_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Dims d = make_dims(cfg);
  const Inputs in = inputs_of(args);
  const bool big = big_d(d);
  Work w = work_of(cfg, args);
  // the tensor-core scan (and its solve) take the B form: every call with this
  // configuration decides the same way, so stages run in separate calls agree
  const bool tc_scan = !big && scan_tc_supported(d) && w.M16 != nullptr;
  w.bform = (tc_scan || big) ? 1 : 0;  // the d = 256 scan takes the B form too
  // d = 256: the VDA stages only (the softmax stage has no kernel at this size)
  if (big && ((stages & VDN_STAGE_SOFTMAX) || !gram_tc_supported(d))) return VDN_ERR_UNSUPPORTED;
  cudaError_t e = cudaSuccess;
  if (cudaMemsetAsync(w.status, 0, 256, s) != cudaSuccess) return VDN_ERR_CUDA;
  TextFork fork;
  if (stages & VDN_STAGE_TEXT) {
    cudaStream_t ts = s;
    if ((stages & VDN_STAGE_SOLVE) && d.update == 0 && gram_tc_supported(d) && fork.open(d, s)) ts = fork.side;
    if (d.L > 0 && gram_tc_supported(d)) {
      if ((e = launch_text_gram_tc(d, in, w, ts)) != cudaSuccess) return VDN_ERR_CUDA;
      e = big ? launch_solve_big(d, w, ts, true) : launch_text_solve_sweep(d, w, ts);
      if (e != cudaSuccess) return VDN_ERR_CUDA;
    } else if ((e = launch_text(d, in, w, ts)) != cudaSuccess) {
      return VDN_ERR_CUDA;
    }
  }
  if (stages & VDN_STAGE_SOLVE) {
    if (d.update != 0) {
      if (launch_variant_maps(d, in, w, s) != cudaSuccess) return VDN_ERR_CUDA;
    } else if (gram_tc_supported(d)) {
      if ((e = launch_gram_tc(d, in, w, s)) != cudaSuccess) return VDN_ERR_CUDA;
      e = big ? launch_solve_big(d, w, s, false) : launch_solve_inplace(d, w, s);
      if (e != cudaSuccess) return VDN_ERR_CUDA;
    } else if ((e = launch_solve_simt(d, in, w, s)) != cudaSuccess) {
      return VDN_ERR_CUDA;
    }
  }
  if (fork.join() != cudaSuccess) return VDN_ERR_CUDA;  // the scans start from the text state
  if (big && (stages & VDN_STAGE_SCAN)) {
    e = (scan256_tc_supported(d) && w.M16 != nullptr) ? launch_scan256_tc(d, in, w, s) : launch_scan_big(d, in, w, s);
    if (e != cudaSuccess) return VDN_ERR_CUDA;
  } else if (stages & VDN_STAGE_SCAN) {
    // the tensor-core scan reads the bf16 split of M that the sweep solve
    // writes; with enough chunks it first composes each chunk's frame maps
    // and steps by whole chunks
    if (tc_scan) {
      int dev = 0, sms = 0;
      if (cudaGetDevice(&dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return VDN_ERR_CUDA;
      const bool chunks = use_chunk_scan(d, sms);
      if (chunks && launch_compose_tc(d, in, w, s) != cudaSuccess) return VDN_ERR_CUDA;
      e = launch_scan_tc(d, in, w, s, chunks);
    } else {
      e = launch_scan_simt(d, in, w, s);
    }
    if (e != cudaSuccess) return VDN_ERR_CUDA;
  }
  if (stages & VDN_STAGE_SOFTMAX) {
    e = softmax_tc_supported(d) ? launch_softmax_tc(d, in, w, s) : launch_softmax_simt(d, in, w, s);
    if (e != cudaSuccess) return VDN_ERR_CUDA;
  }
  if (big && (stages & VDN_STAGE_READ)) {
    // the tensor-core read writes y rows with 32-byte stores; else the chunked SIMT read
    e = (read_tc_supported(d) && aligned(in.y, 32)) ? launch_read_tc(d, in, w, w.R16, s) : launch_read_big(d, in, w, s);
    if (e != cudaSuccess) return VDN_ERR_CUDA;
  } else if (stages & VDN_STAGE_READ) {
    // the tensor-core read writes y rows with 32-byte stores
    e = (read_tc_supported(d) && aligned(in.y, 32)) ? launch_read_tc(d, in, w, w.R16, s)
                                                    : launch_read_simt(d, in, w, s);
    if (e != cudaSuccess) return VDN_ERR_CUDA;
  }
  return VDN_OK;
}

vdn_status vdn_hybrid_attn_fwd(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, vdn_stream_t stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  st = check_args(cfg, args, VDN_STAGE_ALL);
  if (st != VDN_OK) return st;
  return vdn_hybrid_attn_fwd_stages(cfg, args, VDN_STAGE_ALL, stream);
}

vdn_status vdn_hybrid_device_status(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, vdn_stream_t stream,
                                    unsigned* where) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!args || !args->workspace) return VDN_ERR_INVALID_ARG;
  const Work w = work_of(cfg, args);
  uint32_t host[2] = {0, 0};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host, w.status, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return VDN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return VDN_ERR_CUDA;
  if (where) *where = host[1];
  return host[0] ? VDN_ERR_TIMEOUT : VDN_OK;
}

size_t vdn_hybrid_lin_bwd_workspace_size(const vdn_hybrid_cfg* cfg) {
  if (check_bwd_cfg(cfg) != VDN_OK) return 0;
  return lin_bwd_workspace(make_dims(cfg), nullptr);
}

}  // extern "C"

namespace {

// Everything vdn_hybrid_lin_bwd checks before launching.
vdn_status lin_bwd_checks(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, const vdn_lin_grads* g) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!args || !g) return VDN_ERR_INVALID_ARG;
  const void* req[] = {args->q, args->k, args->v, args->gate_lin, g->dy, g->dq, g->dk, g->dv, g->dgate_lin};
  for (const void* p : req)
    if (!p || !aligned(p, 16)) return VDN_ERR_INVALID_ARG;
  if (!args->beta || !args->alpha || !g->dbeta || !g->dalpha) return VDN_ERR_INVALID_ARG;
  if (!aligned(args->beta, 4) || !aligned(args->alpha, 4) || !aligned(g->dbeta, 4) || !aligned(g->dalpha, 4))
    return VDN_ERR_INVALID_ARG;
  if (args->rms_weight && !aligned(args->rms_weight, 4)) return VDN_ERR_INVALID_ARG;
  if (args->fwd_init && !aligned(args->fwd_init, 16)) return VDN_ERR_INVALID_ARG;
  if ((g->drms_weight && !aligned(g->drms_weight, 4)) || (g->dfwd_init && !aligned(g->dfwd_init, 16)))
    return VDN_ERR_INVALID_ARG;
  vdn_workspace_layout L;
  layout_of(cfg, &L);
  if (!args->workspace || !aligned(args->workspace, kAlign) || args->workspace_bytes < L.total)
    return VDN_ERR_WORKSPACE;
  const Dims d = make_dims(cfg);
  if (!g->workspace || !aligned(g->workspace, kAlign) || g->workspace_bytes < lin_bwd_workspace(d, nullptr))
    return VDN_ERR_WORKSPACE;
  return VDN_OK;
}

// The linear branch's launches (arguments already checked); grad_acc adds its
// dq, dk, dv into the outputs instead of overwriting them.
vdn_status lin_bwd_launch(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, const vdn_lin_grads* g,
                          cudaStream_t s, bool grad_acc) {
  Dims d = make_dims(cfg);
  d.grad_acc = grad_acc ? 1 : 0;
  Work w = work_of(cfg, args);
  // the forward's choice of write form (B_t or C_t in the C_t slot)
  w.bform = (scan_tc_supported(d) && w.M16 != nullptr) ? 1 : 0;
  LinBwdArgs a{g->dy, g->dq, g->dk, g->dv, g->dbeta, g->dalpha, g->dgate_lin, g->drms_weight, g->dfwd_init,
               g->workspace, w.status};
  if (cudaMemsetAsync(w.status, 0, 256, s) != cudaSuccess) return VDN_ERR_CUDA;
  return launch_lin_bwd(d, inputs_of(args), w, a, s) == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

size_t sm_bwd_scratch(const Dims& d) {
  const size_t a = sm_bwd_workspace(d, nullptr), b = sm_bwd_tc_workspace(d, nullptr);
  return a > b ? a : b;
}

// Everything vdn_hybrid_sm_bwd checks before launching.
vdn_status sm_bwd_checks(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, const vdn_sm_grads* g) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!args || !g) return VDN_ERR_INVALID_ARG;
  const void* req[] = {args->q, args->k, args->v, args->gate_sm, g->dy, g->dq, g->dk, g->dv, g->dgate_sm};
  for (const void* p : req)
    if (!p || !aligned(p, 16)) return VDN_ERR_INVALID_ARG;
  const Dims d = make_dims(cfg);
  if (g->sm_lse && !aligned(g->sm_lse, 4)) return VDN_ERR_INVALID_ARG;
  if ((long long)d.T * d.N > (1LL << 40)) return VDN_ERR_UNSUPPORTED;
  if (!g->workspace || !aligned(g->workspace, kAlign) || g->workspace_bytes < sm_bwd_scratch(d))
    return VDN_ERR_WORKSPACE;
  return VDN_OK;
}

vdn_status sm_bwd_launch(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, const vdn_sm_grads* g,
                         cudaStream_t s) {
  const Dims d = make_dims(cfg);
  char* base = static_cast<char*>(g->workspace);
  if (sm_bwd_tc_supported(d)) {
    size_t off[8];
    sm_bwd_tc_workspace(d, off);
    SmTcArgs a{g->dy, g->dq, g->dk, g->dv, g->dgate_sm, base + off[1], base + off[2], base + off[3], base + off[4],
               reinterpret_cast<float*>(base + off[5]), reinterpret_cast<float*>(base + off[6]),
               reinterpret_cast<unsigned*>(base + off[7]), reinterpret_cast<uint32_t*>(base + off[0]), g->sm_lse};
    if (cudaMemsetAsync(base + off[0], 0, kAlign, s) != cudaSuccess ||
        cudaMemsetAsync(base + off[7], 0, kAlign, s) != cudaSuccess)
      return VDN_ERR_CUDA;
    return launch_sm_bwd_tc(d, inputs_of(args), a, s) == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
  }
  if (cudaMemsetAsync(base, 0, kAlign, s) != cudaSuccess) return VDN_ERR_CUDA;  // no status on this path
  SmBwdArgs a{g->dy, g->dq, g->dk, g->dv, g->dgate_sm, base + kAlign};
  return launch_sm_bwd(d, inputs_of(args), a, s) == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

// The whole-core backward shares one scratch region between the branches,
// which run one after the other on the stream: the softmax branch's layout
// from byte 0 (its status words in the first 256 bytes), the linear branch's
// from byte 256, so that the softmax branch's status words survive it.
size_t whole_bwd_scratch(const Dims& d) {
  const size_t a = sm_bwd_scratch(d), b = kAlign + lin_bwd_workspace(d, nullptr);
  return a > b ? a : b;
}

}  // namespace

extern "C" {

vdn_status vdn_hybrid_lin_bwd(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, const vdn_lin_grads* g,
                              vdn_stream_t stream) {
  const vdn_status st = lin_bwd_checks(cfg, args, g);
  if (st != VDN_OK) return st;
  return lin_bwd_launch(cfg, args, g, reinterpret_cast<cudaStream_t>(stream), false);
}

size_t vdn_hybrid_sm_bwd_workspace_size(const vdn_hybrid_cfg* cfg) {
  if (check_bwd_cfg(cfg) != VDN_OK) return 0;
  return sm_bwd_scratch(make_dims(cfg));
}

vdn_status vdn_hybrid_sm_bwd(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, const vdn_sm_grads* g,
                             vdn_stream_t stream) {
  const vdn_status st = sm_bwd_checks(cfg, args, g);
  if (st != VDN_OK) return st;
  return sm_bwd_launch(cfg, args, g, reinterpret_cast<cudaStream_t>(stream));
}

size_t vdn_hybrid_bwd_workspace_size(const vdn_hybrid_cfg* cfg) {
  if (check_bwd_cfg(cfg) != VDN_OK) return 0;
  return whole_bwd_scratch(make_dims(cfg));
}

vdn_status vdn_hybrid_bwd(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, const vdn_hybrid_grads* g,
                          vdn_stream_t stream) {
  vdn_status st = check_bwd_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!args || !g) return VDN_ERR_INVALID_ARG;
  const Dims d = make_dims(cfg);
  if (!g->workspace || !aligned(g->workspace, kAlign) || g->workspace_bytes < whole_bwd_scratch(d))
    return VDN_ERR_WORKSPACE;
  vdn_sm_grads sg{g->dy, g->dq, g->dk, g->dv, g->dgate_sm, g->workspace, g->workspace_bytes, g->sm_lse};
  vdn_lin_grads lg{g->dy, g->dq, g->dk, g->dv, g->dbeta, g->dalpha, g->dgate_lin, g->drms_weight, g->dfwd_init,
                   static_cast<char*>(g->workspace) + kAlign, g->workspace_bytes - kAlign};
  if ((st = sm_bwd_checks(cfg, args, &sg)) != VDN_OK) return st;
  if ((st = lin_bwd_checks(cfg, args, &lg)) != VDN_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the softmax branch writes dq, dk, dv; the linear branch adds its share
  if ((st = sm_bwd_launch(cfg, args, &sg, s)) != VDN_OK) return st;
  return lin_bwd_launch(cfg, args, &lg, s, true);
}

vdn_status vdn_text_cross_attn(const vdn_hybrid_cfg* cfg, const vdn_hybrid_args* args, vdn_stream_t stream) {
  vdn_status st = check_cfg(cfg);
  if (st != VDN_OK) return st;
  if (!args) return VDN_ERR_INVALID_ARG;
  if (cfg->L <= 0) return VDN_ERR_INVALID_ARG;
  const void* req[] = {args->q, args->text_k, args->text_v, args->y};
  for (const void* p : req)
    if (!p || !aligned(p, 16)) return VDN_ERR_INVALID_ARG;
  if (!args->workspace || !aligned(args->workspace, kAlign) || args->workspace_bytes < kAlign) return VDN_ERR_WORKSPACE;
  const Dims d = make_dims(cfg);
  if (!softmax_tc_supported(d)) return VDN_ERR_UNSUPPORTED;  // bf16, d = 64 or 128
  if ((long long)d.B * d.L + 256 >= (1LL << 31)) return VDN_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Work w{};
  w.status = static_cast<uint32_t*>(args->workspace);  // the status words (as in the core's layout)
  if (cudaMemsetAsync(w.status, 0, kAlign, s) != cudaSuccess) return VDN_ERR_CUDA;
  return launch_text_xattn_tc(d, inputs_of(args), w, s) == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

vdn_status vdn_out_proj(const vdn_proj_cfg* cfg, const void* y, const void* w, void* out, vdn_stream_t stream) {
  if (!cfg || !y || !w || !out) return VDN_ERR_INVALID_ARG;
  if (cfg->M < 1 || cfg->K < 8 || cfg->N < 8 || cfg->K % 8 || cfg->N % 8) return VDN_ERR_INVALID_ARG;
  if (cfg->out_dtype != VDN_F32 && cfg->out_dtype != VDN_BF16) return VDN_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(w, 16) || !aligned(out, 16)) return VDN_ERR_INVALID_ARG;
  return out_proj(cfg->M, cfg->K, cfg->N, cfg->out_dtype, y, w, out, reinterpret_cast<cudaStream_t>(stream));
}

vdn_status vdn_quantize_fp8(const void* x, int x_dtype, size_t n, void* q, float* scale, vdn_stream_t stream) {
  if (!x || !q || !scale || n == 0 || n > (size_t)1 << 62) return VDN_ERR_INVALID_ARG;
  if (x_dtype != VDN_F32 && x_dtype != VDN_BF16) return VDN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale, 4)) return VDN_ERR_INVALID_ARG;
  return quantize_fp8(x, x_dtype, (long long)n, q, scale, reinterpret_cast<cudaStream_t>(stream));
}

vdn_status vdn_out_proj_fp8(const vdn_proj_cfg* cfg, const void* y, const void* w_t, const float* scales, void* out,
                            vdn_stream_t stream) {
  if (!cfg || !y || !w_t || !scales || !out) return VDN_ERR_INVALID_ARG;
  if (cfg->M < 1 || cfg->K < 16 || cfg->N < 16 || cfg->K % 16 || cfg->N % 16) return VDN_ERR_INVALID_ARG;
  if (cfg->out_dtype != VDN_F32 && cfg->out_dtype != VDN_BF16) return VDN_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(w_t, 16) || !aligned(out, 16) || !aligned(scales, 8)) return VDN_ERR_INVALID_ARG;
  return out_proj(cfg->M, cfg->K, cfg->N, cfg->out_dtype, y, w_t, out, reinterpret_cast<cudaStream_t>(stream), scales);
}

vdn_status vdn_proj_device_status(vdn_stream_t stream, unsigned* where) {
  uint32_t* st = status_of_proj();
  if (!st) return VDN_ERR_CUDA;
  uint32_t host[2] = {0, 0};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host, st, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return VDN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return VDN_ERR_CUDA;
  if (where) *where = host[1];
  return host[0] ? VDN_ERR_TIMEOUT : VDN_OK;
}

const char* vdn_status_string(vdn_status s) {
  switch (s) {
    case VDN_OK: return "ok";
    case VDN_ERR_INVALID_ARG: return "invalid argument";
    case VDN_ERR_UNSUPPORTED: return "configuration not supported by this build";
    case VDN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case VDN_ERR_CUDA: return "CUDA error";
    case VDN_ERR_TIMEOUT: return "a bounded device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
