"""ctypes binding of ``libvdn_hybrid.so`` (the C ABI in ``include/vdn_hybrid.h``).

Argument marshalling only: every step of the hybrid attention core runs in
the library's CUDA kernels.  Names follow the C entry points.  Torch is used
for device memory and streams; the functions accept torch tensors and pass
their device pointers.  There is no fallback: if the library is missing the
first call raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, fields

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvdn_hybrid.so")

VDN_OK, VDN_ERR_INVALID_ARG, VDN_ERR_UNSUPPORTED, VDN_ERR_WORKSPACE, VDN_ERR_CUDA, VDN_ERR_TIMEOUT = range(6)
VDN_F32, VDN_BF16 = 0, 1
STAGE_TEXT, STAGE_SOLVE, STAGE_SCAN, STAGE_SOFTMAX, STAGE_READ = 1, 2, 4, 8, 16
STAGE_ALL = 31
STAGE_SOFTMAX_BWD = 32  # vdn_hybrid_stage_impl key of the softmax branch's backward

EXPORTED = ("vdn_hybrid_attn_workspace_size", "vdn_hybrid_workspace_layout", "vdn_hybrid_attn_fwd",
            "vdn_hybrid_attn_fwd_stages", "vdn_hybrid_device_status", "vdn_hybrid_stage_impl",
            "vdn_status_string", "vdn_hybrid_attn_fwd_noalloc", "vdn_hybrid_noalloc_device_status", "vdn_out_proj", "vdn_text_cross_attn",
            "vdn_quantize_fp8", "vdn_out_proj_fp8", "vdn_hybrid_lin_bwd_workspace_size", "vdn_hybrid_lin_bwd",
            "vdn_hybrid_sm_bwd_workspace_size", "vdn_hybrid_sm_bwd", "vdn_hybrid_bwd_workspace_size", "vdn_hybrid_bwd",
            "vdn_debug_set_read_wait_limit", "vdn_proj_device_status")
NOALLOC_SCRATCH_BYTES = 16 << 20


class VdnCfg(C.Structure):
    _fields_ = [("B", C.c_int), ("T", C.c_int), ("N", C.c_int), ("H", C.c_int), ("d_k", C.c_int),
                ("d_v", C.c_int), ("L", C.c_int), ("chunk", C.c_int), ("anchors", C.c_int),
                ("dtype", C.c_int), ("softmax_scale", C.c_float), ("rms_eps", C.c_float),
                ("out_mode", C.c_int), ("y_dtype", C.c_int), ("scan_mode", C.c_int),
                ("update", C.c_int)]


class VdnArgs(C.Structure):
    _fields_ = [("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p), ("beta", C.c_void_p),
                ("alpha", C.c_void_p), ("gate_sm", C.c_void_p), ("gate_lin", C.c_void_p),
                ("text_k", C.c_void_p), ("text_v", C.c_void_p), ("text_beta", C.c_void_p),
                ("init_state", C.c_void_p), ("rms_weight", C.c_void_p), ("y", C.c_void_p),
                ("workspace", C.c_void_p), ("workspace_bytes", C.c_size_t), ("fwd_init", C.c_void_p),
                ("sm_lse", C.c_void_p)]


class VdnLinGrads(C.Structure):
    """Mirror of ``vdn_lin_grads``."""
    _fields_ = [("dy", C.c_void_p), ("dq", C.c_void_p), ("dk", C.c_void_p), ("dv", C.c_void_p),
                ("dbeta", C.c_void_p), ("dalpha", C.c_void_p), ("dgate_lin", C.c_void_p),
                ("drms_weight", C.c_void_p), ("dfwd_init", C.c_void_p), ("workspace", C.c_void_p),
                ("workspace_bytes", C.c_size_t)]


class VdnSmGrads(C.Structure):
    """Mirror of ``vdn_sm_grads``."""
    _fields_ = [("dy", C.c_void_p), ("dq", C.c_void_p), ("dk", C.c_void_p), ("dv", C.c_void_p),
                ("dgate_sm", C.c_void_p), ("workspace", C.c_void_p), ("workspace_bytes", C.c_size_t),
                ("sm_lse", C.c_void_p)]


class VdnGrads(C.Structure):
    """Mirror of ``vdn_hybrid_grads`` (the whole core's backward)."""
    _fields_ = [("dy", C.c_void_p), ("dq", C.c_void_p), ("dk", C.c_void_p), ("dv", C.c_void_p),
                ("dbeta", C.c_void_p), ("dalpha", C.c_void_p), ("dgate_lin", C.c_void_p), ("dgate_sm", C.c_void_p),
                ("drms_weight", C.c_void_p), ("dfwd_init", C.c_void_p), ("workspace", C.c_void_p),
                ("workspace_bytes", C.c_size_t), ("sm_lse", C.c_void_p)]


class ProjCfg(C.Structure):
    """Mirror of ``vdn_proj_cfg``."""
    _fields_ = [("M", C.c_int), ("K", C.c_int), ("N", C.c_int), ("out_dtype", C.c_int)]


class VdnLayout(C.Structure):
    _fields_ = [(n, C.c_size_t) for n in ("status", "half_text", "frame_M", "frame_C", "fwd_snap",
                                          "bwd_snap", "read_table", "read_table_bf16", "text_gram", "frame_M16",
                                          "chunk_P16", "chunk_C", "chunk_lam", "total")]


@dataclass
class HybridCfg:
    """Mirror of ``vdn_hybrid_cfg``."""
    B: int
    T: int
    N: int
    H: int
    d_k: int
    d_v: int
    L: int = 0
    chunk: int = 5
    anchors: int = 4
    dtype: int = VDN_F32
    softmax_scale: float = 0.0
    rms_eps: float = 0.0
    out_mode: int = 0
    y_dtype: int = VDN_F32
    scan_mode: int = 0
    update: int = 0  # 0 joint solve, 1 frame-level independent writes (1/N), 2 token-wise delta rule

    def c(self) -> VdnCfg:
        return VdnCfg(**{f.name: getattr(self, f.name) for f in fields(self)})

    @property
    def C(self) -> int:
        return -(-self.T // self.chunk)


class VdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def lib() -> C.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run video_diffusion_hybrid_b200/build.py "
                               "(there is no CPU fallback)")
        L = C.CDLL(LIB_PATH)
        L.vdn_hybrid_attn_workspace_size.restype = C.c_size_t
        L.vdn_hybrid_attn_workspace_size.argtypes = [C.POINTER(VdnCfg)]
        L.vdn_hybrid_workspace_layout.restype = C.c_int
        L.vdn_hybrid_workspace_layout.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnLayout)]
        L.vdn_hybrid_attn_fwd.restype = C.c_int
        L.vdn_hybrid_attn_fwd.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.c_void_p]
        L.vdn_hybrid_attn_fwd_stages.restype = C.c_int
        L.vdn_hybrid_attn_fwd_stages.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.c_uint, C.c_void_p]
        L.vdn_hybrid_device_status.restype = C.c_int
        L.vdn_hybrid_device_status.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.c_void_p,
                                               C.POINTER(C.c_uint)]
        L.vdn_hybrid_stage_impl.restype = C.c_int
        L.vdn_hybrid_stage_impl.argtypes = [C.POINTER(VdnCfg), C.c_uint]
        L.vdn_hybrid_attn_fwd_noalloc.restype = C.c_int
        L.vdn_hybrid_attn_fwd_noalloc.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.c_void_p]
        L.vdn_hybrid_noalloc_device_status.restype = C.c_int
        L.vdn_hybrid_noalloc_device_status.argtypes = [C.c_void_p, C.POINTER(C.c_uint)]
        L.vdn_text_cross_attn.restype = C.c_int
        L.vdn_text_cross_attn.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.c_void_p]
        L.vdn_quantize_fp8.restype = C.c_int
        L.vdn_quantize_fp8.argtypes = [C.c_void_p, C.c_int, C.c_size_t, C.c_void_p, C.c_void_p, C.c_void_p]
        L.vdn_out_proj_fp8.restype = C.c_int
        L.vdn_out_proj_fp8.argtypes = [C.POINTER(ProjCfg), C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.c_void_p]
        L.vdn_out_proj.restype = C.c_int
        L.vdn_out_proj.argtypes = [C.POINTER(ProjCfg), C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
        L.vdn_hybrid_lin_bwd_workspace_size.restype = C.c_size_t
        L.vdn_hybrid_lin_bwd_workspace_size.argtypes = [C.POINTER(VdnCfg)]
        L.vdn_hybrid_lin_bwd.restype = C.c_int
        L.vdn_hybrid_lin_bwd.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.POINTER(VdnLinGrads), C.c_void_p]
        L.vdn_hybrid_sm_bwd_workspace_size.restype = C.c_size_t
        L.vdn_hybrid_sm_bwd_workspace_size.argtypes = [C.POINTER(VdnCfg)]
        L.vdn_hybrid_sm_bwd.restype = C.c_int
        L.vdn_hybrid_sm_bwd.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.POINTER(VdnSmGrads), C.c_void_p]
        L.vdn_hybrid_bwd_workspace_size.restype = C.c_size_t
        L.vdn_hybrid_bwd_workspace_size.argtypes = [C.POINTER(VdnCfg)]
        L.vdn_hybrid_bwd.restype = C.c_int
        L.vdn_hybrid_bwd.argtypes = [C.POINTER(VdnCfg), C.POINTER(VdnArgs), C.POINTER(VdnGrads), C.c_void_p]
        L.vdn_proj_device_status.restype = C.c_int
        L.vdn_proj_device_status.argtypes = [C.c_void_p, C.POINTER(C.c_uint)]
        L.vdn_debug_set_read_wait_limit.restype = C.c_int
        L.vdn_debug_set_read_wait_limit.argtypes = [C.c_ulonglong]
        L.vdn_status_string.restype = C.c_char_p
        L.vdn_status_string.argtypes = [C.c_int]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().vdn_status_string(status).decode()


def vdn_hybrid_attn_workspace_size(cfg: HybridCfg) -> int:
    c = cfg.c()
    return int(lib().vdn_hybrid_attn_workspace_size(C.byref(c)))


def vdn_hybrid_workspace_layout(cfg: HybridCfg) -> dict:
    c, out = cfg.c(), VdnLayout()
    st = lib().vdn_hybrid_workspace_layout(C.byref(c), C.byref(out))
    if st != VDN_OK:
        raise VdnError(st, "vdn_hybrid_workspace_layout")
    return {n: int(getattr(out, n)) for n, _ in VdnLayout._fields_}


def vdn_out_proj(M: int, K: int, N: int, out_dtype: int, y, w, out, stream=None, check: bool = True) -> int:
    """out[M, N] = y[M, K] w[K, N] (device pointers or tensors)."""
    c = ProjCfg(M=M, K=K, N=N, out_dtype=out_dtype)
    st = lib().vdn_out_proj(C.byref(c), _ptr(y), _ptr(w), _ptr(out), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_out_proj")
    return st


def vdn_quantize_fp8(x, x_dtype: int, n: int, q, scale, stream=None, check: bool = True) -> int:
    """q = e4m3(x / s), s = amax|x| / 448 into scale (device pointers or tensors)."""
    st = lib().vdn_quantize_fp8(_ptr(x), x_dtype, n, _ptr(q), _ptr(scale), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_quantize_fp8")
    return st


def vdn_out_proj_fp8(M: int, K: int, N: int, out_dtype: int, y, w_t, scales, out, stream=None,
                     check: bool = True) -> int:
    """out[M, N] = (s_y y)(s_w w) with e4m3 y [M, K], w_t [N, K] and scales {s_y, s_w}."""
    c = ProjCfg(M=M, K=K, N=N, out_dtype=out_dtype)
    st = lib().vdn_out_proj_fp8(C.byref(c), _ptr(y), _ptr(w_t), _ptr(scales), _ptr(out), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_out_proj_fp8")
    return st


def vdn_text_cross_attn(cfg: HybridCfg, args: VdnArgs, stream=None, check: bool = True) -> int:
    """Text cross-attention: args.q, text_k, text_v in, args.y out, args.workspace (status words)."""
    c = cfg.c()
    st = lib().vdn_text_cross_attn(C.byref(c), C.byref(args), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_text_cross_attn")
    return st


def vdn_hybrid_stage_impl(cfg: HybridCfg, stage: int) -> int:
    c = cfg.c()
    return int(lib().vdn_hybrid_stage_impl(C.byref(c), stage))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def make_args(q, k, v, beta, alpha, gate_sm, gate_lin, y, workspace, workspace_bytes=None,
              text_k=None, text_v=None, text_beta=None, init_state=None, rms_weight=None,
              fwd_init=None, sm_lse=None) -> VdnArgs:
    """Build a ``vdn_hybrid_args`` from torch tensors (or raw integer device
    pointers).  The caller keeps the tensors alive for the call."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return VdnArgs(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(gate_sm), _ptr(gate_lin),
                   _ptr(text_k), _ptr(text_v), _ptr(text_beta), _ptr(init_state), _ptr(rms_weight),
                   _ptr(y), _ptr(workspace), int(workspace_bytes), _ptr(fwd_init), _ptr(sm_lse))


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def vdn_hybrid_attn_fwd(cfg: HybridCfg, args: VdnArgs, stream=None, check: bool = True) -> int:
    c = cfg.c()
    st = lib().vdn_hybrid_attn_fwd(C.byref(c), C.byref(args), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_hybrid_attn_fwd")
    return st


def vdn_hybrid_attn_fwd_stages(cfg: HybridCfg, args: VdnArgs, stages: int, stream=None, check: bool = True) -> int:
    c = cfg.c()
    st = lib().vdn_hybrid_attn_fwd_stages(C.byref(c), C.byref(args), stages, _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_hybrid_attn_fwd_stages")
    return st


def vdn_hybrid_device_status(cfg: HybridCfg, args: VdnArgs, stream=None) -> tuple:
    c, where = cfg.c(), C.c_uint(0)
    st = lib().vdn_hybrid_device_status(C.byref(c), C.byref(args), _stream_handle(stream), C.byref(where))
    return st, int(where.value)


def vdn_hybrid_noalloc_device_status(stream=None) -> tuple:
    """(status, kernel tag) of the last no-alloc call on the current device
    (synchronises the stream)."""
    where = C.c_uint(0)
    st = lib().vdn_hybrid_noalloc_device_status(_stream_handle(stream), C.byref(where))
    return st, int(where.value)


def vdn_hybrid_attn_fwd_noalloc(cfg: HybridCfg, args: VdnArgs, stream=None, check: bool = True) -> int:
    """The core with the library's own fixed scratch (args.workspace must be
    None, workspace_bytes 0), for callers that cannot allocate."""
    c = cfg.c()
    st = lib().vdn_hybrid_attn_fwd_noalloc(C.byref(c), C.byref(args), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_hybrid_attn_fwd_noalloc")
    return st


def vdn_hybrid_lin_bwd_workspace_size(cfg: HybridCfg) -> int:
    c = cfg.c()
    return int(lib().vdn_hybrid_lin_bwd_workspace_size(C.byref(c)))


def make_lin_grads(dy, dq, dk, dv, dbeta, dalpha, dgate_lin, workspace, workspace_bytes=None, drms_weight=None,
                   dfwd_init=None) -> VdnLinGrads:
    """Build a ``vdn_lin_grads`` from torch tensors (or raw device pointers)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return VdnLinGrads(_ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dalpha), _ptr(dgate_lin),
                       _ptr(drms_weight), _ptr(dfwd_init), _ptr(workspace), int(workspace_bytes))


def vdn_hybrid_lin_bwd(cfg: HybridCfg, args: VdnArgs, grads: VdnLinGrads, stream=None, check: bool = True) -> int:
    """Backward of the linear branch; args.workspace holds the forward's."""
    c = cfg.c()
    st = lib().vdn_hybrid_lin_bwd(C.byref(c), C.byref(args), C.byref(grads), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_hybrid_lin_bwd")
    return st


def vdn_hybrid_sm_bwd_workspace_size(cfg: HybridCfg) -> int:
    c = cfg.c()
    return int(lib().vdn_hybrid_sm_bwd_workspace_size(C.byref(c)))


def make_sm_grads(dy, dq, dk, dv, dgate_sm, workspace, workspace_bytes=None, sm_lse=None) -> VdnSmGrads:
    """Build a ``vdn_sm_grads`` from torch tensors (or raw device pointers)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return VdnSmGrads(_ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgate_sm), _ptr(workspace), int(workspace_bytes),
                      _ptr(sm_lse))


def vdn_hybrid_sm_bwd(cfg: HybridCfg, args: VdnArgs, grads: VdnSmGrads, stream=None, check: bool = True) -> int:
    """Backward of the windowed softmax branch (recomputes its statistics)."""
    c = cfg.c()
    st = lib().vdn_hybrid_sm_bwd(C.byref(c), C.byref(args), C.byref(grads), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_hybrid_sm_bwd")
    return st


def vdn_hybrid_bwd_workspace_size(cfg: HybridCfg) -> int:
    c = cfg.c()
    return int(lib().vdn_hybrid_bwd_workspace_size(C.byref(c)))


def make_grads(dy, dq, dk, dv, dbeta, dalpha, dgate_lin, dgate_sm, workspace, workspace_bytes=None, drms_weight=None,
               dfwd_init=None, sm_lse=None) -> VdnGrads:
    """Build a ``vdn_hybrid_grads`` from torch tensors (or raw device pointers)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return VdnGrads(_ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dalpha), _ptr(dgate_lin),
                    _ptr(dgate_sm), _ptr(drms_weight), _ptr(dfwd_init), _ptr(workspace), int(workspace_bytes),
                    _ptr(sm_lse))


def vdn_hybrid_bwd(cfg: HybridCfg, args: VdnArgs, grads: VdnGrads, stream=None, check: bool = True) -> int:
    """The whole core's backward (both branches, dq / dk / dv summed on the
    device); args.workspace holds the forward's."""
    c = cfg.c()
    st = lib().vdn_hybrid_bwd(C.byref(c), C.byref(args), C.byref(grads), _stream_handle(stream))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_hybrid_bwd")
    return st


TAG_READ = 3  # VDN_TAG_READ


def vdn_debug_set_read_wait_limit(cycles: int, check: bool = True) -> int:
    """Wait limit (SM clock cycles) of the state read's epilogue warps on the
    current device; 0 = the default.  Failure-path tests only."""
    st = lib().vdn_debug_set_read_wait_limit(int(cycles))
    if check and st != VDN_OK:
        raise VdnError(st, "vdn_debug_set_read_wait_limit")
    return st


def vdn_proj_device_status(stream=None) -> tuple:
    """(status, kernel tag) of the last output projection on the current
    device (synchronises the stream)."""
    where = C.c_uint(0)
    st = lib().vdn_proj_device_status(_stream_handle(stream), C.byref(where))
    return st, where.value
