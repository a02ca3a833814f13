"""Host-side checks of the C ABI: the library loads, exports every function
the header declares, sizes its workspace, and rejects bad arguments before
touching the GPU (no compute call here: these run without a device)."""
import ctypes as C
import os
import re

import pytest

from video_diffusion_hybrid_b200 import _lib as L
from video_diffusion_hybrid_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build()
    return L.lib()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(vdn_\w+)\s*\(", src, flags=re.M))
    return names


def test_exports_every_declared_symbol():
    declared = _declared()
    assert declared == set(L.EXPORTED)
    lib = L.lib()
    for name in declared:
        assert hasattr(lib, name), name


def _cfg(**kw):
    base = dict(B=1, T=90, N=1008, H=24, d_k=128, d_v=128, L=512, dtype=L.VDN_BF16)
    base.update(kw)
    return L.HybridCfg(**base)


def test_workspace_size_and_layout():
    cfg = _cfg()
    size = L.vdn_hybrid_attn_workspace_size(cfg)
    lay = L.vdn_hybrid_workspace_layout(cfg)
    assert lay["total"] == size
    dd = 128 * 128 * 4
    assert lay["frame_C"] - lay["frame_M"] >= 90 * 24 * dd
    assert lay["read_table"] - lay["bwd_snap"] >= 24 * 19 * dd
    if cfg.dtype == L.VDN_BF16 and cfg.d_k == 128:  # bf16 hi/lo of every frame's M; the chunk maps
        assert lay["chunk_P16"] - lay["frame_M16"] >= 90 * 24 * dd
        assert lay["chunk_C"] - lay["chunk_P16"] >= 18 * 24 * dd
        assert lay["chunk_lam"] - lay["chunk_C"] >= 2 * 18 * 24 * dd
        assert lay["total"] - lay["chunk_lam"] >= 18 * 24 * 4
    offs = [lay[k] for k in ("status", "half_text", "frame_M", "frame_C", "fwd_snap", "bwd_snap", "read_table",
                             "read_table_bf16", "text_gram", "frame_M16", "chunk_P16", "chunk_C", "chunk_lam",
                             "total")]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    # d = 256, bf16: M's split for the tensor-core scan, no chunk maps
    big = L.vdn_hybrid_workspace_layout(_cfg(d_k=256, d_v=256))
    assert big["chunk_P16"] - big["frame_M16"] >= 90 * 24 * 2 * 256 * 256 * 2
    assert big["chunk_P16"] == big["chunk_C"] == big["chunk_lam"] == big["total"]
    f32 = L.vdn_hybrid_workspace_layout(_cfg(dtype=L.VDN_F32))
    assert f32["frame_M16"] == f32["total"]


@pytest.mark.parametrize("kw,status", [
    (dict(T=1), L.VDN_ERR_INVALID_ARG), (dict(N=0), L.VDN_ERR_INVALID_ARG), (dict(anchors=2), L.VDN_ERR_INVALID_ARG),
    (dict(dtype=7), L.VDN_ERR_INVALID_ARG), (dict(out_mode=3), L.VDN_ERR_INVALID_ARG),
    (dict(L=-1), L.VDN_ERR_INVALID_ARG), (dict(chunk=0), L.VDN_ERR_INVALID_ARG),
    (dict(d_k=48, d_v=48), L.VDN_ERR_UNSUPPORTED), (dict(d_v=64), L.VDN_ERR_UNSUPPORTED),
    (dict(chunk=4), L.VDN_ERR_UNSUPPORTED), (dict(B=3000, H=24), L.VDN_ERR_UNSUPPORTED),
    (dict(scan_mode=3), L.VDN_ERR_INVALID_ARG), (dict(scan_mode=-1), L.VDN_ERR_INVALID_ARG),
    (dict(update=3), L.VDN_ERR_INVALID_ARG), (dict(update=-1), L.VDN_ERR_INVALID_ARG),
    (dict(update=2, d_k=256, d_v=256), L.VDN_ERR_UNSUPPORTED),
])
def test_bad_config_rejected(kw, status):
    cfg = _cfg(**kw)
    assert L.vdn_hybrid_attn_workspace_size(cfg) == 0
    with pytest.raises(L.VdnError) as e:
        L.vdn_hybrid_workspace_layout(cfg)
    assert e.value.status == status


def _fake_args(cfg, **over):
    """Aligned but never dereferenced pointer values: every test below fails
    validation before a launch."""
    p = 1 << 20
    a = dict(q=p, k=p, v=p, beta=p, alpha=p, gate_sm=p, gate_lin=p, y=p, workspace=p,
             workspace_bytes=L.vdn_hybrid_attn_workspace_size(cfg), text_k=p, text_v=p, text_beta=p)
    a.update(over)
    return L.make_args(**a)


@pytest.mark.parametrize("over,status", [
    (dict(q=None), L.VDN_ERR_INVALID_ARG), (dict(y=None), L.VDN_ERR_INVALID_ARG),
    (dict(k=(1 << 20) + 2), L.VDN_ERR_INVALID_ARG), (dict(text_k=None), L.VDN_ERR_INVALID_ARG),
    (dict(init_state=1 << 20), L.VDN_ERR_INVALID_ARG), (dict(workspace=None), L.VDN_ERR_WORKSPACE),
    (dict(workspace=(1 << 20) + 16), L.VDN_ERR_WORKSPACE), (dict(workspace_bytes=1024), L.VDN_ERR_WORKSPACE),
    # the carried forward state: 16-byte aligned and outside the workspace
    (dict(fwd_init=(1 << 24) + 4), L.VDN_ERR_INVALID_ARG), (dict(fwd_init=(1 << 20) + 4096), L.VDN_ERR_INVALID_ARG),
])
def test_bad_args_rejected_before_launch(over, status):
    cfg = _cfg()
    args = _fake_args(cfg, **over)
    assert L.vdn_hybrid_attn_fwd(cfg, args, stream=0, check=False) == status
    assert L.vdn_hybrid_attn_fwd_stages(cfg, args, L.STAGE_SOFTMAX, stream=0, check=False) == status


def test_d256_softmax_refused_before_launch():
    """d = 256 runs the Video Delta Attention stages only: a call that asks for
    the softmax is refused during validation, before any launch."""
    cfg = _cfg(d_k=256, d_v=256)
    args = _fake_args(cfg)
    assert L.vdn_hybrid_attn_fwd(cfg, args, stream=0, check=False) == L.VDN_ERR_UNSUPPORTED
    assert L.vdn_hybrid_attn_fwd_stages(cfg, args, L.STAGE_SOFTMAX | L.STAGE_READ, stream=0, check=False) == \
        L.VDN_ERR_UNSUPPORTED


def test_text_pointers_forbidden_without_text():
    cfg = _cfg(L=0)
    assert L.vdn_hybrid_attn_fwd(cfg, _fake_args(cfg), stream=0, check=False) == L.VDN_ERR_INVALID_ARG


def test_bad_stage_mask_rejected():
    cfg = _cfg()
    for mask in (0, 32, 0xFFFF):
        assert L.vdn_hybrid_attn_fwd_stages(cfg, _fake_args(cfg), mask, stream=0, check=False) == \
            L.VDN_ERR_INVALID_ARG


def test_null_struct_pointers():
    lib = L.lib()
    assert lib.vdn_hybrid_attn_fwd(None, None, None) == L.VDN_ERR_INVALID_ARG
    assert lib.vdn_hybrid_attn_workspace_size(None) == 0
    c = _cfg().c()
    assert lib.vdn_hybrid_attn_fwd(C.byref(c), None, None) == L.VDN_ERR_INVALID_ARG


def test_status_strings_and_stage_impl():
    for s in range(6):
        assert L.status_string(s) and L.status_string(s) != "unknown status"
    assert L.status_string(99) == "unknown status"
    cfg = _cfg()
    for st in (L.STAGE_TEXT, L.STAGE_SOLVE, L.STAGE_SCAN, L.STAGE_READ, L.STAGE_SOFTMAX):
        assert L.vdn_hybrid_stage_impl(cfg, st) in (0, 1)
    assert L.vdn_hybrid_stage_impl(cfg, 3) == -1
    # d = 256: the Video Delta Attention stages only, bf16 inputs only
    big = _cfg(d_k=256, d_v=256)
    assert L.vdn_hybrid_stage_impl(big, L.STAGE_SOFTMAX) == -1
    for st in (L.STAGE_TEXT, L.STAGE_SOLVE, L.STAGE_SCAN, L.STAGE_READ):
        assert L.vdn_hybrid_stage_impl(big, st) in (0, 1)
    assert L.vdn_hybrid_attn_workspace_size(big) > 0
    assert L.vdn_hybrid_stage_impl(_cfg(d_k=256, d_v=256, dtype=L.VDN_F32), L.STAGE_SOLVE) == -1
    # the ablation writes: their own per-frame map kernel, then the SIMT scan
    for u in (1, 2):
        v = _cfg(update=u, d_k=128, d_v=128)
        assert L.vdn_hybrid_stage_impl(v, L.STAGE_SOLVE) == 2
        assert L.vdn_hybrid_stage_impl(v, L.STAGE_SCAN) == 0
    assert L.vdn_hybrid_attn_workspace_size(_cfg(d_k=256, d_v=256, dtype=L.VDN_F32)) == 0


def test_out_proj_bad_args_rejected():
    """vdn_out_proj validates before any launch (no device needed)."""
    p = 1 << 20
    for M, K, N, od, y, w, o in [(0, 64, 64, 0, p, p, p), (8, 60, 64, 0, p, p, p), (8, 64, 12, 0, p, p, p),
                                 (8, 64, 64, 7, p, p, p), (8, 64, 64, 0, None, p, p), (8, 64, 64, 0, p + 8, p, p)]:
        assert L.vdn_out_proj(M, K, N, od, y, w, o, stream=0, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.lib().vdn_out_proj(None, None, None, None, None) == L.VDN_ERR_INVALID_ARG


def test_text_cross_attn_rejected_before_launch():
    p = 1 << 20
    def call(cfg, **over):
        a = dict(q=p, k=None, v=None, beta=None, alpha=None, gate_sm=None, gate_lin=None, y=p, workspace=p,
                 workspace_bytes=256, text_k=p, text_v=p)
        a.update(over)
        return L.vdn_text_cross_attn(cfg, L.make_args(**a), stream=0, check=False)
    assert call(_cfg(L=0)) == L.VDN_ERR_INVALID_ARG
    assert call(_cfg(), text_k=None) == L.VDN_ERR_INVALID_ARG
    assert call(_cfg(), y=p + 4) == L.VDN_ERR_INVALID_ARG
    assert call(_cfg(), workspace_bytes=128) == L.VDN_ERR_WORKSPACE
    assert call(_cfg(dtype=L.VDN_F32)) == L.VDN_ERR_UNSUPPORTED
    assert call(_cfg(d_k=32, d_v=32)) == L.VDN_ERR_UNSUPPORTED


def test_fp8_entries_reject_bad_args():
    p = 1 << 20
    assert L.vdn_quantize_fp8(p, L.VDN_BF16, 0, p, p, stream=0, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.vdn_quantize_fp8(p, 7, 16, p, p, stream=0, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.vdn_quantize_fp8(None, L.VDN_F32, 16, p, p, stream=0, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.vdn_out_proj_fp8(8, 24, 32, 0, p, p, p, p, stream=0, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.vdn_out_proj_fp8(8, 32, 32, 0, p, p, None, p, stream=0, check=False) == L.VDN_ERR_INVALID_ARG


def test_lin_bwd_workspace_size():
    """Every state of both scans ([B,H,T+1,d,d] twice), three d x d matrices
    per frame-head and the RMS partials, each region 256-byte aligned."""
    cfg = _cfg()
    dd = 128 * 128 * 4
    want = 2 * 24 * 91 * dd + 3 * 90 * 24 * dd + 90 * 24 * 128 * 4
    assert L.vdn_hybrid_lin_bwd_workspace_size(cfg) == want
    for kw in (dict(update=1), dict(update=2), dict(d_k=256, d_v=256), dict(T=1), dict(T=70000, N=8, H=2)):
        assert L.vdn_hybrid_lin_bwd_workspace_size(_cfg(**kw)) == 0
        assert L.vdn_hybrid_sm_bwd_workspace_size(_cfg(**kw)) == 0


def _fake_grads(cfg, **over):
    p = 1 << 26
    g = dict(dy=p, dq=p, dk=p, dv=p, dbeta=p, dalpha=p, dgate_lin=p, workspace=p,
             workspace_bytes=L.vdn_hybrid_lin_bwd_workspace_size(cfg))
    g.update(over)
    return L.make_lin_grads(**g)


@pytest.mark.parametrize("over,status", [
    (dict(dy=None), L.VDN_ERR_INVALID_ARG), (dict(dq=(1 << 26) + 4), L.VDN_ERR_INVALID_ARG),
    (dict(dbeta=None), L.VDN_ERR_INVALID_ARG), (dict(dalpha=(1 << 26) + 2), L.VDN_ERR_INVALID_ARG),
    (dict(dfwd_init=(1 << 26) + 4), L.VDN_ERR_INVALID_ARG), (dict(workspace=None), L.VDN_ERR_WORKSPACE),
    (dict(workspace=(1 << 26) + 64), L.VDN_ERR_WORKSPACE), (dict(workspace_bytes=4096), L.VDN_ERR_WORKSPACE),
])
def test_lin_bwd_bad_grads_rejected_before_launch(over, status):
    cfg = _cfg()
    assert L.vdn_hybrid_lin_bwd(cfg, _fake_args(cfg), _fake_grads(cfg, **over), stream=0, check=False) == status


def test_lin_bwd_bad_config_and_forward_workspace_rejected():
    cfg = _cfg()
    assert L.vdn_hybrid_lin_bwd(cfg, _fake_args(cfg, workspace_bytes=1024), _fake_grads(cfg), stream=0,
                                check=False) == L.VDN_ERR_WORKSPACE
    assert L.vdn_hybrid_lin_bwd(cfg, _fake_args(cfg, gate_lin=None), _fake_grads(cfg), stream=0,
                                check=False) == L.VDN_ERR_INVALID_ARG
    for kw in (dict(update=1), dict(d_k=256, d_v=256)):
        c = _cfg(**kw)
        assert L.vdn_hybrid_lin_bwd(c, _fake_args(c), _fake_grads(cfg), stream=0, check=False) == \
            L.VDN_ERR_UNSUPPORTED
    lib = L.lib()
    c = cfg.c()
    assert lib.vdn_hybrid_lin_bwd(C.byref(c), None, None, None) == L.VDN_ERR_INVALID_ARG


def test_sm_bwd_workspace_and_rejections():
    cfg = _cfg()
    rows = 90 * 1008 * 24
    up = lambda x: (x + 255) // 256 * 256
    # the tensor-core layout (status, fp16 q, k, v, dO, LSE, Delta, max |dO|) is the larger
    assert L.vdn_hybrid_sm_bwd_workspace_size(cfg) == 256 + 4 * up(rows * 128 * 2) + 2 * up(rows * 4) + 256
    for kw in (dict(update=1), dict(d_k=256, d_v=256)):
        assert L.vdn_hybrid_sm_bwd_workspace_size(_cfg(**kw)) == 0
    p = 1 << 26
    good = dict(dy=p, dq=p, dk=p, dv=p, dgate_sm=p, workspace=p, workspace_bytes=L.vdn_hybrid_sm_bwd_workspace_size(cfg))
    for over, status in ((dict(dy=None), L.VDN_ERR_INVALID_ARG), (dict(dgate_sm=p + 8), L.VDN_ERR_INVALID_ARG),
                         (dict(workspace=None), L.VDN_ERR_WORKSPACE), (dict(workspace_bytes=64), L.VDN_ERR_WORKSPACE)):
        g = L.make_sm_grads(**{**good, **over})
        assert L.vdn_hybrid_sm_bwd(cfg, _fake_args(cfg), g, stream=0, check=False) == status
    assert L.vdn_hybrid_sm_bwd(cfg, _fake_args(cfg, gate_sm=None), L.make_sm_grads(**good), stream=0,
                               check=False) == L.VDN_ERR_INVALID_ARG
    c = _cfg(update=2)
    assert L.vdn_hybrid_sm_bwd(c, _fake_args(c), L.make_sm_grads(**good), stream=0, check=False) == \
        L.VDN_ERR_UNSUPPORTED


def test_sm_lse_pointers_validated_before_launch():
    """The forward's optional log-sum-exp output and the softmax backward's
    matching input: a misaligned pointer is refused before any launch."""
    cfg = _cfg()
    p = 1 << 26
    assert L.vdn_hybrid_attn_fwd(cfg, _fake_args(cfg, sm_lse=(1 << 24) + 2), stream=0, check=False) == \
        L.VDN_ERR_INVALID_ARG
    good = dict(dy=p, dq=p, dk=p, dv=p, dgate_sm=p, workspace=p,
                workspace_bytes=L.vdn_hybrid_sm_bwd_workspace_size(cfg))
    g = L.make_sm_grads(**good, sm_lse=p + 2)
    assert L.vdn_hybrid_sm_bwd(cfg, _fake_args(cfg), g, stream=0, check=False) == L.VDN_ERR_INVALID_ARG


def test_whole_bwd_workspace_and_rejections():
    """vdn_hybrid_bwd: its scratch is the larger of the softmax branch's and
    256 bytes plus the linear branch's; every check of either branch runs
    before the first launch (a bad pointer of one branch stops the call)."""
    cfg = _cfg()
    sm, lin = L.vdn_hybrid_sm_bwd_workspace_size(cfg), L.vdn_hybrid_lin_bwd_workspace_size(cfg)
    assert L.vdn_hybrid_bwd_workspace_size(cfg) == max(sm, 256 + lin)
    for kw in (dict(update=1), dict(d_k=256, d_v=256), dict(T=1)):
        assert L.vdn_hybrid_bwd_workspace_size(_cfg(**kw)) == 0
    p = 1 << 26
    good = dict(dy=p, dq=p, dk=p, dv=p, dbeta=p, dalpha=p, dgate_lin=p, dgate_sm=p, workspace=p,
                workspace_bytes=L.vdn_hybrid_bwd_workspace_size(cfg))
    for over, status in ((dict(dy=None), L.VDN_ERR_INVALID_ARG), (dict(dgate_sm=p + 8), L.VDN_ERR_INVALID_ARG),
                         (dict(dgate_lin=None), L.VDN_ERR_INVALID_ARG), (dict(dalpha=p + 2), L.VDN_ERR_INVALID_ARG),
                         (dict(dfwd_init=p + 4), L.VDN_ERR_INVALID_ARG), (dict(sm_lse=p + 2), L.VDN_ERR_INVALID_ARG),
                         (dict(workspace=None), L.VDN_ERR_WORKSPACE), (dict(workspace=p + 128), L.VDN_ERR_WORKSPACE),
                         (dict(workspace_bytes=max(sm, 256 + lin) - 1), L.VDN_ERR_WORKSPACE)):
        g = L.make_grads(**{**good, **over})
        assert L.vdn_hybrid_bwd(cfg, _fake_args(cfg), g, stream=0, check=False) == status, over
    g = L.make_grads(**good)
    assert L.vdn_hybrid_bwd(cfg, _fake_args(cfg, gate_sm=None), g, stream=0, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.vdn_hybrid_bwd(cfg, _fake_args(cfg, gate_lin=None), g, stream=0, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.vdn_hybrid_bwd(cfg, _fake_args(cfg, workspace_bytes=1024), g, stream=0, check=False) == \
        L.VDN_ERR_WORKSPACE
    c = _cfg(update=2)
    assert L.vdn_hybrid_bwd(c, _fake_args(c), g, stream=0, check=False) == L.VDN_ERR_UNSUPPORTED
    lib = L.lib()
    cc = cfg.c()
    assert lib.vdn_hybrid_bwd(C.byref(cc), None, None, None) == L.VDN_ERR_INVALID_ARG


def test_read_wait_limit_hook_rejects_out_of_range():
    """The failure-path hook refuses a limit above the default (about one
    second of clock cycles) before touching the device."""
    assert L.vdn_debug_set_read_wait_limit(2_000_000_001, check=False) == L.VDN_ERR_INVALID_ARG
    assert L.vdn_debug_set_read_wait_limit(2 ** 63, check=False) == L.VDN_ERR_INVALID_ARG


def _header_struct_fields(name):
    """Field names, in order, of `typedef struct { ... } name;` in the header."""
    src = open(os.path.join(ROOT, "include", "vdn_hybrid.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    m = re.search(r"typedef struct \{([^{}]*)\}\s*" + name + r"\s*;", src)
    assert m, name
    fields = []
    for decl in m.group(1).split(";"):
        decl = decl.strip()
        if not decl:
            continue
        # "const void *q, *k, *v" -> q, k, v ; "size_t workspace_bytes" -> workspace_bytes
        head, *rest = decl.split(",")
        fields.append(re.findall(r"(\w+)\s*$", head)[0])
        fields += [re.sub(r"[\s\*]", "", r) for r in rest]
    return fields


@pytest.mark.parametrize("cname,pystruct", [
    ("vdn_hybrid_cfg", L.VdnCfg), ("vdn_hybrid_args", L.VdnArgs), ("vdn_lin_grads", L.VdnLinGrads),
    ("vdn_sm_grads", L.VdnSmGrads), ("vdn_proj_cfg", L.ProjCfg), ("vdn_workspace_layout", L.VdnLayout),
    ("vdn_hybrid_grads", L.VdnGrads),
])
def test_ctypes_mirrors_follow_the_header(cname, pystruct):
    """The binding's structs list the header's fields in the same order (a
    mismatch would hand the library wrong pointers)."""
    assert [f for f, _ in pystruct._fields_] == _header_struct_fields(cname)
