"""ctypes binding of libnsa_b200.so.

Argument marshalling only: each function passes device pointers (torch tensors
or raw integers), sizes and the stream to the C entry point of the same name
and raises ``NsaError`` on a non-zero status.  Every step of the computation
runs in the library's CUDA kernels; importing this module fails loudly when
the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .workloads import Workload

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnsa_b200.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with "
                      "`python -m dynamic_block_sparse_scoring_b200.build` (needs nvcc)")
lib = ctypes.CDLL(_LIB_PATH)

NSA_BR_CMP, NSA_BR_SEL, NSA_BR_WIN, NSA_PER_HEAD_SELECT = 1, 2, 4, 8
NSA_SCORE_PROB, NSA_SCORE_CMP, NSA_SINK_SHIFT, NSA_DEBUG_CHECKS = 16, 32, 16, 64
STATUS = {0: "NSA_OK", 1: "NSA_ERR_INVALID_ARG", 2: "NSA_ERR_UNSUPPORTED", 3: "NSA_ERR_WORKSPACE",
          4: "NSA_ERR_CUDA", 5: "NSA_ERR_TIMEOUT"}


class NsaConfig(ctypes.Structure):
    """Mirror of ``nsa_config`` in include/nsa.h."""
    _fields_ = [("batch", ctypes.c_int32), ("seqlen_q", ctypes.c_int32),
                ("seqlen_kv", ctypes.c_int32), ("q_pos0", ctypes.c_int32),
                ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32), ("d_qk", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("sel_block", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("window", ctypes.c_int32), ("cmp_block", ctypes.c_int32),
                ("cmp_stride", ctypes.c_int32), ("scale", ctypes.c_float),
                ("flags", ctypes.c_uint32)]


class NsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib.nsa_status_string(status).decode()
        if status == 4:
            msg += ": " + lib.nsa_last_cuda_error().decode()
        super().__init__(f"{fn} returned {status} ({msg})")


_vp, _sz = ctypes.c_void_p, ctypes.c_size_t
_cfgp = ctypes.POINTER(NsaConfig)
_SIGS = {
    "nsa_workspace_size": [_cfgp, ctypes.POINTER(_sz)],
    "nsa_workspace_size_min": [_cfgp, ctypes.POINTER(_sz)],
    "nsa_pool_kv": [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp],
    "nsa_append_kv": [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "nsa_score_blocks": [_cfgp, _vp, _vp, _vp, _vp],
    "nsa_topk_select": [_cfgp, _vp, _vp, _vp, _vp, _vp],
    "nsa_score_blocks_ex": [_cfgp, _vp, _vp, _vp, _vp, _vp],
    "nsa_topk_select_ex": [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp],
    "nsa_sparse_attn_fwd": [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "nsa_sparse_attn_fwd_noalloc": [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "nsa_get_device_status": [ctypes.POINTER(ctypes.c_int32)],
    "nsa_attn_plan": [_cfgp, ctypes.c_int, _sz, ctypes.POINTER(ctypes.c_int32),
                      ctypes.POINTER(ctypes.c_int32)],
    "nsa_timing_enable": [ctypes.c_int32],
    "nsa_check_bounded_wait": [ctypes.c_uint64, _vp],
    "nsa_set_wait_limit_ns": [ctypes.c_uint64],
    "nsa_bwd_workspace_size": [_cfgp, ctypes.POINTER(_sz)],
    "nsa_sparse_attn_bwd": [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                            _sz, _vp],
    "nsa_timing_read": [ctypes.c_int32, ctypes.POINTER(ctypes.c_float),
                        ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_int32)],
}
for _name, _args in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int
lib.nsa_status_string.argtypes = [ctypes.c_int]
lib.nsa_status_string.restype = ctypes.c_char_p
lib.nsa_last_cuda_error.argtypes = []
lib.nsa_last_cuda_error.restype = ctypes.c_char_p

EXPORTS = list(_SIGS) + ["nsa_status_string", "nsa_last_cuda_error"]


def config(wl: Workload, **override) -> NsaConfig:
    """nsa_config for a workload (fields may be overridden by keyword)."""
    f = dict(batch=wl.batch, seqlen_q=wl.seqlen_q, seqlen_kv=wl.seqlen_kv, q_pos0=wl.q_pos0,
             h_q=wl.h_q, h_kv=wl.h_kv, d_qk=wl.d_qk, d_v=wl.d_v, sel_block=wl.sel_block,
             top_k=wl.top_k, window=wl.window, cmp_block=wl.cmp_block,
             cmp_stride=wl.cmp_stride, scale=wl.scale, flags=wl.flags)
    f.update(override)
    return NsaConfig(**f)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != 0:
        raise NsaError(fn, status)


def nsa_status_string(status: int) -> str:
    return lib.nsa_status_string(status).decode()


PATHS = {0: "rowwise", 1: "query-major", 2: "block-major", 3: "split-k", 4: "decode"}


def nsa_attn_plan(cfg: NsaConfig, select_inside: bool, ws_bytes: int):
    """(path name, kernels launched) nsa_sparse_attn_fwd uses for this call shape."""
    path, n = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("nsa_attn_plan", lib.nsa_attn_plan(ctypes.byref(cfg), int(select_inside), ws_bytes,
                                              ctypes.byref(path), ctypes.byref(n)))
    return PATHS[path.value], n.value


def nsa_bwd_workspace_size(cfg: NsaConfig) -> int:
    n = _sz(0)
    _check("nsa_bwd_workspace_size", lib.nsa_bwd_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def nsa_sparse_attn_bwd(cfg, q, k, v, kcmp, vcmp, gates, idx, d_out, dq, dk, dv, dgates=None,
                        workspace=None, ws_bytes=0, stream=None):
    _check("nsa_sparse_attn_bwd",
           lib.nsa_sparse_attn_bwd(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(kcmp),
                                   _ptr(vcmp), _ptr(gates), _ptr(idx), _ptr(d_out), _ptr(dq),
                                   _ptr(dk), _ptr(dv), _ptr(dgates), _ptr(workspace), ws_bytes,
                                   _stream(stream)))


def nsa_check_bounded_wait(limit_ns: int, stream=None):
    _check("nsa_check_bounded_wait", lib.nsa_check_bounded_wait(limit_ns, _stream(stream)))


def nsa_set_wait_limit_ns(limit_ns: int):
    _check("nsa_set_wait_limit_ns", lib.nsa_set_wait_limit_ns(limit_ns))


def nsa_get_device_status() -> int:
    """Reads and clears the device status word (0 = OK, 5 = a bounded wait timed out)."""
    v = ctypes.c_int32(0)
    _check("nsa_get_device_status", lib.nsa_get_device_status(ctypes.byref(v)))
    return v.value


TIMING_MAX_STAGES = 8


def nsa_timing_enable(on: bool):
    """Start / stop recording stage events in this thread's nsa_sparse_attn_fwd calls."""
    _check("nsa_timing_enable", lib.nsa_timing_enable(int(bool(on))))


def nsa_timing_read():
    """[(stage name, ms)] of this thread's most recent timed nsa_sparse_attn_fwd call."""
    ms = (ctypes.c_float * TIMING_MAX_STAGES)()
    names = (ctypes.c_char_p * TIMING_MAX_STAGES)()
    n = ctypes.c_int32(0)
    _check("nsa_timing_read", lib.nsa_timing_read(TIMING_MAX_STAGES, ms, names, ctypes.byref(n)))
    return [(names[i].decode(), float(ms[i])) for i in range(min(n.value, TIMING_MAX_STAGES))]


def nsa_workspace_size(cfg: NsaConfig) -> int:
    n = _sz(0)
    _check("nsa_workspace_size", lib.nsa_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def nsa_workspace_size_min(cfg: NsaConfig) -> int:
    n = _sz(0)
    _check("nsa_workspace_size_min", lib.nsa_workspace_size_min(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def nsa_pool_kv(cfg, k, v, kbar, kcmp=None, vcmp=None, stream=None):
    _check("nsa_pool_kv", lib.nsa_pool_kv(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(kbar),
                                          _ptr(kcmp), _ptr(vcmp), _stream(stream)))


def nsa_append_kv(cfg, k, v, k_new, v_new, kbar=None, kcmp=None, vcmp=None, stream=None):
    """Append cfg.seqlen_q tokens per sequence at KV position cfg.q_pos0 and refresh the
    pooled tokens they complete (cfg.seqlen_kv = cache rows per plane)."""
    _check("nsa_append_kv", lib.nsa_append_kv(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(k_new),
                                              _ptr(v_new), _ptr(kbar), _ptr(kcmp), _ptr(vcmp),
                                              _stream(stream)))


def nsa_score_blocks_ex(cfg, q, kbar, kcmp, scores, stream=None):
    _check("nsa_score_blocks_ex", lib.nsa_score_blocks_ex(ctypes.byref(cfg), _ptr(q), _ptr(kbar),
                                                          _ptr(kcmp), _ptr(scores), _stream(stream)))


def nsa_topk_select_ex(cfg, q, kbar, kcmp, scores, idx, stream=None):
    _check("nsa_topk_select_ex", lib.nsa_topk_select_ex(ctypes.byref(cfg), _ptr(q), _ptr(kbar),
                                                        _ptr(kcmp), _ptr(scores), _ptr(idx),
                                                        _stream(stream)))


def nsa_score_blocks(cfg, q, kbar, scores, stream=None):
    _check("nsa_score_blocks", lib.nsa_score_blocks(ctypes.byref(cfg), _ptr(q), _ptr(kbar),
                                                    _ptr(scores), _stream(stream)))


def nsa_topk_select(cfg, q, kbar, scores, idx, stream=None):
    _check("nsa_topk_select", lib.nsa_topk_select(ctypes.byref(cfg), _ptr(q), _ptr(kbar),
                                                  _ptr(scores), _ptr(idx), _stream(stream)))


def nsa_sparse_attn_fwd(cfg, q, k, v, kbar, kcmp, vcmp, gates, idx, out, workspace=None,
                        ws_bytes=0, stream=None):
    _check("nsa_sparse_attn_fwd",
           lib.nsa_sparse_attn_fwd(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(kbar),
                                   _ptr(kcmp), _ptr(vcmp), _ptr(gates), _ptr(idx), _ptr(out),
                                   _ptr(workspace), ws_bytes, _stream(stream)))


def nsa_sparse_attn_fwd_noalloc(cfg, q, k, v, kbar, kcmp, vcmp, gates, out, stream=None):
    """Forward with internal selection and no workspace (the library's own scratch array)."""
    _check("nsa_sparse_attn_fwd_noalloc",
           lib.nsa_sparse_attn_fwd_noalloc(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(kbar), _ptr(kcmp), _ptr(vcmp), _ptr(gates),
                                           _ptr(out), _stream(stream)))


# ---------------------------------------------------------------------------
# Buffer shapes and a convenience forward that allocates outputs with torch
# ---------------------------------------------------------------------------

def pooled_shapes(cfg: NsaConfig):
    nb_full = cfg.seqlen_kv // cfg.sel_block
    n_cmp = 0
    if cfg.flags & NSA_BR_CMP and cfg.seqlen_kv >= cfg.cmp_block:
        n_cmp = (cfg.seqlen_kv - cfg.cmp_block) // cfg.cmp_stride + 1
    return {"kbar": (cfg.batch, cfg.h_kv, nb_full, cfg.d_qk),
            "kcmp": (cfg.batch, cfg.h_kv, n_cmp, cfg.d_qk),
            "vcmp": (cfg.batch, cfg.h_kv, n_cmp, cfg.d_v)}


def h_sel(cfg: NsaConfig) -> int:
    return cfg.h_q if cfg.flags & NSA_PER_HEAD_SELECT else cfg.h_kv


def alloc_pooled(cfg: NsaConfig, device):
    sh = pooled_shapes(cfg)
    return {"kbar": torch.empty(sh["kbar"], dtype=torch.float32, device=device),
            "kcmp": torch.empty(sh["kcmp"], dtype=torch.bfloat16, device=device),
            "vcmp": torch.empty(sh["vcmp"], dtype=torch.bfloat16, device=device)}


def forward(cfg: NsaConfig, q, k, v, gates=None, idx=None, stream=None, pooled=None, out=None,
            workspace=None):
    """Pool K/V (unless ``pooled`` is given), select blocks and run the gated forward.

    Returns (out, pooled).  All tensors live on the same CUDA device.
    """
    dev = q.device
    if pooled is None:
        pooled = alloc_pooled(cfg, dev)
        nsa_pool_kv(cfg, k, v, pooled["kbar"], pooled["kcmp"], pooled["vcmp"], stream)
    if out is None:
        out = torch.empty(cfg.batch, cfg.seqlen_q, cfg.h_q, cfg.d_v, dtype=torch.bfloat16,
                          device=dev)
    ws = nsa_workspace_size(cfg)
    if workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev) if ws else None
    else:
        ws = workspace.numel() * workspace.element_size()
    nsa_sparse_attn_fwd(cfg, q, k, v, pooled["kbar"], pooled["kcmp"], pooled["vcmp"], gates, idx,
                        out, workspace, ws, stream)
    return out, pooled
