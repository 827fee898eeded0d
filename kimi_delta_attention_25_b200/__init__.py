"""libkda: B200 (sm_100a) kernels for the KDA (Kimi Delta Attention) hot path.

Thin Python binding over the C ABI in ``include/libkda.h``: argument
marshalling only. PyTorch supplies device memory and streams; every step of
the computation runs in the CUDA kernels of ``libkda.so``. There is no CPU
fallback: if the library is missing or no CUDA device is present, calls raise.

Names follow the C entry points:

* ``chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None)`` -> ``(out, S_final)``
* ``decode_step(q, k, v, log_alpha, beta, S)`` -> ``out`` (``S`` updated in place)
* ``chunk_prep(q, k, log_alpha, beta, workspace, ...)`` and ``chunk_scan(v, workspace, ...)``:
  the two passes of ``chunk_fwd`` for bf16 inputs, one call each
* ``chunk_fwd_workspace_size``, ``workspace_status``, ``status_string``
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = ["chunk_fwd", "chunk_prep", "chunk_scan", "decode_step", "chunk_fwd_workspace_size", "workspace_status",
           "status_string", "library_path", "load", "KDAError", "cu_seqlens_from_mask", "unpad", "pad",
           "chunk_fwd_noalloc", "noalloc_status",
           "KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_CUDA", "KDA_ERR_TIMEOUT"]

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(5)
KDA_F32, KDA_BF16 = 0, 1

_PKG = os.path.dirname(os.path.abspath(__file__))
# KDA_LIBRARY selects another build of the same ABI (the debug build libkda_debug.so, which checks
# every global index); by default the release build next to this file.
library_path = os.environ.get("KDA_LIBRARY") or os.path.join(_PKG, "libkda.so")
_lib = None

# Every entry point declared in include/libkda.h.
EXPORTS = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_decode_step",
           "kda_chunk_fwd_layer_workspace_size", "kda_chunk_fwd_layer", "kda_chunk_prep_layer",
           "kda_chunk_scan_layer", "kda_decode_step_layer", "kda_short_conv", "kda_short_conv_step",
           "kda_state_affine",
           "kda_workspace_status", "kda_status_string", "kda_version", "kda_chunk_fwd_noalloc",
           "kda_chunk_prep", "kda_chunk_scan", "kda_selftest_wait_timeout",
           "kda_chunk_bwd_workspace_size", "kda_chunk_bwd", "kda_chunk_bwd_phase",
           "kda_chunk_fwd_noalloc_status", "kda_chunk_fwd_kernel_launches")


class LayerOpts(ctypes.Structure):
    """``kda_layer_opts_t``: the layer's gate producers and output norm (device pointers)."""
    _fields_ = [("gate_f", ctypes.c_void_p), ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("beta_logits", ctypes.c_void_p), ("out_gate", ctypes.c_void_p),
                ("norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float)]


_LAYER_KEYS = ("gate_f", "A_log", "dt_bias", "beta_logits", "out_gate", "norm_weight")


def _layer_opts(layer):
    """A ``LayerOpts`` from a dict of tensors (keys of ``_LAYER_KEYS`` plus ``norm_eps``), or None."""
    if not layer or not any(layer.get(k) is not None for k in ("gate_f", "beta_logits", "out_gate")):
        return None
    o = LayerOpts()
    for key in _LAYER_KEYS:
        t = layer.get(key)
        if t is not None:
            _need_cuda(t)
            setattr(o, key, t.data_ptr())
    o.norm_eps = float(layer.get("norm_eps", 1e-5))
    return o


class KDAError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s: %s (status %d)" % (where, status_string(code), code))
        self.code = code


def load():
    """Load ``libkda.so`` (built in-tree by ``python -m kimi_delta_attention_25_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError("libkda.so not found at %s; build it with "
                           "`python -m kimi_delta_attention_25_b200.build`" % library_path)
    lib = ctypes.CDLL(library_path)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.kda_chunk_fwd_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.kda_chunk_fwd_workspace_size.restype = Z
    lib.kda_chunk_fwd_kernel_launches.argtypes = [I, I, I, I, I]
    lib.kda_chunk_fwd_kernel_launches.restype = I
    lib.kda_chunk_fwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]
    lib.kda_chunk_fwd.restype = I
    lib.kda_decode_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P]
    lib.kda_decode_step.restype = I
    lib.kda_workspace_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    lib.kda_workspace_status.restype = I
    lib.kda_status_string.argtypes = [I]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.restype = I
    lib.kda_chunk_fwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
    lib.kda_chunk_fwd_noalloc.restype = I
    lib.kda_chunk_fwd_noalloc_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
    lib.kda_chunk_fwd_noalloc_status.restype = I
    lib.kda_chunk_prep.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, Z, P]
    lib.kda_chunk_prep.restype = I
    lib.kda_chunk_scan.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, Z, P]
    lib.kda_chunk_scan.restype = I
    lib.kda_selftest_wait_timeout.argtypes = [P, Z, ctypes.c_longlong, P]
    lib.kda_selftest_wait_timeout.restype = I
    lib.kda_chunk_bwd_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.kda_chunk_bwd_workspace_size.restype = Z
    lib.kda_chunk_bwd.argtypes = [P] * 15 + [I] * 7 + [P, Z, P]
    lib.kda_chunk_bwd.restype = I
    lib.kda_chunk_bwd_phase.argtypes = [I] + [P] * 15 + [I] * 7 + [P, Z, P]
    lib.kda_chunk_bwd_phase.restype = I
    LP = ctypes.POINTER(LayerOpts)
    lib.kda_chunk_fwd_layer_workspace_size.argtypes = [I, I, I, I, I, I, I, LP]
    lib.kda_chunk_fwd_layer_workspace_size.restype = Z
    lib.kda_chunk_fwd_layer.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, LP, P, Z, P]
    lib.kda_chunk_fwd_layer.restype = I
    lib.kda_chunk_prep_layer.argtypes = [P, P, P, P, P, I, I, I, I, I, I, LP, P, Z, P]
    lib.kda_chunk_prep_layer.restype = I
    lib.kda_chunk_scan_layer.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, LP, P, Z, P]
    lib.kda_chunk_scan_layer.restype = I
    lib.kda_decode_step_layer.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, LP, P]
    lib.kda_decode_step_layer.restype = I
    lib.kda_short_conv.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
    lib.kda_short_conv.restype = I
    lib.kda_short_conv_step.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P]
    lib.kda_short_conv_step.restype = I
    lib.kda_state_affine.argtypes = [P, P, P, P, I, I, I, P]
    lib.kda_state_affine.restype = I
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().kda_status_string(int(code)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise TypeError("q/k/v must be float32 or bfloat16, got %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libkda takes CUDA tensors only (no CPU fallback)")
        if t is not None and not t.is_contiguous():
            raise ValueError("libkda takes contiguous tensors only")


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def chunk_fwd_workspace_size(B, T, H, N, dk=128, dv=128, dtype=torch.bfloat16) -> int:
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(load().kda_chunk_fwd_workspace_size(B, T, H, N, dk, dv, code))


def chunk_fwd_kernel_launches(B, T, H, N, dtype=torch.bfloat16) -> int:
    """Kernels one ``chunk_fwd`` call with these sizes launches (``kda_chunk_fwd_kernel_launches``)."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(load().kda_chunk_fwd_kernel_launches(B, T, H, N, code))


def chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, out=None, S_final=None,
              workspace=None, want_state=True, out_dtype=torch.float32, return_workspace=False, layer=None):
    """Chunkwise KDA prefill. Shapes: q, k, log_alpha [B,T,H,dk]; v [B,T,H,dv];
    beta [B,T,H]; S0 [N,H,dk,dv] fp32 or None; cu_seqlens int32 [N+1] or None.
    Returns (out [B,T,H,dv] in out_dtype (or the dtype of a given ``out``),
    S_final [N,H,dk,dv] fp32 or None), and the workspace as a third element when
    ``return_workspace`` (its status word holds the device-side checks: ``workspace_status``).
    Without a ``workspace`` argument each call takes a fresh one from torch's caching allocator
    (about 1 KiB per token and head for bf16 inputs); a caller that runs many calls passes its own.
    ``layer`` (a dict with any of gate_f, A_log, dt_bias, beta_logits, out_gate, norm_weight,
    norm_eps) selects ``kda_chunk_fwd_layer``: the gate producers (log_alpha and/or beta may then be
    None) and the gated output norm, fused into the kernels."""
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=out_dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    _need_cuda(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final)
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    code = _dtype_code(q)
    opts = _layer_opts(layer)
    if opts is None:
        ws_bytes = lib.kda_chunk_fwd_workspace_size(B, T, H, N, dk, dv, code)
    else:
        ws_bytes = lib.kda_chunk_fwd_layer_workspace_size(B, T, H, N, dk, dv, code, ctypes.byref(opts))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(cu_seqlens), _ptr(out),
            _ptr(S_final), B, T, H, N, dk, dv, code, _dtype_code(out))
    if opts is None:
        st = lib.kda_chunk_fwd(*args, _ptr(workspace), workspace.numel(), _stream(q.device))
    else:
        st = lib.kda_chunk_fwd_layer(*args, ctypes.byref(opts), _ptr(workspace), workspace.numel(),
                                     _stream(q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd" if opts is None else "kda_chunk_fwd_layer")
    return (out, S_final, workspace) if return_workspace else (out, S_final)


def chunk_prep(q, k, log_alpha, beta, workspace, cu_seqlens=None, layer=None):
    """``kda_chunk_prep``: first pass of the bf16 prefill (everything that does not depend on the
    state), written into ``workspace`` (uint8, ``chunk_fwd_workspace_size(...)`` bytes)."""
    lib = load()
    B, T, H, dk = q.shape
    N = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    _need_cuda(q, k, log_alpha, beta, cu_seqlens, workspace)
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16:
        raise TypeError("chunk_prep takes bfloat16 q and k")
    opts = _layer_opts(layer)
    args = (_ptr(q), _ptr(k), _ptr(log_alpha), _ptr(beta), _ptr(cu_seqlens), B, T, H, N, dk, dk)
    if opts is None:
        st = lib.kda_chunk_prep(*args, _ptr(workspace), workspace.numel(), _stream(q.device))
    else:
        st = lib.kda_chunk_prep_layer(*args, ctypes.byref(opts), _ptr(workspace), workspace.numel(),
                                      _stream(q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_prep")
    return workspace


def chunk_scan(v, workspace, S0=None, cu_seqlens=None, out=None, S_final=None, want_state=True,
               out_dtype=torch.float32, layer=None):
    """``kda_chunk_scan``: second pass of the bf16 prefill, after ``chunk_prep`` on the same
    workspace and sizes. Returns (out, S_final) like ``chunk_fwd``."""
    lib = load()
    B, T, H, dv = v.shape
    N = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=out_dtype, device=v.device)
    if S_final is None and want_state:
        S_final = torch.empty(N, H, dv, dv, dtype=torch.float32, device=v.device)
    _need_cuda(v, S0, cu_seqlens, out, S_final, workspace)
    if v.dtype != torch.bfloat16:
        raise TypeError("chunk_scan takes bfloat16 v")
    opts = _layer_opts(layer)
    args = (_ptr(v), _ptr(S0), _ptr(cu_seqlens), _ptr(out), _ptr(S_final), B, T, H, N, dv, dv, _dtype_code(out))
    if opts is None:
        st = lib.kda_chunk_scan(*args, _ptr(workspace), workspace.numel(), _stream(v.device))
    else:
        st = lib.kda_chunk_scan_layer(*args, ctypes.byref(opts), _ptr(workspace), workspace.numel(),
                                      _stream(v.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_scan")
    return out, S_final


def chunk_bwd_workspace_size(B, T, H, N, dk=128, dv=128) -> int:
    return int(load().kda_chunk_bwd_workspace_size(B, T, H, N, dk, dv))


def chunk_bwd(q, k, v, log_alpha, beta, dout, S0=None, dS_final=None, cu_seqlens=None,
              want_dS0=True, grads=None, workspace=None, phase=None, return_workspace=False):
    """``kda_chunk_bwd``: gradients of a loss with gradients ``dout`` (w.r.t. every output, dtype of
    q) and ``dS_final`` (w.r.t. the final states, fp32 or None) through ``chunk_fwd`` with the same
    inputs. Returns a dict of fp32 tensors dq, dk, dv, dlog_alpha, dbeta and dS0 (None unless
    ``want_dS0``). ``grads`` may supply those tensors (same keys) to be written in place.
    ``phase`` (0, 1 or 2) runs one of the three kernels only (``kda_chunk_bwd_phase``); the phases
    must then run in order on the same ``grads`` and ``workspace``. With ``return_workspace`` the
    result is ``(grads, workspace)``."""
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    dev = q.device
    g = dict(grads) if grads is not None else {}
    f32 = dict(dtype=torch.float32, device=dev)
    g.setdefault("dq", torch.empty(B, T, H, dk, **f32))
    g.setdefault("dk", torch.empty(B, T, H, dk, **f32))
    g.setdefault("dv", torch.empty(B, T, H, dv, **f32))
    g.setdefault("dlog_alpha", torch.empty(B, T, H, dk, **f32))
    g.setdefault("dbeta", torch.empty(B, T, H, **f32))
    if want_dS0:
        g.setdefault("dS0", torch.empty(N, H, dk, dv, **f32))
    else:
        g["dS0"] = None
    _need_cuda(q, k, v, log_alpha, beta, dout, S0, dS_final, cu_seqlens, *g.values())
    if dout.dtype != q.dtype:
        raise TypeError("dout must have the dtype of q")
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"):
        if g[key] is not None and g[key].dtype != torch.float32:
            raise TypeError("%s must be float32" % key)
    ws_bytes = lib.kda_chunk_bwd_workspace_size(B, T, H, N, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(cu_seqlens), _ptr(dout),
            _ptr(dS_final), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]),
            _ptr(g["dbeta"]), _ptr(g["dS0"]), B, T, H, N, dk, dv, _dtype_code(q), _ptr(workspace),
            workspace.numel(), _stream(dev))
    if phase is None:
        st = lib.kda_chunk_bwd(*args)
    else:
        st = lib.kda_chunk_bwd_phase(int(phase), *args)
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_bwd")
    return (g, workspace) if return_workspace else g


def selftest_wait_timeout(workspace: torch.Tensor, budget_cycles: int) -> None:
    """``kda_selftest_wait_timeout``: one bounded device wait on a barrier nothing arrives on; the
    workspace status word then reads ``KDA_ERR_TIMEOUT`` (check it with ``workspace_status``)."""
    _need_cuda(workspace)
    st = load().kda_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(budget_cycles),
                                          _stream(workspace.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_selftest_wait_timeout")


def workspace_status(workspace: torch.Tensor) -> int:
    """Device status word of a workspace after a kda_chunk_fwd call (syncs the stream)."""
    v = ctypes.c_int32(0)
    st = load().kda_workspace_status(_ptr(workspace), _stream(workspace.device), ctypes.byref(v))
    if st != KDA_OK:
        raise KDAError(st, "kda_workspace_status")
    return int(v.value)


def decode_step(q, k, v, log_alpha, beta, S, out=None, out_dtype=torch.float32, layer=None):
    """One decode step: q, k, log_alpha [N,H,dk]; v [N,H,dv]; beta [N,H]; S [N,H,dk,dv] fp32
    (updated in place). Returns out [N,H,dv] in out_dtype (or the dtype of a given ``out``).
    ``layer`` as for ``chunk_fwd`` (tensors shaped [N,H,...]) selects ``kda_decode_step_layer``."""
    lib = load()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty(N, H, dv, dtype=out_dtype, device=q.device)
    _need_cuda(q, k, v, log_alpha, beta, S, out)
    opts = _layer_opts(layer)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(out), N, H, dk, dv,
            _dtype_code(q), _dtype_code(out))
    if opts is None:
        st = lib.kda_decode_step(*args, _stream(q.device))
    else:
        st = lib.kda_decode_step_layer(*args, ctypes.byref(opts), _stream(q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_decode_step")
    return out


def chunk_fwd_noalloc(q, k, v, log_alpha, beta, out, S_final=None, S0=None, cu_seqlens=None):
    """``kda_chunk_fwd_noalloc``: the chunked prefill without a workspace, for callers that may not
    allocate device memory (for example while a CUDA graph is being captured). ``out`` (and
    ``S_final`` if wanted) must be given; nothing is allocated here or in the library."""
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    _need_cuda(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final)
    st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                                   _ptr(cu_seqlens), _ptr(out), _ptr(S_final), B, T, H, N, dk, dv,
                                   _dtype_code(q), _dtype_code(out), _stream(q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_noalloc")
    return out, S_final


def noalloc_status(device=None) -> int:
    """``kda_chunk_fwd_noalloc_status``: the device-side check result of the last
    ``chunk_fwd_noalloc`` call on the current device (syncs the current stream)."""
    v = ctypes.c_int32(0)
    st = load().kda_chunk_fwd_noalloc_status(_stream(device), ctypes.byref(v))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_noalloc_status")
    return int(v.value)


# ---- padding-mask form -> packed sequences -------------------------------------------------------
# The layer can receive a batch as a [batch, seq_len] 0/1 attention mask (1 = real token, 0 =
# padding; the lpnh.cn Kimi Linear article, sec. 5, gives this form). libkda takes packed sequences
# instead: the real tokens of every row one after another (B = 1) with cu_seqlens offsets. These
# helpers only move data (index selects); every step of the computation runs in libkda.

def cu_seqlens_from_mask(mask: torch.Tensor):
    """``mask`` [B, T] of 0/1 (bool or integer). Returns ``(cu_seqlens, indices)``: int32 [B+1]
    offsets of each row's real tokens in the packed order, and int64 [total] flat indices
    (row * T + t) of those tokens, in row order and, within a row, in token order. Padding may sit
    anywhere in a row (left, right or between tokens); its positions are dropped."""
    if mask.dim() != 2:
        raise ValueError("mask must be [batch, seq_len]")
    m = mask.to(torch.bool)
    lens = m.sum(dim=1, dtype=torch.int64)
    cu = torch.zeros(m.shape[0] + 1, dtype=torch.int64, device=m.device)
    cu[1:] = torch.cumsum(lens, 0)
    indices = torch.nonzero(m.reshape(-1), as_tuple=False).reshape(-1)
    return cu.to(torch.int32), indices


def unpad(x: torch.Tensor, indices: torch.Tensor) -> torch.Tensor:
    """[B, T, ...] -> [1, total, ...]: the real tokens (``indices`` from ``cu_seqlens_from_mask``)
    packed in order, contiguous, ready for ``chunk_fwd(..., cu_seqlens=...)``."""
    B, T = x.shape[:2]
    return x.reshape(B * T, *x.shape[2:]).index_select(0, indices).unsqueeze(0).contiguous()


def pad(y: torch.Tensor, indices: torch.Tensor, B: int, T: int, fill: float = 0.0) -> torch.Tensor:
    """Inverse of ``unpad``: [1, total, ...] -> [B, T, ...] with ``fill`` at the padding positions."""
    flat = torch.full((B * T, *y.shape[2:]), fill, dtype=y.dtype, device=y.device)
    flat.index_copy_(0, indices, y.reshape(-1, *y.shape[2:]))
    return flat.reshape(B, T, *y.shape[2:])


# ---- short causal convolution and state composition --------------------------------------------

def short_conv(x, weight, bias=None, conv_state=None, cu_seqlens=None, out=None, conv_state_out=None,
               activation="silu", normalize_head_dim=0):
    """``kda_short_conv``: x [B,T,D] (float32 or bfloat16, D a multiple of 128), weight [D,K] fp32,
    bias [D] fp32 or None, conv_state [N,D,K-1] fp32 or None (zeros). Returns (y [B,T,D] in x's
    dtype, conv_state_out [N,D,K-1] or None); pass ``conv_state_out=conv_state`` to update in place,
    or ``conv_state_out=True`` for a new tensor. ``normalize_head_dim=128`` L2-normalises each head."""
    lib = load()
    B, T, D = x.shape
    K = weight.shape[1]
    N = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    if out is None:
        out = torch.empty_like(x)
    if conv_state_out is True:
        conv_state_out = torch.empty(N, D, K - 1, dtype=torch.float32, device=x.device)
    _need_cuda(x, weight, bias, conv_state, cu_seqlens, out, conv_state_out)
    st = lib.kda_short_conv(_ptr(x), _ptr(weight), _ptr(bias), _ptr(conv_state), _ptr(conv_state_out),
                            _ptr(cu_seqlens), _ptr(out), B, T, N, D, K, 1 if activation == "silu" else 0,
                            int(normalize_head_dim), _dtype_code(x), _stream(x.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_short_conv")
    return out, conv_state_out


def short_conv_step(x, weight, conv_state, bias=None, out=None, activation="silu", normalize_head_dim=0):
    """``kda_short_conv_step``: one token per sequence, x [N,D]; conv_state [N,D,K-1] fp32 is
    updated in place. Returns y [N,D]."""
    lib = load()
    N, D = x.shape
    K = weight.shape[1]
    if out is None:
        out = torch.empty_like(x)
    _need_cuda(x, weight, bias, conv_state, out)
    st = lib.kda_short_conv_step(_ptr(x), _ptr(weight), _ptr(bias), _ptr(conv_state), _ptr(out), N, D, K,
                                 1 if activation == "silu" else 0, int(normalize_head_dim), _dtype_code(x),
                                 _stream(x.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_short_conv_step")
    return out


def state_affine(Phi, S_in, Psi=None, out=None):
    """``kda_state_affine``: Phi [H,dk,dk] @ S_in [H,dk,dv] + Psi per head (fp32)."""
    lib = load()
    H, dk, dv = S_in.shape
    if out is None:
        out = torch.empty_like(S_in)
    _need_cuda(Phi, S_in, Psi, out)
    st = lib.kda_state_affine(_ptr(Phi), _ptr(S_in), _ptr(Psi), _ptr(out), H, dk, dv, _stream(S_in.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_state_affine")
    return out

