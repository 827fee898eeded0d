"""Python side of the float64 KDA oracle (test infrastructure only).

``forward`` runs the C recurrence in ``kda_ref.c`` through ctypes;
``forward_numpy`` is an independent numpy statement of the same definition:

    S <- (I - beta_t k_t k_t^T) Diag(exp(log_alpha_t)) S + beta_t k_t v_t^T ;  o_t = S^T q_t

(channel-wise forget gate and delta erase term: KimiLinear KDA/MLA tutorial
(icman.com.cn), sec. 2 and sec. 5; KDA as fine-grained-gated Gated DeltaNet:
"Kimi Linear" article (jdon.com)). Inputs are whatever the caller passes,
upcast exactly to float64; nothing here rounds to bf16.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_ref.c")
_LIB = os.path.join(_HERE, "_kda_ref.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ``kda_ref.c`` (gcc -O2, no fast-math) next to itself; return the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.kda_oracle_forward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, I]
            lib.kda_oracle_forward.restype = I
            lib.kda_oracle_online_cores.restype = I
            _lib = lib
    return _lib


def online_cores() -> int:
    return int(_load().kda_oracle_online_cores())


def _f32(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, nthreads=0,
            want_out=True, want_state=True):
    """Float64 recurrence. Arrays are numpy (or anything ``np.asarray`` accepts).

    q, k, log_alpha: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H];
    S0: [N, H, dk, dv] or None; cu_seqlens: int [N+1] or None.
    Returns (out [B, T, H, dv] float64 or None, S_final [N, H, dk, dv] float64 or None).
    """
    q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and la.shape == q.shape
    assert v.shape == (B, T, H, dv) and be.shape == (B, T, H)
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        N = cu.shape[0] - 1
    else:
        N = B
    s0 = None
    if S0 is not None:
        s0 = np.ascontiguousarray(np.asarray(S0, dtype=np.float64))
        assert s0.shape == (N, H, dk, dv)
    out = np.empty((B, T, H, dv), dtype=np.float64) if want_out else None
    sf = np.empty((N, H, dk, dv), dtype=np.float64) if want_state else None
    rc = _load().kda_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(s0),
                                    _ptr(cu), B, T, H, N, dk, dv, _ptr(out), _ptr(sf),
                                    int(nthreads))
    if rc != 0:
        raise ValueError("kda_oracle_forward rejected its arguments")
    return out, sf


def forward_numpy(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None):
    """The same definition in numpy, one token at a time (small cases only)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    la = np.asarray(log_alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(b, 0, T) for b in range(B)]
    else:
        cu = [int(x) for x in cu_seqlens]
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    N = len(spans)
    out = np.zeros((B, T, H, dv))
    Sf = np.zeros((N, H, dk, dv))
    for n, (b, t0, t1) in enumerate(spans):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[n, h], dtype=np.float64)
            for t in range(t0, t1):
                kt, vt, qt = k[b, t, h], v[b, t, h], q[b, t, h]
                A = (np.eye(dk) - be[b, t, h] * np.outer(kt, kt)) @ np.diag(np.exp(la[b, t, h]))
                S = A @ S + be[b, t, h] * np.outer(kt, vt)
                out[b, t, h] = S.T @ qt
            Sf[n, h] = S
    return out, Sf
