"""Chunkwise form of the KDA recurrence in float64 (test infrastructure only).

This restates, in plain numpy, the chunk algebra that follows from the
token-by-token definition (see ``ref.py``). The pages name the technique --
chunk-parallel prefill with a WY representation, chunk size 64 (KimiLinear
KDA/MLA tutorial (icman.com.cn), sec. 3 config and sec. 6 tuning notes) -- but
print no formula, so the steps below are derived here from the definition.

Within one chunk of L <= C tokens (rows r = 0..L-1), with S the state entering
the chunk and all products per key channel c:

  g_r      = sum_{j<=r} log_alpha_j                   (cumulative log-decay)
  Kt_r     = k_r * exp(g_r)         Kh_r = k_r * exp(-g_r)
  Qt_r     = q_r * exp(g_r)         Kend_r = k_r * exp(g_{L-1} - g_r)
  A        = StrictLower(diag(beta) Kt Kh^T)          (A_ri = beta_r sum_c k_rc k_ic exp(g_rc - g_ic), i < r)
  Tm       = (I + A)^{-1}                             (unit lower triangular)
  W        = Tm diag(beta) Kt ,   U' = Tm diag(beta) V
  U        = U' - W S                                 (the per-token delta-rule writes u_r)
  O        = Qt S + tril(Qt Kh^T) U                   (diagonal included)
  S_next   = Diag(exp(g_{L-1})) S + Kend^T U

Derivation sketch: unrolling the recurrence inside the chunk gives
S_r = Diag(e^{g_r}) S + sum_{i<=r} Diag(e^{g_r - g_i}) k_i u_i^T with
u_r = beta_r (v_r - (Diag(alpha_r) S_{r-1})^T k_r); collecting the u_r gives the
unit lower-triangular system (I + A) U = diag(beta)(V - Kt S).
"""
from __future__ import annotations

import numpy as np


def _chunk(S, q, k, v, la, be):
    L = q.shape[0]
    g = np.cumsum(la, axis=0)
    Kt = k * np.exp(g)
    Kh = k * np.exp(-g)
    Qt = q * np.exp(g)
    Kend = k * np.exp(g[L - 1][None, :] - g)
    A = np.tril(be[:, None] * (Kt @ Kh.T), -1)
    Tm = np.linalg.inv(np.eye(L) + A)
    W = Tm @ (be[:, None] * Kt)
    Up = Tm @ (be[:, None] * v)
    U = Up - W @ S
    O = Qt @ S + np.tril(Qt @ Kh.T) @ U
    S_next = np.exp(g[L - 1])[:, None] * S + Kend.T @ U
    return O, S_next


def forward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, chunk=64):
    """Same arguments and results as ``ref.forward_numpy``, computed chunk by chunk."""
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
    out = np.zeros((B, T, H, dv))
    Sf = np.zeros((len(spans), H, dk, dv))
    for n, (b, t0, t1) in enumerate(spans):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[n, h], dtype=np.float64)
            for s in range(t0, t1, chunk):
                e = min(s + chunk, t1)
                O, S = _chunk(S, q[b, s:e, h], k[b, s:e, h], v[b, s:e, h], la[b, s:e, h], be[b, s:e, h])
                out[b, s:e, h] = O
            Sf[n, h] = S
    return out, Sf


def decode_step(S, q, k, v, log_alpha, beta):
    """One token per (sequence, head): the chunk form with L = 1.

    S: [N, H, dk, dv]; q, k, log_alpha: [N, H, dk]; v: [N, H, dv]; beta: [N, H].
    S' = Diag(alpha) S; w = S'^T k; u = beta (v - w); S_new = S' + k u^T;
    o = S'^T q + (q . k) u. Returns (o, S_new).
    """
    S = np.asarray(S, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    a = np.exp(np.asarray(log_alpha, dtype=np.float64))
    be = np.asarray(beta, dtype=np.float64)
    Sp = a[..., :, None] * S
    w = np.einsum("nhi,nhij->nhj", k, Sp)
    u = be[..., None] * (v - w)
    S_new = Sp + k[..., :, None] * u[..., None, :]
    o = np.einsum("nhi,nhij->nhj", q, Sp) + np.einsum("nhi,nhi->nh", q, k)[..., None] * u
    return o, S_new


def _chunk_backward(S, dSn, dO, q, k, v, la, be):
    """Gradients through one chunk of the chunk form above, given the state S entering it, the
    gradient dSn reaching the state leaving it and the gradient dO of its outputs. Reverse-mode
    chain rule through the chunk-form lines, last line first. Returns (dq, dk, dv, dla, dbe, dS)
    with dS the gradient reaching S."""
    L = q.shape[0]
    g = np.cumsum(la, axis=0)
    E = np.exp(g)
    Kt, Kh, Qt = k * E, k / E, q * E
    Kend = k * np.exp(g[L - 1][None, :] - g)
    gam = np.exp(g[L - 1])
    Pm = Kt @ Kh.T
    Tm = np.linalg.inv(np.eye(L) + np.tril(be[:, None] * Pm, -1))
    Tb = Tm * be[None, :]
    R = v - Kt @ S
    U = Tb @ R
    Mm = np.tril(Qt @ Kh.T)
    # S_next = Diag(gam) S + Kend^T U ;  O = Qt S + Mm U
    dU = Mm.T @ dO + Kend @ dSn
    dMm = np.tril(dO @ U.T)
    dQt = dO @ S.T + dMm @ Kh
    dKh = dMm.T @ Qt
    dKend = U @ dSn.T
    dgam = np.sum(dSn * S, axis=1)
    # U = Tb R,  R = V - Kt S
    dR = Tb.T @ dU
    dTb = dU @ R.T
    dS = gam[:, None] * dSn + Qt.T @ dO - Kt.T @ dR
    dv = dR
    dKt = -dR @ S.T
    # Tb = Tm diag(beta),  Tm = (I + A)^{-1},  A = StrictLower(diag(beta) Kt Kh^T)
    dbe = np.sum(dTb * Tm, axis=0)
    dTm = dTb * be[None, :]
    dA = np.tril(-Tm.T @ dTm @ Tm.T, -1)
    dbe += np.sum(dA * Pm, axis=1)
    dPm = be[:, None] * dA
    dKt += dPm @ Kh
    dKh += dPm.T @ Kt
    # back to the raw inputs through the decay scalings and g = cumsum(log_alpha)
    dq = dQt * E
    dk = dKt * E + dKh / E + dKend * np.exp(g[L - 1][None, :] - g)
    dg = dQt * Qt + dKt * Kt - dKh * Kh - dKend * Kend
    dg[L - 1] += np.sum(dKend * Kend, axis=0) + dgam * gam
    dla = np.cumsum(dg[::-1], axis=0)[::-1]
    return dq, dk, dv, dla, dbe, dS


def _chunk_backward_regrouped(S, dSn, dO, q, k, v, la, be):
    """The same gradients as ``_chunk_backward``, regrouped the way the GPU backward computes them:
    no inverse is formed -- Y = (I + A)^{-T} dU comes from one triangular solve -- and every sum
    over the value channels is a dense product:
      dU = M^T dO + Kend dSn,  Y = (I + A)^{-T} dU,  dV = diag(beta) Y,
      dS = Diag(gamma) dSn + Qt^T dO - Kt^T dV,
      dM = tril(dO U^T),  dA = -StrictLower(Y U^T),  dP = diag(beta) dA,
      dQt = dO S^T + dM Kh,  dKt = -diag(beta) Y S^T + dP Kh,  dKh = dM^T Qt + dP^T Kt,
      dKend = U dSn^T,  dgamma = rowsum(dSn * S),  dbeta = rowsum(R * Y) + rowsum(dA * Kt Kh^T).
    (From Tb = Tm diag(beta) and U = Tb R: Tm^T dTm Tm^T = Y U^T and sum_i dTb_ij Tm_ij =
    sum_v R_jv Y_jv.)"""
    L = q.shape[0]
    g = np.cumsum(la, axis=0)
    E = np.exp(g)
    Kt, Kh, Qt = k * E, k / E, q * E
    gam = E[L - 1]
    Kend = Kh * gam[None, :]
    P = Kt @ Kh.T
    A = np.tril(be[:, None] * P, -1)
    M = np.tril(Qt @ Kh.T)
    R = v - Kt @ S
    U = np.linalg.solve(np.eye(L) + A, be[:, None] * R)
    dU = M.T @ dO + Kend @ dSn
    Y = np.linalg.solve((np.eye(L) + A).T, dU)
    dv = be[:, None] * Y
    dS = gam[:, None] * dSn + Qt.T @ dO - Kt.T @ dv
    dM = np.tril(dO @ U.T)
    dA = -np.tril(Y @ U.T, -1)
    dP = be[:, None] * dA
    dQt = dO @ S.T + dM @ Kh
    dKt = -be[:, None] * (Y @ S.T) + dP @ Kh
    dKh = dM.T @ Qt + dP.T @ Kt
    dKend = U @ dSn.T
    dgam = np.sum(dSn * S, axis=1)
    dbe = np.sum(R * Y, axis=1) + np.sum(dA * P, axis=1)
    dq = dQt * E
    dk = dKt * E + (dKh + dKend * gam[None, :]) / E
    dg = dQt * Qt + dKt * Kt - dKh * Kh - dKend * Kend
    dg[L - 1] += np.sum(dKend * Kend, axis=0) + dgam * gam
    dla = np.cumsum(dg[::-1], axis=0)[::-1]
    return dq, dk, dv, dla, dbe, dS


def _chunk_backward_scan_form(S, dSn, dO, q, k, v, la, be):
    """The regrouped gradients with the serial part in the shape of the forward's state scan: every
    state-independent product is formed ahead (Tm = (I + A)^{-1} explicitly), so that only two
    products per chunk involve the carried state gradient dSn --
      seeds (no dSn):  Y0 = Tm^T M^T dO,   G0 = Qt^T dO
      operands:        Kp = Tm^T Kend,     Bk = diag(beta) Kt
      chain:           Y = Y0 + Kp dSn,    dS = Diag(gamma) dSn + G0 - Bk^T Y
    (from dU = M^T dO + Kend dSn and Y = Tm^T dU) -- mirroring U = Tb V - W S and
    S' = Diag(gamma) S + Kend^T U forward. The rest is as ``_chunk_backward_regrouped``."""
    L = q.shape[0]
    g = np.cumsum(la, axis=0)
    E = np.exp(g)
    Kt, Kh, Qt = k * E, k / E, q * E
    gam = E[L - 1]
    Kend = Kh * gam[None, :]
    P = Kt @ Kh.T
    Tm = np.linalg.inv(np.eye(L) + np.tril(be[:, None] * P, -1))
    M = np.tril(Qt @ Kh.T)
    Kp, Bk = Tm.T @ Kend, be[:, None] * Kt
    Y0, G0 = Tm.T @ (M.T @ dO), Qt.T @ dO
    Y = Y0 + Kp @ dSn
    dS = gam[:, None] * dSn + G0 - Bk.T @ Y
    R = v - Kt @ S
    U = Tm @ (be[:, None] * R)
    dv = be[:, None] * Y
    dM = np.tril(dO @ U.T)
    dA = -np.tril(Y @ U.T, -1)
    dP = be[:, None] * dA
    dQt = dO @ S.T + dM @ Kh
    dKt = -be[:, None] * (Y @ S.T) + dP @ Kh
    dKh = dM.T @ Qt + dP.T @ Kt
    dKend = U @ dSn.T
    dgam = np.sum(dSn * S, axis=1)
    dbe = np.sum(R * Y, axis=1) + np.sum(dA * P, axis=1)
    dq = dQt * E
    dk = dKt * E + (dKh + dKend * gam[None, :]) / E
    dg = dQt * Qt + dKt * Kt - dKh * Kh - dKend * Kend
    dg[L - 1] += np.sum(dKend * Kend, axis=0) + dgam * gam
    dla = np.cumsum(dg[::-1], axis=0)[::-1]
    return dq, dk, dv, dla, dbe, dS


_BACKWARD_FORMS = {"plain": "_chunk_backward", "regrouped": "_chunk_backward_regrouped",
                   "scan": "_chunk_backward_scan_form"}


def backward(q, k, v, log_alpha, beta, dout, S0=None, dS_final=None, cu_seqlens=None, chunk=64,
             form="plain"):
    """The gradients of ``backward.backward`` (same arguments and result), computed chunk by
    chunk: a forward sweep keeps the state entering every chunk, then a reverse sweep over the
    chunks carries the state gradient dS and differentiates each chunk on its own. ``form`` picks
    the per-chunk algebra: "plain" (chain rule line by line), "regrouped" (the current GPU
    backward's) or "scan" (the state-gradient scan in the forward scan's shape)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    la = np.asarray(log_alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(b, 0, T) for b in range(B)]
    else:
        cu = [int(x) for x in cu_seqlens]
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    res = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dlog_alpha=np.zeros_like(la),
               dbeta=np.zeros_like(be), dS0=np.zeros((len(spans), H, dk, dv)))
    for n, (b, t0, t1) in enumerate(spans):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[n, h], dtype=np.float64)
            bounds = [(s, min(s + chunk, t1)) for s in range(t0, t1, chunk)]
            states = []
            for s, e in bounds:
                states.append(S)
                S = _chunk(S, q[b, s:e, h], k[b, s:e, h], v[b, s:e, h], la[b, s:e, h], be[b, s:e, h])[1]
            dS = np.zeros((dk, dv)) if dS_final is None else np.array(dS_final[n, h], dtype=np.float64)
            for (s, e), Sc in zip(reversed(bounds), reversed(states)):
                f = globals()[_BACKWARD_FORMS[form]]
                r = f(Sc, dS, dout[b, s:e, h], q[b, s:e, h], k[b, s:e, h], v[b, s:e, h],
                      la[b, s:e, h], be[b, s:e, h])
                res["dq"][b, s:e, h], res["dk"][b, s:e, h], res["dv"][b, s:e, h] = r[0], r[1], r[2]
                res["dlog_alpha"][b, s:e, h], res["dbeta"][b, s:e, h] = r[3], r[4]
                dS = r[5]
            res["dS0"][n, h] = dS
    return res
