"""Float64 gradients of the KDA recurrence (test infrastructure only).

The forward definition, per sequence and head, one token t at a time (channel-wise forget
gate and delta-rule erase/write: KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 2 and 5;
"Kimi Linear" article (jdon.com), KDA as fine-grained-gated Gated DeltaNet), written in the
intermediate quantities that the reverse sweep needs:

    a_t = exp(log_alpha_t)                    (per key channel)
    P_t = Diag(a_t) S_{t-1}                   (decayed state)
    w_t = P_t^T k_t                           (what the state currently returns for k_t)
    u_t = beta_t (v_t - w_t)                  (the delta-rule write)
    S_t = P_t + k_t u_t^T
    o_t = S_t^T q_t

This is the same map as S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T.
The pages print no backward pass; the gradients below are the chain rule applied to those six
lines in reverse order (reverse-mode differentiation of the definition), for a scalar loss L
whose gradients with respect to every o_t (``dout``) and to the final state (``dS_final``) are
given. With G the running dL/dS_t:

    G     += q_t do_t^T ;           dq_t  = S_t do_t
    dP     = G ;                    dk_t  = G u_t ;           du = G^T k_t
    dv_t   = beta_t du ;            dbeta_t = du . (v_t - w_t) ;   dw = -beta_t du
    dP    += k_t dw^T ;             dk_t += P_t dw
    dlog_alpha_t = rowsum(dP * P_t) (elementwise product, summed over the value channels)
    G      = Diag(a_t) dP           (dL/dS_{t-1});   dS0 = G after the first token

Memory only: the states S_t are needed in reverse order, so they are recomputed one
64-token segment at a time from stored segment-start states; the arithmetic is that of the
definition, token by token.

Parity status: pinned by tests that do not go through this file -- central finite differences
of the forward oracle, reverse-mode autograd of a float64 torch statement of the definition, and
closed forms (beta = 0) -- see ``tests/test_oracle_backward.py``.
"""
from __future__ import annotations

import numpy as np

_SEG = 64


def _spans(B, T, cu_seqlens):
    if cu_seqlens is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(x) for x in cu_seqlens]
    return [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def _step(S, k, v, la, be):
    """One token of the definition; returns (P, w, u, S_new)."""
    P = np.exp(la)[:, None] * S
    w = P.T @ k
    u = be * (v - w)
    return P, w, u, P + np.outer(k, u)


def backward_head(q, k, v, la, be, S0, dout, dSf):
    """Gradients for one (sequence, head). q, k, la: [L, dk]; v, dout: [L, dv]; be: [L];
    S0, dSf: [dk, dv] (None = zero). Returns (dq, dk, dv, dla, dbe, dS0)."""
    q, k, v, la = (np.asarray(x, dtype=np.float64) for x in (q, k, v, la))
    be = np.asarray(be, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    L, dk_ = q.shape
    dv_ = v.shape[1]
    S = np.zeros((dk_, dv_)) if S0 is None else np.array(S0, dtype=np.float64)
    # forward sweep, keeping the state entering each segment
    starts = []
    for s in range(0, L, _SEG):
        starts.append(S.copy())
        for t in range(s, min(s + _SEG, L)):
            S = _step(S, k[t], v[t], la[t], be[t])[3]
    G = np.zeros((dk_, dv_)) if dSf is None else np.array(dSf, dtype=np.float64)
    gq = np.zeros_like(q)
    gk = np.zeros_like(k)
    gv = np.zeros_like(v)
    gla = np.zeros_like(la)
    gbe = np.zeros_like(be)
    for si in range(len(starts) - 1, -1, -1):
        s = si * _SEG
        e = min(s + _SEG, L)
        # recompute the segment's per-token quantities from its start state
        Sprev = starts[si]
        rec = []
        for t in range(s, e):
            P, w, u, Snew = _step(Sprev, k[t], v[t], la[t], be[t])
            rec.append((P, w, u, Snew))
            Sprev = Snew
        for t in range(e - 1, s - 1, -1):
            P, w, u, St = rec[t - s]
            G = G + np.outer(q[t], dout[t])
            gq[t] = St @ dout[t]
            dP = G
            gk[t] = G @ u
            du = G.T @ k[t]
            gv[t] = be[t] * du
            gbe[t] = du @ (v[t] - w)
            dw = -be[t] * du
            dP = dP + np.outer(k[t], dw)
            gk[t] += P @ dw
            gla[t] = np.sum(dP * P, axis=1)
            G = np.exp(la[t])[:, None] * dP
    return gq, gk, gv, gla, gbe, G


def backward(q, k, v, log_alpha, beta, dout, S0=None, dS_final=None, cu_seqlens=None, heads=None):
    """Gradients of L = sum(dout * out) + sum(dS_final * S_final) for the whole batch.

    Shapes as in ``ref.forward``: q, k, log_alpha [B, T, H, dk]; v, dout [B, T, H, dv];
    beta [B, T, H]; S0, dS_final [N, H, dk, dv] or None (zero); cu_seqlens [N+1] or None.
    ``heads``: restrict to these head indices (the other heads' gradients are left zero).
    Returns a dict of float64 arrays dq, dk, dv, dlog_alpha, dbeta (input shapes) and dS0
    [N, H, dk, dv].
    """
    q = np.asarray(q, dtype=np.float64)
    B, T, H, dk_ = q.shape
    dv_ = np.asarray(v).shape[-1]
    spans = _spans(B, T, cu_seqlens)
    res = dict(dq=np.zeros((B, T, H, dk_)), dk=np.zeros((B, T, H, dk_)), dv=np.zeros((B, T, H, dv_)),
               dlog_alpha=np.zeros((B, T, H, dk_)), dbeta=np.zeros((B, T, H)),
               dS0=np.zeros((len(spans), H, dk_, dv_)))
    for n, (b, t0, t1) in enumerate(spans):
        for h in (range(H) if heads is None else heads):
            g = backward_head(q[b, t0:t1, h], np.asarray(k)[b, t0:t1, h], np.asarray(v)[b, t0:t1, h],
                              np.asarray(log_alpha)[b, t0:t1, h], np.asarray(beta)[b, t0:t1, h],
                              None if S0 is None else np.asarray(S0)[n, h],
                              np.asarray(dout)[b, t0:t1, h],
                              None if dS_final is None else np.asarray(dS_final)[n, h])
            res["dq"][b, t0:t1, h], res["dk"][b, t0:t1, h], res["dv"][b, t0:t1, h] = g[0], g[1], g[2]
            res["dlog_alpha"][b, t0:t1, h], res["dbeta"][b, t0:t1, h] = g[3], g[4]
            res["dS0"][n, h] = g[5]
    return res
