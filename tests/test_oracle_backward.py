"""Pins for the float64 backward oracle (``oracle/backward.py``): gradients fixed by the forward
definition and by calculus, never by the backward code itself.

* central finite differences of the forward definition (numpy statement, float64), element by
  element on a tiny case and along random directions on a case that spans several 64-token
  segments, two sequences and an empty one;
* reverse-mode autograd (torch, float64, CPU) of an independent torch statement of the
  definition -- mechanical differentiation instead of the hand-derived chain rule;
* closed forms: beta = 0 (pure decay, every gradient in closed form) and alpha = 1 with
  orthonormal keys and S0 = 0 (plain linear attention, whose dv, dq and dbeta are textbook).
The last test plants slips in a copy of the backward oracle and checks the pins catch them.
"""
import math

import numpy as np
import pytest
import torch

from oracle import backward as bw
from oracle import ref


def rel_err(x, r):
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    rms = math.sqrt(float(np.mean(r * r))) if r.size else 0.0
    return float(np.max(np.abs(x - r))) / (rms if rms > 0 else 1.0) if r.size else 0.0


def _inputs(B, T, H, dk, dv, seed, n_seqs=None, alpha=(0.8, 0.99)):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    la = np.log(rng.uniform(alpha[0], alpha[1], (B, T, H, dk)))
    be = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    N = B if n_seqs is None else len(n_seqs) - 1
    S0 = 0.3 * rng.standard_normal((N, H, dk, dv))
    dout = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((N, H, dk, dv))
    return dict(q=q, k=k, v=v, log_alpha=la, beta=be, S0=S0, cu_seqlens=n_seqs), dout, dSf


def _loss(x, dout, dSf):
    out, Sf = ref.forward_numpy(**x)
    return float(np.sum(out * dout) + np.sum(Sf * dSf))


NAMES = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_alpha", "dlog_alpha"), ("beta", "dbeta"), ("S0", "dS0")]


def test_backward_equals_finite_differences_elementwise():
    x, dout, dSf = _inputs(1, 5, 1, 3, 2, seed=1)
    g = bw.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf)
    eps = 1e-6
    for name, gname in NAMES:
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            xp = {key: (None if val is None else np.array(val, copy=True)) for key, val in x.items()}
            xm = {key: (None if val is None else np.array(val, copy=True)) for key, val in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (_loss(xp, dout, dSf) - _loss(xm, dout, dSf)) / (2 * eps)
        assert np.max(np.abs(g[gname] - fd)) < 1e-7 * max(1.0, np.max(np.abs(fd))), name


def test_backward_equals_finite_differences_directional_varlen():
    cu = [0, 70, 70, 140]                       # three sequences, one empty; 70 > one segment
    x, dout, dSf = _inputs(1, 140, 2, 6, 4, seed=2, n_seqs=cu)
    g = bw.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf,
                    cu_seqlens=cu)
    rng = np.random.default_rng(3)
    eps = 1e-6
    for name, gname in NAMES:
        d = rng.standard_normal(x[name].shape)
        xp = dict(x)
        xm = dict(x)
        xp[name] = x[name] + eps * d
        xm[name] = x[name] - eps * d
        fd = (_loss(xp, dout, dSf) - _loss(xm, dout, dSf)) / (2 * eps)
        an = float(np.sum(g[gname] * d))
        assert abs(an - fd) < 1e-7 * max(1.0, abs(fd)), (name, an, fd)
    # the empty sequence passes its final-state gradient straight through
    assert np.array_equal(g["dS0"][1], dSf[1])


def _torch_forward(q, k, v, la, be, S0):
    """Independent torch statement of the definition for one (sequence, head)."""
    S = S0
    outs = []
    I = torch.eye(q.shape[1], dtype=torch.float64)
    for t in range(q.shape[0]):
        A = (I - be[t] * torch.outer(k[t], k[t])) @ torch.diag(torch.exp(la[t]))
        S = A @ S + be[t] * torch.outer(k[t], v[t])
        outs.append(S.T @ q[t])
    return torch.stack(outs), S


@pytest.mark.parametrize("T", [1, 64, 130])
def test_backward_equals_autograd(T):
    x, dout, dSf = _inputs(1, T, 1, 16, 12, seed=4 + T)
    tens = {n: torch.tensor(x[n][0, :, 0], requires_grad=True) for n in ("q", "k", "v", "log_alpha")}
    tens["beta"] = torch.tensor(x["beta"][0, :, 0], requires_grad=True)
    tens["S0"] = torch.tensor(x["S0"][0, 0], requires_grad=True)
    out, Sf = _torch_forward(tens["q"], tens["k"], tens["v"], tens["log_alpha"], tens["beta"], tens["S0"])
    L = (out * torch.tensor(dout[0, :, 0])).sum() + (Sf * torch.tensor(dSf[0, 0])).sum()
    L.backward()
    g = bw.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf)
    for name, gname in NAMES:
        mine = g[gname][0, 0] if name == "S0" else g[gname][0, :, 0]
        assert rel_err(mine, tens[name].grad.numpy()) < 1e-12, name


def test_beta_zero_closed_form_gradients():
    """beta = 0: S_t = Diag(e^{G_t}) S0 with G_t = sum_{j<=t} log_alpha_j, o_t = S_t^T q_t, so
    L = sum_t q_t^T Diag(e^{G_t}) S0 do_t + <dSf, Diag(e^{G_T}) S0>. Then dv = 0, dk = 0 (k and v
    only enter through beta), dq_t = S_t do_t, dS0 = sum_t e^{G_t} q_t do_t^T + Diag(e^{G_T}) dSf,
    dlog_alpha_j = sum_{t>=j} e^{G_t} q_t (S0 do_t) + e^{G_T} rowsum(dSf * S0), and
    dbeta_t = (v_t - P_t^T k_t) . (G_t^T k_t) with G_t the gradient reaching S_t."""
    T, dk, dv = 20, 5, 4
    x, dout, dSf = _inputs(1, T, 1, dk, dv, seed=7)
    x["beta"] = np.zeros_like(x["beta"])
    g = bw.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf)
    q, k, v, la, S0 = x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0], x["log_alpha"][0, :, 0], x["S0"][0, 0]
    do, dS = dout[0, :, 0], dSf[0, 0]
    G = np.cumsum(la, axis=0)
    E = np.exp(G)                                              # [T, dk]
    assert np.max(np.abs(g["dv"])) == 0 and np.max(np.abs(g["dk"])) == 0
    dq = np.stack([(E[t][:, None] * S0) @ do[t] for t in range(T)])
    dS0 = sum(np.outer(E[t] * q[t], do[t]) for t in range(T)) + E[-1][:, None] * dS
    c = np.stack([E[t] * q[t] * (S0 @ do[t]) for t in range(T)])   # [T, dk]
    dla = np.cumsum(c[::-1], axis=0)[::-1] + E[-1] * np.sum(dS * S0, axis=1)
    dbe = np.zeros(T)
    for t in range(T):
        # gradient reaching S_t: later reads, decayed back to t, plus the final-state term
        Gt = sum(np.outer(np.exp(G[r] - G[t]) * q[r], do[r]) for r in range(t, T)) + np.exp(G[-1] - G[t])[:, None] * dS
        Pt = E[t][:, None] * S0
        dbe[t] = (v[t] - Pt.T @ k[t]) @ (Gt.T @ k[t])
    assert rel_err(g["dq"][0, :, 0], dq) < 1e-13
    assert rel_err(g["dS0"][0, 0], dS0) < 1e-13
    assert rel_err(g["dlog_alpha"][0, :, 0], dla) < 1e-13
    assert rel_err(g["dbeta"][0, :, 0], dbe) < 1e-13


def test_linear_attention_closed_form_gradients():
    """alpha = 1, S0 = 0, mutually orthonormal keys: every erase term is zero, u_i = beta_i v_i and
    o_t = sum_{i<=t} beta_i (q_t . k_i) v_i (linear attention). Its gradients: dv_i = beta_i
    sum_{t>=i} (q_t . k_i) do_t, dq_t = sum_{i<=t} beta_i (v_i . do_t) k_i, dbeta_i = v_i .
    sum_{t>=i} (q_t . k_i) do_t."""
    T, d, dv = 12, 16, 5
    rng = np.random.default_rng(8)
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    k = Qm[:T][None, :, None, :]
    q = rng.standard_normal((1, T, 1, d))
    v = rng.standard_normal((1, T, 1, dv))
    be = rng.uniform(0.1, 0.9, (1, T, 1))
    la = np.zeros((1, T, 1, d))
    dout = rng.standard_normal((1, T, 1, dv))
    g = bw.backward(q, k, v, la, be, dout)
    K, Q, V, b, do = k[0, :, 0], q[0, :, 0], v[0, :, 0], be[0, :, 0], dout[0, :, 0]
    QK = Q @ K.T                                               # [t, i] = q_t . k_i
    causal = np.tril(np.ones((T, T)))
    dv_ref = b[:, None] * ((QK * causal).T @ do)
    dq_ref = ((do @ V.T) * causal * b[None, :]) @ K
    dbe_ref = np.sum(V * ((QK * causal).T @ do), axis=1)
    assert rel_err(g["dv"][0, :, 0], dv_ref) < 1e-13
    assert rel_err(g["dq"][0, :, 0], dq_ref) < 1e-13
    assert rel_err(g["dbeta"][0, :, 0], dbe_ref) < 1e-13


# --- the pins catch plausible slips ---------------------------------------------------------

_BACKWARD_HEAD = bw.backward_head


def _slipped_head(slip):
    def f(q, k, v, la, be, S0, dout, dSf):
        gq, gk, gv, gla, gbe, gS0 = _BACKWARD_HEAD(q, k, v, la, be, S0, dout, dSf)
        if slip == "dla_uses_prev_state":      # rowsum(dP * S_{t-1}) instead of dP * P_t
            gla = gla / np.exp(np.asarray(la))
        elif slip == "dk_drops_erase_term":
            S = np.zeros((q.shape[1], v.shape[1])) if S0 is None else np.array(S0)
            # dk without its P_t dw term
            gk2 = np.zeros_like(gk)
            G = np.array(dSf) if dSf is not None else np.zeros_like(S)
            states = [S]
            for t in range(q.shape[0]):
                states.append(bw._step(states[-1], k[t], v[t], la[t], be[t])[3])
            for t in range(q.shape[0] - 1, -1, -1):
                P, w, u, St = bw._step(states[t], k[t], v[t], la[t], be[t])
                G = G + np.outer(q[t], dout[t])
                gk2[t] = G @ u
                du = G.T @ k[t]
                dP = G + np.outer(k[t], -be[t] * du)
                G = np.exp(la[t])[:, None] * dP
            gk = gk2
        elif slip == "dbeta_sign":
            gbe = -gbe
        elif slip == "dS0_undecayed":
            gS0 = gS0 / np.exp(np.asarray(la[0]))[:, None]
        return gq, gk, gv, gla, gbe, gS0
    return f


@pytest.mark.parametrize("slip", ["dla_uses_prev_state", "dk_drops_erase_term", "dbeta_sign", "dS0_undecayed"])
def test_pins_reject_planted_slips(slip, monkeypatch):
    monkeypatch.setattr(bw, "backward_head", _slipped_head(slip))
    with pytest.raises(AssertionError):
        test_backward_equals_autograd(64)


@pytest.mark.parametrize("T,d,C,cu", [(1, 8, 64, None), (130, 16, 64, None), (200, 32, 64, [0, 70, 70, 200]),
                                      (37, 8, 8, None)])
def test_chunked_backward_equals_token_backward(T, d, C, cu):
    """The chunk-form gradients (the algebra the GPU backward follows) equal the token-level
    reverse sweep, across chunk boundaries, a ragged tail and an empty sequence."""
    from oracle import chunked
    x, dout, dSf = _inputs(1, T, 2, d, d - 3, seed=T, n_seqs=cu)
    a = bw.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf,
                    cu_seqlens=cu)
    b = chunked.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf,
                         cu_seqlens=cu, chunk=C)
    for key in a:
        assert rel_err(b[key], a[key]) < 1e-12, key
