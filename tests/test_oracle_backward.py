"""Pins for the float64 backward oracle (``oracle/backward.py``): gradients fixed by the forward
definition and by calculus, never by the backward code itself.

* central finite differences of the forward definition (numpy statement, float64), element by
  element on a tiny case and along random directions on a case that spans several 64-token
  segments, two sequences and an empty one;
* reverse-mode autograd (torch, float64, CPU) of an independent torch statement of the
  definition -- mechanical differentiation instead of the hand-derived chain rule;
* closed forms: beta = 0 (pure decay, every gradient in closed form) and alpha = 1 with
  orthonormal keys and S0 = 0 (plain linear attention, whose dv, dq and dbeta are textbook);
* exact directional derivatives: dual numbers over rationals stepped through the definition with
  explicit transition matrices, on the exact inputs of the golden fixture.
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
    with pytest.raises(AssertionError):
        test_backward_equals_exact_directional_derivatives_on_the_golden_inputs()


@pytest.mark.parametrize("form", ["plain", "regrouped", "scan"])
@pytest.mark.parametrize("T,d,C,cu", [(1, 8, 64, None), (130, 16, 64, None), (200, 32, 64, [0, 70, 70, 200]),
                                      (37, 8, 8, None)])
def test_chunked_backward_equals_token_backward(T, d, C, cu, form):
    """The chunk-form gradients -- plain, regrouped (the algebra the GPU backward follows) and in
    the scan shape (two state products per chunk) -- equal the token-level reverse sweep, across
    chunk boundaries, a ragged tail and an empty sequence."""
    from oracle import chunked
    x, dout, dSf = _inputs(1, T, 2, d, d - 3, seed=T, n_seqs=cu)
    a = bw.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf,
                    cu_seqlens=cu)
    b = chunked.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_final=dSf,
                         cu_seqlens=cu, chunk=C, form=form)
    for key in a:
        assert rel_err(b[key], a[key]) < 1e-12, key


# --- exact directional derivatives: dual numbers over rationals ------------------------------

class _Dual:
    """a + b eps with eps^2 = 0, over Fractions: forward-mode derivative in exact arithmetic."""
    __slots__ = ("a", "b")

    def __init__(self, a, b=0):
        from fractions import Fraction
        self.a, self.b = Fraction(a), Fraction(b)

    @staticmethod
    def lift(x):
        return x if isinstance(x, _Dual) else _Dual(x)

    def __add__(self, o):
        o = _Dual.lift(o)
        return _Dual(self.a + o.a, self.b + o.b)

    __radd__ = __add__

    def __sub__(self, o):
        o = _Dual.lift(o)
        return _Dual(self.a - o.a, self.b - o.b)

    def __rsub__(self, o):
        return _Dual.lift(o) - self

    def __mul__(self, o):
        o = _Dual.lift(o)
        return _Dual(self.a * o.a, self.a * o.b + self.b * o.a)

    __rmul__ = __mul__


def _exact_jvp(q, k, v, alpha, beta, S0, dout, dSf, direction):
    """Exact d/d(eps) of L = sum dout * o + sum dSf * S_final for one (sequence, head) when every
    input x moves to x + eps * direction[x]; log_alpha moving by eps * delta moves alpha by
    eps * alpha * delta. The recurrence is stepped with explicit transition matrices
    (I - beta k k^T) Diag(alpha), straight from the definition."""
    T, dk, dv = len(q), len(q[0]), len(v[0])
    D = lambda name, *ix: 0 if name not in direction else direction[name][ix]  # noqa: E731

    def dual(x, name, *ix):
        return _Dual(x, D(name, *ix))

    S = [[dual(S0[i][j], "S0", i, j) for j in range(dv)] for i in range(dk)]
    L = _Dual(0)
    for t in range(T):
        qt = [dual(q[t][i], "q", t, i) for i in range(dk)]
        kt = [dual(k[t][i], "k", t, i) for i in range(dk)]
        vt = [dual(v[t][j], "v", t, j) for j in range(dv)]
        at = [_Dual(alpha[t][i], alpha[t][i] * D("log_alpha", t, i)) for i in range(dk)]
        bt = dual(beta[t], "beta", t)
        A = [[((1 if i == c else 0) - bt * kt[i] * kt[c]) * at[c] for c in range(dk)] for i in range(dk)]
        S = [[sum((A[i][c] * S[c][j] for c in range(dk)), _Dual(0)) + bt * kt[i] * vt[j] for j in range(dv)]
             for i in range(dk)]
        for j in range(dv):
            o = sum((S[i][j] * qt[i] for i in range(dk)), _Dual(0))
            L = L + o * dout[t][j]
    for i in range(dk):
        for j in range(dv):
            L = L + S[i][j] * dSf[i][j]
    return L.b


def test_backward_equals_exact_directional_derivatives_on_the_golden_inputs():
    """On the exact rational inputs of tests/golden/brute_tiny.json (two packed sequences, two
    heads, d_k = 3, d_v = 2), every gradient of the float64 backward oracle, contracted with a
    rational direction, equals the exact directional derivative of the definition."""
    import json
    import os
    import random
    from fractions import Fraction as F
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "brute_tiny.json")
    with open(path) as f:
        gd = json.load(f)
    fr = lambda a: np.vectorize(lambda x: F(x), otypes=[object])(np.array(a, dtype=object))  # noqa: E731
    q, k, v = fr(gd["q"]), fr(gd["k"]), fr(gd["v"])                 # [T][H][d]
    alpha, beta, S0 = fr(gd["alpha"]), fr(gd["beta"]), fr(gd["S0"])
    cu = gd["cu_seqlens"]
    T, H = q.shape[0], q.shape[1]
    rnd = random.Random(11)
    rat = lambda *shape: np.vectorize(lambda _: F(rnd.randint(-6, 6), 4), otypes=[object])(  # noqa: E731
        np.zeros(shape))
    dout, dSf = rat(T, H, v.shape[2]), rat(len(cu) - 1, H, k.shape[2], v.shape[2])
    fl = lambda a: np.vectorize(float)(a).astype(np.float64)  # noqa: E731
    g = bw.backward(fl(q)[None], fl(k)[None], fl(v)[None], np.log(fl(alpha))[None], fl(beta)[None],
                    fl(dout)[None], S0=fl(S0), dS_final=fl(dSf), cu_seqlens=cu)
    for n in range(len(cu) - 1):
        t0, t1 = cu[n], cu[n + 1]
        for h in range(H):
            seq = lambda a: [list(a[t, h]) for t in range(t0, t1)]  # noqa: E731
            args = (seq(q), seq(k), seq(v), seq(alpha), [beta[t, h] for t in range(t0, t1)],
                    [list(r) for r in S0[n, h]], seq(dout), [list(r) for r in dSf[n, h]])
            for name, gname in NAMES:
                if name == "S0":
                    d = rat(k.shape[2], v.shape[2])
                    mine = float(np.sum(g["dS0"][n, h] * fl(d)))
                elif name == "beta":
                    d = rat(t1 - t0)
                    mine = float(np.sum(g["dbeta"][0, t0:t1, h] * fl(d)))
                else:
                    width = v.shape[2] if name == "v" else k.shape[2]
                    d = rat(t1 - t0, width)
                    mine = float(np.sum(g[gname][0, t0:t1, h] * fl(d)))
                exact = _exact_jvp(*args, direction={name: d})
                assert abs(mine - float(exact)) <= 1e-12 * max(1.0, abs(float(exact))), (n, h, name, mine, exact)
