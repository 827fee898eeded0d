"""Pins of the layer-level oracle functions (oracle/layer.py) against values fixed by hand, closed
forms, a library routine and planted slips. CPU only."""
import math

import numpy as np
import pytest

from oracle import layer

RNG = np.random.default_rng(7)


# ---- gated RMSNorm output (o_norm = FusedRMSNormGated, sigmoid gate) ----------------------------

def test_gated_rmsnorm_worked_example():
    # o = (3, 4): mean of squares 12.5, rms 5/sqrt(2); w = (1, 2); g = 0 -> sigmoid 1/2; eps = 0:
    # y = (3 sqrt(2)/10, 4 sqrt(2)/5), worked out by hand
    y = layer.gated_rmsnorm([3.0, 4.0], [0.0, 0.0], [1.0, 2.0], 0.0)
    assert np.allclose(y, [0.42426406871192851, 1.1313708498984760], rtol=0, atol=1e-15)
    # g = ln 3 -> sigmoid 3/4; w = (2, 0.5); o = (-1, 1, 1, -1): rms 1 -> y = (-1.5, 0.375, 0.375, -1.5)... per channel
    y = layer.gated_rmsnorm([-1.0, 1.0, 1.0, -1.0], [math.log(3.0)] * 4, [2.0, 0.5, 0.5, 2.0], 0.0)
    assert np.allclose(y, [-1.5, 0.375, 0.375, -1.5], rtol=0, atol=1e-15)
    # eps inside the root: o = (3, 4), eps = 37.5 -> sqrt(12.5 + 37.5) = 5 sqrt(2); w = 1, g = 0:
    # y = (3 sqrt(2)/20, 4 sqrt(2)/20)
    y = layer.gated_rmsnorm([3.0, 4.0], [0.0, 0.0], [1.0, 1.0], 37.5)
    assert np.allclose(y, [0.21213203435596426, 0.28284271247461901], rtol=0, atol=1e-15)


def test_gated_rmsnorm_closed_forms():
    o = RNG.normal(size=(5, 128))
    w = RNG.uniform(0.5, 1.5, size=128)
    big = np.full_like(o, 60.0)
    y = layer.gated_rmsnorm(o, big, w, 0.0)                      # open gate: plain RMSNorm times w
    assert np.allclose(np.mean((y / w) ** 2, axis=-1), 1.0, atol=1e-12)
    assert np.allclose(layer.gated_rmsnorm(o, -big, w, 0.0), 0.0, atol=1e-20)   # closed gate
    a = np.array([[2.5], [-0.3]])
    g = RNG.normal(size=(2, 128))
    y = layer.gated_rmsnorm(np.repeat(a, 128, axis=1), g, w, 0.0)   # constant vector: sign(a) w sigma(g)
    assert np.allclose(y, np.sign(a) * w / (1 + np.exp(-g)), atol=1e-14)
    g = RNG.normal(size=o.shape)
    assert np.allclose(layer.gated_rmsnorm(7.0 * o, g, w, 0.0), layer.gated_rmsnorm(o, g, w, 0.0), atol=1e-13)
    # eps dominates: y ~ o w sigma(g) / sqrt(eps)
    assert np.allclose(layer.gated_rmsnorm(1e-6 * o, g, w, 1.0), 1e-6 * o * w / (1 + np.exp(-g)), rtol=1e-9)


def _planted_norms():
    sig = lambda g: 1 / (1 + np.exp(-np.asarray(g)))  # noqa: E731
    return {
        "sum instead of mean": lambda o, g, w, e: o / np.sqrt(np.sum(np.square(o), -1, keepdims=True) + e) * w * sig(g),
        "no gate": lambda o, g, w, e: o / np.sqrt(np.mean(np.square(o), -1, keepdims=True) + e) * w,
        "no weight": lambda o, g, w, e: o / np.sqrt(np.mean(np.square(o), -1, keepdims=True) + e) * sig(g),
        "eps outside the root": lambda o, g, w, e: o / (np.sqrt(np.mean(np.square(o), -1, keepdims=True)) + e) * w * sig(g),
        "swish gate": lambda o, g, w, e: o / np.sqrt(np.mean(np.square(o), -1, keepdims=True) + e) * w * np.asarray(g) * sig(g),
    }


@pytest.mark.parametrize("slip", list(_planted_norms()))
def test_gated_rmsnorm_pins_reject_planted_slips(slip):
    f = _planted_norms()[slip]
    o1 = np.array([3.0, 4.0]); g1 = np.zeros(2); w1 = np.array([1.0, 2.0])
    o2 = np.array([-1.0, 1.0, 1.0, -1.0]); g2 = np.full(4, math.log(3.0)); w2 = np.array([2.0, 0.5, 0.5, 2.0])
    ok1 = np.allclose(f(o1, g1, w1, 0.0), [0.42426406871192851, 1.1313708498984760], atol=1e-12)
    ok2 = np.allclose(f(o2, g2, w2, 0.0), [-1.5, 0.375, 0.375, -1.5], atol=1e-12)
    o3 = RNG.normal(size=128) * 1e-6; g3 = RNG.normal(size=128); w3 = np.ones(128)
    ok3 = np.allclose(f(o3, g3, w3, 1.0), o3 * w3 / (1 + np.exp(-g3)), rtol=1e-9)
    ok4 = np.allclose(f(o1, g1, np.ones(2), 37.5), [0.21213203435596426, 0.28284271247461901], atol=1e-12)
    assert not (ok1 and ok2 and ok3 and ok4), slip


# ---- fused gate producer (A_log, dt_bias, softplus) and the write gate ---------------------------

def test_kda_gate_exact_values():
    # A_log = 0 and f + dt_bias = 0: rate 1, step softplus(0) = ln 2 -> alpha = 1/2 exactly
    la = layer.kda_gate(np.zeros((1, 2, 3)), np.zeros(2), np.zeros((2, 3)))
    assert np.allclose(la, -math.log(2.0), atol=1e-15)
    # A_log = ln 2, f + dt_bias = ln(e - 1): step 1 -> log alpha = -2
    f = np.full((1, 1, 4), math.log(math.e - 1.0) - 0.25)
    la = layer.kda_gate(f, [math.log(2.0)], np.full((1, 4), 0.25))
    assert np.allclose(la, -2.0, atol=1e-14)


def test_kda_gate_limits_and_layout():
    f = RNG.normal(size=(3, 2, 5))
    dt = RNG.normal(size=(2, 5))
    # A_log -> -inf: the decay rate vanishes, alpha -> 1
    assert np.allclose(layer.kda_gate(f, [-60.0, -60.0], dt), 0.0, atol=1e-20)
    # large f + dt_bias: softplus is linear -> log alpha = -exp(A_log) (f + dt_bias)
    A = np.array([0.3, -1.2])
    la = layer.kda_gate(f + 50.0, A, dt)
    assert np.allclose(la, -np.exp(A)[:, None] * (f + 50.0 + dt), rtol=1e-15)
    # very negative f + dt_bias: softplus(x) ~ e^x -> alpha -> 1 from below
    la = layer.kda_gate(f - 60.0, A, dt)
    assert np.all(la < 0) and np.allclose(la / (-np.exp(A)[:, None] * np.exp(f - 60.0 + dt)), 1.0, atol=1e-12)
    # per-head rate, per (head, channel) bias: swapping heads of A_log changes only that head
    la1 = layer.kda_gate(f, A, dt)
    la2 = layer.kda_gate(f, A[::-1], dt)
    assert np.allclose(la1[:, 0] * np.exp(A[1] - A[0]), la2[:, 0])
    assert np.allclose(layer.kda_gate(f, A, dt.reshape(-1)), la1)      # flat [H * d_k] bias


def test_beta_gate_values():
    assert layer.beta_gate(0.0) == 0.5
    assert abs(layer.beta_gate(math.log(3.0)) - 0.75) < 1e-15
    assert abs(layer.beta_gate(-math.log(3.0)) - 0.25) < 1e-15


# ---- short causal convolution (kernel 4) with conv states ----------------------------------------

def test_short_conv_taps_and_history():
    x = RNG.normal(size=(9, 6))
    w_now = np.zeros((6, 4)); w_now[:, 3] = 1.0                      # newest tap only: identity
    y, st = layer.short_conv(x, w_now, activation=None)
    assert np.array_equal(y, x)
    assert np.array_equal(st[0], x[-3:].T)                            # state = last 3 inputs
    w_old = np.zeros((6, 4)); w_old[:, 0] = 1.0                       # oldest tap: shift by 3
    hist = RNG.normal(size=(1, 6, 3))
    y, _ = layer.short_conv(x, w_old, conv_state=hist, activation=None)
    assert np.array_equal(y[3:], x[:-3])
    assert np.array_equal(y[:3], hist[0].T)                           # the history, oldest first


def test_short_conv_matches_numpy_convolve():
    x = RNG.normal(size=(40, 3))
    w = RNG.normal(size=(3, 4))
    b = RNG.normal(size=3)
    y, _ = layer.short_conv(x, w, bias=b, activation=None)
    for c in range(3):
        ref = np.convolve(x[:, c], w[c, ::-1])[:40] + b[c]           # zero history, causal
        assert np.allclose(y[:, c], ref, atol=1e-13)
    ys, _ = layer.short_conv(x, w, bias=b, activation="silu")
    assert np.allclose(ys, y / (1 + np.exp(-y)), atol=1e-14)


def test_short_conv_split_continuation_and_packing():
    x = RNG.normal(size=(30, 5))
    w = RNG.normal(size=(5, 4))
    y, st = layer.short_conv(x, w)
    for cut in (1, 2, 3, 17):
        ya, sa = layer.short_conv(x[:cut], w)
        yb, sb = layer.short_conv(x[cut:], w, conv_state=sa)
        assert np.allclose(np.concatenate([ya, yb]), y, atol=1e-14)
        assert np.allclose(sb, st, atol=0)
    cu = [0, 7, 7, 8, 30]                                              # packed, with empty and 1-token
    states = RNG.normal(size=(4, 5, 3))
    yp, sp = layer.short_conv(x, w, conv_state=states, cu_seqlens=cu)
    for n in range(4):
        yn, sn = layer.short_conv(x[cu[n]:cu[n + 1]], w, conv_state=states[n:n + 1])
        assert np.allclose(yp[cu[n]:cu[n + 1]], yn, atol=1e-14)
        assert np.allclose(sp[n], sn[0], atol=0)
    assert np.array_equal(sp[1], states[1])                            # empty sequence keeps its state
    assert np.array_equal(sp[2][:, :2], states[2][:, 1:]) and np.array_equal(sp[2][:, 2], x[7])


def test_l2_normalize():
    x = RNG.normal(size=(4, 128))
    y = layer.l2_normalize(x, eps=0.0)
    assert np.allclose(np.sum(y * y, axis=-1), 1.0, atol=1e-14)
    assert np.allclose(layer.l2_normalize(np.array([3.0, 4.0]), eps=0.0), [0.6, 0.8], atol=1e-15)
