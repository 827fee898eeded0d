"""The KDA layer's element-wise neighbours of the recurrence, in float64 (test infrastructure only:
tests, the smoke check and the benchmark's CPU baseline use it; the CUDA path never does).

The pages name these pieces of the Kimi Linear KDA layer but print no formula for any of them
(lpnh.cn "Kimi Linear KDA/NoPE" article, sec. 3: the KDA module holds A_log, dt_bias,
f_a_proj/f_b_proj, b_proj, g_a_proj/g_b_proj; its output norm o_norm is FusedRMSNormGated with the
activation fixed to sigmoid; the layer config sets short_conv_kernel_size 4; sec. 6: the cache
keeps conv_states beside recurrent_states). The readings below are the plainest ones the names
support; each function states its reading.

* ``gated_rmsnorm``  -- the output norm: y = o / sqrt(mean_c o_c^2 + eps) * w * sigmoid(g), over
  the value channels of one head (the layer normalises each head's d_v-vector; w has d_v entries
  shared by all heads).
* ``kda_gate``       -- the channel-wise forget gate from the decay parameters: with the low-rank
  projection output f (one value per head and key channel), log alpha = -exp(A_log[h]) *
  softplus(f + dt_bias[h, c]). A_log is the log of a per-head decay rate and dt_bias a per-channel
  time-step bias, read in the continuous-to-discrete form their names describe
  (alpha = exp(-rate * step), step = softplus(f + bias) > 0, so 0 < alpha < 1).
* ``beta_gate``      -- the write gate beta = sigmoid(b) of the b_proj output.
* ``short_conv``     -- the causal depthwise convolution of kernel size K = 4 in front of q, k and v:
  y_t,c = act(bias_c + sum_{j=0}^{K-1} w_c,j x_{t-K+1+j},c), taps ordered oldest to newest,
  inputs before the first token of a sequence taken from that sequence's conv state (the last
  K-1 inputs seen before it, oldest first; zeros for a fresh sequence), act = SiLU or identity.
  The new conv state is the last K-1 inputs of the sequence (including the old state when the
  sequence is shorter than K-1).
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def sigmoid(x):
    x = _f64(x)
    return 0.5 * (1.0 + np.tanh(0.5 * x))        # the logistic function, overflow-free


def softplus(x):
    x = _f64(x)
    return np.logaddexp(0.0, x)                   # log(1 + e^x)


def gated_rmsnorm(o, g, w, eps):
    """o, g: [..., d_v]; w: [d_v]. Returns o / sqrt(mean(o^2) + eps) * w * sigmoid(g)."""
    o, g, w = _f64(o), _f64(g), _f64(w)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + float(eps)) * w * sigmoid(g)


def kda_gate(f, A_log, dt_bias):
    """f: [..., H, d_k]; A_log: [H]; dt_bias: [H, d_k] (or [H * d_k]). Returns log alpha, same
    shape as f: -exp(A_log[h]) * softplus(f + dt_bias[h, c])."""
    f, A_log, dt_bias = _f64(f), _f64(A_log), _f64(dt_bias)
    H, dk = f.shape[-2], f.shape[-1]
    dt_bias = dt_bias.reshape(H, dk)
    return -np.exp(A_log)[:, None] * softplus(f + dt_bias)


def beta_gate(b):
    """beta = sigmoid(b)."""
    return sigmoid(b)


def silu(x):
    x = _f64(x)
    return x * sigmoid(x)


def short_conv(x, weight, bias=None, conv_state=None, cu_seqlens=None, activation="silu"):
    """Causal depthwise convolution over tokens, one sequence at a time.

    x [T_total, D] (packed tokens, D channels); weight [D, K] (tap j multiplies the input K-1-j
    tokens back); bias [D] or None; conv_state [N, D, K-1] (inputs before each sequence, oldest
    first) or None for zeros; cu_seqlens [N+1] or None (one sequence). Returns (y [T_total, D],
    new_state [N, D, K-1])."""
    x, weight, bias = _f64(x), _f64(weight), _f64(bias)
    T, D = x.shape
    K = weight.shape[1]
    cu = [0, T] if cu_seqlens is None else [int(v) for v in cu_seqlens]
    N = len(cu) - 1
    st = np.zeros((N, D, K - 1)) if conv_state is None else _f64(conv_state).copy()
    y = np.zeros((T, D))
    new = np.zeros((N, D, K - 1))
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        ext = np.concatenate([st[n].T, x[a:b]], axis=0)      # [K-1 + L, D]: history then tokens
        for t in range(b - a):
            acc = np.zeros(D) if bias is None else bias.copy()
            for j in range(K):
                acc = acc + weight[:, j] * ext[t + j]
            y[a + t] = silu(acc) if activation == "silu" else acc
        new[n] = ext[ext.shape[0] - (K - 1):].T
    return y, new


def l2_normalize(x, eps=1e-6):
    """x / sqrt(sum x^2 + eps) over the last axis (the unit-norm precondition on q and k)."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
