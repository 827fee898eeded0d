"""Seeded synthetic inputs for the KDA (Kimi Delta Attention) hot path.

This module only draws random numbers. It holds none of the method's
arithmetic, so both the float64 oracle (``oracle/``) and the CUDA path
(``kimi_delta_attention_25_b200``) can be fed from it without sharing code.

The five workloads follow the shapes the source pages give for a KDA layer
(head_dim 128, 16 or 32 heads, chunk 64; "Kimi Linear" config sections of the
icman.com.cn and lpnh.cn tutorials, section 3): two single-sequence prefills,
one 128K-token prefill, one packed variable-length prefill and one large
decode batch.

Recipe (one ``torch.Generator`` per tensor stream, seeded with the config
seed; draw order q, k, v, log_alpha, beta, S0):

* q, k ~ N(0, 1) in fp32, L2-normalised over the head dimension in fp32,
  then rounded to the input dtype (round-to-nearest-even). The normalisation
  is a precondition of the layer (the erase term needs unit keys), not part
  of the recurrence.
* v ~ N(0, 1), rounded to the input dtype.
* log_alpha = log(U(lo, hi)) in fp32, per token, head and key channel.
* beta = sigmoid(N(0, 1)) in fp32, per token and head.
* S0 = 0, or N(0, 0.1^2) in fp32 (0.1 is the standard deviation).
* decode step s draws q, k, v, log_alpha, beta with seed 1000 + s.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_prefill", "make_decode_state",
           "make_decode_step", "varlen_lengths", "to_dtype", "make_layer_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int                 # tokens per batch row (total packed tokens when varlen)
    H: int
    dk: int = 128
    dv: int = 128
    dtype: str = "bf16"    # q, k, v, out
    alpha_lo: float = 0.9
    alpha_hi: float = 0.999
    s0_std: float = 0.0    # 0 -> S0 = 0
    n_seqs: int = 0        # >0: packed variable-length sequences (B must be 1)
    len_lo: int = 0
    len_hi: int = 0
    decode_steps: int = 0  # >0: decode workload (N = B sequences, one token per step)
    seed: int = 0


WORKLOADS = {
    "fp32_t256_h2": Workload("fp32_t256_h2", B=1, T=256, H=2, dtype="f32"),
    "bf16_t8k_h16": Workload("bf16_t8k_h16", B=1, T=8192, H=16),
    "bf16_t128k_h32": Workload("bf16_t128k_h32", B=1, T=131072, H=32,
                               alpha_lo=0.95, alpha_hi=0.9999, s0_std=0.1),
    "bf16_varlen8_262k_h32": Workload("bf16_varlen8_262k_h32", B=1, T=262144, H=32,
                                      alpha_lo=0.95, alpha_hi=0.9999, s0_std=0.1,
                                      n_seqs=8, len_lo=4096, len_hi=65536),
    "decode_n256_h32": Workload("decode_n256_h32", B=256, T=1, H=32,
                                alpha_lo=0.95, alpha_hi=0.9999, s0_std=0.1,
                                decode_steps=1000),
}


def to_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def varlen_lengths(n: int, total: int, lo: int, hi: int, seed: int = 0) -> List[int]:
    """n lengths in [lo, hi] summing to ``total``.

    Draw n integers uniformly in [lo, hi], rescale to the total, floor, clamp
    to [lo, hi], then move the remainder one token at a time over the
    sequences in index order (skipping any that would leave [lo, hi]).
    """
    if not (n * lo <= total <= n * hi):
        raise ValueError("total not reachable with lengths in [lo, hi]")
    g = _gen("cpu", seed)
    raw = torch.randint(lo, hi + 1, (n,), generator=g).tolist()
    s = sum(raw)
    lens = [min(hi, max(lo, (x * total) // s)) for x in raw]
    rem = total - sum(lens)
    i = 0
    while rem != 0:
        step = 1 if rem > 0 else -1
        if lo <= lens[i] + step <= hi:
            lens[i] += step
            rem -= step
        i = (i + 1) % n
    return lens


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def make_prefill(w: Workload, device="cpu", T: Optional[int] = None, H: Optional[int] = None,
                 seed: Optional[int] = None):
    """Inputs of one prefill call, laid out ``[B, T, H, d]`` (last dim fastest).

    Returns a dict with q, k, v (input dtype), log_alpha [B,T,H,dk] fp32,
    beta [B,T,H] fp32, S0 [N,H,dk,dv] fp32 (or None when S0 = 0),
    cu_seqlens int32 [N+1] (or None) and the per-sequence lengths.
    ``T``/``H`` override the workload's sizes (smaller parity cases).
    """
    T = w.T if T is None else T
    H = w.H if H is None else H
    seed = w.seed if seed is None else seed
    dt = to_dtype(w.dtype)
    B, dk, dv = w.B, w.dk, w.dv
    g = _gen(device, seed)
    q = _unit_rows(torch.randn(B, T, H, dk, generator=g, device=device)).to(dt)
    k = _unit_rows(torch.randn(B, T, H, dk, generator=g, device=device)).to(dt)
    v = torch.randn(B, T, H, dv, generator=g, device=device).to(dt)
    u = torch.rand(B, T, H, dk, generator=g, device=device)
    log_alpha = torch.log(w.alpha_lo + (w.alpha_hi - w.alpha_lo) * u)
    beta = torch.sigmoid(torch.randn(B, T, H, generator=g, device=device))
    lens = None
    cu = None
    if w.n_seqs > 0:
        if B != 1:
            raise ValueError("packed sequences need B == 1")
        if T == w.T:
            lens = varlen_lengths(w.n_seqs, T, w.len_lo, w.len_hi, seed)
        else:  # scaled-down parity case: same rule, bounds scaled with T
            lo = max(0, (w.len_lo * T) // w.T)
            hi = max(lo, (w.len_hi * T) // w.T)
            lens = varlen_lengths(w.n_seqs, T, lo, hi, seed)
        offs = [0]
        for L in lens:
            offs.append(offs[-1] + L)
        cu = torch.tensor(offs, dtype=torch.int32, device=device)
    N = len(lens) if lens is not None else B
    S0 = None
    if w.s0_std > 0:
        S0 = w.s0_std * torch.randn(N, H, dk, dv, generator=g, device=device)
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S0=S0,
                cu_seqlens=cu, lens=lens)


def make_decode_state(w: Workload, device="cpu", N: Optional[int] = None,
                      H: Optional[int] = None) -> torch.Tensor:
    """Initial fp32 decode state ``[N, H, dk, dv]`` ~ N(0, s0_std^2), seed = workload seed."""
    N = w.B if N is None else N
    H = w.H if H is None else H
    g = _gen(device, w.seed)
    return w.s0_std * torch.randn(N, H, w.dk, w.dv, generator=g, device=device)


def make_decode_step(w: Workload, step: int, device="cpu", N: Optional[int] = None,
                     H: Optional[int] = None):
    """Single-token inputs of decode step ``step``: q, k, v ``[N, H, d]``, log_alpha
    ``[N, H, dk]``, beta ``[N, H]``; seed 1000 + step."""
    N = w.B if N is None else N
    H = w.H if H is None else H
    dt = to_dtype(w.dtype)
    g = _gen(device, 1000 + step)
    q = _unit_rows(torch.randn(N, H, w.dk, generator=g, device=device)).to(dt)
    k = _unit_rows(torch.randn(N, H, w.dk, generator=g, device=device)).to(dt)
    v = torch.randn(N, H, w.dv, generator=g, device=device).to(dt)
    u = torch.rand(N, H, w.dk, generator=g, device=device)
    log_alpha = torch.log(w.alpha_lo + (w.alpha_hi - w.alpha_lo) * u)
    beta = torch.sigmoid(torch.randn(N, H, generator=g, device=device))
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta)


def make_layer_inputs(B: int, T: int, H: int, dtype: str = "bf16", device="cpu", seed: int = 0,
                      dk: int = 128, dv: int = 128):
    """Inputs of the layer's gate producers and output norm (synthetic, seeded; draw order f,
    A_log, dt_bias, b, g, w): the decay-gate projection output f ~ N(0, 0.5^2) [B,T,H,dk], the
    per-head A_log ~ U(0, 2) [H], the per-channel dt_bias ~ U(-6, -3) [H*dk], the write-gate logits
    b ~ N(0, 1) [B,T,H], the output gate g ~ N(0, 1) [B,T,H,dv] and the norm weight
    w ~ U(0.5, 1.5) [dv]. f, b and g take the input dtype (rounded from fp32); A_log, dt_bias and w
    stay fp32. (With these ranges the decay per token lies between about e^-0.4 and e^-0.0003.)"""
    dt = to_dtype(dtype)
    g = _gen(device, seed)
    f = (0.5 * torch.randn(B, T, H, dk, generator=g, device=device)).to(dt)
    A_log = 2.0 * torch.rand(H, generator=g, device=device)
    dt_bias = -6.0 + 3.0 * torch.rand(H * dk, generator=g, device=device)
    b = torch.randn(B, T, H, generator=g, device=device).to(dt)
    og = torch.randn(B, T, H, dv, generator=g, device=device).to(dt)
    w = 0.5 + torch.rand(dv, generator=g, device=device)
    return dict(gate_f=f, A_log=A_log, dt_bias=dt_bias, beta_logits=b, out_gate=og, norm_weight=w)

