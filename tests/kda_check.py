"""Helpers shared by the GPU parity tests: run the float64 oracle on torch inputs and compare.

Error metric: max |x - ref| <= tol * RMS(ref), evaluated separately for the outputs and for the
final state, RMS over the whole compared reference tensor. tol = 1e-4 for fp32 inputs and 2e-2
for bf16 inputs with fp32 state.
"""
import math

import numpy as np
import torch

from oracle import ref

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def np32(t):
    return None if t is None else t.detach().float().cpu().numpy()


def rel_err(x, r):
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    rms = math.sqrt(float(np.mean(r * r)))
    return float(np.max(np.abs(x - r))) / (rms if rms > 0 else 1.0)


# Every comparison made through the helpers below, as (test, what, max|err|/RMS(ref), tol); the
# test session prints them and, when KDA_MARGINS_FILE is set, writes them there as JSON lines.
MARGINS = []


def _record(what, e, tol):
    import os
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    MARGINS.append({"test": test, "what": what, "err_over_rms": e, "tol": tol})
    print("margin %-60s %-28s max|err|/RMS = %.3e (tol %.0e)" % (test[-60:], what, e, tol))


def assert_close(x, r, tol, what):
    e = rel_err(x, r)
    _record(what, e, tol)
    assert np.all(np.isfinite(np.asarray(x, dtype=np.float64))), "%s: non-finite values" % what
    assert e <= tol, "%s: max|err|/RMS(ref) = %.3e > %.1e" % (what, e, tol)
    return e


def assert_close_bf16_out(x, r, tol, what):
    """For a bf16-stored result: the stated bound plus the rounding of the storage format
    itself (round-to-nearest-even to bf16 moves a value y by at most 2^-8 |y|), elementwise:
    |x - r| <= tol * RMS(r) * (1 + 2^-8) + 2^-8 |r|."""
    x = np.asarray(x, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    rms = math.sqrt(float(np.mean(r * r))) if r.size else 0.0
    slack = np.abs(x - r) - (tol * rms * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(r))
    worst = float(np.max(slack)) if r.size else -1.0
    e = rel_err(x, r)
    _record(what, e, tol)
    assert np.all(np.isfinite(x)), "%s: non-finite values" % what
    assert worst <= 0, "%s: exceeds tol*RMS + bf16 rounding by %.3e (RMS %.3e)" % (what, worst, rms)
    return e


def oracle_prefill(d, heads=None, nthreads=0):
    """Oracle on the inputs of ``kda_inputs.make_prefill`` (torch, any device), optionally
    restricted to a list of heads. Returns (out, S_final) float64 numpy arrays."""
    sel = (lambda t: t) if heads is None else (lambda t: t[:, :, heads])
    q, k, v, la = (np32(sel(d[x])) for x in ("q", "k", "v", "log_alpha"))
    be = np32(d["beta"] if heads is None else d["beta"][:, :, heads])
    S0 = None
    if d.get("S0") is not None:
        S0 = d["S0"].double().cpu().numpy()
        if heads is not None:
            S0 = S0[:, heads]
    cu = None if d.get("cu_seqlens") is None else d["cu_seqlens"].cpu().numpy()
    return ref.forward(q, k, v, la, be, S0=S0, cu_seqlens=cu, nthreads=nthreads)


def to_device(d, device):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
