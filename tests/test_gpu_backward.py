"""GPU parity of the backward pass: libkda's kda_chunk_bwd (through its C ABI) against the float64
backward oracle (token-level reverse sweep) on the same seeded inputs and output gradients.

The library computes in fp32 for either input dtype; the bar is the forward's: max|err| <= tol *
RMS(ref) per gradient, tol = 1e-4 for fp32 inputs and 2e-2 for bf16 inputs (the reference is fed
the same bf16-rounded values, so both are in practice limited by fp32 arithmetic).
"""
import numpy as np
import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda
from oracle import backward as bw
from tests.kda_check import TOL, assert_close, np32, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kimi_delta_attention_25_b200 import build
    build.build()
    kda.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _with_output_grads(d, seed, with_dSf=True):
    g = torch.Generator().manual_seed(seed)
    B, T, H, dv = d["v"].shape
    N = B if d["cu_seqlens"] is None else d["cu_seqlens"].shape[0] - 1
    d["dout"] = torch.randn(B, T, H, dv, generator=g).to(d["q"].dtype)
    d["dS_final"] = torch.randn(N, H, 128, dv, generator=g) if with_dSf else None
    return d


def _oracle(d, heads=None):
    c = lambda t: None if t is None else t.detach().float().cpu().numpy()  # noqa: E731
    return bw.backward(c(d["q"]), c(d["k"]), c(d["v"]), c(d["log_alpha"]), c(d["beta"]), c(d["dout"]),
                       S0=c(d["S0"]), dS_final=c(d["dS_final"]),
                       cu_seqlens=None if d["cu_seqlens"] is None else d["cu_seqlens"].cpu().numpy(),
                       heads=heads)


def _run(d, tol, heads=None, want_dS0=True):
    gd = to_device(d, DEV)
    g, ws = kda.chunk_bwd(gd["q"], gd["k"], gd["v"], gd["log_alpha"], gd["beta"], gd["dout"], S0=gd["S0"],
                          dS_final=gd["dS_final"], cu_seqlens=gd["cu_seqlens"], want_dS0=want_dS0,
                          return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_OK
    r = _oracle(d, heads=heads)
    errs = {}
    for name in GRADS:
        if name == "dS0" and not want_dS0:
            assert g["dS0"] is None
            continue
        x, ref = np32(g[name]), r[name]
        if heads is not None:
            x, ref = x[:, :, heads] if name != "dS0" else x[:, heads], ref[:, :, heads] if name != "dS0" else ref[:, heads]
        errs[name] = assert_close(x, ref, tol, name)
    return errs


@pytest.mark.parametrize("T", [1, 64, 150])
def test_fp32_small(T):
    w = K.Workload("bwd_fp32", B=2, T=T, H=2, dtype="f32", s0_std=0.1)
    _run(_with_output_grads(K.make_prefill(w, seed=31 + T), seed=T), TOL[torch.float32])


def test_bf16_ragged_heads():
    w = K.Workload("bwd_bf16", B=1, T=1000, H=3, dtype="bf16", s0_std=0.1)
    _run(_with_output_grads(K.make_prefill(w, seed=32), seed=2), TOL[torch.bfloat16])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_with_empty_sequences(dtype):
    lens = [70, 0, 1, 64, 0, 129]
    cu = torch.tensor(np.cumsum([0] + lens), dtype=torch.int32)
    w = K.Workload("bwd_varlen", B=1, T=int(cu[-1]), H=2, dtype=dtype, s0_std=0.1)
    d = K.make_prefill(w, seed=33)
    d["S0"] = 0.1 * torch.randn(len(lens), 2, 128, 128, generator=torch.Generator().manual_seed(4))
    d["cu_seqlens"] = cu
    d = _with_output_grads(d, seed=3)
    _run(d, TOL[K.to_dtype(dtype)])


def test_packed_sequences_across_token_ranges():
    """Few (sequence, head) chains and enough chunks: the forward records come from the two passes
    pipelined over token ranges, with sequences that start, end or lie inside a range and the state
    carried between ranges; gradients against the oracle on two of the four heads."""
    lens = [1000, 0, 3000, 64, 5000, 70]
    cu = torch.tensor(np.cumsum([0] + lens), dtype=torch.int32)
    w = K.Workload("bwd_packed", B=1, T=int(cu[-1]), H=4, dtype="bf16", s0_std=0.1)
    d = K.make_prefill(w, seed=39)
    d["S0"] = 0.1 * torch.randn(len(lens), 4, 128, 128, generator=torch.Generator().manual_seed(6))
    d["cu_seqlens"] = cu
    d = _with_output_grads(d, seed=12)
    assert kda.chunk_fwd_kernel_launches(1, int(cu[-1]), 4, len(lens), torch.bfloat16) > 2   # pipelined
    _run(d, TOL[torch.bfloat16], heads=[0, 3])


def test_zero_state_and_no_state_gradients():
    w = K.Workload("bwd_nostate", B=1, T=200, H=2, dtype="bf16")
    d = _with_output_grads(K.make_prefill(w, seed=34), seed=5, with_dSf=False)
    assert d["S0"] is None and d["dS_final"] is None
    _run(d, TOL[torch.bfloat16], want_dS0=False)


def test_beta_zero_gives_zero_key_and_value_gradients():
    """beta = 0: k and v enter only through the write, so their gradients vanish exactly."""
    w = K.Workload("bwd_beta0", B=1, T=130, H=2, dtype="f32", s0_std=0.5)
    d = K.make_prefill(w, seed=35)
    d["beta"] = torch.zeros_like(d["beta"])
    d = _with_output_grads(d, seed=6)
    gd = to_device(d, DEV)
    g = kda.chunk_bwd(gd["q"], gd["k"], gd["v"], gd["log_alpha"], gd["beta"], gd["dout"], S0=gd["S0"],
                      dS_final=gd["dS_final"])
    assert float(g["dv"].abs().max()) == 0.0
    r = _oracle(d)
    assert float(np.abs(r["dk"]).max()) == 0.0
    assert float(g["dk"].abs().max()) < 1e-5 * float(np.sqrt(np.mean(r["dq"] ** 2)))
    for name in ("dq", "dlog_alpha", "dbeta", "dS0"):
        assert_close(np32(g[name]), r[name], TOL[torch.float32], name)


def test_invalid_cu_seqlens_flagged_on_device():
    w = K.Workload("bwd_bad", B=1, T=128, H=2, dtype="bf16")
    d = to_device(_with_output_grads(K.make_prefill(w, seed=36), seed=7), DEV)
    cu = torch.tensor([0, 100, 50, 128], dtype=torch.int32, device=DEV)
    _, ws = kda.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["dout"], cu_seqlens=cu,
                          return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_ERR_INVALID_ARG


def test_decay_outside_range_is_reported():
    """A chunk whose cumulative log-decay falls below -80 in some channel cannot be factored in
    fp32 (e^{-g} overflows): the backward reports KDA_ERR_UNSUPPORTED in its status word instead
    of returning non-finite gradients silently."""
    w = K.Workload("bwd_too_strong", B=1, T=128, H=2, dtype="bf16", alpha_lo=0.2, alpha_hi=0.25)
    d = to_device(_with_output_grads(K.make_prefill(w, seed=38), seed=11), DEV)
    _, ws = kda.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["dout"], return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.slow
def test_bf16_t8k_h16_sampled_heads():
    w = K.WORKLOADS["bf16_t8k_h16"]
    d = _with_output_grads(K.make_prefill(w), seed=8)
    _run(d, TOL[torch.bfloat16], heads=[0, 15])


def test_phases_one_by_one_equal_one_call_bitwise():
    w = K.Workload("bwd_phases", B=1, T=300, H=2, dtype="bf16", s0_std=0.1)
    d = to_device(_with_output_grads(K.make_prefill(w, seed=37), seed=9), DEV)
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["dout"])
    kw = dict(S0=d["S0"], dS_final=d["dS_final"])
    ref = kda.chunk_bwd(*args, **kw)
    g = None
    ws = None
    for phase in range(3):
        g, ws = kda.chunk_bwd(*args, **kw, grads=g, workspace=ws, phase=phase, return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_OK
    for name in GRADS:
        assert torch.equal(g[name], ref[name]), name


@pytest.mark.slow
def test_bf16_t128k_h32_sampled_head():
    """The benchmark workload (128K tokens, 32 heads, bf16) in the benchmark's launch configuration;
    one head is recomputed by the oracle (heads are independent)."""
    w = K.WORKLOADS["bf16_t128k_h32"]
    d = K.make_prefill(w, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(10)
    B, T, H, D = d["v"].shape
    d["dout"] = torch.randn(B, T, H, D, generator=g, device=DEV).to(torch.bfloat16)
    d["dS_final"] = torch.randn(B, H, D, D, generator=g, device=DEV)
    gr, ws = kda.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["dout"], S0=d["S0"],
                           dS_final=d["dS_final"], return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_OK
    h = 7
    sub = {x: d[x][:, :, h:h + 1].contiguous() for x in ("q", "k", "v", "log_alpha", "beta", "dout")}
    sub["S0"] = d["S0"][:, h:h + 1].contiguous()
    sub["dS_final"] = d["dS_final"][:, h:h + 1].contiguous()
    sub["cu_seqlens"] = None
    r = _oracle(sub)
    for name in GRADS:
        x = gr[name][:, h:h + 1] if name == "dS0" else gr[name][:, :, h:h + 1]
        assert_close(np32(x), r[name], TOL[torch.bfloat16], name)
