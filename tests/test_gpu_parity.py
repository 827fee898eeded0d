"""GPU parity: libkda (through its C ABI) against the float64 oracle on the same seeded inputs.

Sizes span several 64-token chunks and a ragged tail; the full-size workloads are checked on
sampled heads / sequences that the oracle recomputes from scratch. Tolerances: max|err| <=
1e-4 * RMS(ref) for fp32 inputs, <= 2e-2 * RMS(ref) for bf16 inputs (fp32 state), applied to
the outputs and to the final state separately.
"""
import numpy as np
import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda
from oracle import ref
from tests.kda_check import TOL, assert_close, assert_close_bf16_out, np32, oracle_prefill, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kimi_delta_attention_25_b200 import build
    build.build()
    kda.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _run_check(d, tol, heads=None, check_state=True, out_dtype=torch.float32):
    g = to_device(d, DEV)
    out, Sf, ws = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                                cu_seqlens=g["cu_seqlens"], out_dtype=out_dtype, return_workspace=True)
    assert out.dtype == out_dtype
    assert kda.workspace_status(ws) == kda.KDA_OK
    ro, rs = oracle_prefill(d, heads=heads)
    o = out if heads is None else out[:, :, heads]
    s = Sf if heads is None else Sf[:, heads]
    if out_dtype == torch.bfloat16:
        e1 = assert_close_bf16_out(np32(o), ro, tol, "out (bf16)")
    else:
        e1 = assert_close(np32(o), ro, tol, "out")
    e2 = assert_close(np32(s), rs, tol, "S_final") if check_state else 0.0
    return e1, e2


# ---- the small workloads, whole ------------------------------------------------------------

def test_fp32_t256_h2_whole():
    w = K.WORKLOADS["fp32_t256_h2"]
    _run_check(K.make_prefill(w), TOL[torch.float32])


def test_bf16_t8k_h16_whole():
    w = K.WORKLOADS["bf16_t8k_h16"]
    _run_check(K.make_prefill(w, device=DEV), TOL[torch.bfloat16])


def test_bf16_t8k_h16_whole_bf16_out():
    w = K.WORKLOADS["bf16_t8k_h16"]
    _run_check(K.make_prefill(w, device=DEV), TOL[torch.bfloat16], out_dtype=torch.bfloat16)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200])
def test_ragged_lengths(dtype, T):
    w = K.Workload("ragged", B=2, T=T, H=3, dtype=dtype, alpha_lo=0.9, alpha_hi=0.999, s0_std=0.1)
    _run_check(K.make_prefill(w, seed=T), TOL[K.to_dtype(dtype)])
    _run_check(K.make_prefill(w, seed=T), TOL[K.to_dtype(dtype)], out_dtype=torch.bfloat16)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_varlen_with_empty_sequences(dtype):
    torch.manual_seed(0)
    lens = [70, 0, 1, 64, 0, 129]
    cu = torch.tensor(np.cumsum([0] + lens), dtype=torch.int32)
    T = int(cu[-1])
    w = K.Workload("varlen", B=1, T=T, H=2, dtype=dtype, s0_std=0.1)
    d = K.make_prefill(w, seed=3)
    d["S0"] = 0.1 * torch.randn(len(lens), 2, 128, 128)
    d["cu_seqlens"] = cu
    _run_check(d, TOL[K.to_dtype(dtype)])


def test_zero_initial_state_and_no_final_state():
    w = K.Workload("nostate", B=1, T=100, H=2, dtype="bf16")
    d = to_device(K.make_prefill(w, seed=5), DEV)
    out, Sf = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], want_state=False)
    assert Sf is None
    ro, _ = oracle_prefill(d)
    assert_close(np32(out), ro, TOL[torch.bfloat16], "out")


def test_invalid_cu_seqlens_flagged_on_device():
    w = K.Workload("bad", B=1, T=128, H=2, dtype="bf16")
    d = to_device(K.make_prefill(w, seed=6), DEV)
    for bad in ([0, 100, 50, 128], [0, 64, 129], [1, 64, 128]):
        cu = torch.tensor(bad, dtype=torch.int32, device=DEV)
        ws = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu_seqlens=cu,
                           return_workspace=True)[2]
        assert kda.workspace_status(ws) == kda.KDA_ERR_INVALID_ARG
    cu = torch.tensor([0, 64, 128], dtype=torch.int32, device=DEV)
    ws = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu_seqlens=cu, return_workspace=True)[2]
    assert kda.workspace_status(ws) == kda.KDA_OK


# ---- properties ----------------------------------------------------------------------------

def test_causality_bitwise():
    w = K.Workload("causal", B=1, T=200, H=2, dtype="bf16", s0_std=0.1)
    d = to_device(K.make_prefill(w, seed=7), DEV)
    o1, _ = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    t = 130
    v2 = d["v"].clone()
    v2[:, t + 1:] += 1.0
    k2 = d["k"].clone()
    k2[:, t + 1:] = k2[:, t + 1:].flip(-1)
    o2, _ = kda.chunk_fwd(d["q"], k2, v2, d["log_alpha"], d["beta"], S0=d["S0"])
    assert torch.equal(o1[:, :t + 1], o2[:, :t + 1])
    assert not torch.equal(o1[:, t + 1:], o2[:, t + 1:])


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_two_pass_calls_equal_chunk_fwd_bitwise(out_dtype):
    """kda_chunk_prep then kda_chunk_scan (varlen, ragged, with an empty sequence) give exactly
    what one kda_chunk_fwd call gives."""
    w = K.Workload("twopass", B=1, T=700, H=3, dtype="bf16", s0_std=0.1)
    d = to_device(K.make_prefill(w, seed=11), DEV)
    cu = torch.tensor([0, 130, 130, 451, 700], dtype=torch.int32, device=DEV)
    S0 = torch.randn(4, 3, 128, 128, device=DEV) * 0.1
    o1, s1 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=S0, cu_seqlens=cu,
                           out_dtype=out_dtype)
    ws = torch.empty(kda.chunk_fwd_workspace_size(1, 700, 3, 4), dtype=torch.uint8, device=DEV)
    kda.chunk_prep(d["q"], d["k"], d["log_alpha"], d["beta"], ws, cu_seqlens=cu)
    o2, s2 = kda.chunk_scan(d["v"], ws, S0=S0, cu_seqlens=cu, out_dtype=out_dtype)
    assert kda.workspace_status(ws) == kda.KDA_OK
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)


def test_split_continuation():
    w = K.Workload("split", B=1, T=300, H=2, dtype="f32", s0_std=0.1)
    d = to_device(K.make_prefill(w, seed=8), DEV)
    o, s = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    c = 100
    part = lambda x, sl: x[:, sl].contiguous()  # noqa: E731
    a, sa = kda.chunk_fwd(*(part(d[x], slice(0, c)) for x in ("q", "k", "v", "log_alpha", "beta")),
                          S0=d["S0"])
    b, sb = kda.chunk_fwd(*(part(d[x], slice(c, None)) for x in ("q", "k", "v", "log_alpha", "beta")),
                          S0=sa)
    assert_close(np32(torch.cat([a, b], 1)), np32(o), 1e-5, "out")
    assert_close(np32(sb), np32(s), 1e-5, "S_final")


def test_decode_steps_equal_chunked_prefill():
    w = K.Workload("dec_vs_chunk", B=1, T=70, H=3, dtype="f32", s0_std=0.1)
    d = to_device(K.make_prefill(w, seed=9), DEV)
    o, s = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    S = d["S0"].clone()
    outs = []
    for t in range(w.T):
        x = {n: d[n][:, t].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
        outs.append(kda.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S))
    assert_close(np32(torch.stack(outs, 1)), np32(o), 1e-4, "out")
    assert_close(np32(S), np32(s), 1e-4, "S")


# ---- decode --------------------------------------------------------------------------------

@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_small(dtype, out_dtype):
    w = K.Workload("dec", B=5, T=1, H=3, dtype=dtype, alpha_lo=0.95, alpha_hi=0.9999, s0_std=0.1)
    S = K.make_decode_state(w, N=5, H=3)
    Sg = S.to(DEV)
    Sd = S.double().numpy()
    for step in range(3):
        x = K.make_decode_step(w, step, N=5, H=3)
        g = to_device(x, DEV)
        o = kda.decode_step(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], Sg, out_dtype=out_dtype)
        cu = np.arange(6)
        ro, Sd = ref.forward(np32(x["q"])[None], np32(x["k"])[None], np32(x["v"])[None],
                             np32(x["log_alpha"])[None], np32(x["beta"])[None], S0=Sd, cu_seqlens=cu)
        if out_dtype == torch.bfloat16:
            assert_close_bf16_out(np32(o), ro[0], TOL[K.to_dtype(dtype)], "out step %d" % step)
        else:
            assert_close(np32(o), ro[0], TOL[K.to_dtype(dtype)], "out step %d" % step)
    assert_close(np32(Sg), Sd, TOL[K.to_dtype(dtype)], "S")


# ---- full-size workloads, sampled ----------------------------------------------------------

@pytest.mark.slow
def test_bf16_t128k_h32_sampled_heads():
    """The benchmark workload as the benchmark runs it (one kda_chunk_fwd with bf16 outputs, the
    launch configuration bench.py times) and with fp32 outputs; five heads recomputed by the oracle."""
    w = K.WORKLOADS["bf16_t128k_h32"]
    d = K.make_prefill(w, device=DEV)
    heads = [0, 7, 13, 24, 31]
    ro, rs = oracle_prefill(d, heads=heads)
    tol = TOL[torch.bfloat16]
    for od in (torch.bfloat16, torch.float32):
        out, Sf, ws = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"],
                                    out_dtype=od, return_workspace=True)
        assert kda.workspace_status(ws) == kda.KDA_OK
        o = np32(out[:, :, heads])
        if od == torch.bfloat16:
            assert_close_bf16_out(o, ro, tol, "out (bf16)")
        else:
            assert_close(o, ro, tol, "out (fp32)")
        assert_close(np32(Sf[:, heads]), rs, tol, "S_final (%s out)" % str(od)[6:])
        del out, Sf, ws


@pytest.mark.slow
def test_bf16_varlen8_262k_h32_sampled_sequences():
    w = K.WORKLOADS["bf16_varlen8_262k_h32"]
    d = K.make_prefill(w, device=DEV)
    g = d
    cu = d["cu_seqlens"].tolist()
    pairs = [(1, 0), (0, 21), (7, 31), (4, 12)]
    refs = {}
    for n, h in pairs:
        sl = slice(cu[n], cu[n + 1])
        sub = {x: d[x][:, sl][:, :, [h]] for x in ("q", "k", "v", "log_alpha", "beta")}
        sub["S0"] = d["S0"][n:n + 1, [h]]
        sub["cu_seqlens"] = None
        refs[(n, h)] = oracle_prefill(sub)
    for od in (torch.bfloat16, torch.float32):
        out, Sf, ws = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                                    cu_seqlens=g["cu_seqlens"], out_dtype=od, return_workspace=True)
        assert kda.workspace_status(ws) == kda.KDA_OK
        for n, h in pairs:
            sl = slice(cu[n], cu[n + 1])
            ro, rs = refs[(n, h)]
            o = np32(out[:, sl][:, :, [h]])
            if od == torch.bfloat16:
                assert_close_bf16_out(o, ro, TOL[torch.bfloat16], "out (bf16) seq %d head %d" % (n, h))
            else:
                assert_close(o, ro, TOL[torch.bfloat16], "out seq %d head %d" % (n, h))
            assert_close(np32(Sf[n:n + 1, [h]]), rs, TOL[torch.bfloat16], "S_final seq %d head %d" % (n, h))
        del out, Sf, ws


@pytest.mark.slow
def test_decode_n256_h32_1000_steps_sampled():
    w = K.WORKLOADS["decode_n256_h32"]
    S = K.make_decode_state(w, device=DEV)
    pairs = [(0, 0), (3, 17), (100, 5), (128, 31), (255, 0), (255, 31), (17, 9), (200, 22)]
    ni = torch.tensor([p[0] for p in pairs])
    hi = torch.tensor([p[1] for p in pairs])
    Sd = S[ni, hi].double().cpu().numpy()[:, None]          # [P, 1, dk, dv]
    cu = np.arange(len(pairs) + 1)
    tol = TOL[torch.bfloat16]
    for step in range(w.decode_steps):
        x = K.make_decode_step(w, step, device=DEV)
        o = kda.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
        sub = {n: np32(x[n][ni, hi]) for n in ("q", "k", "v", "log_alpha", "beta")}
        ro, Sd = ref.forward(sub["q"][None, :, None], sub["k"][None, :, None], sub["v"][None, :, None],
                             sub["log_alpha"][None, :, None], sub["beta"][None, :, None],
                             S0=Sd, cu_seqlens=cu)
        if step % 50 == 49:
            assert_close(np32(o[ni, hi]), ro[0, :, 0], tol, "out step %d" % step)
    assert_close(np32(S[ni, hi]), Sd[:, 0], tol, "S after 1000 steps")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("lo,hi", [(0.3, 0.7), (0.8, 0.9), (0.85, 0.95)])
def test_fast_forgetting_channels(dtype, lo, hi):
    """Channel gates that forget fast within a chunk (alpha ~ U(0.3, 0.7): the cumulative
    log-decay of one 64-token chunk reaches about -47; U(0.8, 0.9): about -11): the gate is
    channel-wise so that some channels can forget quickly (KimiLinear tutorial (icman.com.cn),
    sec. 1-2). The intra-chunk product runs on tf32 operands, so these stay inside the range."""
    w = K.Workload("fast_forget", B=1, T=1000, H=3, dtype=dtype, alpha_lo=lo, alpha_hi=hi, s0_std=0.1)
    for od in (torch.float32, torch.bfloat16):
        _run_check(K.make_prefill(w, seed=12), TOL[K.to_dtype(dtype)], out_dtype=od)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decay_outside_range_is_reported(dtype):
    """A chunk whose cumulative log-decay falls below -80 in some channel (alpha ~ U(0.2, 0.25):
    about -95 per 64 tokens) cannot be factored in fp32; the call still returns KDA_OK (the check
    needs device data) and the workspace status word reads KDA_ERR_UNSUPPORTED."""
    w = K.Workload("too_strong", B=1, T=128, H=2, dtype=dtype, alpha_lo=0.2, alpha_hi=0.25)
    d = to_device(K.make_prefill(w, seed=13), DEV)
    ws = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], return_workspace=True)[2]
    assert kda.workspace_status(ws) == kda.KDA_ERR_UNSUPPORTED
    # the first 40 tokens alone stay inside the range (about -60)
    part = {x: d[x][:, :40].contiguous() for x in ("q", "k", "v", "log_alpha", "beta")}
    ws = kda.chunk_fwd(part["q"], part["k"], part["v"], part["log_alpha"], part["beta"],
                       return_workspace=True)[2]
    assert kda.workspace_status(ws) == kda.KDA_OK


# ---- degenerate cases of the method, against closed forms ----------------------------------

def _closed_form_out(S_seq, q):
    """o_t = S_t^T q_t for a list of per-token states [T, dk, dv] and queries [T, dk]."""
    return np.einsum("tkv,tk->tv", S_seq, q)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_beta_zero_is_pure_decay(dtype):
    """With beta = 0 the delta-rule write vanishes and the recurrence is S_t = Diag(alpha_t) S_{t-1}:
    the state is S0 scaled per key channel by the running product of the decays, and the output
    reads that state (the gated delta rule of Kimi Linear, section 3.1, with the write term zero)."""
    w = K.Workload("beta0", B=1, T=200, H=2, dtype=dtype, alpha_lo=0.9, alpha_hi=0.999, s0_std=0.5)
    d = K.make_prefill(w, seed=21)
    d["beta"] = torch.zeros_like(d["beta"])
    g = to_device(d, DEV)
    out, Sf, ws = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                                return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_OK
    tol = TOL[K.to_dtype(dtype)]
    q = d["q"].double().numpy()[0]
    G = np.cumsum(d["log_alpha"].double().numpy()[0], axis=0)       # [T, H, dk]
    S0 = d["S0"].double().numpy()[0]                                 # [H, dk, dv]
    for h in range(w.H):
        S_seq = np.exp(G[:, h, :, None]) * S0[h][None]
        assert_close(np32(out[0, :, h]), _closed_form_out(S_seq, q[:, h]), tol, "out h%d" % h)
        assert_close(np32(Sf[0, h]), S_seq[-1], tol, "S_final h%d" % h)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [100, 128])
def test_no_decay_unit_beta_one_hot_keys_overwrite_rows(dtype, T):
    """alpha = 1 (DeltaNet) and beta = 1 with one-hot keys k_t = e_{p(t)}: each update
    (I - k k^T) S + k v^T replaces row p(t) of the state by v_t, so S_t is S0 with the rows
    p(1..t) overwritten (the delta rule of Kimi Linear, section 3.1, at its fixed point)."""
    w = K.Workload("overwrite", B=1, T=T, H=2, dtype=dtype, s0_std=0.5)
    d = K.make_prefill(w, seed=22)
    dt = K.to_dtype(dtype)
    gen = torch.Generator().manual_seed(22)
    k = torch.zeros(1, T, w.H, 128)
    perms = [torch.randperm(128, generator=gen)[:T] for _ in range(w.H)]
    for h in range(w.H):
        k[0, torch.arange(T), h, perms[h]] = 1.0
    d["k"] = k.to(dt)
    d["log_alpha"] = torch.zeros_like(d["log_alpha"])
    d["beta"] = torch.ones_like(d["beta"])
    g = to_device(d, DEV)
    out, Sf, ws = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                                return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_OK
    tol = TOL[dt]
    q = d["q"].double().numpy()[0]
    v = d["v"].double().numpy()[0]
    for h in range(w.H):
        S = d["S0"].double().numpy()[0, h].copy()
        S_seq = np.empty((T, 128, 128))
        for t in range(T):
            S[int(perms[h][t])] = v[t, h]
            S_seq[t] = S
        assert_close(np32(out[0, :, h]), _closed_form_out(S_seq, q[:, h]), tol, "out h%d" % h)
        assert_close(np32(Sf[0, h]), S, tol, "S_final h%d" % h)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_no_decay_is_deltanet(dtype):
    """log alpha = 0: the per-chunk decay factors are all 1 and the path computes DeltaNet;
    checked against the oracle on random inputs with a ragged tail."""
    w = K.Workload("deltanet", B=2, T=150, H=2, dtype=dtype, s0_std=0.1)
    d = K.make_prefill(w, seed=23)
    d["log_alpha"] = torch.zeros_like(d["log_alpha"])
    _run_check(d, TOL[K.to_dtype(dtype)])
