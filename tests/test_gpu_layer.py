"""GPU parity of the layer options (kda_chunk_fwd_layer, kda_decode_step_layer): the gate producers
(log_alpha from f, A_log, dt_bias; beta from its logits) and the gated RMSNorm of the outputs, each
against the float64 oracle composed from oracle/layer.py and the recurrence oracle. Tolerances as
for the plain prefill (1e-4 of RMS for fp32 inputs, 2e-2 for bf16 inputs, plus the bf16 rounding
of a bf16-stored result), applied to the normalised outputs and to the final state."""
import numpy as np
import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda
from oracle import layer as L
from oracle import ref
from tests.kda_check import TOL, assert_close, assert_close_bf16_out, np32, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kimi_delta_attention_25_b200 import build
    build.build()
    kda.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _inputs(dtype, T, H, seed, lens=None, s0=0.1):
    w = K.Workload("layer", B=1, T=T, H=H, dtype=dtype, alpha_lo=0.9, alpha_hi=0.999, s0_std=s0)
    d = K.make_prefill(w, seed=seed)
    lay = K.make_layer_inputs(1, T, H, dtype=dtype, seed=seed + 100)
    if lens is not None:
        d["cu_seqlens"] = torch.tensor(np.cumsum([0] + lens), dtype=torch.int32)
        d["S0"] = s0 * torch.randn(len(lens), H, 128, 128, generator=torch.Generator().manual_seed(seed))
    return d, lay


def _oracle(d, lay, use_gate, use_beta, use_norm, eps):
    la = L.kda_gate(np32(lay["gate_f"]), np32(lay["A_log"]), np32(lay["dt_bias"])) if use_gate \
        else np32(d["log_alpha"])
    be = L.beta_gate(np32(lay["beta_logits"])) if use_beta else np32(d["beta"])
    S0 = None if d.get("S0") is None else d["S0"].double().cpu().numpy()
    cu = None if d.get("cu_seqlens") is None else d["cu_seqlens"].cpu().numpy()
    o, s = ref.forward(np32(d["q"]), np32(d["k"]), np32(d["v"]), la, be, S0=S0, cu_seqlens=cu)
    if use_norm:
        o = L.gated_rmsnorm(o, np32(lay["out_gate"]), np32(lay["norm_weight"]), eps)
    return o, s


def _run(d, lay, use_gate, use_beta, use_norm, out_dtype, eps=1e-5):
    g = to_device(d, DEV)
    ly = to_device(lay, DEV)
    opts = {"norm_eps": eps}
    if use_gate:
        opts.update(gate_f=ly["gate_f"], A_log=ly["A_log"], dt_bias=ly["dt_bias"])
    if use_beta:
        opts["beta_logits"] = ly["beta_logits"]
    if use_norm:
        opts.update(out_gate=ly["out_gate"], norm_weight=ly["norm_weight"])
    out, Sf, ws = kda.chunk_fwd(g["q"], g["k"], g["v"], None if use_gate else g["log_alpha"],
                                None if use_beta else g["beta"], S0=g["S0"], cu_seqlens=g["cu_seqlens"],
                                out_dtype=out_dtype, return_workspace=True, layer=opts)
    assert kda.workspace_status(ws) == kda.KDA_OK
    return out, Sf


def _check(d, lay, flags, out_dtype, dtype):
    tol = TOL[K.to_dtype(dtype)]
    out, Sf = _run(d, lay, *flags, out_dtype=out_dtype)
    ro, rs = _oracle(d, lay, *flags, eps=1e-5)
    if out_dtype == torch.bfloat16:
        assert_close_bf16_out(np32(out), ro, tol, "out (bf16)")
    else:
        assert_close(np32(out), ro, tol, "out")
    assert_close(np32(Sf), rs, tol, "S_final")


FLAGS = {"gates": (True, True, False), "norm": (False, False, True), "all": (True, True, True),
         "decay_gate_only": (True, False, False)}


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("which", list(FLAGS))
def test_layer_prefill_packed_ragged(which, dtype, out_dtype):
    """Packed sequences with an empty one and ragged chunk tails, several chunks each."""
    d, lay = _inputs(dtype, T=70 + 1 + 200 + 129, H=3, seed=41, lens=[70, 0, 1, 200, 129])
    _check(d, lay, FLAGS[which], out_dtype, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layer_prefill_batch_rows(dtype):
    w = K.Workload("layer_b", B=2, T=260, H=2, dtype=dtype, s0_std=0.1)
    d = K.make_prefill(w, seed=43)
    lay = K.make_layer_inputs(2, 260, 2, dtype=dtype, seed=143)
    _check(d, lay, FLAGS["all"], torch.float32, dtype)


def test_layer_two_passes_equal_one_call_bitwise():
    d, lay = _inputs("bf16", T=450, H=2, seed=44, lens=[130, 0, 320])
    g, ly = to_device(d, DEV), to_device(lay, DEV)
    opts = dict(gate_f=ly["gate_f"], A_log=ly["A_log"], dt_bias=ly["dt_bias"], beta_logits=ly["beta_logits"],
                out_gate=ly["out_gate"], norm_weight=ly["norm_weight"], norm_eps=1e-5)
    o1, s1 = kda.chunk_fwd(g["q"], g["k"], g["v"], None, None, S0=g["S0"], cu_seqlens=g["cu_seqlens"],
                           out_dtype=torch.bfloat16, layer=opts)
    ws = torch.empty(kda.chunk_fwd_workspace_size(1, 450, 2, 3), dtype=torch.uint8, device=DEV)
    kda.chunk_prep(g["q"], g["k"], None, None, ws, cu_seqlens=g["cu_seqlens"], layer=opts)
    o2, s2 = kda.chunk_scan(g["v"], ws, S0=g["S0"], cu_seqlens=g["cu_seqlens"], out_dtype=torch.bfloat16,
                            layer=opts)
    assert kda.workspace_status(ws) == kda.KDA_OK
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_norm_closed_gate_and_open_gate():
    """A very negative output gate closes every output (y = 0 exactly in fp32 up to the gate's
    underflow); a very positive one leaves plain RMSNorm times w: mean((y / w)^2) = 1 per token
    (eps = 0)."""
    d, lay = _inputs("bf16", T=200, H=2, seed=45)
    g, ly = to_device(d, DEV), to_device(lay, DEV)
    for sign in (-1.0, 1.0):
        og = torch.full_like(ly["out_gate"], 60.0 * sign)
        out, _ = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                               layer=dict(out_gate=og, norm_weight=ly["norm_weight"], norm_eps=0.0))
        if sign < 0:
            assert float(out.abs().max()) < 1e-20
        else:
            ms = ((out / ly["norm_weight"]) ** 2).mean(-1)
            assert float((ms - 1).abs().max()) < 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layer_decode_steps(dtype):
    N, H, steps = 5, 3, 4
    w = K.Workload("layer_dec", B=N, T=1, H=H, dtype=dtype, alpha_lo=0.95, alpha_hi=0.9999, s0_std=0.1)
    S = K.make_decode_state(w, N=N, H=H)
    Sg = S.to(DEV)
    Sd = S.double().numpy()
    tol = TOL[K.to_dtype(dtype)]
    for step in range(steps):
        x = K.make_decode_step(w, step, N=N, H=H)
        lay = K.make_layer_inputs(N, 1, H, dtype=dtype, seed=200 + step)
        lay1 = {k: (v[:, 0] if k in ("gate_f", "beta_logits", "out_gate") else v) for k, v in lay.items()}
        g, ly = to_device(x, DEV), to_device(lay1, DEV)
        o = kda.decode_step(g["q"], g["k"], g["v"], None, None, Sg,
                            layer=dict(gate_f=ly["gate_f"], A_log=ly["A_log"], dt_bias=ly["dt_bias"],
                                       beta_logits=ly["beta_logits"], out_gate=ly["out_gate"],
                                       norm_weight=ly["norm_weight"], norm_eps=1e-5))
        la = L.kda_gate(np32(lay1["gate_f"]), np32(lay1["A_log"]), np32(lay1["dt_bias"]))
        be = L.beta_gate(np32(lay1["beta_logits"]))
        ro, Sd = ref.forward(np32(x["q"])[None], np32(x["k"])[None], np32(x["v"])[None], la[None], be[None],
                             S0=Sd, cu_seqlens=np.arange(N + 1))
        y = L.gated_rmsnorm(ro[0], np32(lay1["out_gate"]), np32(lay1["norm_weight"]), 1e-5)
        assert_close(np32(o), y, tol, "out step %d" % step)
    assert_close(np32(Sg), Sd, tol, "S")


def test_layer_host_checks():
    d, lay = _inputs("bf16", T=64, H=1, seed=46)
    g, ly = to_device(d, DEV), to_device(lay, DEV)
    with pytest.raises(kda.KDAError) as e:
        kda.chunk_fwd(g["q"], g["k"], g["v"], None, g["beta"], layer=dict(gate_f=ly["gate_f"], A_log=ly["A_log"]))
    assert e.value.code == kda.KDA_ERR_INVALID_ARG
    with pytest.raises(kda.KDAError) as e:
        kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                      layer=dict(out_gate=ly["out_gate"], norm_weight=ly["norm_weight"], norm_eps=-1.0))
    assert e.value.code == kda.KDA_ERR_INVALID_ARG


@pytest.mark.slow
def test_layer_bf16_t128k_h32_sampled_heads():
    """The benchmark workload with every layer option on (gates produced in the preparation pass,
    the output norm in the scan's cluster epilogue), bf16 outputs; two heads recomputed."""
    w = K.WORKLOADS["bf16_t128k_h32"]
    d = K.make_prefill(w, device=DEV)
    lay = K.make_layer_inputs(1, w.T, w.H, dtype="bf16", device=DEV, seed=7)
    opts = dict(lay, norm_eps=1e-5)
    out, Sf, ws = kda.chunk_fwd(d["q"], d["k"], d["v"], None, None, S0=d["S0"], out_dtype=torch.bfloat16,
                                return_workspace=True, layer=opts)
    assert kda.workspace_status(ws) == kda.KDA_OK
    heads = [0, 31]
    sub = {x: d[x][:, :, heads] for x in ("q", "k", "v")}
    sub["S0"] = d["S0"][:, heads]
    sub["cu_seqlens"] = None
    sl = {"gate_f": lay["gate_f"][:, :, heads], "A_log": lay["A_log"][heads],
          "dt_bias": lay["dt_bias"].view(w.H, 128)[heads], "beta_logits": lay["beta_logits"][:, :, heads],
          "out_gate": lay["out_gate"][:, :, heads], "norm_weight": lay["norm_weight"]}
    ro, rs = _oracle(sub, sl, True, True, True, eps=1e-5)
    assert_close_bf16_out(np32(out[:, :, heads]), ro, TOL[torch.bfloat16], "out (bf16, gated norm)")
    assert_close(np32(Sf[:, heads]), rs, TOL[torch.bfloat16], "S_final")
