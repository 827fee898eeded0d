"""GPU parity of the short causal convolution (kda_short_conv, kda_short_conv_step), the state
composition (kda_state_affine) and context-parallel prefill (segments run one after the other on
one GPU, composed through their affine state maps), against the float64 oracle."""
import numpy as np
import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda
from kimi_delta_attention_25_b200 import cp
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


def _conv_inputs(dtype, lens, D=256, K=4, seed=0):
    g = torch.Generator().manual_seed(seed)
    T = sum(lens)
    x = torch.randn(1, T, D, generator=g).to(K_DT[dtype])
    w = 0.5 * torch.randn(D, K, generator=g)
    b = 0.1 * torch.randn(D, generator=g)
    st = torch.randn(len(lens), D, K - 1, generator=g)
    cu = torch.tensor(np.cumsum([0] + lens), dtype=torch.int32)
    return x, w, b, st, cu


K_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("act,norm", [("silu", 0), (None, 0), ("silu", 128)])
def test_short_conv_packed_with_states(dtype, act, norm):
    lens = [70, 0, 1, 2, 200, 3]
    x, w, b, st, cu = _conv_inputs(dtype, lens, seed=1)
    xg, wg, bg, stg, cug = (t.to(DEV) for t in (x, w, b, st, cu))
    y, st_new = kda.short_conv(xg, wg, bg, conv_state=stg, cu_seqlens=cug, conv_state_out=True,
                               activation=act or "none", normalize_head_dim=norm)
    ry, rst = L.short_conv(np32(x)[0], np32(w), np32(b), conv_state=np32(st), cu_seqlens=cu.numpy(),
                           activation=act)
    if norm:
        ry = L.l2_normalize(ry.reshape(ry.shape[0], -1, norm)).reshape(ry.shape)
    tol = 1e-5 if dtype == "f32" else 0.0
    if dtype == "bf16":
        assert_close_bf16_out(np32(y)[0], ry, 1e-5, "y (bf16)")
    else:
        assert_close(np32(y)[0], ry, tol, "y")
    assert np.array_equal(np32(st_new), rst.astype(np.float32)), "conv state"
    # in place: the state buffer updated by the same call gives the same outputs and state
    st2 = stg.clone()
    y2, _ = kda.short_conv(xg, wg, bg, conv_state=st2, cu_seqlens=cug, conv_state_out=st2,
                           activation=act or "none", normalize_head_dim=norm)
    assert torch.equal(y2, y) and torch.equal(st2, st_new)


def test_short_conv_batch_rows_and_zero_state():
    x = torch.randn(3, 50, 128, generator=torch.Generator().manual_seed(2))
    w = torch.randn(128, 4, generator=torch.Generator().manual_seed(3))
    y, _ = kda.short_conv(x.to(DEV), w.to(DEV))
    for bi in range(3):
        ry, _ = L.short_conv(x[bi].numpy(), w.numpy())
        assert_close(np32(y[bi]), ry, 1e-5, "y row %d" % bi)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_short_conv_steps_equal_prefill(dtype):
    """Decode steps from a conv state continue a prefill exactly as one longer prefill does."""
    lens = [5, 9]
    x, w, b, st, cu = _conv_inputs(dtype, lens, D=128, seed=4)
    xg, wg, bg, stg = (t.to(DEV) for t in (x, w, b, st))
    y_all, st_all = kda.short_conv(xg, wg, bg, conv_state=stg, cu_seqlens=cu.to(DEV), conv_state_out=True)
    # prefill the first 3 tokens of each sequence, then step the rest one token at a time
    first = [3, 3]
    cu1 = torch.tensor(np.cumsum([0] + first), dtype=torch.int32)
    x1 = torch.cat([x[:, int(cu[i]):int(cu[i]) + first[i]] for i in range(2)], 1).contiguous()
    _, s = kda.short_conv(x1.to(DEV), wg, bg, conv_state=stg, cu_seqlens=cu1.to(DEV), conv_state_out=True)
    for t in range(3, 9):
        rows = [i for i in range(2) if t < lens[i]]
        xt = torch.stack([x[0, int(cu[i]) + t] for i in range(2)]).to(DEV)
        s_before = s.clone()
        yt = kda.short_conv_step(xt, wg, s, bias=bg)
        for i in rows:
            assert torch.allclose(yt[i].float(), y_all[0, int(cu[i]) + t].float(), rtol=1e-6, atol=1e-6)
        for i in range(2):
            if i not in rows:
                s[i] = s_before[i]
    assert torch.allclose(s[1], st_all[1])


def test_state_affine_matches_float64():
    g = torch.Generator().manual_seed(5)
    Phi = torch.randn(3, 128, 128, generator=g)
    S = torch.randn(3, 128, 128, generator=g)
    Psi = torch.randn(3, 128, 128, generator=g)
    out = kda.state_affine(Phi.to(DEV), S.to(DEV), Psi.to(DEV))
    ref_ = np.einsum("hij,hjk->hik", Phi.double().numpy(), S.double().numpy()) + Psi.double().numpy()
    assert_close(np32(out), ref_, 1e-5, "Phi S + Psi")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_context_parallel_segments_on_one_gpu(dtype):
    """One 1000-token sequence split into 3 segments: each segment's (Phi, Psi) from the kernels,
    composed with kda_state_affine, then each segment run from its entering state; the outputs and
    the final state match one oracle run over the whole sequence."""
    w = K.Workload("cp", B=1, T=1000, H=2, dtype=dtype, alpha_lo=0.95, alpha_hi=0.9999, s0_std=0.1)
    d = K.make_prefill(w, seed=51)
    g = to_device(d, DEV)
    cuts = [0, 320, 321, 1000]
    ops = cp.KernelOps(out_dtype=torch.float32)
    segs = [{x: g[x][:, cuts[r]:cuts[r + 1]].contiguous() for x in ("q", "k", "v", "log_alpha", "beta")}
            for r in range(3)]
    maps = [ops.segment_map(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"]) for s in segs]
    outs, S_leave = [], None
    for r in range(3):
        S_in = cp.entering_state([m[0] for m in maps], [m[1] for m in maps], g["S0"][0], r, ops)
        o, S_leave = ops.prefill(**{x: segs[r][x] for x in ("q", "k", "v", "log_alpha", "beta")},
                                 S0=S_in.unsqueeze(0).contiguous())
        outs.append(o)
    out = torch.cat(outs, 1)
    ro, rs = ref.forward(np32(d["q"]), np32(d["k"]), np32(d["v"]), np32(d["log_alpha"]), np32(d["beta"]),
                         S0=d["S0"].double().numpy())
    tol = TOL[K.to_dtype(dtype)]
    assert_close(np32(out), ro, tol, "out")
    assert_close(np32(S_leave), rs, tol, "S_final")
