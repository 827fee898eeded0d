"""kda_chunk_fwd_noalloc, the prefill entry point for callers that cannot allocate device memory
(code hosted by a runtime that owns all device memory, or a process whose footprint is capped).

Called through the C ABI twice in a row on each case, every result is checked against the float64
oracle within the tolerance the parity tests use (2e-2 of RMS for bf16 inputs, 1e-4 for fp32), and
the device-side checks are read back from the library's shared status word with
kda_chunk_fwd_noalloc_status. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda
from tests.kda_check import TOL, assert_close, oracle_prefill, np32, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kimi_delta_attention_25_b200 import build
    build.build()
    kda.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _call_noalloc(lib, d, out, S_final):
    P = ctypes.c_void_p
    B, T, H, dk = d["q"].shape
    cu = d.get("cu_seqlens")
    N = B if cu is None else cu.shape[0] - 1
    ptr = lambda t: None if t is None else P(t.data_ptr())  # noqa: E731
    stream = P(torch.cuda.current_stream().cuda_stream)
    dt = kda.KDA_BF16 if d["q"].dtype == torch.bfloat16 else kda.KDA_F32
    od = kda.KDA_BF16 if out.dtype == torch.bfloat16 else kda.KDA_F32
    return lib.kda_chunk_fwd_noalloc(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["log_alpha"]),
                                     ptr(d["beta"]), ptr(d.get("S0")), ptr(cu), ptr(out), ptr(S_final),
                                     B, T, H, N, dk, d["v"].shape[-1], dt, od, stream)


def _status(lib):
    v = ctypes.c_int32(-1)
    assert lib.kda_chunk_fwd_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                            ctypes.byref(v)) == kda.KDA_OK
    return int(v.value)


def _check_two_calls(d, heads, tol):
    lib = kda.load()
    g = to_device(d, DEV)
    N = g["q"].shape[0] if g.get("cu_seqlens") is None else g["cu_seqlens"].shape[0] - 1
    H = g["q"].shape[2]
    ro, rs = oracle_prefill(d, heads=heads)
    for call in range(2):                                  # two consecutive calls, same inputs
        out = torch.full(g["v"].shape, float("nan"), dtype=torch.float32, device=DEV)
        S_final = torch.full((N, H, 128, 128), float("nan"), device=DEV)
        assert _call_noalloc(lib, g, out, S_final) == kda.KDA_OK
        assert _status(lib) == kda.KDA_OK
        assert_close(np32(out[:, :, heads]), ro, tol, "out (call %d)" % call)
        assert_close(np32(S_final[:, heads]), rs, tol, "S_final (call %d)" % call)


def test_noalloc_bf16_varlen_matches_oracle_on_two_calls():
    w = K.WORKLOADS["bf16_varlen8_262k_h32"]
    d = K.make_prefill(w, T=3000, H=4, seed=31)
    _check_two_calls(d, [0, 3], TOL[torch.bfloat16])


def test_noalloc_fp32_ragged_with_empty_sequence_matches_oracle():
    lens = [70, 0, 1, 130]
    w = K.Workload("noalloc_f32", B=1, T=sum(lens), H=2, dtype="f32", s0_std=0.1)
    d = K.make_prefill(w, seed=33)
    d["S0"] = 0.1 * torch.randn(len(lens), 2, 128, 128, generator=torch.Generator().manual_seed(33))
    d["cu_seqlens"] = torch.tensor(np.cumsum([0] + lens), dtype=torch.int32)
    _check_two_calls(d, [0, 1], TOL[torch.float32])


def test_noalloc_status_reports_device_side_checks():
    lib = kda.load()
    w = K.Workload("noalloc_bad", B=1, T=128, H=2, dtype="bf16")
    g = to_device(K.make_prefill(w, seed=34), DEV)
    out = torch.empty(g["v"].shape, dtype=torch.float32, device=DEV)
    g["cu_seqlens"] = torch.tensor([0, 100, 50, 128], dtype=torch.int32, device=DEV)
    assert _call_noalloc(lib, g, out, None) == kda.KDA_OK
    assert _status(lib) == kda.KDA_ERR_INVALID_ARG
    # the f16 operands of this entry point need the decay of one chunk to stay above e^-9.0
    ws = K.Workload("noalloc_strong", B=1, T=128, H=2, dtype="bf16", alpha_lo=0.5, alpha_hi=0.6)
    g = to_device(K.make_prefill(ws, seed=35), DEV)
    assert _call_noalloc(lib, g, out, None) == kda.KDA_OK
    assert _status(lib) == kda.KDA_ERR_UNSUPPORTED
    # the next call clears the shared status word
    g = to_device(K.make_prefill(w, seed=36), DEV)
    assert _call_noalloc(lib, g, out, None) == kda.KDA_OK
    assert _status(lib) == kda.KDA_OK
