"""kda_chunk_fwd_noalloc, the prefill entry point for callers that cannot allocate device memory
(inside a CUDA-graph capture, or hosted by a runtime that owns all device memory): called through
the C ABI twice in a row, each result must match kda_chunk_fwd's on the same inputs within the
tolerance the parity tests use. This file is collected last on purpose."""
import ctypes

import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda
from tests.kda_check import TOL, assert_close, np32

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
    cu = d["cu_seqlens"]
    N = B if cu is None else cu.shape[0] - 1
    ptr = lambda t: None if t is None else P(t.data_ptr())  # noqa: E731
    stream = P(torch.cuda.current_stream().cuda_stream)
    return lib.kda_chunk_fwd_noalloc(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["log_alpha"]),
                                     ptr(d["beta"]), ptr(d["S0"]), ptr(cu), ptr(out), ptr(S_final),
                                     B, T, H, N, dk, d["v"].shape[-1], kda.KDA_BF16, 0, stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    lib = kda.load()
    w = K.WORKLOADS["bf16_varlen8_262k_h32"]
    tol = TOL[torch.bfloat16]
    for seed in (31, 32):                                 # two consecutive calls
        d = K.make_prefill(w, device=DEV, T=3000, H=4, seed=seed)
        ref_out, ref_S = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"],
                                       cu_seqlens=d["cu_seqlens"])
        assert kda.workspace_status(kda.chunk_fwd.last_workspace) == kda.KDA_OK
        out = torch.full_like(ref_out, float("nan"))
        S_final = torch.full_like(ref_S, float("nan"))
        assert _call_noalloc(lib, d, out, S_final) == kda.KDA_OK
        torch.cuda.synchronize()
        assert_close(np32(out), np32(ref_out), tol, "out (call with seed %d)" % seed)
        assert_close(np32(S_final), np32(ref_S), tol, "S_final (call with seed %d)" % seed)
