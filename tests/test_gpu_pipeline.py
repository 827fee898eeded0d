"""GPU tests of the pipelined prefill: with few (sequence, head) chains kda_chunk_fwd runs its two
passes over token ranges (the scan of one range beside the preparation of the next ones) and
carries the state between ranges. Packed sequences whose ranges cross sequence boundaries (one
empty, one of a single chunk) against the float64 oracle; bitwise equality with the two passes run
one after the other; the carry kept in the workspace when no final state is asked for; an
in-place state (S0 and S_final the same buffer)."""
import numpy as np
import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda
from tests.kda_check import TOL, assert_close, assert_close_bf16_out, np32, oracle_prefill, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"
LENS = [1000, 0, 3000, 64, 5000, 70]
H = 4


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kimi_delta_attention_25_b200 import build
    build.build()
    kda.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _inputs(seed=21):
    T = int(sum(LENS))
    w = K.Workload("pipe", B=1, T=T, H=H, dtype="bf16", s0_std=0.1)
    d = K.make_prefill(w, seed=seed)
    d["cu_seqlens"] = torch.tensor(np.cumsum([0] + LENS), dtype=torch.int32)
    d["S0"] = 0.1 * torch.randn(len(LENS), H, 128, 128, generator=torch.Generator().manual_seed(seed))
    return d


def test_this_size_is_pipelined():
    T = int(sum(LENS))
    assert kda.chunk_fwd_kernel_launches(1, T, H, len(LENS)) > 2
    assert kda.chunk_fwd_kernel_launches(1, 262144, 32, 8) == 2      # many chains: no pipeline


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_pipelined_packed_matches_oracle(out_dtype):
    d = _inputs()
    g = to_device(d, DEV)
    out, Sf, ws = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                                cu_seqlens=g["cu_seqlens"], out_dtype=out_dtype, return_workspace=True)
    assert kda.workspace_status(ws) == kda.KDA_OK
    ro, rs = oracle_prefill(d)
    if out_dtype == torch.bfloat16:
        assert_close_bf16_out(np32(out), ro, TOL[torch.bfloat16], "out (bf16, pipelined)")
    else:
        assert_close(np32(out), ro, TOL[torch.bfloat16], "out (pipelined)")
    assert_close(np32(Sf), rs, TOL[torch.bfloat16], "S_final (pipelined)")


def test_pipelined_equals_two_passes_bitwise():
    g = to_device(_inputs(seed=22), DEV)
    N, T = len(LENS), int(sum(LENS))
    o1, s1 = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                           cu_seqlens=g["cu_seqlens"], out_dtype=torch.bfloat16)
    ws = torch.empty(kda.chunk_fwd_workspace_size(1, T, H, N), dtype=torch.uint8, device=DEV)
    kda.chunk_prep(g["q"], g["k"], g["log_alpha"], g["beta"], ws, cu_seqlens=g["cu_seqlens"])
    o2, s2 = kda.chunk_scan(g["v"], ws, S0=g["S0"], cu_seqlens=g["cu_seqlens"], out_dtype=torch.bfloat16)
    assert kda.workspace_status(ws) == kda.KDA_OK
    assert torch.equal(o1, o2)
    assert torch.equal(s1, s2)


def test_pipelined_without_final_state_and_in_place():
    g = to_device(_inputs(seed=23), DEV)
    o1, s1 = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                           cu_seqlens=g["cu_seqlens"])
    # no final state: the state between ranges lives in the workspace
    o2, s2 = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"],
                           cu_seqlens=g["cu_seqlens"], want_state=False)
    assert s2 is None
    assert torch.equal(o1, o2)
    # S0 and S_final the same buffer
    S = g["S0"].clone()
    o3, s3 = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=S, S_final=S,
                           cu_seqlens=g["cu_seqlens"])
    assert s3.data_ptr() == S.data_ptr()
    assert torch.equal(o1, o3)
    assert torch.equal(s1, S)
