"""Failure detection on the GPU without a fault: a bounded device wait that nothing satisfies runs
out, records KDA_ERR_TIMEOUT in the workspace status word, and leaves the CUDA context usable."""
import pytest
import torch

import kda_inputs as K
import kimi_delta_attention_25_b200 as kda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kimi_delta_attention_25_b200 import build
    build.build()
    kda.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    kda.selftest_wait_timeout(ws, 2_000_000)              # ~1 ms of polling at ~2 GHz
    assert kda.workspace_status(ws) == kda.KDA_ERR_TIMEOUT
    # the same workspace is cleared and reused by an ordinary call
    w = K.Workload("after_timeout", B=1, T=130, H=2, dtype="bf16", s0_std=0.1)
    d = K.make_prefill(w, device="cuda", seed=3)
    big = torch.empty(kda.chunk_fwd_workspace_size(1, 130, 2, 1), dtype=torch.uint8, device="cuda")
    out, Sf = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], workspace=big)
    assert kda.workspace_status(big) == kda.KDA_OK
    assert torch.isfinite(out).all() and torch.isfinite(Sf).all()
