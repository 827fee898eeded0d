"""The seeded input generator: shapes, dtypes, ranges and the packed-length rule."""
import torch

import kda_inputs as K


def test_varlen_rule_meets_bounds_and_total():
    lens = K.varlen_lengths(8, 262144, 4096, 65536, 0)
    assert sum(lens) == 262144 and len(lens) == 8
    assert all(4096 <= L <= 65536 for L in lens)
    assert lens == K.varlen_lengths(8, 262144, 4096, 65536, 0)   # deterministic


def test_prefill_inputs_follow_the_recipe():
    w = K.WORKLOADS["bf16_t128k_h32"]
    d = K.make_prefill(w, T=300, H=3)
    assert d["q"].dtype == torch.bfloat16 and d["q"].shape == (1, 300, 3, 128)
    n = torch.linalg.vector_norm(d["k"].float(), dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)
    a = torch.exp(d["log_alpha"])
    assert a.min() >= 0.95 - 1e-6 and a.max() <= 0.9999 + 1e-6
    assert 0 < d["beta"].min() and d["beta"].max() < 1
    assert d["S0"].shape == (1, 3, 128, 128) and abs(d["S0"].std().item() - 0.1) < 0.01
    d2 = K.make_prefill(w, T=300, H=3)
    assert torch.equal(d["v"], d2["v"]) and torch.equal(d["S0"], d2["S0"])


def test_varlen_inputs_pack_sequences():
    w = K.WORKLOADS["bf16_varlen8_262k_h32"]
    d = K.make_prefill(w, T=4096, H=2)
    cu = d["cu_seqlens"].tolist()
    assert cu[0] == 0 and cu[-1] == 4096 and len(cu) == 9
    assert all(b >= a for a, b in zip(cu, cu[1:]))
    assert d["S0"].shape == (8, 2, 128, 128)


def test_decode_inputs():
    w = K.WORKLOADS["decode_n256_h32"]
    s = K.make_decode_state(w, N=4, H=2)
    x = K.make_decode_step(w, 3, N=4, H=2)
    assert s.shape == (4, 2, 128, 128) and s.dtype == torch.float32
    assert x["q"].shape == (4, 2, 128) and x["beta"].shape == (4, 2)
    y = K.make_decode_step(w, 4, N=4, H=2)
    assert not torch.equal(x["v"], y["v"])
