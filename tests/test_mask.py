"""The padding-mask helpers of the binding: a [batch, seq_len] 0/1 attention mask (the form the
lpnh.cn Kimi Linear article, sec. 5, gives) becomes packed sequences with cu_seqlens, and back.
Host logic only (CPU tensors)."""
import numpy as np
import torch

import kimi_delta_attention_25_b200 as kda


def test_right_left_and_inner_padding():
    mask = torch.tensor([[1, 1, 1, 0, 0],
                         [0, 0, 1, 1, 1],
                         [0, 0, 0, 0, 0],
                         [1, 0, 1, 0, 1]])
    cu, idx = kda.cu_seqlens_from_mask(mask)
    assert cu.dtype == torch.int32
    assert cu.tolist() == [0, 3, 6, 6, 9]
    assert idx.tolist() == [0, 1, 2, 7, 8, 9, 15, 17, 19]


def test_unpad_pad_round_trip_keeps_token_order():
    g = torch.Generator().manual_seed(0)
    B, T, H, D = 3, 7, 2, 4
    x = torch.randn(B, T, H, D, generator=g)
    mask = (torch.rand(B, T, generator=g) > 0.4).to(torch.int64)
    cu, idx = kda.cu_seqlens_from_mask(mask)
    packed = kda.unpad(x, idx)
    assert packed.shape == (1, int(cu[-1]), H, D) and packed.is_contiguous()
    for b in range(B):
        rows = x[b][mask[b].bool()]
        assert torch.equal(packed[0, int(cu[b]):int(cu[b + 1])], rows)
    back = kda.pad(packed, idx, B, T, fill=float("nan"))
    m = mask.bool()
    assert torch.equal(back[m], x[m])
    assert bool(torch.isnan(back[~m]).all())


def test_per_token_scalars_and_bool_mask():
    beta = torch.arange(12, dtype=torch.float32).reshape(2, 6, 1)
    mask = torch.tensor([[True, False, True, True, False, False], [False] * 5 + [True]])
    cu, idx = kda.cu_seqlens_from_mask(mask)
    assert cu.tolist() == [0, 3, 4]
    assert kda.unpad(beta, idx)[0, :, 0].tolist() == [0.0, 2.0, 3.0, 11.0]
    assert np.array_equal(kda.pad(kda.unpad(beta, idx), idx, 2, 6)[mask].numpy(), beta[mask].numpy())
