"""Context-parallel prefill: one sequence split into consecutive token segments, one per rank.

The recurrence is linear in the state, so each segment maps the state entering it to the state
leaving it affinely, S -> Phi S + Psi, with Phi the product of the segment's transitions
(I - beta k k^T) Diag(alpha) and Psi the segment's final state from a zero start. Every rank
computes its segment's (Phi, Psi) from its own tokens, the ranks exchange them (one all-gather of
2 x H x 128 x 128 fp32 per rank), each rank composes the maps of the ranks before it to find the
state entering its segment, and runs its segment from that state. The pages do not describe this
split (the layer runs on one device there); it follows from the recurrence.

The per-segment work runs in libkda's kernels on the rank's own GPU; the all-gather goes through
torch.distributed (NCCL over NVLink between GPUs; gloo in the CPU tests). ``ops`` lets a test put
other implementations of the three local steps behind the same host logic.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist


class KernelOps:
    """The three local steps through libkda: the segment's affine map, a prefill from a given
    state, and the composition S -> Phi S + Psi."""

    def __init__(self, out_dtype=torch.bfloat16):
        self.out_dtype = out_dtype

    def segment_map(self, q, k, v, log_alpha, beta):
        import kimi_delta_attention_25_b200 as kda
        B, T, H, D = q.shape
        dev = q.device
        ws = torch.empty(max(256, kda.chunk_fwd_workspace_size(B, T, H, B, dtype=q.dtype)), dtype=torch.uint8,
                         device=dev)
        eye = torch.eye(D, dtype=torch.float32, device=dev).expand(B, H, D, D).contiguous()
        zero_v = torch.zeros_like(v)
        # Phi: the segment run from S0 = I with v = 0; Psi: from S0 = 0 with the real v
        _, phi = kda.chunk_fwd(q, k, zero_v, log_alpha, beta, S0=eye, workspace=ws, out_dtype=torch.float32)
        _, psi = kda.chunk_fwd(q, k, v, log_alpha, beta, S0=None, workspace=ws, out_dtype=torch.float32)
        return phi[0], psi[0]

    def prefill(self, q, k, v, log_alpha, beta, S0):
        import kimi_delta_attention_25_b200 as kda
        return kda.chunk_fwd(q, k, v, log_alpha, beta, S0=S0, out_dtype=self.out_dtype)

    def compose(self, Phi, S, Psi):
        import kimi_delta_attention_25_b200 as kda
        return kda.state_affine(Phi, S, Psi)


def entering_state(phis, psis, S0, rank, ops):
    """State entering segment ``rank``: S0 pushed through the maps of segments 0 .. rank-1."""
    S = S0
    for r in range(rank):
        S = ops.compose(phis[r], S, psis[r])
    return S


def context_parallel_prefill(q, k, v, log_alpha, beta, S0: Optional[torch.Tensor] = None, group=None,
                             ops=None):
    """This rank's segment of one sequence (B = 1; tensors [1, T_local, H, d], segments in rank
    order). S0 [1, H, dk, dv] is the sequence's initial state (all ranks pass the same, or None).
    Returns (out of this segment, the state leaving this segment); the last rank's second value is
    the sequence's final state. Every rank must call this (it contains one all-gather)."""
    ops = ops or KernelOps()
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    H, D = q.shape[2], q.shape[3]
    phi, psi = ops.segment_map(q, k, v, log_alpha, beta)
    both = torch.stack([phi, psi]).contiguous()                 # [2, H, dk, dv]
    if world > 1:
        gathered = [torch.empty_like(both) for _ in range(world)]
        dist.all_gather(gathered, both, group=group)
    else:
        gathered = [both]
    start = torch.zeros(H, D, D, dtype=torch.float32, device=q.device) if S0 is None else S0[0]
    S_in = entering_state([g[0] for g in gathered], [g[1] for g in gathered], start, rank, ops)
    return ops.prefill(q, k, v, log_alpha, beta, S_in.unsqueeze(0).contiguous())
