"""Context-parallel prefill (kimi_delta_attention_25_b200/cp.py) on CPU: one sequence split into
consecutive segments over 2 and 3 gloo ranks. The host logic (each rank's segment map, the
all-gather of (Phi, Psi), the composition of the earlier ranks' maps, the run from the composed
entering state) is exercised with the float64 oracle standing in for the kernels of the three local
steps; the concatenated outputs and the last rank's final state must equal one oracle run over the
whole sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(T=250, H=2, d=8):
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, T, H, d)).astype(np.float32)
    k = rng.standard_normal((1, T, H, d)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, d)).astype(np.float32)
    la = np.log(rng.uniform(0.9, 1.0, (1, T, H, d))).astype(np.float32)
    be = rng.uniform(0, 1, (1, T, H)).astype(np.float32)
    S0 = rng.standard_normal((1, H, d, d))
    return q, k, v, la, be, S0


class OracleOps:
    """The three local steps of cp.context_parallel_prefill in float64 on the host (oracle)."""

    def segment_map(self, q, k, v, log_alpha, beta):
        from oracle import ref
        H, d = q.shape[2], q.shape[3]
        a = [t.numpy() for t in (q, k, v, log_alpha, beta)]
        eye = np.broadcast_to(np.eye(d), (1, H, d, d))
        _, phi = ref.forward(a[0], a[1], np.zeros_like(a[2]), a[3], a[4], S0=eye)
        _, psi = ref.forward(*a)
        return torch.from_numpy(phi[0]), torch.from_numpy(psi[0])

    def prefill(self, q, k, v, log_alpha, beta, S0):
        from oracle import ref
        out, sf = ref.forward(*[t.numpy() for t in (q, k, v, log_alpha, beta)], S0=S0.numpy())
        return torch.from_numpy(out), torch.from_numpy(sf)

    def compose(self, Phi, S, Psi):
        return torch.matmul(Phi.double(), S.double()) + Psi.double()


def _worker(rank, world, port, cuts, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from kimi_delta_attention_25_b200 import cp
        q, k, v, la, be, S0 = _inputs()
        sl = slice(cuts[rank], cuts[rank + 1])
        seg = [torch.from_numpy(np.ascontiguousarray(a[:, sl])) for a in (q, k, v, la, be)]
        out, S_leave = cp.context_parallel_prefill(*seg, S0=torch.from_numpy(S0), ops=OracleOps())
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, out.numpy(), S_leave.numpy()))
        if rank == 0:
            q_out.put(gathered)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 120, 250], [0, 64, 65, 250]])
def test_context_parallel_equals_one_pass(cuts):
    from oracle import ref
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    gathered = q_out.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    gathered.sort(key=lambda g: g[0])
    out = np.concatenate([g[1] for g in gathered], axis=1)
    q, k, v, la, be, S0 = _inputs()
    ro, rs = ref.forward(q, k, v, la, be, S0=S0)
    assert np.max(np.abs(out - ro)) <= 1e-11 * np.sqrt(np.mean(ro ** 2))
    assert np.max(np.abs(gathered[-1][2] - rs)) <= 1e-11 * np.sqrt(np.mean(rs ** 2))
    # every rank's leaving state is the state after its last token
    for g in gathered[:-1]:
        _, rs_cut = ref.forward(q[:, :cuts[g[0] + 1]], k[:, :cuts[g[0] + 1]], v[:, :cuts[g[0] + 1]],
                                la[:, :cuts[g[0] + 1]], be[:, :cuts[g[0] + 1]], S0=S0)
        assert np.max(np.abs(g[2] - rs_cut)) <= 1e-11 * np.sqrt(np.mean(rs_cut ** 2))
