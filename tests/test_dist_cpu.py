"""The N > 1 path on CPU: world_size 2 over gloo.

Sequences and heads are independent, so ranks share nothing but the timing reduction. These tests
run two CPU ranks that each take their share of a packed batch (``shard.balance_sequences``),
compute it with the float64 oracle, and all-gather the results: the union must reproduce a
single-process run bit for bit. They also check the MAX timing reduction and the per-rank seeds
of the weak-scaling benchmark.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from kimi_delta_attention_25_b200 import shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(5)
    lens = [37, 5, 64, 0, 101, 12, 70]
    T, H, d = sum(lens), 2, 8
    q = rng.standard_normal((1, T, H, d)).astype(np.float32)
    k = rng.standard_normal((1, T, H, d)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, d)).astype(np.float32)
    la = np.log(rng.uniform(0.9, 1.0, (1, T, H, d))).astype(np.float32)
    be = rng.uniform(0, 1, (1, T, H)).astype(np.float32)
    S0 = rng.standard_normal((len(lens), H, d, d))
    return lens, q, k, v, la, be, S0


def _worker(rank, world, port, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import ref
        lens, q, k, v, la, be, S0 = _inputs()
        offs = shard.pack_offsets(lens)
        mine = shard.balance_sequences(lens, world)[rank]
        # pack this rank's sequences and run them
        sl = [slice(offs[i], offs[i + 1]) for i in mine]
        cat = lambda a: np.concatenate([a[:, s] for s in sl], axis=1) if sl else a[:, :0]  # noqa: E731
        my_lens = [lens[i] for i in mine]
        out, Sf = ref.forward(cat(q), cat(k), cat(v), cat(la), cat(be), S0=S0[mine],
                              cu_seqlens=shard.pack_offsets(my_lens))
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, out, Sf))
        t = shard.max_over_ranks(1.5 + rank)
        if rank == 0:
            q_out.put((gathered, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_single_process_result():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    gathered, t = q_out.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert t == 2.5                                     # MAX over the ranks' timings

    from oracle import ref
    lens, q, k, v, la, be, S0 = _inputs()
    out_ref, S_ref = ref.forward(q, k, v, la, be, S0=S0, cu_seqlens=shard.pack_offsets(lens))
    offs = shard.pack_offsets(lens)
    seen = []
    for mine, out, Sf in gathered:
        pos = 0
        for j, i in enumerate(mine):
            L = lens[i]
            np.testing.assert_array_equal(out[:, pos:pos + L], out_ref[:, offs[i]:offs[i + 1]])
            np.testing.assert_array_equal(Sf[j], S_ref[i])
            pos += L
        seen += mine
    assert sorted(seen) == list(range(len(lens)))


def test_balance_sequences_is_a_partition_and_balanced():
    lens = [18991, 15538, 40614, 37040, 39372, 55389, 35869, 19331]
    for world in (1, 2, 3, 4, 8, 16):
        shards = shard.balance_sequences(lens, world)
        flat = sorted(i for s in shards for i in s)
        assert flat == list(range(len(lens)))
        loads = [sum(lens[i] for i in s) for s in shards]
        # longest-first greedy: the spread never exceeds the longest sequence
        assert max(loads) - min(loads) <= max(lens)
        assert shards == shard.balance_sequences(lens, world)      # deterministic


def test_rank_seeds_are_distinct_and_start_at_the_base():
    assert [shard.rank_seed(0, r) for r in range(4)] == [0, 1, 2, 3]
    assert shard.max_over_ranks(3.25) == 3.25                       # no process group: identity
    with pytest.raises(ValueError):
        shard.balance_sequences([1, 2], 0)
