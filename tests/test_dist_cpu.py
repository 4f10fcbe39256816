"""The N>1 path on CPU: two gloo ranks shard heads, compute their slice (with
the oracle standing in for the GPU kernel), gather, and reduce timings."""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tiled_attention_12_b200.dist import (aggregate_throughput, gather_heads, max_over_ranks, shard_heads,
                                          shard_range)


def test_shard_range_covers_everything_once():
    for n in (1, 2, 7, 64, 100):
        for world in (1, 2, 3, 8):
            parts = [shard_range(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [e - s for s, e in parts]
            assert max(sizes) - min(sizes) <= 1


def test_aggregate_throughput_is_weak_scaling():
    assert aggregate_throughput(1e12, 10, 4, 1000.0) == pytest.approx(40.0)
    assert aggregate_throughput(1e12, 10, 1, 1000.0) == pytest.approx(10.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out):
    import torch.distributed as dist

    from oracle import attention_ref
    from tiled_attention_12_b200.synth import Case, make_qkv

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = Case("d", 2, 3, 40, 16, True, seed=9)
        q, k, v = make_qkv(c)
        ql, kl, vl = (shard_heads(t, rank, world) for t in (q, k, v))
        o, lse = attention_ref(ql, kl, vl, c.softmax_scale, True)      # this rank's heads only
        o_all = gather_heads(torch.from_numpy(o), c.B, c.H)
        l_all = gather_heads(torch.from_numpy(lse), c.B, c.H)
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            o_ref, l_ref = attention_ref(q, k, v, c.softmax_scale, True)
            out.put((float(np.abs(o_all.numpy() - o_ref).max()), float(np.abs(l_all.numpy() - l_ref).max()), t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_gather_and_reduce():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    o_err, l_err, t = out.get(timeout=10)
    assert o_err == 0.0 and l_err == 0.0
    assert t == 2.0
