"""The ring attention schedule and transfers on CPU: gloo ranks run
ring_attention with the oracle standing in for the two GPU calls (attention
of one block, merge of one partial), and every rank's rows must equal plain
attention over the whole sequence."""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tiled_attention_12_b200.ring import ring_steps


def test_zigzag_pieces_cover_the_causal_triangle_once():
    """Over all steps, rank r's two query chunks meet every key chunk at or
    before them exactly once, and the work per rank is equal."""
    from tiled_attention_12_b200.ring import chunk_pairs
    for world in (1, 2, 3, 4, 8):
        work = []
        for rank in range(world):
            seen, units = set(), 0.0
            own = (rank, 2 * world - 1 - rank)
            for src, _ in ring_steps(rank, world, True):
                other = (src, 2 * world - 1 - src)
                for qa, kb, mode in chunk_pairs(rank, src, world, True, True):
                    qc, kc = own[qa], other[kb]
                    assert (qc, kc) not in seen and kc <= qc and (mode == "causal") == (kc == qc)
                    seen.add((qc, kc))
                    units += 0.5 if mode == "causal" else 1.0
            assert seen == {(qc, kc) for qc in own for kc in range(qc + 1)}
            work.append(units)
        assert max(work) == min(work)


def test_ring_steps_visit_every_block_once():
    for world in (1, 2, 3, 8):
        for rank in range(world):
            srcs = [s for s, _ in ring_steps(rank, world, False)]
            assert sorted(srcs) == list(range(world)) and srcs[0] == rank
            assert all(m == "full" for _, m in ring_steps(rank, world, False))
            for src, mode in ring_steps(rank, world, True):
                assert mode == ("full" if src < rank else "causal" if src == rank else "skip")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _attend_cpu(q, k, v, causal, scale):
    from oracle import attention_ref

    o, lse = attention_ref(q, k, v, scale, causal, workers=1)
    return torch.from_numpy(o).to(q.dtype), torch.from_numpy(lse).to(torch.float32)


def _merge_cpu(o_part, lse_part, o_acc, lse_acc, o_out, first):
    from oracle import merge_partials_ref

    if first:
        o, lse = o_part.double().numpy(), lse_part.double().numpy()
    else:
        o, lse = merge_partials_ref(o_acc, lse_acc, o_part, lse_part)
    lse_acc.copy_(torch.from_numpy(np.asarray(lse)))
    (o_out if o_out is not None else o_acc).copy_(torch.from_numpy(np.asarray(o)))


def _rank(rank, world, causal, port, out, zigzag=False):
    import torch.distributed as dist

    from oracle import attention_ref
    from tiled_attention_12_b200.ring import ring_attention

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, n, d = 1, 2, 8, 4
        g = torch.Generator().manual_seed(3)
        q, k, v = (torch.randn((B, H, n * world, d), generator=g) for _ in range(3))
        if zigzag:  # chunks rank and 2*world-1-rank of 2*world
            c = n // 2
            sl = torch.cat((torch.arange(rank * c, (rank + 1) * c),
                            torch.arange((2 * world - 1 - rank) * c, (2 * world - rank) * c)))
        else:
            sl = torch.arange(rank * n, (rank + 1) * n)
        o, lse = ring_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                                causal=causal, softmax_scale=0.5, attend=_attend_cpu, merge=_merge_cpu, zigzag=zigzag)
        ro, rl = attention_ref(q, k, v, 0.5, causal, workers=1)
        out.put((rank, float(np.abs(o.double().numpy() - ro[:, :, sl.numpy()]).max()),
                 float(np.abs(lse.double().numpy() - rl[:, :, sl.numpy()]).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("zigzag", [False, True])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ring_equals_plain_attention(world, causal, zigzag):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, causal, port, out, zigzag)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(out.get(timeout=10) for _ in range(world))
    assert [g[0] for g in got] == list(range(world))
    for _, o_err, l_err in got:
        assert o_err < 1e-5 and l_err < 1e-5
