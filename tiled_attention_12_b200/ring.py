"""Ring (sequence-parallel) attention over torch.distributed.

"深度解析注意力机制的变体与演进", section Ring Attention: the sequence is split
over the devices of a ring; each device attends its own query block and the
devices pass blocks around the ring, so a sequence too long for one device's
memory is processed in pieces.  Reading used here: the key/value blocks
travel (one hop per step, to the next rank), each rank keeps its query block,
and the partial results are combined with the online-softmax renormalisation
in log-sum-exp form (fa_merge_partial).

Layout: rank r holds rows [r*n, (r+1)*n) of Q, K and V ([B, H, n, d], the
same n on every rank).  With the causal mask a key block from an earlier rank
is attended in full, the rank's own block with the causal mask, and a later
one not at all (its contribution is empty), so every step is one plain
fa_fwd call.

Each step's transfer (one send to rank+1 and one receive from rank-1 of the
packed K/V block, NCCL peer-to-peer on NVLink) is posted before the step's
attention and waited for after it, so it overlaps the compute.  Every rank
posts the same transfers in the same order; there is no other collective.

``attend`` and ``merge`` default to the CUDA library (fa_fwd,
fa_merge_partial); tests on CPU replace them to exercise the transfer
schedule with the gloo backend.
"""

from __future__ import annotations


def ring_steps(rank: int, world: int, causal: bool):
    """[(source_rank, mode)] for the K/V block held at each step: step s holds
    the block that started on rank (rank - s) mod world.  mode is "full",
    "causal" (the rank's own block under the causal mask) or "skip"."""
    steps = []
    for s in range(world):
        src = (rank - s + world) % world
        if causal and src > rank:
            steps.append((src, "skip"))
        elif causal and src == rank:
            steps.append((src, "causal"))
        else:
            steps.append((src, "full"))
    return steps


def _cuda_attend(q, k, v, causal, softmax_scale):
    from .binding import fa_fwd

    return fa_fwd(q, k, v, causal=causal, softmax_scale=softmax_scale)


def _cuda_merge(o_part, lse_part, o_acc, lse_acc, o_out, first):
    from .binding import fa_merge_partial

    return fa_merge_partial(o_part, lse_part, o_acc, lse_acc, o_out=o_out, first=first)


class _Accumulator:
    """fp32 running (O, LSE) of the local query block across ring steps."""

    def __init__(self, q, merge):
        import torch

        B, H, n, d = q.shape
        self.o_acc = torch.empty((B, H, n, d), device=q.device, dtype=torch.float32)
        self.lse = torch.empty((B, H, n), device=q.device, dtype=torch.float32)
        self.merge = merge
        self.count = 0

    def add(self, o_part, lse_part, o_out=None):
        self.merge(o_part, lse_part, self.o_acc, self.lse, o_out, self.count == 0)
        self.count += 1


def _run_steps(q, blocks, steps, causal, softmax_scale, attend, merge, out):
    """Attend q to each block of `steps` (block fetched by blocks(i)) and merge;
    the last contributing step writes the 16-bit result into `out`."""
    acc = _Accumulator(q, merge)
    live = [i for i, (_, mode) in enumerate(steps) if mode != "skip"]
    for i, (_, mode) in enumerate(steps):
        k, v = blocks(i)
        if mode == "skip":
            continue
        o_part, lse_part = attend(q, k, v, mode == "causal", softmax_scale)
        acc.add(o_part, lse_part, out if i == live[-1] else None)
    return out, acc.lse


def ring_attention(q, k, v, causal: bool = False, softmax_scale=None, group=None, attend=None, merge=None):
    """This rank's rows of softmax(scale Q K^T [+ causal]) V over the whole
    ring's sequence.  q, k, v: this rank's [B, H, n, d] contiguous blocks.
    Returns (o [B, H, n, d] in q's dtype, lse [B, H, n] fp32)."""
    import torch
    import torch.distributed as dist

    attend = attend or _cuda_attend
    merge = merge or _cuda_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    steps = ring_steps(rank, world, causal)
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world

    # double-buffered packed K/V: [2, B, H, n, d]
    bufs = [torch.stack((k, v)), torch.empty((2,) + tuple(k.shape), device=k.device, dtype=k.dtype)]
    pending = [None]

    def blocks(i):
        if pending[0] is not None:          # the transfer posted at step i - 1
            for req in pending[0]:
                req.wait()
            pending[0] = None
        cur = bufs[i % 2]
        if i + 1 < world:                   # forward this block, receive the next
            ops = [dist.P2POp(dist.isend, cur, nxt, group), dist.P2POp(dist.irecv, bufs[(i + 1) % 2], prv, group)]
            pending[0] = dist.batch_isend_irecv(ops)
        return cur[0], cur[1]

    out = torch.empty_like(q)
    o, lse = _run_steps(q, blocks, steps, causal, softmax_scale, attend, merge, out)
    if pending[0] is not None:
        for req in pending[0]:
            req.wait()
    return o, lse


def ring_attention_emulated(q, k, v, world: int, causal: bool = False, softmax_scale=None):
    """The ring on one device: the full [B, H, N, d] tensors are cut into
    `world` equal sequence blocks and every rank's steps run one after the
    other (no rank waits on another).  Returns (o, lse) for the whole
    sequence.  It runs exactly the per-rank attention and merge calls of
    ring_attention, without the transfers."""
    import torch

    B, H, N, d = q.shape
    if N % world:
        raise ValueError("the sequence length must split into equal blocks")
    n = N // world
    blk = [slice(r * n, (r + 1) * n) for r in range(world)]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    for rank in range(world):
        steps = ring_steps(rank, world, causal)
        qr = q[:, :, blk[rank]].contiguous()
        kv = {src: (k[:, :, blk[src]].contiguous(), v[:, :, blk[src]].contiguous())
              for src, mode in steps if mode != "skip"}
        out = torch.empty_like(qr)
        _, lr = _run_steps(qr, lambda i: kv.get(steps[i][0], (None, None)), steps, causal, softmax_scale,
                           _cuda_attend, _cuda_merge, out)
        o[:, :, blk[rank]] = out
        lse[:, :, blk[rank]] = lr
    return o, lse
