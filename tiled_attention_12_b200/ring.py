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

Zig-zag layout (``zigzag=True``, for the causal mask): with contiguous blocks
rank world-1 attends to every block and rank 0 to one, so the causal work is
unbalanced.  Cutting the sequence into 2*world chunks and giving rank r the
chunks r and 2*world-1-r (stacked as its [B, H, 2c, d] block) equalises it.
Each pair of (query chunk, key chunk) is again full, causal (same chunk) or
empty (a later key chunk), so every piece is one plain fa_fwd call, merged
into the accumulator of its query chunk.
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


def chunk_pairs(rank: int, src: int, world: int, zigzag: bool, causal: bool):
    """Pieces of one ring step: [(query part, key part, mode)] where a part
    indexes the rank's block (0: the whole block, or with zigzag 0/1: its
    first/second chunk) and mode is "full" or "causal" (empty pieces are left
    out)."""
    if not zigzag or not causal:  # without the mask the whole block pair is one full piece
        mode = "causal" if causal and src == rank else "full"
        return [] if causal and src > rank else [(None, None, mode)]
    own = (rank, 2 * world - 1 - rank)
    other = (src, 2 * world - 1 - src)
    pieces = []
    for qa, qc in enumerate(own):
        for kb, kc in enumerate(other):
            if not causal or kc < qc:
                pieces.append((qa, kb, "full"))
            elif kc == qc:
                pieces.append((qa, kb, "causal"))
    return pieces


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


def _run_steps(q, blocks, pieces, softmax_scale, attend, merge, out):
    """Attend the rank's query block to the key/value block each step brings
    (blocks(i)), piece by piece (pieces[i] from chunk_pairs), merging into one
    accumulator per query part; each part's last piece writes its 16-bit rows
    into `out`.  Returns (out, lse)."""
    import torch

    n_parts = 1 if all(p[0] is None for ps in pieces for p in ps) else 2
    c = q.shape[2] // n_parts
    # chunk views, no copies: the attention call takes strided views
    qs = [q] if n_parts == 1 else [q[:, :, :c], q[:, :, c:]]
    outs = [out] if n_parts == 1 else [torch.empty_like(qs[0]), torch.empty_like(qs[1])]
    accs = [_Accumulator(x, merge) for x in qs]
    last = {}
    for i, ps in enumerate(pieces):
        for p in ps:
            last[p[0] or 0] = (i, p)
    for i, ps in enumerate(pieces):
        k, v = blocks(i)
        for p in ps:
            qa, kb, mode = p
            qa = qa or 0
            kk, vv = (k, v) if kb is None else (k[:, :, kb * c:(kb + 1) * c], v[:, :, kb * c:(kb + 1) * c])
            o_part, lse_part = attend(qs[qa], kk, vv, mode == "causal", softmax_scale)
            accs[qa].add(o_part, lse_part, outs[qa] if last[qa] == (i, p) else None)
    if n_parts == 1:
        return out, accs[0].lse
    out[:, :, :c] = outs[0]
    out[:, :, c:] = outs[1]
    return out, torch.cat((accs[0].lse, accs[1].lse), dim=2)


def ring_attention(q, k, v, causal: bool = False, softmax_scale=None, group=None, attend=None, merge=None,
                   zigzag: bool = False):
    """This rank's rows of softmax(scale Q K^T [+ causal]) V over the whole
    ring's sequence.  q, k, v: this rank's [B, H, n, d] contiguous blocks
    (zigzag: its two chunks stacked, n even).  Returns (o [B, H, n, d] in q's
    dtype, lse [B, H, n] fp32) for the same rows."""
    import torch
    import torch.distributed as dist

    attend = attend or _cuda_attend
    merge = merge or _cuda_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    steps = ring_steps(rank, world, causal)
    pieces = [chunk_pairs(rank, src, world, zigzag, causal) for src, _ in steps]
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
    o, lse = _run_steps(q, blocks, pieces, softmax_scale, attend, merge, out)
    if pending[0] is not None:
        for req in pending[0]:
            req.wait()
    return o, lse


def ring_attention_emulated(q, k, v, world: int, causal: bool = False, softmax_scale=None, zigzag: bool = False,
                            rank_ms=None):
    """The ring on one device: the full [B, H, N, d] tensors are cut into the
    ranks' blocks (contiguous, or zig-zag chunk pairs) and every rank's steps
    run one after the other (no rank waits on another).  It runs exactly the
    per-rank attention and merge calls of ring_attention, without the
    transfers.  With ``rank_ms`` a list, each rank's device time (CUDA events)
    is appended to it: the maximum is the compute time of a real ring.
    Returns (o, lse) for the whole sequence."""
    import torch

    B, H, N, d = q.shape
    parts = 2 * world if zigzag else world
    if N % parts:
        raise ValueError("the sequence length must split into equal blocks")
    c = N // parts
    if zigzag:
        rows = [torch.cat((torch.arange(r * c, (r + 1) * c), torch.arange((parts - 1 - r) * c, (parts - r) * c)))
                for r in range(world)]
    else:
        rows = [torch.arange(r * c, (r + 1) * c) for r in range(world)]
    rows = [r.to(q.device) for r in rows]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    blk = {r: (k[:, :, rows[r]].contiguous(), v[:, :, rows[r]].contiguous()) for r in range(world)}
    for rank in range(world):
        steps = ring_steps(rank, world, causal)
        pieces = [chunk_pairs(rank, src, world, zigzag, causal) for src, _ in steps]
        qr = q[:, :, rows[rank]].contiguous()
        out = torch.empty_like(qr)
        if rank_ms is not None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
        _, lr = _run_steps(qr, lambda i: blk[steps[i][0]], pieces, softmax_scale, _cuda_attend, _cuda_merge, out)
        if rank_ms is not None:
            e1.record()
            torch.cuda.synchronize()
            rank_ms.append(e0.elapsed_time(e1))
        o[:, :, rows[rank]] = out
        lse[:, :, rows[rank]] = lr
    return o, lse
