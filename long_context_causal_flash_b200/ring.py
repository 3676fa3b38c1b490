"""Context-parallel ring attention over a causal sequence sharded across ranks.

The 1,048,576-token training runs of maxtext PR #4929 ("Effect") use context
parallelism, and its code review names the ring attention path (``use_tokamax_ring``).
Here a sequence is cut into equal chunks and every rank holds the query rows, keys and
values of its chunks:

* ``layout="contiguous"``: ``world`` chunks, rank ``r`` holds chunk ``r``;
* ``layout="zigzag"``: ``2 world`` chunks, rank ``r`` holds chunks ``r`` and
  ``2 world - 1 - r`` (in that order), so every rank attends to the same number of
  visible chunk pairs (with contiguous chunks rank ``r`` has ``r + 1`` and the last
  rank does ``world`` times the work of the first).

At ring step ``s = 0 .. world - 1`` rank ``r`` holds the key/value shard of rank
``src = (r - s) mod world`` and passes it on to rank ``r + 1`` while it computes, for
each of its query chunks ``qc`` and each key chunk ``kc`` of that shard:

* ``kc == qc``: the diagonal block, causal (``gqa_attn_fwd_offset``, offset 0);
* ``kc < qc``: a block wholly before the queries, every key visible (offset
  ``(qc - kc) C`` for chunks of ``C`` positions);
* ``kc > qc``: wholly after them, nothing to compute.

Partial results merge exactly by their log-sum-exps (``gqa_attn_merge``) into an fp32
accumulator per query chunk; a last merge writes ``out`` in the input dtype.  The
transport is torch.distributed point-to-point (NCCL send / receive over NVLink into the
receiver's own buffers): each step posts the next shard's send and receive before
computing on the current one, so the transfer overlaps the compute.  No kernel here
reads another GPU's memory.

The backward (``ring_attention_backward``) walks the same schedule with the whole
sequence's ``out`` and ``lse`` of each rank's rows: each visible block's gradients
(``gqa_attn_bwd_offset``) add to this rank's dq and to dk / dv accumulators (fp32)
that travel with the key/value shard, one step behind it: a step's contributions are
computed while the shard's accumulators are still on their way from the previous rank,
then added to them and passed on; after the last step they reach the shard's owner.
"""

from __future__ import annotations

import torch

from . import bwd_offset, fwd_offset, merge

LAYOUTS = ("contiguous", "zigzag")


def chunks_of(rank: int, world: int, layout: str = "contiguous"):
    """Global chunk ids held by `rank`, in the order its shard stores them."""
    if layout == "contiguous":
        return (rank,)
    if layout == "zigzag":
        return (rank, 2 * world - 1 - rank)
    raise ValueError(f"layout must be one of {LAYOUTS}")


def ring_schedule(rank: int, world: int, layout: str = "contiguous"):
    """Per ring step ``s``: ``(src, blocks)``: the rank whose key/value shard this rank
    holds at step ``s``, and the visible blocks ``(q_local, k_local, offset_in_chunks)``
    to compute on it (local = index of the chunk within a shard)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    mine = chunks_of(rank, world, layout)
    out = []
    for s in range(world):
        src = (rank - s) % world
        theirs = chunks_of(src, world, layout)
        blocks = [(qi, kj, qc - kc) for qi, qc in enumerate(mine) for kj, kc in enumerate(theirs) if kc <= qc]
        out.append((src, blocks))
    return out


def _gpu_block(q, k, v, q_pos_offset):
    return fwd_offset(q, k, v, q_pos_offset=q_pos_offset)


class _GpuAccumulator:
    """fp32 running (out, lse) of one query chunk, merged on the GPU."""

    def __init__(self, q):
        self.q = q
        self.o = None
        self.lse = None

    def add(self, o_b, lse_b):
        if self.o is None:
            self.o, self.lse = merge(None, None, o_b, lse_b)
        else:
            merge(self.o, self.lse, o_b, lse_b, out=self.o, lse_out=self.lse)

    def result(self):
        out = torch.empty_like(self.q)
        lse = torch.empty(self.lse.shape, dtype=torch.float32, device=self.lse.device)
        merge(self.o, self.lse, None, None, out=out, lse_out=lse)
        return out, lse


def _chunk(t, i, n):
    """Chunk i of n along the sequence axis of a [B, H, L, d] shard, contiguous."""
    C = t.shape[2] // n
    return t[:, :, i * C:(i + 1) * C].contiguous()


def _accumulate(q, kv_steps, rank, world, layout, block, accumulator):
    n = len(chunks_of(rank, world, layout))
    C = q.shape[2] // n
    qs = [_chunk(q, i, n) for i in range(n)] if n > 1 else [q]
    accs = [accumulator(qc) for qc in qs]
    for (src, blocks), (k, v) in zip(ring_schedule(rank, world, layout), kv_steps):
        ks = [_chunk(k, j, n) for j in range(n)] if n > 1 else [k]
        vs = [_chunk(v, j, n) for j in range(n)] if n > 1 else [v]
        for qi, kj, off in blocks:
            o_b, lse_b = block(qs[qi], ks[kj], vs[kj], off * C)
            accs[qi].add(o_b, lse_b)
    results = [a.result() for a in accs]
    if n == 1:
        return results[0]
    return torch.cat([r[0] for r in results], dim=2), torch.cat([r[1] for r in results], dim=2)


def _ring_kv(k, v, rank, world, group):
    """The key/value shard held at each step, rotated one rank per step.  Shards arrive
    in two buffers of this function's own, used in turn; the caller's ``k`` and ``v``
    are only sent, never written."""
    import torch.distributed as dist

    cur = (k, v)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)] if world > 1 else []
    to_rank = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    from_rank = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    for s in range(world):
        reqs = []
        nxt = None
        if s < world - 1:
            nxt = bufs[s % 2]  # sent during step s - 1 at the latest, and waited for then
            ops = [dist.P2POp(dist.isend, cur[0], to_rank, group), dist.P2POp(dist.isend, cur[1], to_rank, group),
                   dist.P2POp(dist.irecv, nxt[0], from_rank, group), dist.P2POp(dist.irecv, nxt[1], from_rank, group)]
            reqs = dist.batch_isend_irecv(ops)
        yield cur
        for r in reqs:
            r.wait()
        if nxt is not None:
            cur = nxt


def ring_attention(q, k, v, *, group=None, layout="contiguous", block=None, accumulator=None):
    """Causal attention of this rank's shard over the whole sharded sequence.

    ``q`` ``[B, Hq, Ls, d]`` and ``k``/``v`` ``[B, Hkv, Ls, d]`` are this rank's shard
    (contiguous, equal length on every rank; for ``layout="zigzag"`` its two chunks in
    the order of ``chunks_of``, see ``shard``).  Returns ``(out, lse)`` of this rank's
    query rows in the same order.  Every rank of ``group`` must call it (each step
    sends and receives).  ``block(q, k, v, q_pos_offset) -> (out, lse)`` and
    ``accumulator(q)`` default to the CUDA library (``gqa_attn_fwd_offset``,
    ``gqa_attn_merge``)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if k.shape[2] != q.shape[2] or v.shape != k.shape:
        raise ValueError("q, k and v must hold shards of the same length")
    if q.shape[2] % len(chunks_of(rank, world, layout)):
        raise ValueError("the shard length must split into the layout's chunks")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k and v must be contiguous")
    return _accumulate(q, _ring_kv(k, v, rank, world, group), rank, world, layout, block or _gpu_block,
                       accumulator or _GpuAccumulator)


def _gpu_block_bwd(q, k, v, out, lse, dout, q_pos_offset):
    return bwd_offset(q, k, v, out, lse, dout, q_pos_offset=q_pos_offset)


def _chunk_views(t, n):
    """The n equal chunks of a shard along the sequence axis, as views."""
    C = t.shape[2] // n
    return [t[:, :, i * C:(i + 1) * C] for i in range(n)]


def _acc_dtype(dtype):
    """Gradient accumulators: fp32, or the inputs' own precision when it is higher."""
    return torch.float64 if dtype == torch.float64 else torch.float32


def _add_block_grads(blocks, n, C, qs, outs, lses, douts, k, v, dq_acc, dk_acc, dv_acc, block_bwd):
    """Adds the gradients of one ring step's visible blocks: dq to this rank's chunks,
    dk / dv to the accumulators of the key/value shard held at this step."""
    ks = [_chunk(k, j, n) for j in range(n)] if n > 1 else [k]
    vs = [_chunk(v, j, n) for j in range(n)] if n > 1 else [v]
    dqs, dks, dvs = _chunk_views(dq_acc, n), _chunk_views(dk_acc, n), _chunk_views(dv_acc, n)
    for qi, kj, off in blocks:
        dq_b, dk_b, dv_b = block_bwd(qs[qi], ks[kj], vs[kj], outs[qi], lses[qi], douts[qi], off * C)
        dqs[qi] += dq_b
        dks[kj] += dk_b
        dvs[kj] += dv_b


def ring_attention_backward(q, k, v, out, lse, dout, *, group=None, layout="contiguous", block_bwd=None):
    """Gradients ``(dq, dk, dv)`` of this rank's shard for a loss over the whole
    sharded sequence, from ``ring_attention``'s ``out`` and ``lse`` of this rank's rows
    and the upstream gradient ``dout`` of those rows (shard layouts as for
    ``ring_attention``).  Every rank of ``group`` must call it.  ``block_bwd(q, k, v,
    out, lse, dout, q_pos_offset) -> (dq, dk, dv)`` defaults to the CUDA library
    (``gqa_attn_bwd_offset``).  Partial gradients are summed in fp32 (fp64 for fp64
    inputs) and returned in the inputs' dtype."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if k.shape[2] != q.shape[2] or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("q, out, dout and k, v must hold shards of the same length")
    n = len(chunks_of(rank, world, layout))
    if q.shape[2] % n:
        raise ValueError("the shard length must split into the layout's chunks")
    C = q.shape[2] // n
    block_bwd = block_bwd or _gpu_block_bwd
    qs = [_chunk(q, i, n) for i in range(n)] if n > 1 else [q]
    outs = [_chunk(out, i, n) for i in range(n)] if n > 1 else [out]
    douts = [_chunk(dout, i, n) for i in range(n)] if n > 1 else [dout]
    lses = [lse[:, :, i * C:(i + 1) * C].contiguous() for i in range(n)] if n > 1 else [lse]
    acc = dict(dtype=_acc_dtype(q.dtype), device=q.device)
    dq = torch.zeros(q.shape, **acc)
    cur_kv = (k, v)
    to_rank = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    from_rank = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    pending = None  # the accumulators of the shard held next, in flight from the previous rank
    for s, (src, blocks) in enumerate(ring_schedule(rank, world, layout)):
        kv_reqs = []
        nxt_kv = None
        if s < world - 1:  # the next shard moves while this one is computed
            nxt_kv = (torch.empty_like(k), torch.empty_like(v))
            kv_reqs = dist.batch_isend_irecv(
                [dist.P2POp(dist.isend, cur_kv[0], to_rank, group), dist.P2POp(dist.isend, cur_kv[1], to_rank, group),
                 dist.P2POp(dist.irecv, nxt_kv[0], from_rank, group),
                 dist.P2POp(dist.irecv, nxt_kv[1], from_rank, group)])
        # this step's dk / dv contributions, computed while the shard's accumulators
        # (sent by the previous rank after its step s - 1) are still arriving
        part = (torch.zeros(k.shape, **acc), torch.zeros(v.shape, **acc))
        _add_block_grads(blocks, n, C, qs, outs, lses, douts, cur_kv[0], cur_kv[1], dq, part[0], part[1],
                         block_bwd)
        if pending is not None:
            reqs, arrived = pending
            for r in reqs:
                r.wait()
            part[0].add_(arrived[0])
            part[1].add_(arrived[1])
        if world > 1:  # pass them on (after the last step they reach their owner)
            arrived = (torch.empty_like(part[0]), torch.empty_like(part[1]))
            pending = (dist.batch_isend_irecv(
                [dist.P2POp(dist.isend, part[0], to_rank, group), dist.P2POp(dist.isend, part[1], to_rank, group),
                 dist.P2POp(dist.irecv, arrived[0], from_rank, group),
                 dist.P2POp(dist.irecv, arrived[1], from_rank, group)]), arrived)
        for r in kv_reqs:
            r.wait()
        if nxt_kv is not None:
            cur_kv = nxt_kv
    if pending is None:  # one rank: the accumulators never left
        own = part
    else:
        reqs, own = pending
        for r in reqs:
            r.wait()
    return dq.to(q.dtype), own[0].to(k.dtype), own[1].to(v.dtype)


class _RingAttention(torch.autograd.Function):
    """ring_attention as the forward, ring_attention_backward as the backward."""

    @staticmethod
    def forward(ctx, q, k, v, group, layout, block, accumulator, block_bwd):
        out, lse = ring_attention(q, k, v, group=group, layout=layout, block=block, accumulator=accumulator)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.cfg = (group, layout, block_bwd)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, _dlse):
        q, k, v, out, lse = ctx.saved_tensors
        group, layout, block_bwd = ctx.cfg
        dq, dk, dv = ring_attention_backward(q, k, v, out, lse, dout.to(q.dtype).contiguous(), group=group,
                                             layout=layout, block_bwd=block_bwd)
        return dq, dk, dv, None, None, None, None, None


def ring_attention_autograd(q, k, v, *, group=None, layout="contiguous", block=None, accumulator=None,
                            block_bwd=None):
    """Differentiable ``ring_attention``: returns ``out`` of this rank's rows; autograd's
    backward runs ``ring_attention_backward`` (every rank of ``group`` must take part in
    the backward, as in the forward).  The block functions default to the CUDA
    library's."""
    out, _ = _RingAttention.apply(q, k, v, group, layout, block, accumulator, block_bwd)
    return out


def ring_attention_backward_single_device(q, k, v, out, lse, dout, world, *, layout="contiguous", block_bwd=None):
    """Every rank's ring backward on one device, one after another, from the full
    ``[B, H, L, d]`` tensors and the whole sequence's ``out`` / ``lse`` (no transport:
    each shard's dk / dv accumulate in place).  Returns the full ``(dq, dk, dv)``."""
    block_bwd = block_bwd or _gpu_block_bwd
    acc = dict(dtype=_acc_dtype(q.dtype), device=q.device)
    dqs, dks, dvs = [], [], []
    n = len(chunks_of(0, world, layout))
    for r in range(world):
        dks.append(torch.zeros(shard(k, r, world, layout).shape, **acc))
        dvs.append(torch.zeros(shard(v, r, world, layout).shape, **acc))
    for rank in range(world):
        qr, outr, doutr, lser = (shard(x, rank, world, layout) for x in (q, out, dout, lse))
        C = qr.shape[2] // n
        qs = [_chunk(qr, i, n) for i in range(n)] if n > 1 else [qr]
        outs = [_chunk(outr, i, n) for i in range(n)] if n > 1 else [outr]
        douts = [_chunk(doutr, i, n) for i in range(n)] if n > 1 else [doutr]
        lses = [lser[:, :, i * C:(i + 1) * C].contiguous() for i in range(n)] if n > 1 else [lser]
        dq = torch.zeros(qr.shape, **acc)
        for src, blocks in ring_schedule(rank, world, layout):
            ks, vs = shard(k, src, world, layout), shard(v, src, world, layout)
            _add_block_grads(blocks, n, C, qs, outs, lses, douts, ks, vs, dq, dks[src], dvs[src], block_bwd)
        dqs.append(dq)
    return (unshard(dqs, world, layout).to(q.dtype), unshard(dks, world, layout).to(k.dtype),
            unshard(dvs, world, layout).to(v.dtype))


def shard(x, rank, world, layout="contiguous"):
    """This rank's shard of a full ``[B, H, L, d]`` (or ``[B, H, L]``) tensor."""
    ids = chunks_of(rank, world, layout)
    n_all = world * len(ids)
    C = x.shape[2] // n_all
    if x.shape[2] != C * n_all:
        raise ValueError("the sequence length must split into equal chunks")
    return torch.cat([x[:, :, c * C:(c + 1) * C] for c in ids], dim=2).contiguous()


def unshard(parts, world, layout="contiguous"):
    """The full tensor from every rank's shard (``parts[r]`` of rank ``r``)."""
    n = len(chunks_of(0, world, layout))
    C = parts[0].shape[2] // n
    pieces = {}
    for r, p in enumerate(parts):
        for i, c in enumerate(chunks_of(r, world, layout)):
            pieces[c] = p[:, :, i * C:(i + 1) * C]
    return torch.cat([pieces[c] for c in sorted(pieces)], dim=2)


def ring_attention_single_device(q, k, v, world, *, layout="contiguous", block=None, accumulator=None):
    """Every rank's ring computation on one device, one after another, with the shards
    taken from the full ``[B, H, L, d]`` tensors (no transport).  Returns the full
    ``(out, lse)``; equals the causal attention of the whole sequence."""
    outs, lses = [], []
    for rank in range(world):
        kv = ((shard(k, src, world, layout), shard(v, src, world, layout)) for src, _ in ring_schedule(rank, world, layout))
        o, lse = _accumulate(shard(q, rank, world, layout), kv, rank, world, layout, block or _gpu_block,
                             accumulator or _GpuAccumulator)
        outs.append(o)
        lses.append(lse)
    return unshard(outs, world, layout), unshard(lses, world, layout)
