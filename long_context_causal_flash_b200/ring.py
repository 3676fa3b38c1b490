"""Context-parallel ring attention over a causal sequence sharded across ranks.

The 1,048,576-token training runs of maxtext PR #4929 ("Effect") use context
parallelism, and its code review names the ring attention path (``use_tokamax_ring``).
Here a sequence of ``L = world * Ls`` positions is cut into contiguous shards: rank
``r`` holds the query rows, keys and values of positions ``[r Ls, (r + 1) Ls)``.  At
ring step ``s = 0 .. world - 1`` rank ``r`` holds the key/value shard of rank
``src = (r - s) mod world`` and passes it on to rank ``r + 1`` while it computes:

* ``src == r``: the diagonal block, causal (``gqa_attn_fwd_offset``, offset 0);
* ``src < r``: a block wholly before the queries, every key visible (offset
  ``(r - src) Ls``);
* ``src > r``: wholly after them, nothing to compute (the shard is only passed on).

Partial results merge exactly by their log-sum-exps (``gqa_attn_merge``) into an fp32
accumulator; the last merge (``src == 0``) writes ``out`` in the input dtype and the
final LSE.  The transport is torch.distributed point-to-point (NCCL send / receive over
NVLink into the receiver's own buffers): each step posts the next shard's send and
receive before computing on the current one, so the transfer overlaps the compute.
No kernel here reads another GPU's memory.

Contiguous shards leave rank ``r`` with ``r + 1`` blocks (rank ``world - 1`` does the
most); the per-rank work is therefore uneven by design of the plainest schedule.
"""

from __future__ import annotations

import torch

from . import fwd_offset, merge


def ring_schedule(rank: int, world: int):
    """Per ring step ``s``: ``(src, offset_in_shards)`` of the key/value shard rank
    ``rank`` holds at step ``s``; the offset is ``None`` when that shard lies wholly
    after the rank's queries (nothing to compute)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    out = []
    for s in range(world):
        src = (rank - s) % world
        out.append((src, rank - src if src <= rank else None))
    return out


def _gpu_block(q, k, v, q_pos_offset):
    return fwd_offset(q, k, v, q_pos_offset=q_pos_offset)


class _GpuAccumulator:
    """fp32 running (out, lse) of one rank, merged on the GPU."""

    def __init__(self, q):
        self.q = q
        self.o = None
        self.lse = None

    def add(self, o_b, lse_b, final):
        if final:
            out = torch.empty_like(self.q)
            lse = torch.empty(lse_b.shape, dtype=torch.float32, device=lse_b.device)
            merge(self.o, self.lse, o_b, lse_b, out=out, lse_out=lse)
            self.o, self.lse = out, lse
        elif self.o is None:
            self.o, self.lse = merge(None, None, o_b, lse_b)
        else:
            merge(self.o, self.lse, o_b, lse_b, out=self.o, lse_out=self.lse)

    def result(self):
        return self.o, self.lse


def _accumulate(q, kv_steps, rank, world, block, accumulator):
    Ls = q.shape[2]
    acc = accumulator(q)
    for (src, off), (k, v) in zip(ring_schedule(rank, world), kv_steps):
        if off is None:
            continue
        o_b, lse_b = block(q, k, v, off * Ls)
        acc.add(o_b, lse_b, final=src == 0)
    return acc.result()


def _ring_kv(k, v, rank, world, group):
    """The key/value shard held at each step, rotated one rank per step."""
    import torch.distributed as dist

    cur = (k, v)
    nxt = (torch.empty_like(k), torch.empty_like(v)) if world > 1 else None
    to_rank = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    from_rank = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    for s in range(world):
        reqs = []
        if s < world - 1:
            ops = [dist.P2POp(dist.isend, cur[0], to_rank, group), dist.P2POp(dist.isend, cur[1], to_rank, group),
                   dist.P2POp(dist.irecv, nxt[0], from_rank, group), dist.P2POp(dist.irecv, nxt[1], from_rank, group)]
            reqs = dist.batch_isend_irecv(ops)
        yield cur
        for r in reqs:
            r.wait()
        if s < world - 1:
            cur, nxt = nxt, cur


def ring_attention(q, k, v, *, group=None, block=None, accumulator=None):
    """Causal attention of this rank's shard over the whole sharded sequence.

    ``q`` ``[B, Hq, Ls, d]`` and ``k``/``v`` ``[B, Hkv, Ls, d]`` are this rank's shard
    (contiguous, equal length on every rank).  Returns ``(out, lse)`` of this rank's
    query rows.  Every rank of ``group`` must call it (each step sends and receives).
    ``block(q, k, v, q_pos_offset) -> (out, lse)`` and ``accumulator(q)`` default to the
    CUDA library (``gqa_attn_fwd_offset``, ``gqa_attn_merge``)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if k.shape[2] != q.shape[2] or v.shape != k.shape:
        raise ValueError("q, k and v must hold shards of the same length")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k and v must be contiguous")
    return _accumulate(q, _ring_kv(k, v, rank, world, group), rank, world, block or _gpu_block,
                       accumulator or _GpuAccumulator)


def ring_attention_single_device(q, k, v, world, *, block=None, accumulator=None):
    """Every rank's ring computation on one device, one after another, with the shards
    sliced from the full ``[B, H, world * Ls, d]`` tensors (no transport).  Returns the
    full ``(out, lse)``; equals the causal attention of the whole sequence."""
    L = q.shape[2]
    if L % world or k.shape[2] != L:
        raise ValueError("the sequence length must split into `world` equal shards")
    Ls = L // world
    shard = lambda t, r: t[:, :, r * Ls:(r + 1) * Ls].contiguous()  # noqa: E731
    outs, lses = [], []
    for rank in range(world):
        kv = ((shard(k, src), shard(v, src)) for src, _ in ring_schedule(rank, world))
        o, lse = _accumulate(shard(q, rank), kv, rank, world, block or _gpu_block, accumulator or _GpuAccumulator)
        outs.append(o)
        lses.append(lse)
    return torch.cat(outs, dim=2), torch.cat(lses, dim=2)
