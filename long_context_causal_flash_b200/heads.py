"""Forward and backward attention sharded across ranks by key/value head group.

Grouped-query attention splits into independent problems along its key/value heads:
query head h reads only key/value head h / G (kev PR #202, "Why fp32 fell to the L x
L kernel": 16 query heads share 4 key/value heads).  With ``world`` ranks, rank ``r``
takes a contiguous range of key/value heads and the G query heads of each, computes
them with the library's forward, and nothing crosses between ranks on the data path.
``gather=True`` adds one all-gather per output (torch.distributed, NCCL on GPUs) for
a caller that wants the whole ``out`` / ``lse`` on every rank.  The backward splits
the same way: a key/value head's gradient sums over its own G query heads only, which
sit on the same rank, so dK and dV need no reduction across ranks either.
"""

from __future__ import annotations

import torch

from . import bwd, fwd


def head_range(rank: int, world: int, Hkv: int):
    """Key/value heads ``[g0, g1)`` of ``rank``: consecutive, as equal as possible
    (the first ``Hkv % world`` ranks take one more); empty when ``world > Hkv`` and
    ``rank >= Hkv``."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    if Hkv < 1:
        raise ValueError("Hkv must be positive")
    base, extra = divmod(Hkv, world)
    g0 = rank * base + min(rank, extra)
    return g0, g0 + base + (1 if rank < extra else 0)


def shard_heads(q, k, v, rank: int, world: int):
    """This rank's query heads and key/value heads of ``[B, H, L, d]`` tensors, as
    contiguous tensors (``q``: the G query heads of every key/value head it holds).
    With B = 1 a head range of a contiguous tensor is already contiguous and is
    returned as a view (no copy); with B > 1 it is copied."""
    Hq, Hkv = q.shape[1], k.shape[1]
    if Hkv < 1 or Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    g0, g1 = head_range(rank, world, Hkv)
    return (q[:, g0 * G:g1 * G].contiguous(), k[:, g0:g1].contiguous(), v[:, g0:g1].contiguous())


def shard_query_heads(x, rank: int, world: int, Hkv: int):
    """This rank's query heads of a tensor laid out like ``q`` along dim 1 (``out``,
    ``dout`` ``[B, Hq, L, d]`` or ``lse`` ``[B, Hq, L]``), contiguous."""
    Hq = x.shape[1]
    if Hkv < 1 or Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    g0, g1 = head_range(rank, world, Hkv)
    return x[:, g0 * G:g1 * G].contiguous()


def fwd_head_sharded(q, k, v, *, group=None, gather=False, attention=None, presharded=False, **kwargs):
    """Attention of this rank's head groups.

    By default ``q``/``k``/``v`` are the full ``[B, H, L, d]`` tensors on this rank's
    device (every rank passes the same ones) and this rank's heads are taken from them
    (``shard_heads``: a view for B = 1, a copy for B > 1, so a rank then holds the full
    inputs plus, for B > 1, its shard).  With ``presharded=True`` they are already this
    rank's shard (the G query heads of each of its key/value heads, as ``shard_heads``
    returns) and are used as they are: a rank then holds only its own share, 1 / world
    of the inputs.

    Returns ``(out, lse)`` of this rank's query heads, or, with ``gather=True``, the
    full ``out`` ``[B, Hq, Lq, d]`` and ``lse`` ``[B, Hq, Lq]`` on every rank (needs
    every shard to have the same shape: ``Hkv`` divisible by the world size).
    ``attention(q, k, v, **kwargs) -> (out, lse)`` defaults to the CUDA library's
    ``fwd``; ``kwargs`` (mask, offsets, segment ids, splits, fp32_path) pass through.
    Every rank of ``group`` must call it when ``gather`` is set."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if presharded:
        qs, ks, vs = q, k, v
    else:
        if gather and k.shape[1] % world:
            raise ValueError("gather needs Hkv divisible by the world size")
        qs, ks, vs = shard_heads(q, k, v, rank, world)
    run = attention or fwd
    if qs.shape[1] == 0:
        out = torch.empty(qs.shape, dtype=q.dtype, device=q.device)
        lse = torch.empty(qs.shape[:3], dtype=torch.float32, device=q.device)
    else:
        out, lse = run(qs, ks, vs, **kwargs)
    if not gather:
        return out, lse
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return torch.cat(outs, dim=1), torch.cat(lses, dim=1)


def bwd_head_sharded(q, k, v, out, lse, dout, *, group=None, gather=False, backward=None, presharded=False,
                     **kwargs):
    """Gradients of this rank's head groups: ``(dq, dk, dv)`` of its query heads and
    key/value heads, from the forward's ``out`` / ``lse`` and the output gradient
    ``dout``.

    Arguments as in ``fwd_head_sharded``: full tensors (``q``, ``out``, ``dout`` with
    all Hq query heads, ``lse`` ``[B, Hq, Lq]``, ``k`` / ``v`` with all Hkv heads) from
    which this rank takes its heads, or with ``presharded=True`` this rank's shards.
    ``gather=True`` all-gathers the three gradients so every rank holds the full ``dq``
    ``[B, Hq, Lq, d]``, ``dk`` and ``dv`` ``[B, Hkv, Lk, d]``.  ``backward(q, k, v, out,
    lse, dout, **kwargs) -> (dq, dk, dv)`` defaults to the CUDA library's ``bwd``.
    Every rank of ``group`` must call it when ``gather`` is set."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    Hkv = k.shape[1]
    if presharded:
        qs, ks, vs, os_, ls, ds = q, k, v, out, lse, dout
    else:
        if gather and Hkv % world:
            raise ValueError("gather needs Hkv divisible by the world size")
        qs, ks, vs = shard_heads(q, k, v, rank, world)
        os_, ls, ds = (shard_query_heads(x, rank, world, Hkv) for x in (out, lse, dout))
    run = backward or bwd
    if ks.shape[1] == 0:
        dq, dk, dv = torch.empty_like(qs), torch.empty_like(ks), torch.empty_like(vs)
    else:
        dq, dk, dv = run(qs, ks, vs, os_, ls, ds, **kwargs)
    if not gather:
        return dq, dk, dv
    res = []
    for g in (dq, dk, dv):
        parts = [torch.empty_like(g) for _ in range(world)]
        dist.all_gather(parts, g.contiguous(), group=group)
        res.append(torch.cat(parts, dim=1))
    return tuple(res)
