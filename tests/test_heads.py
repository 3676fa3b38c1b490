"""Attention sharded by key/value head group (long_context_causal_flash_b200.heads),
forward and backward: the partition and the gather on CPU gloo ranks with the fp64
oracle as each rank's attention, and the CUDA shards of one process put back together
against the unsharded CUDA call."""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from long_context_causal_flash_b200 import heads, inputs  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_head_range_partitions_the_heads():
    for Hkv in (1, 2, 3, 4, 8, 16):
        for world in (1, 2, 3, 4, 5, 8):
            ranges = [heads.head_range(r, world, Hkv) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))       # contiguous
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    assert heads.head_range(3, 4, 4) == (3, 4)
    assert heads.head_range(5, 8, 4) == (4, 4)  # more ranks than heads: empty
    with pytest.raises(ValueError):
        heads.head_range(2, 2, 4)
    with pytest.raises(ValueError):
        heads.head_range(0, 0, 4)


def test_shard_heads_takes_each_groups_query_heads():
    q = torch.arange(1 * 16 * 3 * 2, dtype=torch.float32).reshape(1, 16, 3, 2)
    k = torch.arange(1 * 4 * 3 * 2, dtype=torch.float32).reshape(1, 4, 3, 2)
    qs, ks, vs = heads.shard_heads(q, k, k, 1, 2)
    assert torch.equal(qs, q[:, 8:16]) and torch.equal(ks, k[:, 2:4]) and torch.equal(vs, k[:, 2:4])
    assert qs.is_contiguous() and ks.is_contiguous()
    with pytest.raises(ValueError):
        heads.shard_heads(q[:, :15], k, k, 0, 2)


def _oracle_attention(q, k, v, **kw):
    out, lse = oracle.attention(q, k, v, **kw)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _rank_main(rank, world, port, gather, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = inputs.qkv(1, 16, 4, 40, 70, 256, dtype=torch.float64)
        out, lse = heads.fwd_head_sharded(q, k, v, gather=gather, attention=_oracle_attention, q_pos_offset=30)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out.numpy(), lse=lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,gather", [(2, True), (4, True), (3, False)])
def test_head_sharded_ranks_reproduce_the_full_attention(tmp_path, world, gather):
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, gather, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v = inputs.qkv(1, 16, 4, 40, 70, 256, dtype=torch.float64)
    ref_out, ref_lse = oracle.attention(q, k, v, q_pos_offset=30)
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    if gather:
        for p in parts:  # every rank holds the whole result
            np.testing.assert_allclose(p["out"], ref_out, rtol=0, atol=1e-13)
            np.testing.assert_allclose(p["lse"], ref_lse, rtol=0, atol=1e-13)
    else:
        out = np.concatenate([p["out"] for p in parts], axis=1)
        lse = np.concatenate([p["lse"] for p in parts], axis=1)
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-13)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("world", [2, 4])
def test_cuda_shards_concatenate_to_the_full_call(cuda_device, dtype, world):
    """Every rank's share computed by the CUDA forward (one process, ranks in turn),
    put back together along the head axis, equals the unsharded call bit for bit: the
    kernels compute each key/value head group alone, whatever other heads the call
    holds.  Causal, segmented and shared-prefix branch masks."""
    import long_context_causal_flash_b200 as gqa

    dev = cuda_device
    S, nb, bl = 200, 3, 48
    cases = []
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, 300, 300, 256, dtype=dtype))
    cases.append(((q, k, v), {}))
    ids = torch.as_tensor(inputs.segment_ids([90, 7, 150, 53]), device=dev)
    cases.append(((q, k, v), {"seg_q": ids, "seg_kv": ids}))
    qb, kb, vb = (t.to(dev) for t in inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256, dtype=dtype))
    sq, skv = (torch.as_tensor(x, device=dev) for x in inputs.branch_ids(S, nb, bl))
    cases.append(((qb, kb, vb), {"mask_kind": "prefix_branch", "q_pos_offset": S, "seg_q": sq, "seg_kv": skv}))
    for (q, k, v), kw in cases:
        full_out, full_lse = gqa.fwd(q, k, v, **kw)
        outs, lses = [], []
        for r in range(world):
            qs, ks, vs = heads.shard_heads(q, k, v, r, world)
            o, l = gqa.fwd(qs, ks, vs, **kw)
            outs.append(o)
            lses.append(l)
        torch.cuda.synchronize()
        assert torch.equal(torch.cat(outs, 1), full_out) and torch.equal(torch.cat(lses, 1), full_lse), kw.keys()


def _oracle_backward(q, k, v, out, lse, dout, **kw):
    return tuple(torch.from_numpy(g) for g in oracle.attention_backward(q, k, v, dout, **kw))


def _bwd_rank_main(rank, world, port, gather, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = inputs.qkv(1, 16, 4, 40, 70, 256, dtype=torch.float64)
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7), dtype=torch.float64)
        out = torch.zeros_like(q)  # unused by the oracle's backward (it recomputes P)
        lse = torch.zeros(q.shape[:3], dtype=torch.float64)
        dq, dk, dv = heads.bwd_head_sharded(q, k, v, out, lse, dout, gather=gather, backward=_oracle_backward,
                                            q_pos_offset=30)
        np.savez(os.path.join(out_dir, f"bwd{rank}.npz"), dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,gather", [(2, True), (4, False)])
def test_head_sharded_backward_reproduces_the_full_gradients(tmp_path, world, gather):
    """Gradients per rank (the fp64 oracle's backward as each rank's), gathered or
    concatenated along the head axis, equal the unsharded gradients: a key/value head's
    gradient sums over its own query heads only, all on one rank."""
    port = _free_port()
    mp.start_processes(_bwd_rank_main, args=(world, port, gather, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v = inputs.qkv(1, 16, 4, 40, 70, 256, dtype=torch.float64)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7), dtype=torch.float64)
    ref = oracle.attention_backward(q, k, v, dout, q_pos_offset=30)
    parts = [np.load(tmp_path / f"bwd{r}.npz") for r in range(world)]
    for i, name in enumerate(("dq", "dk", "dv")):
        got = parts[0][name] if gather else np.concatenate([p[name] for p in parts], axis=1)
        np.testing.assert_allclose(got, ref[i], rtol=0, atol=1e-12, err_msg=name)
        if gather:
            for p in parts[1:]:
                assert np.array_equal(p[name], got), name


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("world", [2, 4])
def test_cuda_backward_shards_concatenate_to_the_full_call(cuda_device, dtype, world):
    """Each rank's gradients from the CUDA backward (one process, ranks in turn),
    concatenated along the head axis, equal the unsharded backward bit for bit, for
    causal, segmented and shared-prefix branch masks."""
    import long_context_causal_flash_b200 as gqa

    dev = cuda_device
    S, nb, bl = 200, 3, 48
    cases = []
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, 300, 300, 256, dtype=dtype))
    cases.append(((q, k, v), {}))
    ids = torch.as_tensor(inputs.segment_ids([90, 7, 150, 53]), device=dev)
    cases.append(((q, k, v), {"seg_q": ids, "seg_kv": ids}))
    qb, kb, vb = (t.to(dev) for t in inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256, dtype=dtype))
    sq, skv = (torch.as_tensor(x, device=dev) for x in inputs.branch_ids(S, nb, bl))
    cases.append(((qb, kb, vb), {"mask_kind": "prefix_branch", "q_pos_offset": S, "seg_q": sq, "seg_kv": skv}))
    for (q, k, v), kw in cases:
        out, lse = gqa.fwd(q, k, v, **kw)
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(5)).to(dtype).to(dev)
        full = gqa.bwd(q, k, v, out, lse, dout, **kw)
        parts = []
        for r in range(world):
            qs, ks, vs = heads.shard_heads(q, k, v, r, world)
            os_, ls, ds = (heads.shard_query_heads(x, r, world, 4) for x in (out, lse, dout))
            parts.append(gqa.bwd(qs, ks, vs, os_, ls, ds, **kw))
        torch.cuda.synchronize()
        for i, name in enumerate(("dq", "dk", "dv")):
            assert torch.equal(torch.cat([p[i] for p in parts], 1), full[i]), (name, kw.keys())
