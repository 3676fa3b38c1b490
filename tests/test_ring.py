"""Context-parallel ring attention: the host logic on CPU (gloo ranks) and the CUDA
compute on one GPU.

CPU (no GPU): `ring.ring_attention` runs on 2 and 3 gloo ranks with the transport it
uses on GPUs (torch.distributed point-to-point) and the per-block compute and merge
supplied by the fp64 oracle (oracle.attention_block, oracle.merge_partials); every
rank's result must equal the oracle's attention over the whole sequence.  This checks
the schedule (which shard arrives at which step, the offsets, the skipped blocks), the
buffer rotation and the accumulation order.

GPU: `ring.ring_attention_single_device` runs every rank's schedule on one device with
the library's gqa_attn_fwd_offset and gqa_attn_merge, compared with the oracle.  (No
test here runs several ranks' kernels against one another on one GPU.)

The backward (`ring.ring_attention_backward`) is tested the same two ways: on gloo
ranks with the oracle's block backward (oracle.attention_block_backward) as each
block's compute, and on one GPU with the library's gqa_attn_bwd_offset, both against
the oracle's whole-sequence backward; gqa_attn_bwd_offset alone against the oracle's
block backward.
"""

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
from long_context_causal_flash_b200 import inputs, ring  # noqa: E402
from tests._helpers import to64  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_schedule():
    assert ring.ring_schedule(0, 1) == [(0, [(0, 0, 0)])]
    assert ring.ring_schedule(0, 3) == [(0, [(0, 0, 0)]), (2, []), (1, [])]
    assert ring.ring_schedule(2, 3) == [(2, [(0, 0, 0)]), (1, [(0, 0, 1)]), (0, [(0, 0, 2)])]
    for layout in ring.LAYOUTS:
        for world in (2, 4, 7):
            counts = []
            for r in range(world):
                steps = ring.ring_schedule(r, world, layout)
                assert sorted(src for src, _ in steps) == list(range(world))  # every shard once
                mine = ring.chunks_of(r, world, layout)
                seen = set()
                for src, blocks in steps:
                    theirs = ring.chunks_of(src, world, layout)
                    for qi, kj, off in blocks:
                        assert off == mine[qi] - theirs[kj] >= 0                  # offsets in chunks
                        seen.add((mine[qi], theirs[kj]))
                # every visible (query chunk, key chunk) pair of this rank exactly once
                assert seen == {(qc, kc) for qc in mine for kc in range(world * len(mine)) if kc <= qc}
                counts.append(sum(len(b) for _, b in steps))
            if layout == "zigzag":
                assert len(set(counts)) == 1                                     # balanced
            else:
                assert counts == [r + 1 for r in range(world)]
    with pytest.raises(ValueError):
        ring.ring_schedule(3, 3)
    with pytest.raises(ValueError):
        ring.chunks_of(0, 2, "striped")


def test_shard_and_unshard_are_inverse():
    x = torch.arange(2 * 3 * 24 * 2, dtype=torch.float32).reshape(2, 3, 24, 2)
    for layout in ring.LAYOUTS:
        for world in (1, 2, 3):
            parts = [ring.shard(x, r, world, layout) for r in range(world)]
            assert all(p.shape[2] == 24 // world for p in parts)
            assert torch.equal(ring.unshard(parts, world, layout), x)


def _oracle_block(q, k, v, q_pos_offset):
    out, lse = oracle.attention_block(q, k, v, q_pos_offset=q_pos_offset)
    return torch.from_numpy(out), torch.from_numpy(lse)


class _OracleAccumulator:
    def __init__(self, q):
        self.o = np.zeros(tuple(q.shape))
        self.lse = np.full(tuple(q.shape[:3]), -np.inf)

    def add(self, o_b, lse_b):
        self.o, self.lse = oracle.merge_partials(self.o, self.lse, o_b.numpy(), lse_b.numpy())

    def result(self):
        return torch.from_numpy(self.o), torch.from_numpy(self.lse)


def _rank_main(rank, world, port, Ls, layout, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = inputs.qkv(1, 8, 2, world * Ls, world * Ls, 256, dtype=torch.float32)
        qs, ks, vs = (ring.shard(t, rank, world, layout) for t in (q, k, v))
        ks0, vs0 = ks.clone(), vs.clone()
        out, lse = ring.ring_attention(qs, ks, vs, layout=layout, block=_oracle_block, accumulator=_OracleAccumulator)
        # the caller's key / value shard is only sent, never overwritten by the rotation
        assert torch.equal(ks, ks0) and torch.equal(vs, vs0)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out.numpy(), lse=lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(2, "contiguous"), (3, "contiguous"), (2, "zigzag"), (3, "zigzag")])
def test_ring_on_gloo_ranks_equals_full_attention(tmp_path, world, layout):
    Ls = 18
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, Ls, layout, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v = inputs.qkv(1, 8, 2, world * Ls, world * Ls, 256, dtype=torch.float32)
    ref_out, ref_lse = oracle.attention(q, k, v)
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    out = ring.unshard([torch.from_numpy(p["out"]) for p in parts], world, layout).numpy()
    lse = ring.unshard([torch.from_numpy(p["lse"]) for p in parts], world, layout).numpy()
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("world,Ls,layout", [(2, 200, "contiguous"), (4, 130, "contiguous"), (3, 512, "contiguous"),
                                             (2, 200, "zigzag"), (4, 130, "zigzag"), (3, 510, "zigzag")])
def test_ring_single_device_gpu(cuda_device, dtype, world, Ls, layout):
    L = world * Ls
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    dev = torch.device("cuda")
    out, lse = ring.ring_attention_single_device(q.to(dev), k.to(dev), v.to(dev), world, layout=layout)
    torch.cuda.synchronize()
    assert out.dtype == dtype and lse.dtype == torch.float32
    ref_out, ref_lse = oracle.attention(q, k, v)
    tol_out, tol_lse = (2e-5, 1e-5) if dtype == torch.float32 else (2e-2, 2e-3)
    assert float(np.max(np.abs(to64(out) - ref_out))) <= tol_out
    assert float(np.max(np.abs(to64(lse) - ref_lse))) <= tol_lse


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("Lq,Lk,off", [(200, 300, 0), (200, 300, 57), (130, 70, 500), (64, 64, 64), (1, 300, 0),
                                       (300, 1, 5), (257, 129, 128)])
def test_fwd_offset_gpu(cuda_device, dtype, Lq, Lk, off):
    import long_context_causal_flash_b200 as gqa

    q, k, v = inputs.qkv(1, 16, 4, Lq, Lk, 256, dtype=dtype)
    dev = torch.device("cuda")
    out, lse = gqa.fwd_offset(q.to(dev), k.to(dev), v.to(dev), q_pos_offset=off)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.attention_block(q, k, v, q_pos_offset=off)
    tol_out, tol_lse = (2e-5, 1e-5) if dtype == torch.float32 else (2e-2, 2e-3)
    assert float(np.max(np.abs(to64(out) - ref_out))) <= tol_out
    assert float(np.max(np.abs(to64(lse) - ref_lse))) <= tol_lse


@pytest.mark.gpu
@pytest.mark.parametrize("b_dtype,out_dtype", [(torch.float32, torch.float32), (torch.bfloat16, torch.float32),
                                               (torch.bfloat16, torch.bfloat16), (torch.float32, torch.bfloat16)])
def test_merge_gpu(cuda_device, b_dtype, out_dtype):
    import long_context_causal_flash_b200 as gqa

    rows, d = 1000, 256
    g = torch.Generator().manual_seed(11)
    oa = torch.randn((rows, d), generator=g)
    ob = torch.randn((rows, d), generator=g).to(b_dtype)
    la = torch.randn(rows, generator=g) * 3
    lb = torch.randn(rows, generator=g) * 3
    la[::7] = -float("inf")   # rows empty on one side or on both
    lb[::5] = -float("inf")
    dev = torch.device("cuda")
    out, lse = gqa.merge(oa.to(dev), la.to(dev), ob.to(dev), lb.to(dev), out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.merge_partials(oa.numpy(), la.numpy(), ob.float().numpy(), lb.numpy())
    # bf16 output: half an ulp, at most 2^-8 of the value
    tol = 2e-6 if out_dtype == torch.float32 else 2.0 ** -8 * float(np.max(np.abs(ref_out)))
    assert float(np.max(np.abs(to64(out) - ref_out))) <= tol
    assert np.array_equal(np.isinf(to64(lse)), np.isinf(ref_lse))
    fin = np.isfinite(ref_lse)
    assert float(np.max(np.abs(to64(lse)[fin] - ref_lse[fin]))) <= 1e-6

    # one side absent; in place into the fp32 accumulator
    acc, acc_l = oa.to(dev).clone(), la.to(dev).clone()
    gqa.merge(acc, acc_l, None, None, out=acc, lse_out=acc_l)
    gqa.merge(None, None, ob.to(dev), lb.to(dev), out=acc, lse_out=acc_l)
    torch.cuda.synchronize()
    want = np.where(np.isfinite(lb.numpy())[:, None], ob.float().numpy(), 0.0)
    assert float(np.max(np.abs(to64(acc) - want))) <= 1e-7
    gqa.merge(acc, acc_l, ob.to(dev), lb.to(dev), out=acc, lse_out=acc_l)
    torch.cuda.synchronize()
    # merging a result with itself leaves out unchanged and adds ln 2 to its lse
    assert float(np.max(np.abs(to64(acc) - want))) <= 2e-6
    fin = np.isfinite(lb.numpy())
    assert float(np.max(np.abs(to64(acc_l)[fin] - (lb.numpy()[fin] + np.log(2.0))))) <= 1e-5


# ---- the ring backward

def _oracle_block_bwd(q, k, v, out, lse, dout, q_pos_offset):
    return tuple(torch.from_numpy(g) for g in oracle.attention_block_backward(q, k, v, out, lse, dout,
                                                                              q_pos_offset=q_pos_offset))


def _bwd_inputs(world, Ls):
    q, k, v = inputs.qkv(1, 8, 2, world * Ls, world * Ls, 256, dtype=torch.float64)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(21), dtype=torch.float64)
    out, lse = oracle.attention(q, k, v)
    return q, k, v, torch.from_numpy(out), torch.from_numpy(lse), dout


def _bwd_rank_main(rank, world, port, Ls, layout, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        full = _bwd_inputs(world, Ls)
        q, k, v, out, lse, dout = (ring.shard(t, rank, world, layout) for t in full)
        k0, v0 = k.clone(), v.clone()
        dq, dk, dv = ring.ring_attention_backward(q, k, v, out, lse, dout, layout=layout,
                                                  block_bwd=_oracle_block_bwd)
        assert torch.equal(k, k0) and torch.equal(v, v0)
        np.savez(os.path.join(out_dir, f"bwd{rank}.npz"), dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(1, "contiguous"), (2, "contiguous"), (3, "contiguous"), (2, "zigzag"),
                                          (3, "zigzag")])
def test_ring_backward_on_gloo_ranks_equals_full_backward(tmp_path, world, layout):
    """The ring backward's schedule, the dk / dv accumulators travelling with their
    shard and the final transfer home, with the oracle's block backward as each
    block's compute: every rank's gradients, put together, are the whole sequence's."""
    Ls = 12
    port = _free_port()
    mp.start_processes(_bwd_rank_main, args=(world, port, Ls, layout, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v, out, lse, dout = _bwd_inputs(world, Ls)
    ref = oracle.attention_backward(q, k, v, dout)
    parts = [np.load(tmp_path / f"bwd{r}.npz") for r in range(world)]
    for i, name in enumerate(("dq", "dk", "dv")):
        got = ring.unshard([torch.from_numpy(p[name]) for p in parts], world, layout).numpy()
        np.testing.assert_allclose(got, ref[i], rtol=0, atol=1e-12, err_msg=name)


@pytest.mark.parametrize("world,layout", [(2, "contiguous"), (4, "contiguous"), (3, "zigzag")])
def test_ring_backward_single_device_with_oracle_blocks(world, layout):
    Ls = 10
    q, k, v, out, lse, dout = _bwd_inputs(world, Ls)
    got = ring.ring_attention_backward_single_device(q, k, v, out, lse, dout, world, layout=layout,
                                                     block_bwd=_oracle_block_bwd)
    ref = oracle.attention_backward(q, k, v, dout)
    for g, w, name in zip(got, ref, ("dq", "dk", "dv")):
        np.testing.assert_allclose(g.numpy(), w, rtol=0, atol=1e-12, err_msg=name)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("Lq,Lk,off,B,Hq,Hkv", [(200, 300, 0, 1, 16, 4), (200, 300, 57, 1, 16, 4),
                                                (130, 70, 500, 1, 16, 4), (64, 64, 64, 1, 16, 4),
                                                (1, 300, 0, 1, 16, 4), (300, 1, 5, 1, 16, 4),
                                                (257, 129, 128, 1, 16, 4), (300, 300, 0, 1, 16, 4),
                                                (150, 90, 200, 2, 16, 1), (150, 90, 60, 1, 16, 16)])
def test_bwd_offset_gpu(cuda_device, dtype, Lq, Lk, off, B, Hq, Hkv):
    """One block's gradients against the oracle's block backward, with the out / lse of
    a whole sequence in which the block is one key range (here: the oracle's attention
    of the queries over [other keys | this block], so lse covers more than the block)."""
    import long_context_causal_flash_b200 as gqa

    L_all = off + Lq  # positions 0 .. off + Lq - 1; the block's keys sit at 0 .. Lk - 1
    q, k_all, v_all = inputs.qkv(B, Hq, Hkv, Lq, max(L_all, Lk), 256, dtype=dtype)
    k, v = k_all[:, :, :Lk].contiguous(), v_all[:, :, :Lk].contiguous()
    # whole-sequence rows: keys 0 .. off + Lq - 1 (the block is the first Lk of them)
    out, lse = oracle.attention(q, k_all[:, :, :L_all], v_all[:, :, :L_all], q_pos_offset=off)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(9)).to(dtype)
    dev = torch.device("cuda")
    out_d = torch.from_numpy(out).to(dtype).to(dev)
    lse_d = torch.from_numpy(lse).float().to(dev)
    dq, dk, dv = gqa.bwd_offset(q.to(dev), k.to(dev), v.to(dev), out_d, lse_d, dout.to(dev), q_pos_offset=off)
    torch.cuda.synchronize()
    ref = oracle.attention_block_backward(q, k, v, out_d.double().cpu(), lse_d.double().cpu(), dout,
                                          q_pos_offset=off)
    tol = 5e-5 if dtype == torch.float32 else 2e-2
    for g, w, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
        err = float(np.max(np.abs(to64(g) - w))) / max(1.0, float(np.max(np.abs(w))))
        assert err <= tol, (name, err)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("world,Ls,layout,B,Hq,Hkv", [(2, 200, "contiguous", 1, 16, 4), (4, 130, "contiguous", 1, 16, 4),
                                                      (2, 200, "zigzag", 1, 16, 4), (3, 170, "zigzag", 1, 16, 4),
                                                      (2, 96, "zigzag", 2, 16, 1), (3, 64, "contiguous", 1, 16, 16)])
def test_ring_backward_single_device_gpu(cuda_device, dtype, world, Ls, layout, B, Hq, Hkv):
    """Every rank's ring backward on one GPU with the library's blocks, against the
    oracle's whole-sequence backward (group sizes 4, 16 and 1; a batch of two)."""
    import long_context_causal_flash_b200 as gqa

    L = world * Ls
    q, k, v = inputs.qkv(B, Hq, Hkv, L, L, 256, dtype=dtype)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(4)).to(dtype)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    out, lse = gqa.fwd(qd, kd, vd)
    dq, dk, dv = ring.ring_attention_backward_single_device(qd, kd, vd, out, lse, dod, world, layout=layout)
    torch.cuda.synchronize()
    assert dq.dtype == dtype
    ref = oracle.attention_backward(q, k, v, dout)
    tol = 5e-5 if dtype == torch.float32 else 2e-2
    for g, w, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
        err = float(np.max(np.abs(to64(g) - w))) / max(1.0, float(np.max(np.abs(w))))
        assert err <= tol, (name, err)


def _autograd_rank_main(rank, world, port, Ls, layout, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, _, _, dout = _bwd_inputs(world, Ls)
        qs, ks, vs = (ring.shard(t, rank, world, layout).requires_grad_(True) for t in (q, k, v))
        out = ring.ring_attention_autograd(qs, ks, vs, layout=layout, block=_oracle_block,
                                           accumulator=_OracleAccumulator, block_bwd=_oracle_block_bwd)
        (out * ring.shard(dout, rank, world, layout)).sum().backward()
        np.savez(os.path.join(out_dir, f"ag{rank}.npz"), dq=qs.grad.numpy(), dk=ks.grad.numpy(),
                 dv=vs.grad.numpy(), out=out.detach().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(2, "zigzag"), (3, "contiguous")])
def test_ring_autograd_on_gloo_ranks(tmp_path, world, layout):
    """loss.backward() through the differentiable ring on every rank: the gradients of
    each rank's shard, put together, are the whole sequence's (oracle blocks)."""
    Ls = 12
    port = _free_port()
    mp.start_processes(_autograd_rank_main, args=(world, port, Ls, layout, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v, out, _, dout = _bwd_inputs(world, Ls)
    ref = oracle.attention_backward(q, k, v, dout)
    parts = [np.load(tmp_path / f"ag{r}.npz") for r in range(world)]
    got_out = ring.unshard([torch.from_numpy(p["out"]) for p in parts], world, layout).numpy()
    np.testing.assert_allclose(got_out, out.numpy(), rtol=0, atol=1e-12)
    for i, name in enumerate(("dq", "dk", "dv")):
        got = ring.unshard([torch.from_numpy(p[name]) for p in parts], world, layout).numpy()
        np.testing.assert_allclose(got, ref[i], rtol=0, atol=1e-12, err_msg=name)
