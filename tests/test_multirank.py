"""Host logic of the multi-GPU bench path on CPU: two gloo ranks.

Each rank of `bench.py --gpus N` runs an independent replica (its own batch entry,
seeds shifted per rank) and the step time is the maximum over ranks, taken with one
all-reduce of a scalar.  These tests run that logic with the gloo backend on the
host (world size 2), with no GPU.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    from long_context_causal_flash_b200 import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        m = bench._max_over_ranks(times[rank], dist, torch.device("cpu"))
        cfg = bench._config(workloads.by_name("causal_512_f32"), world)
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{m!r} {bench._seed_offset(rank)} {cfg['global_batch']} {cfg['parallelism']}\n")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times", [(3.5, 7.25), (9.0, 1.0)])
def test_step_time_is_max_over_two_gloo_ranks(tmp_path, times):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, times, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    lines = [open(tmp_path / f"rank{r}.txt").read().split(maxsplit=3) for r in range(2)]
    for r, (m, off, gb, par) in enumerate(lines):
        assert float(m) == max(times)           # every rank sees the same maximum
        assert int(off) == 10 * r               # each replica draws its own inputs
        assert int(gb) == 2                     # one batch entry per rank
        assert par.strip().startswith("replicas x2")


def test_single_process_max_is_identity():
    import bench

    assert bench._max_over_ranks(4.25, None, torch.device("cpu")) == 4.25


# ----------------------------------------------------------------------------- one problem over the ranks
def _oracle_attention(q, k, v, **kw):
    import oracle

    out, lse = oracle.attention(q, k, v, **kw)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _oracle_block(q, k, v, q_pos_offset):
    import oracle

    out, lse = oracle.attention_block(q, k, v, q_pos_offset=q_pos_offset)
    return torch.from_numpy(out), torch.from_numpy(lse)


class _OracleAccumulator:
    def __init__(self, q):
        import numpy as np

        self.o = np.zeros(tuple(q.shape))
        self.lse = np.full(tuple(q.shape[:3]), -np.inf)

    def add(self, o_b, lse_b):
        import oracle

        self.o, self.lse = oracle.merge_partials(self.o, self.lse, o_b.numpy(), lse_b.numpy())

    def result(self):
        return torch.from_numpy(self.o), torch.from_numpy(self.lse)


def _sharded_rank_main(rank, world, port, mode, layout, gather, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import numpy as np

    import bench
    from long_context_causal_flash_b200 import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.causal(96, torch.float64)
        step, _ = bench.sharded_setup(mode, w, rank, world, torch.device("cpu"), layout=layout, gather=gather,
                                      attention=_oracle_attention, block=_oracle_block,
                                      accumulator=_OracleAccumulator)
        out, lse = step()
        m = bench._max_over_ranks(float(rank + 1), dist, torch.device("cpu"))
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out.numpy(), lse=lse.numpy(), m=m)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode,layout,gather", [("heads", "zigzag", False), ("heads", "zigzag", True),
                                                ("ring", "zigzag", False), ("ring", "contiguous", False)])
def test_sharded_bench_step_on_two_gloo_ranks(tmp_path, mode, layout, gather):
    """The bench's strong-scaling step (``--shard heads|ring``) on two CPU ranks, with
    the fp64 oracle standing in for the CUDA calls: the ranks' shares put together
    are the whole problem's attention, and the step time is the slower rank's."""
    import numpy as np

    import oracle
    from long_context_causal_flash_b200 import heads, inputs, ring

    world = 2
    port = _free_port()
    mp.start_processes(_sharded_rank_main, args=(world, port, mode, layout, gather, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    q, k, v = inputs.qkv(1, 16, 4, 96, 96, 256, dtype=torch.float64)
    ref_out, ref_lse = oracle.attention(q, k, v)
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    assert all(float(p["m"]) == 2.0 for p in parts)
    if mode == "heads" and gather:
        for p in parts:
            np.testing.assert_allclose(p["out"], ref_out, rtol=0, atol=1e-12)
            np.testing.assert_allclose(p["lse"], ref_lse, rtol=0, atol=1e-12)
    elif mode == "heads":
        G = 4
        for r, p in enumerate(parts):
            g0, g1 = heads.head_range(r, world, 4)
            np.testing.assert_allclose(p["out"], ref_out[:, g0 * G:g1 * G], rtol=0, atol=1e-12)
            np.testing.assert_allclose(p["lse"], ref_lse[:, g0 * G:g1 * G], rtol=0, atol=1e-12)
    else:
        out = ring.unshard([torch.from_numpy(p["out"]) for p in parts], world, layout)
        lse = ring.unshard([torch.from_numpy(p["lse"]) for p in parts], world, layout)
        np.testing.assert_allclose(out.numpy(), ref_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse.numpy(), ref_lse, rtol=0, atol=1e-12)


def _oracle_backward(q, k, v, out, lse, dout, **kw):
    import oracle

    return tuple(torch.from_numpy(g) for g in oracle.attention_backward(q, k, v, dout, **kw))


def _oracle_block_bwd(q, k, v, out, lse, dout, q_pos_offset):
    import oracle

    return tuple(torch.from_numpy(g) for g in oracle.attention_block_backward(q, k, v, out, lse, dout,
                                                                              q_pos_offset=q_pos_offset))


def _sharded_bwd_rank_main(rank, world, port, mode, layout, gather, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import numpy as np

    import bench
    from long_context_causal_flash_b200 import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.causal(96, torch.float64)
        step, _ = bench.sharded_setup(mode, w, rank, world, torch.device("cpu"), layout=layout, gather=gather,
                                      attention=_oracle_attention, block=_oracle_block,
                                      accumulator=_OracleAccumulator, backward=True, backward_fn=_oracle_backward,
                                      block_bwd=_oracle_block_bwd)
        dq, dk, dv = step()
        np.savez(os.path.join(out_dir, f"bwd{rank}.npz"), dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode,layout,gather", [("heads", "zigzag", False), ("heads", "zigzag", True),
                                                ("ring", "zigzag", False), ("ring", "contiguous", False)])
def test_sharded_bench_backward_step_on_two_gloo_ranks(tmp_path, mode, layout, gather):
    """The bench's strong-scaling backward step (``--shard heads|ring --pass bwd``) on
    two CPU ranks with the oracle standing in for the CUDA calls: the ranks' gradients
    put together are the whole problem's, for the seeded upstream gradient."""
    import numpy as np

    import oracle
    from long_context_causal_flash_b200 import inputs, ring

    world = 2
    port = _free_port()
    mp.start_processes(_sharded_bwd_rank_main, args=(world, port, mode, layout, gather, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    q, k, v = inputs.qkv(1, 16, 4, 96, 96, 256, dtype=torch.float64)
    gen = torch.Generator().manual_seed(inputs.SEED_V + 100)
    dout = torch.randn(q.shape, generator=gen, dtype=torch.float32).to(torch.float64)
    ref = oracle.attention_backward(q, k, v, dout)
    parts = [np.load(tmp_path / f"bwd{r}.npz") for r in range(world)]
    for i, name in enumerate(("dq", "dk", "dv")):
        if mode == "heads" and gather:  # every rank holds the whole gradients
            got = parts[0][name]
            assert all(np.array_equal(p[name], got) for p in parts)
        elif mode == "heads":
            got = np.concatenate([p[name] for p in parts], axis=1)
        else:
            got = ring.unshard([torch.from_numpy(p[name]) for p in parts], world, layout).numpy()
        np.testing.assert_allclose(got, ref[i], rtol=0, atol=1e-12, err_msg=name)
