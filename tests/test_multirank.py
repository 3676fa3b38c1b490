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
