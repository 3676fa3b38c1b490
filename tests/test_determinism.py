"""Run-to-run determinism and batch independence of every GPU path.

No kernel accumulates floating point through atomics or in an order that depends on
scheduling (each output row is reduced by one warp in a fixed order; key splits merge
in split order), so the same call must give the same bits every time, and a batch
entry must not depend on the other entries of its batch.  Each case runs twice with
separate workspaces and an unrelated call in between, and compares bit for bit."""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
from long_context_causal_flash_b200 import inputs

pytestmark = pytest.mark.gpu

PATHS = [(torch.float32, "ffma"), (torch.bfloat16, "ffma"), (torch.float32, "tc")]
IDS = ["f32", "bf16", "f32_tc"]


def _ids(x, dev):
    return torch.as_tensor(np.asarray(x), dtype=torch.int32, device=dev)


def _disturb(dev):
    """An unrelated call of another shape between the two runs."""
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, 333, 333, 256, seeds=(7, 8, 9)))
    gqa.fwd(q, k, v)


@pytest.mark.parametrize("dtype,path", PATHS, ids=IDS)
def test_forward_is_bitwise_repeatable(cuda_device, dtype, path):
    dev = cuda_device
    L = 1100
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    ids = _ids(inputs.segment_ids([300, 1, 499, 300]), dev)
    for kw in ({}, {"seg_q": ids, "seg_kv": ids}, {"splits": 3}):
        o1, l1 = gqa.fwd(q, k, v, fp32_path=path, **kw)
        o1, l1 = o1.clone(), l1.clone()
        _disturb(dev)
        o2, l2 = gqa.fwd(q, k, v, fp32_path=path, **kw)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), kw.keys()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_is_bitwise_repeatable(cuda_device, dtype):
    dev = cuda_device
    L = 700
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(dtype).to(dev)
    out, lse = gqa.fwd(q, k, v)
    g1 = [t.clone() for t in gqa.bwd(q, k, v, out, lse, dout)]
    _disturb(dev)
    g2 = gqa.bwd(q, k, v, out, lse, dout)
    torch.cuda.synchronize()
    for a, b, name in zip(g1, g2, ("dq", "dk", "dv")):
        assert torch.equal(a, b), name


@pytest.mark.parametrize("dtype,path", PATHS, ids=IDS)
def test_batch_entries_are_independent(cuda_device, dtype, path):
    """A batch of two equals the two entries called alone, bit for bit."""
    dev = cuda_device
    L = 500
    q, k, v = (t.to(dev) for t in inputs.qkv(2, 16, 4, L, L, 256, dtype=dtype))
    ob, lb = gqa.fwd(q, k, v, fp32_path=path)
    for b in range(2):
        o, l = gqa.fwd(q[b:b + 1].contiguous(), k[b:b + 1].contiguous(), v[b:b + 1].contiguous(), fp32_path=path)
        torch.cuda.synchronize()
        assert torch.equal(o, ob[b:b + 1]) and torch.equal(l, lb[b:b + 1]), b
