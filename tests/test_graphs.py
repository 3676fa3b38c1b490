"""Every entry point is stream-ordered and allocates nothing, so a call can be captured
in a CUDA graph and replayed: after the inputs change in place, the replay must give
the bits an eager call gives on the new inputs."""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
from long_context_causal_flash_b200 import inputs

pytestmark = pytest.mark.gpu


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("dtype,path,seg,splits", [
    (torch.float32, "ffma", False, 1), (torch.bfloat16, "ffma", False, 1), (torch.float32, "tc", False, 1),
    (torch.float32, "ffma", True, 1), (torch.bfloat16, "ffma", True, 1), (torch.float32, "ffma", False, 3),
    (torch.bfloat16, "ffma", False, 3)],
    ids=["f32", "bf16", "f32_tc", "f32_seg", "bf16_seg", "f32_split", "bf16_split"])
def test_forward_replays_in_a_cuda_graph(cuda_device, dtype, path, seg, splits):
    dev = cuda_device
    L = 600
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    q2, k2, v2 = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype, seeds=(11, 12, 13)))
    ids = torch.as_tensor(np.asarray(inputs.segment_ids([200, 1, 399])), dtype=torch.int32, device=dev) if seg \
        else None
    code = gqa.GQA_F32_TC if path == "tc" else dtype
    need = gqa.split_workspace_bytes(1, 16, 4, L, L, splits, 256, code, "causal", seg) if splits > 1 else \
        gqa.workspace_bytes(1, 16, 4, L, L, 256, code, "causal", seg)
    ws = torch.empty(max(256, need), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    g = _capture(lambda: gqa.fwd(q, k, v, seg_q=ids, seg_kv=ids, out=out, lse=lse, workspace=ws, splits=splits,
                                 fp32_path=path))
    for src, dst in ((q2, q), (k2, k), (v2, v)):
        dst.copy_(src)
    g.replay()
    torch.cuda.synchronize()
    assert gqa.status(ws) == 0
    o_e, l_e = gqa.fwd(q2, k2, v2, seg_q=ids, seg_kv=ids, splits=splits, fp32_path=path)
    torch.cuda.synchronize()
    assert torch.equal(out, o_e) and torch.equal(lse, l_e)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_replays_in_a_cuda_graph(cuda_device, dtype):
    dev = cuda_device
    L = 400
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(dtype).to(dev)
    out, lse = gqa.fwd(q, k, v)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bws = torch.empty(max(256, gqa.bwd_workspace_bytes(1, 16, 4, L, L, 256, dtype)), dtype=torch.uint8, device=dev)
    g = _capture(lambda: gqa.bwd(q, k, v, out, lse, dout, dq=dq, dk=dk, dv=dv, workspace=bws))
    dout2 = torch.randn(q.shape, generator=torch.Generator().manual_seed(8)).to(dtype).to(dev)
    dout.copy_(dout2)
    g.replay()
    torch.cuda.synchronize()
    assert gqa.status(bws) == 0
    want = gqa.bwd(q, k, v, out, lse, dout2)
    torch.cuda.synchronize()
    for got, w, name in zip((dq, dk, dv), want, ("dq", "dk", "dv")):
        assert torch.equal(got, w), name
