"""`attention`, the autograd wrapper: its gradients are exactly those of `bwd` called
on the forward's out and LSE, and match the fp64 oracle's backward."""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
import oracle
from long_context_causal_flash_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_autograd_gradients_equal_bwd(cuda_device, dtype):
    dev = cuda_device
    L = 300
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(dtype).to(dev)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    out = gqa.attention(qa, ka, va)
    out.backward(dout)
    ref_out, ref_lse = gqa.fwd(q, k, v)
    dq, dk, dv = gqa.bwd(q, k, v, ref_out, ref_lse, dout)
    torch.cuda.synchronize()
    assert torch.equal(out.detach(), ref_out)
    for got, want, name in ((qa.grad, dq, "dq"), (ka.grad, dk, "dk"), (va.grad, dv, "dv")):
        assert torch.equal(got, want), name


def test_autograd_through_a_loss_matches_the_oracle(cuda_device):
    """A loss that is not a plain inner product (so dout is built by autograd, not
    contiguous-by-construction), segment ids, fp32: gradients against the oracle's."""
    dev = cuda_device
    lengths = [50, 1, 149]
    L = sum(lengths)
    ids = inputs.segment_ids(lengths)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256)
    w = torch.randn(256, 1, generator=torch.Generator().manual_seed(3))
    qa, ka, va = (t.to(dev).requires_grad_(True) for t in (q, k, v))
    tid = torch.as_tensor(np.asarray(ids), dtype=torch.int32, device=dev)
    out, lse = gqa.attention(qa, ka, va, seg_q=tid, seg_kv=tid, return_lse=True)
    assert not lse.requires_grad
    loss = (out.transpose(1, 2) @ w.to(dev)).square().sum()
    loss.backward()
    # the loss's dout, formed on the CPU in fp64 from the kernel's out
    o64 = out.detach().double().cpu()
    dout = (2 * (o64.transpose(1, 2) @ w.double()) @ w.double().T).transpose(1, 2)
    ref = oracle.attention_backward(q, k, v, dout.float(), seg_q=ids, seg_kv=ids)
    for got, want, name in zip((qa.grad, ka.grad, va.grad), ref, ("dq", "dk", "dv")):
        err = float(np.max(np.abs(got.double().cpu().numpy() - want))) / max(1.0, float(np.max(np.abs(want))))
        assert err <= 5e-5, (name, err)
