"""Failure detection without a GPU fault.

Host side: bad arguments come back as status codes (tests/test_abi.py).  Device
side: every mbarrier wait is bounded; the self-test kernel waits on a barrier that
nothing completes, must give up after its budget, record GQA_ERR_DEVICE_TIMEOUT and
leave the context usable for the next call.
"""

import time

import pytest
import torch

import long_context_causal_flash_b200 as gqa
from long_context_causal_flash_b200 import _lib, inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    t0 = time.time()
    st = gqa.selftest_wait(budget_ns=50_000_000)  # 50 ms
    assert st == _lib.GQA_ERR_DEVICE_TIMEOUT
    assert time.time() - t0 < 30
    # the context still works: a normal call succeeds and reports OK
    q, k, v = (t.to(cuda_device) for t in inputs.qkv(1, 16, 4, 64, 64, 256))
    ws = torch.empty(256, dtype=torch.uint8, device=cuda_device)
    out, lse = gqa.fwd(q, k, v, workspace=ws)
    assert gqa.status(ws) == _lib.GQA_OK
    assert torch.isfinite(out).all()


def test_status_word_is_reset_by_each_call(cuda_device):
    ws = torch.empty(256, dtype=torch.uint8, device=cuda_device)
    ws.view(torch.int32)[0] = _lib.GQA_ERR_DEVICE_TIMEOUT
    q, k, v = (t.to(cuda_device) for t in inputs.qkv(1, 16, 4, 10, 10, 256))
    gqa.fwd(q, k, v, workspace=ws)
    assert gqa.status(ws) == _lib.GQA_OK


def test_binding_raises_on_a_rejected_call(cuda_device):
    q = torch.zeros(1, 16, 8, 128, device=cuda_device)  # d = 128 is not supported
    with pytest.raises(gqa.GqaAttnError) as e:
        gqa.fwd(q, q[:, :4].contiguous(), q[:, :4].contiguous())
    assert e.value.status == _lib.GQA_ERR_UNSUPPORTED
