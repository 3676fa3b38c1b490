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


_SKIP_FILL_SCRIPT = r"""
import json, os, sys
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import long_context_causal_flash_b200 as gqa
import oracle
from long_context_causal_flash_b200 import inputs

dev = torch.device("cuda")
L = 512
res = {}


def diff(a, b):
    return float(np.max(np.abs(a.double().cpu().numpy() - b)))


for name, dtype, path in (("fwd_f32_kernel", torch.float32, "ffma"), ("fwd_bf16_kernel", torch.bfloat16, "ffma"),
                          ("fwd_f32_tc_kernel", torch.float32, "tc")):
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    code = gqa.GQA_F32_TC if path == "tc" else dtype
    ws = torch.empty(max(256, gqa.workspace_bytes(1, 16, 4, L, L, 256, code)), dtype=torch.uint8, device=dev)
    os.environ["GQA_ATTN_TEST_SKIP_FILL"] = "1"
    gqa.fwd(q, k, v, workspace=ws, fp32_path=path)
    faulted = gqa.status(ws)
    del os.environ["GQA_ATTN_TEST_SKIP_FILL"]
    out, lse = gqa.fwd(q, k, v, workspace=ws, fp32_path=path)
    after = gqa.status(ws)
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu())
    res[name] = [faulted, after, diff(out, ref_out), diff(lse, ref_lse)]

q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=torch.bfloat16))
dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
out, lse = gqa.fwd(q, k, v)
bws = torch.empty(max(256, gqa.bwd_workspace_bytes(1, 16, 4, L, L, 256, torch.bfloat16)), dtype=torch.uint8,
                  device=dev)
os.environ["GQA_ATTN_TEST_SKIP_FILL"] = "1"
gqa.bwd(q, k, v, out, lse, dout.to(dev), workspace=bws)
faulted = gqa.status(bws)
del os.environ["GQA_ATTN_TEST_SKIP_FILL"]
grads = gqa.bwd(q, k, v, out, lse, dout.to(dev), workspace=bws)
after = gqa.status(bws)
ref = oracle.attention_backward(q.cpu(), k.cpu(), v.cpu(), dout)
rel = max(diff(g, r) / max(1.0, float(np.max(np.abs(r)))) for g, r in zip(grads, ref))
res["bwd_tc_kernel"] = [faulted, after, rel, 0.0]

q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=torch.float32))
dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7))
out, lse = gqa.fwd(q, k, v)
bws = torch.empty(max(256, gqa.bwd_workspace_bytes(1, 16, 4, L, L, 256, torch.float32)), dtype=torch.uint8,
                  device=dev)
os.environ["GQA_ATTN_TEST_SKIP_FILL"] = "1"
gqa.bwd(q, k, v, out, lse, dout.to(dev), workspace=bws)
faulted = gqa.status(bws)
del os.environ["GQA_ATTN_TEST_SKIP_FILL"]
grads = gqa.bwd(q, k, v, out, lse, dout.to(dev), workspace=bws)
after = gqa.status(bws)
ref = oracle.attention_backward(q.cpu(), k.cpu(), v.cpu(), dout)
rel = max(diff(g, r) / max(1.0, float(np.max(np.abs(r)))) for g, r in zip(grads, ref))
res["bwd_dq_kernel + bwd_dkv_kernel"] = [faulted, after, rel, 0.0]
print("RESULT " + json.dumps(res))
"""


def test_attention_kernels_take_their_timeout_exit(cuda_device):
    """A producer that skips one fill (test hook GQA_ATTN_TEST_SKIP_FILL) leaves the
    waits on that fill without an arrival: every attention kernel fed through mbarriers
    must give up after its budget (50 ms here), report GQA_ERR_DEVICE_TIMEOUT through
    its workspace, release its tensor memory and CTA pair partner (where it has them),
    and leave the
    context usable: the next call, without the hook, reports GQA_OK and matches the
    oracle.  Runs in a child process (the budget is read once per process)."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, GQA_ATTN_WAIT_BUDGET_NS="50000000")
    env.pop("GQA_ATTN_TEST_SKIP_FILL", None)
    r = subprocess.run([sys.executable, "-c", _SKIP_FILL_SCRIPT, root], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    tol = {"fwd_f32_kernel": (2e-5, 1e-5), "fwd_bf16_kernel": (2e-2, 2e-3), "fwd_f32_tc_kernel": (2e-5, 1e-5),
           "bwd_tc_kernel": (2e-2, 1.0), "bwd_dq_kernel + bwd_dkv_kernel": (5e-5, 1.0)}
    for name, (faulted, after, d_out, d_lse) in res.items():
        assert faulted == _lib.GQA_ERR_DEVICE_TIMEOUT, (name, faulted)
        assert after == _lib.GQA_OK, (name, after)
        assert d_out <= tol[name][0] and d_lse <= tol[name][1], (name, d_out, d_lse)
