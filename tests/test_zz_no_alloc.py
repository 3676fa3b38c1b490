"""gqa_attn_fwd_static_ws: the forward for callers that cannot allocate device memory.

Such callers (a plug-in inside a framework that owns all device memory, a service
under a fixed post-start-up memory budget, a path that must avoid an allocation's
device synchronisation) provide inputs and outputs but no workspace; the library
then uses its own fixed device scratch.  These tests call the entry point through
the C ABI, twice in a row after one warm-up call, check that device memory in use
does not change around each call, and compare the results with gqa_attn_fwd on the
same inputs bit for bit (both run the same kernels on the same data).
The file is named to be collected last, so a run that stops at its first failure
has run every other test before it.
"""

import ctypes

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
from long_context_causal_flash_b200 import _lib, inputs

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 2 << 20  # GQA_ATTN_STATIC_WORKSPACE_BYTES in include/gqa_attn.h


def _static_ws_fwd(q, k, v, *, out, lse, mask_kind=0, q_pos_offset=0, seg_q=None, seg_kv=None):
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    dt = gqa._dtype_code(q.dtype)
    return _lib.load().gqa_attn_fwd_static_ws(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq, Lk, d, dt,
        mask_kind, q_pos_offset, None if seg_q is None else seg_q.data_ptr(),
        None if seg_kv is None else seg_kv.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same(a_out, a_lse, b_out, b_lse):
    """Same kernels on the same inputs: the results must be identical, bit for bit."""
    assert torch.equal(a_out, b_out) and torch.equal(a_lse, b_lse)


def _outputs(q):
    return torch.empty_like(q), torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)


def _warm_up(call, q):
    """One unmeasured call: the first call on a device looks up the scratch's address,
    which may make the driver load the library's device code (and the scratch) then."""
    out, lse = _outputs(q)
    assert call(out, lse) == _lib.GQA_OK
    torch.cuda.synchronize()


def _no_device_allocation(call):
    """Runs `call` and checks that device memory in use did not change around it, both
    as the driver sees it (cudaMemGetInfo) and as torch's allocator does."""
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    res = call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device memory changed by {free0 - free1} bytes during the call"
    assert torch.cuda.memory_allocated() == alloc0
    return res


@pytest.mark.parametrize("dtype,L,segmented", [(torch.bfloat16, 1000, False), (torch.float32, 777, False),
                                                (torch.float32, 3000, True), (torch.bfloat16, 5000, True)])
def test_matches_the_workspace_entry_point_on_two_calls(cuda_device, dtype, L, segmented):
    q, k, v = (t.to(cuda_device) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    ids = None
    if segmented:
        lengths = inputs.segment_lengths(L, lo=100, hi=900)
        ids = torch.as_tensor(inputs.segment_ids(lengths), device=cuda_device)
    ref_out, ref_lse = gqa.fwd(q, k, v, seg_q=ids, seg_kv=ids)
    _warm_up(lambda out, lse: _static_ws_fwd(q, k, v, seg_q=ids, seg_kv=ids, out=out, lse=lse), q)
    outs = [_outputs(q) for _ in range(2)]  # allocated before the measured calls
    for out, lse in outs:  # the second call finds the scratch holding the first call's tables
        rc = _no_device_allocation(lambda: _static_ws_fwd(q, k, v, seg_q=ids, seg_kv=ids, out=out, lse=lse))
        assert rc == _lib.GQA_OK, _lib.strerror(rc)
        _same(out, lse, ref_out, ref_lse)


def test_prefix_branch_through_the_static_scratch(cuda_device):
    S, nb, bl = 700, 3, 64
    q, k, v = (t.to(cuda_device) for t in inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256))
    sq, skv = (torch.as_tensor(x, device=cuda_device) for x in inputs.branch_ids(S, nb, bl))
    ref_out, ref_lse = gqa.fwd(q, k, v, mask_kind="prefix_branch", q_pos_offset=S, seg_q=sq, seg_kv=skv)
    call = lambda out, lse: _static_ws_fwd(q, k, v, mask_kind=1, q_pos_offset=S, seg_q=sq, seg_kv=skv, out=out,
                                           lse=lse)
    _warm_up(call, q)
    outs = [_outputs(q) for _ in range(2)]
    for out, lse in outs:
        rc = _no_device_allocation(lambda: call(out, lse))
        assert rc == _lib.GQA_OK, _lib.strerror(rc)
        _same(out, lse, ref_out, ref_lse)


def test_rejects_calls_beyond_the_fixed_scratch(cuda_device):
    lib = _lib.load()
    L = 1 << 22  # fp32 with segment ids at 4M tokens needs more than the 2 MiB scratch
    need = lib.gqa_attn_workspace_bytes(1, 16, 4, L, L, 256, 0, 0, 1)
    assert need > STATIC_WS_BYTES
    # rejected on the host before any pointer is used (the values below are never read)
    rc = lib.gqa_attn_fwd_static_ws(16, 16, 16, 16, 16, 1, 16, 4, L, L, 256, 0, 0, 0, 16, 16, None)
    assert rc == _lib.GQA_ERR_WORKSPACE
    # invalid shapes report the same error as gqa_attn_fwd
    rc = lib.gqa_attn_fwd_static_ws(16, 16, 16, 16, 16, 1, 16, 4, 64, 64, 128, 0, 0, 0, None, None, None)
    assert rc == _lib.GQA_ERR_UNSUPPORTED
    assert np.isfinite(need)
