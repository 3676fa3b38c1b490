"""gqa_attn_fwd_static_ws: the forward for callers that cannot allocate device memory.

Such callers (a plug-in inside a framework that owns all device memory, a service
under a fixed post-start-up memory budget, a path that must avoid an allocation's
device synchronisation) provide inputs and outputs but no workspace; the library
then uses its own fixed device scratch.  These tests call the entry point through
the C ABI, twice in a row, and compare it with gqa_attn_fwd on the same inputs.
The file is named to be collected last, so a run that stops at its first failure
has run every other test before it.
"""

import ctypes

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
from long_context_causal_flash_b200 import _lib, inputs
from tests._helpers import TOL

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 2 << 20  # GQA_ATTN_STATIC_WORKSPACE_BYTES in include/gqa_attn.h


def _static_ws_fwd(q, k, v, *, mask_kind=0, q_pos_offset=0, seg_q=None, seg_kv=None):
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    dt = gqa._dtype_code(q.dtype)
    rc = _lib.load().gqa_attn_fwd_static_ws(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq, Lk, d, dt,
        mask_kind, q_pos_offset, None if seg_q is None else seg_q.data_ptr(),
        None if seg_kv is None else seg_kv.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, out, lse


def _close(a_out, a_lse, b_out, b_lse, dtype):
    tol_out, tol_lse = TOL[dtype]
    assert torch.equal(torch.isneginf(a_lse), torch.isneginf(b_lse))
    fin = torch.isfinite(b_lse)
    assert float((a_out.double() - b_out.double()).abs().max()) <= tol_out
    assert float((a_lse[fin].double() - b_lse[fin].double()).abs().max()) <= tol_lse


@pytest.mark.parametrize("dtype,L,segmented", [(torch.bfloat16, 1000, False), (torch.float32, 777, False),
                                                (torch.float32, 3000, True), (torch.bfloat16, 5000, True)])
def test_matches_the_workspace_entry_point_on_two_calls(cuda_device, dtype, L, segmented):
    q, k, v = (t.to(cuda_device) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    ids = None
    if segmented:
        lengths = inputs.segment_lengths(L, lo=100, hi=900)
        ids = torch.as_tensor(inputs.segment_ids(lengths), device=cuda_device)
    ref_out, ref_lse = gqa.fwd(q, k, v, seg_q=ids, seg_kv=ids)
    for _ in range(2):  # the second call finds the scratch holding the first call's tables
        rc, out, lse = _static_ws_fwd(q, k, v, seg_q=ids, seg_kv=ids)
        torch.cuda.synchronize()
        assert rc == _lib.GQA_OK, _lib.strerror(rc)
        _close(out, lse, ref_out, ref_lse, dtype)


def test_prefix_branch_through_the_static_scratch(cuda_device):
    S, nb, bl = 700, 3, 64
    q, k, v = (t.to(cuda_device) for t in inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256))
    sq, skv = (torch.as_tensor(x, device=cuda_device) for x in inputs.branch_ids(S, nb, bl))
    ref_out, ref_lse = gqa.fwd(q, k, v, mask_kind="prefix_branch", q_pos_offset=S, seg_q=sq, seg_kv=skv)
    for _ in range(2):
        rc, out, lse = _static_ws_fwd(q, k, v, mask_kind=1, q_pos_offset=S, seg_q=sq, seg_kv=skv)
        torch.cuda.synchronize()
        assert rc == _lib.GQA_OK
        _close(out, lse, ref_out, ref_lse, torch.float32)


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
