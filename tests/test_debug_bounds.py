"""The bounds-checked build (``build --debug-bounds``, loaded with GQA_ATTN_DEBUG_BOUNDS=1).

In that build the fp32 FFMA kernels (the forward, dQ and dK/dV) check every shared-memory
access against the region it belongs to (Q^T, a ring slot, a warp's P or weight slice)
and every output row index against its buffer; a failed check skips the access and the
kernel reports GQA_ERR_DEVICE_BOUNDS in the status word.  The CPU tests check that the
checked library builds and exports the same C ABI and that a normal build has no checks;
the GPU tests run the checks' self-test (the comparisons alone, on planted out-of-range
values, with no access made) and run the checked library, in a child process, over the
fp32 parity cases (every mask, several tiles with ragged ends, group
sizes 1, 4 and 16, key splits, the backward): each call must report GQA_OK and match the
oracle.
"""

import ctypes
import json
import os
import subprocess
import sys

import pytest

from long_context_causal_flash_b200 import _lib
from long_context_causal_flash_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_exports_the_same_abi():
    path = build(debug_bounds=True)
    assert path.endswith("libgqa_attn_debug_bounds.so")
    lib = ctypes.CDLL(path)
    for name in _lib.SIGNATURES:
        assert hasattr(lib, name), name
    lib.gqa_attn_strerror.restype = ctypes.c_char_p
    assert b"index check" in lib.gqa_attn_strerror(_lib.GQA_ERR_DEVICE_BOUNDS)
    # argument checks come before any CUDA call
    buf = ctypes.create_string_buffer(512)
    ws = (ctypes.addressof(buf) + 15) & ~15
    assert lib.gqa_attn_selftest_bounds(ctypes.c_void_p(ws), ctypes.c_size_t(256), 2, None) == \
        _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_selftest_bounds(ctypes.c_void_p(ws), ctypes.c_size_t(16), 1, None) == _lib.GQA_ERR_WORKSPACE


def test_normal_build_has_no_index_checks():
    """The self-test answers GQA_ERR_UNSUPPORTED, launching nothing, in a normal build."""
    build()
    lib = _lib.load()
    assert _lib.LIB_PATH.endswith("libgqa_attn.so")
    buf = ctypes.create_string_buffer(512)
    ws = (ctypes.addressof(buf) + 15) & ~15
    for planted in (0, 1):
        assert lib.gqa_attn_selftest_bounds(ws, 256, planted, None) == _lib.GQA_ERR_UNSUPPORTED


_CHECKED_SCRIPT = r"""
import json, sys
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import long_context_causal_flash_b200 as gqa
from long_context_causal_flash_b200 import _lib, inputs
import oracle

assert _lib.LIB_PATH.endswith("libgqa_attn_debug_bounds.so"), _lib.LIB_PATH
dev = torch.device("cuda")
res = []


def ids(x):
    return None if x is None else torch.as_tensor(np.asarray(x), dtype=torch.int32, device=dev)


def mk(kind):
    return oracle.MASK_CAUSAL if kind == "causal" else oracle.MASK_PREFIX_BRANCH


def fwd_case(name, Hq, Hkv, Lq, Lk, kind="causal", off=0, seg_q=None, seg_kv=None, splits=1):
    q, k, v = inputs.qkv(1, Hq, Hkv, Lq, Lk, 256)
    has_seg = seg_q is not None
    need = (gqa.workspace_bytes(1, Hq, Hkv, Lq, Lk, 256, torch.float32, kind, has_seg) if splits == 1 else
            gqa.split_workspace_bytes(1, Hq, Hkv, Lq, Lk, splits, 256, torch.float32, kind, has_seg))
    ws = torch.empty(max(256, need), dtype=torch.uint8, device=dev)
    out, lse = gqa.fwd(q.to(dev), k.to(dev), v.to(dev), mask_kind=kind, q_pos_offset=off, seg_q=ids(seg_q),
                       seg_kv=ids(seg_kv), workspace=ws, splits=splits)
    st = gqa.status(ws)
    ro, rl = oracle.attention(q, k, v, mask_kind=mk(kind), q_pos_offset=off, seg_q=seg_q, seg_kv=seg_kv)
    d_out = float(np.max(np.abs(out.double().cpu().numpy() - ro)))
    fin = np.isfinite(rl)
    lc = lse.double().cpu().numpy()
    d_lse = float(np.max(np.abs(lc[fin] - rl[fin]))) if fin.any() else 0.0
    same_inf = bool(np.array_equal(np.isfinite(lc), fin))
    res.append(["fwd " + name, st, d_out, d_lse if same_inf else float("inf")])


def bwd_case(name, Hq, Hkv, Lq, Lk, kind="causal", off=0, seg_q=None, seg_kv=None):
    q, k, v = inputs.qkv(1, Hq, Hkv, Lq, Lk, 256)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(7))
    kw = dict(mask_kind=kind, q_pos_offset=off, seg_q=ids(seg_q), seg_kv=ids(seg_kv))
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out, lse = gqa.fwd(qd, kd, vd, **kw)
    ws = torch.empty(max(256, gqa.bwd_workspace_bytes(1, Hq, Hkv, Lq, Lk, 256, torch.float32, kind,
                                                      seg_q is not None)), dtype=torch.uint8, device=dev)
    grads = gqa.bwd(qd, kd, vd, out, lse, do.to(dev), workspace=ws, **kw)
    st = gqa.status(ws)
    ref = oracle.attention_backward(q, k, v, do, mask_kind=mk(kind), q_pos_offset=off, seg_q=seg_q, seg_kv=seg_kv)
    rel = max(float(np.max(np.abs(g.double().cpu().numpy() - r))) / max(1.0, float(np.max(np.abs(r))))
              for g, r in zip(grads, ref))
    res.append(["bwd " + name, st, rel, 0.0])


S, nb, bl = 300, 3, 40
bq, bkv = inputs.branch_ids(S, nb, bl)
seg = inputs.segment_ids([1, 70, 5, 200, 64, 33])
for L in (1, 2, 65, 257):
    fwd_case(f"causal L={L}", 16, 4, L, L)
fwd_case("causal G=4 L=700", 16, 4, 700, 700)
fwd_case("causal G=16 L=300", 16, 1, 300, 300)
fwd_case("causal G=1 L=500", 16, 16, 500, 500)
fwd_case("rows after a state", 16, 4, 100, 300, off=200)
fwd_case("prefix branch", 16, 4, nb * bl, S + nb * bl, kind="prefix_branch", off=S, seg_q=bq, seg_kv=bkv)
fwd_case("segments", 16, 4, len(seg), len(seg), seg_q=seg, seg_kv=seg)
fwd_case("key splits", 16, 4, 700, 700, splits=3)
for L in (1, 33, 129):
    bwd_case(f"causal L={L}", 16, 4, L, L)
bwd_case("causal G=4 L=500", 16, 4, 500, 500)
bwd_case("causal G=16 L=300", 16, 1, 300, 300)
bwd_case("causal G=1 L=300", 16, 16, 300, 300)
bwd_case("rows after a state", 16, 4, 100, 250, off=150)
bwd_case("prefix branch", 16, 4, nb * bl, S + nb * bl, kind="prefix_branch", off=S, seg_q=bq, seg_kv=bkv)
bwd_case("segments", 16, 4, len(seg), len(seg), seg_q=seg, seg_kv=seg)
for Lq, Lk, off in ((130, 70, 500), (200, 300, 57)):  # key blocks of a sharded sequence
    q, k, v = inputs.qkv(1, 16, 4, Lq, Lk, 256)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    out, lse = gqa.fwd_offset(q.to(dev), k.to(dev), v.to(dev), q_pos_offset=off, workspace=ws)
    st = gqa.status(ws)
    ro, rl = oracle.attention_block(q, k, v, q_pos_offset=off)
    res.append([f"fwd_offset {Lq}/{Lk}/{off}", st, float(np.max(np.abs(out.double().cpu().numpy() - ro))),
                float(np.max(np.abs(lse.double().cpu().numpy() - rl)))])
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(7))
    bws = torch.empty(max(256, gqa.bwd_workspace_bytes(1, 16, 4, Lq, Lq, 256, torch.float32)), dtype=torch.uint8,
                      device=dev)
    grads = gqa.bwd_offset(q.to(dev), k.to(dev), v.to(dev), out, lse, do.to(dev), q_pos_offset=off, workspace=bws)
    st = gqa.status(bws)
    ref = oracle.attention_block_backward(q, k, v, out.double().cpu(), lse.double().cpu(), do, q_pos_offset=off)
    rel = max(float(np.max(np.abs(g.double().cpu().numpy() - r))) / max(1.0, float(np.max(np.abs(r))))
              for g, r in zip(grads, ref))
    res.append([f"bwd_offset {Lq}/{Lk}/{off}", st, rel, 0.0])
print("RESULT " + json.dumps(res))
"""


_SELFTEST_SCRIPT = r"""
import sys
sys.path.insert(0, sys.argv[1])
import long_context_causal_flash_b200 as gqa
print("RESULT", gqa.selftest_bounds(planted=False), gqa.selftest_bounds(planted=True),
      gqa.selftest_bounds(planted=False))
"""


@pytest.mark.gpu
def test_checked_build_reports_a_failed_check(cuda_device):
    """Only the comparisons of the checks run (no access at the planted address): the
    flag stays clear for in-range indices, is set by the planted out-of-range ones, and
    the next call starts clear again."""
    build(debug_bounds=True)
    env = dict(os.environ, GQA_ATTN_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, "-c", _SELFTEST_SCRIPT, ROOT], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1].split()
    assert [int(x) for x in line[1:]] == [_lib.GQA_OK, _lib.GQA_ERR_DEVICE_BOUNDS, _lib.GQA_OK]


@pytest.mark.gpu
def test_checked_build_passes_the_fp32_parity_cases(cuda_device):
    build(debug_bounds=True)
    env = dict(os.environ, GQA_ATTN_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, "-c", _CHECKED_SCRIPT, ROOT], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert len(res) == 24
    for name, st, d_out, d_lse in res:
        assert st == _lib.GQA_OK, (name, st)
        tol_out = 5e-5 if name.startswith("bwd") else 2e-5
        assert d_out <= tol_out and d_lse <= 1e-5, (name, d_out, d_lse)
