"""Exact causal grouped-query attention for B200 (sm_100a) behind a C ABI.

Python binding of libgqa_attn.so (include/gqa_attn.h).  This module only
marshals arguments: every step of the attention runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.

    out, lse = fwd(q, k, v)                                  # causal self-attention
    out, lse = fwd(q, k, v, q_pos_offset=S)                  # one branch after a state
    out, lse = fwd(q, k, v, mask_kind="prefix_branch",
                   q_pos_offset=S, seg_q=ids_q, seg_kv=ids_kv)   # packed branches
    out, lse = fwd(q, k, v, seg_q=ids, seg_kv=ids)           # block-causal packing
    out, lse = fwd(q, k, v, q_pos_offset=S, splits="auto")   # split-KV for short query blocks
    out, lse = fwd(q, k, v, fp32_path="tc")                  # fp32 on the tensor cores (split operands)
    dq, dk, dv = bwd(q, k, v, out, lse, dout)                # gradients from the saved LSE
    out = attention(q, k, v)                                 # differentiable (autograd: fwd + bwd)

q: [B, Hq, Lq, 256], k/v: [B, Hkv, Lk, 256], fp32 or bf16, contiguous CUDA
tensors; Lk = q_pos_offset + Lq.  Returns out (dtype of q) and lse (fp32).
"""

from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (GQA_BF16, GQA_F32, GQA_F32_TC, GQA_MASK_CAUSAL, GQA_MASK_PREFIX_BRANCH,  # noqa: F401
                   GqaAttnError)

__all__ = ["fwd", "fwd_offset", "merge", "bwd", "bwd_offset", "attention", "bwd_workspace_bytes", "fwd_host", "workspace_bytes", "split_hint", "split_workspace_bytes", "tile_sizes",
           "tile_plan", "status", "selftest_wait", "selftest_bounds", "GqaAttnError", "GQA_F32", "GQA_BF16", "GQA_F32_TC"]

_MASKS = {"causal": GQA_MASK_CAUSAL, "prefix_branch": GQA_MASK_PREFIX_BRANCH,
          GQA_MASK_CAUSAL: GQA_MASK_CAUSAL, GQA_MASK_PREFIX_BRANCH: GQA_MASK_PREFIX_BRANCH}
_DTYPES = {torch.float32: GQA_F32, torch.bfloat16: GQA_BF16}


def _mask(mask_kind) -> int:
    try:
        return _MASKS[mask_kind]
    except KeyError:
        raise ValueError(f"mask_kind must be 'causal' or 'prefix_branch', got {mask_kind!r}") from None


def _dtype_code(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    try:
        return _DTYPES[dtype]
    except KeyError:
        raise ValueError(f"dtype must be torch.float32 or torch.bfloat16, got {dtype}") from None


_FP32_PATHS = ("ffma", "tc")


def _call_dtype(dtype, fp32_path) -> int:
    """Library dtype code of a call on tensors of ``dtype``: fp32 tensors run on the
    FFMA kernel (``fp32_path="ffma"``) or on the tensor cores with split operands
    (``"tc"``, GQA_F32_TC)."""
    if fp32_path not in _FP32_PATHS:
        raise ValueError(f"fp32_path must be one of {_FP32_PATHS}, got {fp32_path!r}")
    dt = _dtype_code(dtype)
    if fp32_path == "tc":
        if dt != GQA_F32:
            raise ValueError("fp32_path='tc' applies to fp32 tensors")
        return GQA_F32_TC
    return dt


def _stream_ptr(stream, device) -> ctypes.c_void_p:
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_bytes(B, Hq, Hkv, Lq, Lk, d=256, dtype=torch.float32, mask_kind="causal",
                    has_segments=False) -> int:
    """Device workspace bytes for one call (0 if the shape is rejected)."""
    return int(_lib.load().gqa_attn_workspace_bytes(B, Hq, Hkv, Lq, Lk, d, _dtype_code(dtype),
                                                    _mask(mask_kind), int(bool(has_segments))))


def split_hint(B, Hq, Hkv, Lq, Lk, dtype=torch.float32, mask_kind="causal", has_segments=False) -> int:
    """Key-split count the library suggests for this shape on a B200 (1 = no split)."""
    n = int(_lib.load().gqa_attn_split_hint(B, Hq, Hkv, Lq, Lk, _dtype_code(dtype), _mask(mask_kind),
                                            int(bool(has_segments))))
    _lib.check("gqa_attn_split_hint", min(n, 0))
    return n


def split_workspace_bytes(B, Hq, Hkv, Lq, Lk, splits, d=256, dtype=torch.float32, mask_kind="causal",
                          has_segments=False) -> int:
    """Device workspace bytes for a split-KV call (0 if rejected)."""
    return int(_lib.load().gqa_attn_split_workspace_bytes(B, Hq, Hkv, Lq, Lk, d, _dtype_code(dtype),
                                                          _mask(mask_kind), int(bool(has_segments)),
                                                          int(splits)))


def tile_sizes(dtype=torch.float32, Hq=16, Hkv=4):
    """(query positions per tile, keys per tile) used by the kernel for this dtype and group."""
    br, bc = ctypes.c_int(), ctypes.c_int()
    _lib.check("gqa_attn_tile_sizes",
               _lib.load().gqa_attn_tile_sizes(_dtype_code(dtype), Hq, Hkv, ctypes.byref(br), ctypes.byref(bc)))
    return br.value, bc.value


def _device(device) -> torch.device:
    dev = torch.device(device)
    if dev.type == "cuda" and dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    return dev


def _check_ids(ids, n, device, name):
    if ids is None:
        return None
    if not isinstance(ids, torch.Tensor):
        ids = torch.as_tensor(ids)
    if ids.dtype != torch.int32 or ids.device != device or not ids.is_contiguous() or ids.shape != (n,):
        raise ValueError(f"{name} must be a contiguous int32 tensor of shape ({n},) on {device}")
    return ids


def fwd(q, k, v, *, mask_kind="causal", q_pos_offset=0, seg_q=None, seg_kv=None, out=None, lse=None,
        workspace=None, stream=None, splits=1, fp32_path="ffma"):
    """Attention forward on the GPU; returns ``(out, lse)``.  Asynchronous on ``stream``
    (default: the current stream).  ``out``/``lse``/``workspace`` may be preallocated.
    ``splits`` > 1 (or ``"auto"``: the library's hint) runs the split-KV form.
    ``fp32_path="tc"`` runs fp32 tensors on the tensor cores (GQA_F32_TC: split fp16
    operands, a workspace of about the inputs' size)."""
    if not (isinstance(q, torch.Tensor) and q.is_cuda):
        raise ValueError("fwd takes CUDA tensors; use fwd_host for host tensors")
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.device != dev or t.dim() != 4 or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError(f"{name} must be a contiguous 4-d tensor on {dev} with q's dtype")
    dt = _call_dtype(q.dtype, fp32_path)
    B, Hq, Lq, d = q.shape
    Bk, Hkv, Lk, dk = k.shape
    if v.shape != k.shape or Bk != B or dk != d:
        raise ValueError("k and v must be [B, Hkv, Lk, d] with q's B and d")
    seg_q = _check_ids(seg_q, Lq, dev, "seg_q")
    seg_kv = _check_ids(seg_kv, Lk, dev, "seg_kv")
    m = _mask(mask_kind)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), device=dev, dtype=torch.float32)
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or out.device != dev:
        raise ValueError("out must match q")
    if lse.shape != (B, Hq, Lq) or lse.dtype != torch.float32 or not lse.is_contiguous() or lse.device != dev:
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Lq] tensor on q's device")
    lib = _lib.load()
    has_seg = int(seg_q is not None)
    if splits == "auto":
        splits = split_hint(B, Hq, Hkv, Lq, Lk, dt, m, has_seg)
    splits = int(splits)
    if splits == 1:
        need = int(lib.gqa_attn_workspace_bytes(B, Hq, Hkv, Lq, Lk, d, dt, m, has_seg))
    else:
        need = int(lib.gqa_attn_split_workspace_bytes(B, Hq, Hkv, Lq, Lk, d, dt, m, has_seg, splits))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    sq = None if seg_q is None else seg_q.data_ptr()
    skv = None if seg_kv is None else seg_kv.data_ptr()
    with torch.cuda.device(dev):
        if splits == 1:
            rc = lib.gqa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  B, Hq, Hkv, Lq, Lk, d, dt, m, int(q_pos_offset), sq, skv,
                                  workspace.data_ptr(), workspace.numel(), _stream_ptr(stream, dev))
        else:
            rc = lib.gqa_attn_fwd_split(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                        B, Hq, Hkv, Lq, Lk, d, dt, m, int(q_pos_offset), sq, skv, splits,
                                        workspace.data_ptr(), workspace.numel(), _stream_ptr(stream, dev))
    _lib.check("gqa_attn_fwd" if splits == 1 else "gqa_attn_fwd_split", rc)
    return out, lse


def fwd_offset(q, k, v, *, q_pos_offset, out=None, lse=None, workspace=None, stream=None):
    """Causal attention of ``q`` against a key block that starts ``q_pos_offset`` >= 0
    positions before query row 0 (any key count): ``gqa_attn_fwd_offset``.  Returns
    ``(out, lse)``; asynchronous on ``stream``."""
    if not (isinstance(q, torch.Tensor) and q.is_cuda):
        raise ValueError("fwd_offset takes CUDA tensors")
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.device != dev or t.dim() != 4 or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError(f"{name} must be a contiguous 4-d tensor on {dev} with q's dtype")
    dt = _dtype_code(q.dtype)
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if v.shape != k.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, Hkv, Lk, d] with q's B and d")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Lq), device=dev, dtype=torch.float32) if lse is None else lse
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or out.device != dev:
        raise ValueError("out must match q")
    if lse.shape != (B, Hq, Lq) or lse.dtype != torch.float32 or not lse.is_contiguous() or lse.device != dev:
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Lq] tensor on q's device")
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=dev)
    lib = _lib.load()
    with torch.cuda.device(dev):
        rc = lib.gqa_attn_fwd_offset(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                     B, Hq, Hkv, Lq, Lk, d, dt, int(q_pos_offset), workspace.data_ptr(),
                                     workspace.numel(), _stream_ptr(stream, dev))
    _lib.check("gqa_attn_fwd_offset", rc)
    return out, lse


def merge(o_a, lse_a, o_b, lse_b, *, out=None, lse_out=None, out_dtype=torch.float32, stream=None):
    """Exact merge of two partial results by their log-sum-exps (``gqa_attn_merge``).
    ``o_a`` (fp32) / ``o_b`` (fp32 or bf16) are ``[..., d]`` with LSEs ``[...]``; either
    pair may be ``None`` (empty).  ``out`` may be ``o_a`` (in place, fp32).  Returns
    ``(out, lse_out)``."""
    if (o_a is None) != (lse_a is None) or (o_b is None) != (lse_b is None):
        raise ValueError("each partial is an (o, lse) pair or (None, None)")
    ref_o = o_a if o_a is not None else o_b
    ref_l = lse_a if lse_a is not None else lse_b
    if ref_o is None:
        raise ValueError("merge needs at least one partial result")
    dev = ref_o.device
    rows = ref_l.numel()
    d = ref_o.shape[-1]
    for t in (o_a, lse_a, o_b, lse_b):
        if t is not None and (t.device != dev or not t.is_contiguous()):
            raise ValueError("partials must be contiguous tensors on one device")
    if o_a is not None and (o_a.dtype != torch.float32 or o_a.numel() != rows * d):
        raise ValueError("o_a must be fp32 with lse_a's rows")
    if o_b is not None and o_b.numel() != rows * d:
        raise ValueError("o_b must have lse_b's rows")
    out = torch.empty(ref_o.shape, dtype=out_dtype, device=dev) if out is None else out
    lse_out = torch.empty(ref_l.shape, dtype=torch.float32, device=dev) if lse_out is None else lse_out

    def ptr(t):
        return None if t is None else t.data_ptr()

    lib = _lib.load()
    with torch.cuda.device(dev):
        rc = lib.gqa_attn_merge(ptr(o_a), ptr(lse_a), ptr(o_b), ptr(lse_b), out.data_ptr(), lse_out.data_ptr(),
                                rows, d, _dtype_code(o_b.dtype if o_b is not None else torch.float32),
                                _dtype_code(out.dtype), _stream_ptr(stream, dev))
    _lib.check("gqa_attn_merge", rc)
    return out, lse_out


def bwd_workspace_bytes(B, Hq, Hkv, Lq, Lk, d=256, dtype=torch.float32, mask_kind="causal",
                        has_segments=False) -> int:
    """Device workspace bytes for one backward call (0 if the shape is rejected)."""
    return int(_lib.load().gqa_attn_bwd_workspace_bytes(B, Hq, Hkv, Lq, Lk, d, _dtype_code(dtype),
                                                        _mask(mask_kind), int(bool(has_segments))))


def bwd(q, k, v, out, lse, dout, *, mask_kind="causal", q_pos_offset=0, seg_q=None, seg_kv=None, dq=None,
        dk=None, dv=None, workspace=None, stream=None):
    """Gradients ``(dq, dk, dv)`` of ``sum(out * dout)`` from the forward's ``out`` and
    ``lse``; asynchronous on ``stream``.  Outputs may be preallocated."""
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if not (isinstance(t, torch.Tensor) and t.device == dev and t.is_contiguous() and t.dtype == q.dtype):
            raise ValueError(f"{name} must be a contiguous tensor on {dev} with q's dtype")
    if out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("out and dout must have q's shape")
    dt = _dtype_code(q.dtype)
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if lse.shape != (B, Hq, Lq) or lse.dtype != torch.float32 or not lse.is_contiguous() or lse.device != dev:
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Lq] tensor on q's device")
    seg_q = _check_ids(seg_q, Lq, dev, "seg_q")
    seg_kv = _check_ids(seg_kv, Lk, dev, "seg_kv")
    m = _mask(mask_kind)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t.shape != ref.shape or t.dtype != ref.dtype or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must match {name[1:]}")
    lib = _lib.load()
    need = int(lib.gqa_attn_bwd_workspace_bytes(B, Hq, Hkv, Lq, Lk, d, dt, m, int(seg_q is not None)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = lib.gqa_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                              dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Lq, Lk, d,
                              dt, m, int(q_pos_offset), None if seg_q is None else seg_q.data_ptr(),
                              None if seg_kv is None else seg_kv.data_ptr(), workspace.data_ptr(),
                              workspace.numel(), _stream_ptr(stream, dev))
    _lib.check("gqa_attn_bwd", rc)
    return dq, dk, dv


class _Attention(torch.autograd.Function):
    """fwd as the forward, bwd (from the saved out and LSE) as the backward."""

    @staticmethod
    def forward(ctx, q, k, v, mask_kind, q_pos_offset, seg_q, seg_kv, fp32_path):
        out, lse = fwd(q, k, v, mask_kind=mask_kind, q_pos_offset=q_pos_offset, seg_q=seg_q, seg_kv=seg_kv,
                       fp32_path=fp32_path)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.kw = dict(mask_kind=mask_kind, q_pos_offset=q_pos_offset, seg_q=seg_q, seg_kv=seg_kv)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, _dlse):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = bwd(q, k, v, out, lse, dout.to(q.dtype).contiguous(), **ctx.kw)
        return dq, dk, dv, None, None, None, None, None


def attention(q, k, v, *, mask_kind="causal", q_pos_offset=0, seg_q=None, seg_kv=None, fp32_path="ffma",
              return_lse=False):
    """Differentiable attention for training: ``out`` (and, with ``return_lse``, the
    fp32 ``lse``, which carries no gradient).  The forward is ``fwd``; autograd's
    backward calls ``bwd`` with the saved ``out`` and ``lse`` (gradients of q, k and v,
    none for the segment ids).  Same arguments and layouts as ``fwd``."""
    out, lse = _Attention.apply(q, k, v, mask_kind, q_pos_offset, seg_q, seg_kv, fp32_path)
    return (out, lse) if return_lse else out


def bwd_offset(q, k, v, out, lse, dout, *, q_pos_offset, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """The backward of one ``fwd_offset`` block (queries at ``q_pos_offset`` positions
    after the block's first key, any number of keys): ``(dq, dk, dv)``, the block's
    contributions given the whole sequence's ``out`` and ``lse`` rows; the caller sums
    them over the blocks.  Causal mask, no segment ids, fp32 or bf16."""
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if not (isinstance(t, torch.Tensor) and t.device == dev and t.is_contiguous() and t.dtype == q.dtype):
            raise ValueError(f"{name} must be a contiguous tensor on {dev} with q's dtype")
    if out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("out and dout must have q's shape")
    dt = _dtype_code(q.dtype)
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if lse.shape != (B, Hq, Lq) or lse.dtype != torch.float32 or not lse.is_contiguous() or lse.device != dev:
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Lq] tensor on q's device")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t.shape != ref.shape or t.dtype != ref.dtype or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must match {name[1:]}")
    lib = _lib.load()
    need = int(lib.gqa_attn_bwd_workspace_bytes(B, Hq, Hkv, Lq, Lq, d, dt, GQA_MASK_CAUSAL, 0))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = lib.gqa_attn_bwd_offset(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                     dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Lq,
                                     Lk, d, dt, int(q_pos_offset), workspace.data_ptr(), workspace.numel(),
                                     _stream_ptr(stream, dev))
    _lib.check("gqa_attn_bwd_offset", rc)
    return dq, dk, dv


_SIDE_STREAMS = {}


def _side_streams(dev):
    """Two streams per device (copies in, copies out), created once and reused so that
    the caching allocator's blocks and the streams stay the same from call to call."""
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _SIDE_STREAMS:
        _SIDE_STREAMS[key] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    return _SIDE_STREAMS[key]


def fwd_host(q, k, v, *, device="cuda", mask_kind="causal", q_pos_offset=0, seg_q=None, seg_kv=None,
             out=None, lse=None, stream=None, fp32_path="ffma"):
    """Attention on host tensors: copies inputs to ``device``, runs, copies out/lse back.

    The work is cut into independent pieces, one per (batch entry, key/value head): the
    G query heads of a group, their key/value head and their out / lse rows are
    contiguous in every layout, so each piece moves with plain asynchronous copies.
    Copies in, the attention and copies out run on three streams, piece by piece, so
    the transfers of one piece overlap the attention of another.  Pinned host tensors
    make the copies asynchronous; ``out``/``lse`` may be preallocated (pinned) host
    buffers.  ``fp32_path`` as for ``fwd``.  Returns after the results are on the host.
    """
    _call_dtype(q.dtype, fp32_path)
    dev = _device(device)
    B, Hq, Lq, d = q.shape
    Hkv = k.shape[1]
    if Hkv < 1 or Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    q, k, v = (t.contiguous() for t in (q, k, v))
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, pin_memory=True)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    with torch.cuda.device(dev):
        s_in, s_out = _side_streams(dev)
        with torch.cuda.stream(s):  # device buffers belong to the caller's stream
            dq, dk, dv = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (q, k, v))
            dout = torch.empty(q.shape, dtype=q.dtype, device=dev)
            dlse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=dev)
            dsq = None if seg_q is None else torch.as_tensor(seg_q, dtype=torch.int32).to(dev, non_blocking=True)
            dskv = None if seg_kv is None else torch.as_tensor(seg_kv, dtype=torch.int32).to(dev, non_blocking=True)
        s_in.wait_stream(s)
        for t in (dq, dk, dv, dout, dlse):
            t.record_stream(s_in)
            t.record_stream(s_out)
        for b in range(B):
            for g in range(Hkv):
                hs = slice(g * G, (g + 1) * G)
                with torch.cuda.stream(s_in):
                    dq[b, hs].copy_(q[b, hs], non_blocking=True)
                    dk[b, g].copy_(k[b, g], non_blocking=True)
                    dv[b, g].copy_(v[b, g], non_blocking=True)
                s.wait_stream(s_in)
                with torch.cuda.stream(s):  # the call's workspace lives on s
                    fwd(dq[b:b + 1, hs], dk[b:b + 1, g:g + 1], dv[b:b + 1, g:g + 1], mask_kind=mask_kind,
                        q_pos_offset=q_pos_offset, seg_q=dsq, seg_kv=dskv, out=dout[b:b + 1, hs],
                        lse=dlse[b:b + 1, hs], stream=s, fp32_path=fp32_path)
                s_out.wait_stream(s)
                with torch.cuda.stream(s_out):
                    out[b, hs].copy_(dout[b, hs], non_blocking=True)
                    lse[b, hs].copy_(dlse[b, hs], non_blocking=True)
        s.wait_stream(s_out)
    s_out.synchronize()
    s.synchronize()
    return out, lse


def tile_plan(Hq, Hkv, Lq, Lk, *, dtype=torch.float32, mask_kind="causal", q_pos_offset=0, seg_q=None,
              seg_kv=None, device="cuda", stream=None):
    """Device block-skip plan (debug export): numpy ``classes [nq, nk]`` uint8 and ``ranges [nq, 2]``."""
    dev = _device(device)
    dt = _dtype_code(dtype)
    m = _mask(mask_kind)
    br, bc = tile_sizes(dt, Hq, Hkv)
    nq, nk = -(-Lq // br), -(-Lk // bc)
    seg_q = _check_ids(seg_q, Lq, dev, "seg_q")
    seg_kv = _check_ids(seg_kv, Lk, dev, "seg_kv")
    lib = _lib.load()
    need = int(lib.gqa_attn_workspace_bytes(1, Hq, Hkv, Lq, Lk, 256, dt, m, int(seg_q is not None)))
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    classes = torch.empty(nq * nk, dtype=torch.uint8, device=dev)
    ranges = torch.empty(nq * 2, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        rc = lib.gqa_attn_tile_plan(Hq, Hkv, Lq, Lk, dt, m, int(q_pos_offset),
                                    None if seg_q is None else seg_q.data_ptr(),
                                    None if seg_kv is None else seg_kv.data_ptr(),
                                    ws.data_ptr(), ws.numel(), classes.data_ptr(), ranges.data_ptr(),
                                    _stream_ptr(stream, dev))
    _lib.check("gqa_attn_tile_plan", rc)
    return classes.view(nq, nk).cpu().numpy(), ranges.view(nq, 2).cpu().numpy()


def status(workspace, stream=None) -> int:
    """Device status word of the last call that used ``workspace`` (synchronises)."""
    with torch.cuda.device(workspace.device):
        return int(_lib.load().gqa_attn_status(workspace.data_ptr(), _stream_ptr(stream, workspace.device)))


def selftest_wait(budget_ns=50_000_000, device="cuda") -> int:
    """Runs the bounded-wait self-test; returns the recorded device status (expect -6)."""
    dev = _device(device)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _lib.check("gqa_attn_selftest_wait",
                   _lib.load().gqa_attn_selftest_wait(ws.data_ptr(), ws.numel(), int(budget_ns),
                                                      _stream_ptr(None, dev)))
    return status(ws)


def selftest_bounds(planted=False, device="cuda") -> int:
    """Runs the index-check self-test of a checked build (GQA_ATTN_DEBUG_BOUNDS=1);
    returns the recorded device status: GQA_OK, or GQA_ERR_DEVICE_BOUNDS with
    ``planted``.  Raises GqaAttnError (GQA_ERR_UNSUPPORTED) on a normal build."""
    dev = _device(device)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _lib.check("gqa_attn_selftest_bounds",
                   _lib.load().gqa_attn_selftest_bounds(ws.data_ptr(), ws.numel(), int(bool(planted)),
                                                        _stream_ptr(None, dev)))
    return status(ws)
