"""Exact grouped-query attention in float64: the plain definition.

Test infrastructure (see the package docstring): never imported by the product.

What is computed, and where the pages fix it
--------------------------------------------
* Scores ``s_ij = scale * <q_h,i , k_g,j>`` with ``scale = 1/sqrt(d)`` and the
  softmax over visible keys, ``out = sum_j softmax_j * v_g,j``.  The pages name the
  computation as the attention that SDPA runs, either through the L x L "math"
  kernel or a memory-efficient kernel with the same result (kev PR #202, "Why
  fp32 fell to the L x L kernel" and "Measurements", where the efficient kernel
  matches math to fp32 noise).
* Grouped-query sharing: 16 query heads over 4 key/value heads (kev PR #202, "Why
  fp32 fell to the L x L kernel"; shapes in system1-omni issue #27, "The closest
  planned or implemented model": head_dim 256, 16 query / 4 KV heads).  Query
  head ``h`` reads KV head ``h // (Hq // Hkv)``: consecutive groups, which is the
  convention of the per-head key/value repeat that kev PR #202 ("The change")
  swaps in for grouped attention.
* Causal mask with the query rows placed after ``q_pos_offset`` earlier keys:
  query row ``i`` sits at absolute position ``p = i + q_pos_offset`` and sees keys
  ``j <= p``.  A branch follows its state (system1-omni issue #27, item 3: state
  once, then one branch per question with positions restarting at the state
  length).
* Shared-prefix branch rows (``MASK_PREFIX_BRANCH``): the ``q_pos_offset`` state keys
  are visible to every branch row; a branch key is visible only to rows of the
  same branch (same segment id), causally.  Reading taken: branches do not see one
  another, because each question has its own branch (system1-omni issue #27,
  item 3; kev PR #202, "End to end": the row form re-runs the state per question).
* Segment ids (block-causal packing): a query sees a key only if both carry the
  same id, on top of the causal rule (maxtext PR #4929, description: the
  segmented splash kernel; constant ids give the non-segmented result).
* LSE: natural log of the sum of ``exp`` of the *scaled* scores over visible keys.
  The pages never mention it; this is the flash convention.  A row with no
  visible key has ``out = 0`` and ``LSE = -inf``.

Arithmetic: inputs (fp32, or bf16 values upcast exactly) are converted to float64;
the score rows are one float64 matrix product per head (a library primitive), the
softmax is taken over each full row after subtracting its maximum.  Rows are
processed in chunks so that only ``chunk x Lk`` scores are ever held: memory is
linear in L for the oracle too.
"""

from __future__ import annotations

import math

import numpy as np

MASK_CAUSAL = 0
MASK_PREFIX_BRANCH = 1


def _as_f64(x) -> np.ndarray:
    """Exact conversion of an fp32 / bf16 / fp64 array (numpy or torch) to float64."""
    try:  # torch tensors (bf16 has no numpy dtype: upcast through float32, exact)
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _as_i64(x) -> np.ndarray | None:
    if x is None:
        return None
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.int64)


def visible(rows, Lk, *, mask_kind=MASK_CAUSAL, q_pos_offset=0, seg_q=None, seg_kv=None):
    """Boolean matrix ``[len(rows), Lk]``: may query row ``i`` attend to key ``j``?

    ``visible(i, j) = (j <= p) and (no segment ids or seg_q[i] == seg_kv[j] or j < P0)``
    with ``p = i + q_pos_offset`` and ``P0 = q_pos_offset`` for the shared-prefix
    branch mask, ``P0 = 0`` otherwise (see the module docstring for the sources).
    """
    rows = np.asarray(rows, dtype=np.int64)
    Lk = int(Lk)
    j = np.arange(Lk, dtype=np.int64)[None, :]
    p = rows[:, None] + int(q_pos_offset)
    vis = j <= p
    seg_q = _as_i64(seg_q)
    seg_kv = _as_i64(seg_kv)
    if (seg_q is None) != (seg_kv is None):
        raise ValueError("segment ids must be given for both queries and keys, or neither")
    if mask_kind == MASK_PREFIX_BRANCH and seg_q is None:
        raise ValueError("the shared-prefix branch mask needs segment (branch) ids")
    if seg_q is not None:
        same = seg_q[rows][:, None] == seg_kv[None, :Lk]
        P0 = int(q_pos_offset) if mask_kind == MASK_PREFIX_BRANCH else 0
        vis &= same | (j < P0)
    return vis


def _check_shapes(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, H, L, d]")
    B, Hq, Lq, d = q.shape
    Bk, Hkv, Lk, dk = k.shape
    if v.shape != k.shape or Bk != B or dk != d:
        raise ValueError("k and v must be [B, Hkv, Lk, d] with q's B and d")
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, Hq, Hkv, Lq, Lk, d


def attention(q, k, v, *, mask_kind=MASK_CAUSAL, q_pos_offset=0, seg_q=None, seg_kv=None,
              rows=None, scale=None, chunk=64):
    """Exact attention in float64 for all query rows or the selected ``rows``.

    Args:
      q: ``[B, Hq, Lq, d]``; k, v: ``[B, Hkv, Lk, d]`` (numpy or torch, any float
        dtype; values are converted to float64 exactly).
      mask_kind: ``MASK_CAUSAL`` or ``MASK_PREFIX_BRANCH``.
      q_pos_offset: keys that precede query row 0 (``Lk = q_pos_offset + Lq``).
      seg_q, seg_kv: optional int segment ids of length ``Lq`` / ``Lk`` (shared by
        every batch entry and head).
      rows: optional sorted or unsorted query row indices; default all rows.
      scale: score scale, default ``1/sqrt(d)``.

    Returns:
      ``(out, lse)``: float64 arrays ``[B, Hq, n, d]`` and ``[B, Hq, n]`` where ``n``
      is the number of selected rows.
    """
    B, Hq, Hkv, Lq, Lk, d = _check_shapes(q, k, v)
    if Lk != q_pos_offset + Lq:
        raise ValueError("Lk must equal q_pos_offset + Lq")
    return _attention_rows(q, k, v, mask_kind=mask_kind, q_pos_offset=q_pos_offset, seg_q=seg_q, seg_kv=seg_kv,
                           rows=rows, scale=scale, chunk=chunk)


def _attention_rows(q, k, v, *, mask_kind, q_pos_offset, seg_q, seg_kv, rows, scale, chunk):
    """The body of ``attention`` for any key count: keys ``j <= i + q_pos_offset``."""
    B, Hq, Hkv, Lq, Lk, d = _check_shapes(q, k, v)
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rows = np.arange(Lq, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    n = rows.shape[0]
    sliced = rows.shape[0] < Lq
    # Only the selected query rows are converted, and keys / values only up to the
    # last key any selected row can see, one key/value head at a time.
    q = _as_f64(q[:, :, rows] if sliced else q)
    kmax = min(Lk, int(rows.max()) + int(q_pos_offset) + 1) if n else 0
    out = np.zeros((B, Hq, n, d))
    lse = np.full((B, Hq, n), -np.inf)
    chunks = []
    for c0 in range(0, n, chunk):
        r = rows[c0:c0 + chunk]
        # Keys past the last row's position are hidden for every row of the chunk:
        # leaving them out drops only exp(-inf) = 0 terms.
        kend = min(Lk, int(r.max()) + int(q_pos_offset) + 1)
        vis = visible(r, kend, mask_kind=mask_kind, q_pos_offset=q_pos_offset,
                      seg_q=seg_q, seg_kv=seg_kv)
        chunks.append((c0, r, kend, vis, vis.any(axis=1)))
    for b in range(B):
        for g in range(Hkv):
            kg = _as_f64(k[b, g, :kmax])
            vg = _as_f64(v[b, g, :kmax])
            for c0, r, kend, vis, has_any in chunks:
                qr = np.arange(c0, c0 + len(r)) if sliced else r
                for h in range(g * G, (g + 1) * G):
                    s = (q[b, h, qr] @ kg[:kend].T) * scale
                    s = np.where(vis, s, -np.inf)
                    m = s.max(axis=1)
                    m_safe = np.where(has_any, m, 0.0)
                    e = np.exp(s - m_safe[:, None])  # exp(-inf) = 0 for hidden keys
                    ell = e.sum(axis=1)
                    ell_safe = np.where(has_any, ell, 1.0)
                    o = (e @ vg[:kend]) / ell_safe[:, None]
                    out[b, h, c0:c0 + len(r)] = np.where(has_any[:, None], o, 0.0)
                    lse[b, h, c0:c0 + len(r)] = np.where(has_any, m_safe + np.log(ell_safe), -np.inf)
    return out, lse


def probabilities(q, k, *, b, h, row, mask_kind=MASK_CAUSAL, q_pos_offset=0, seg_q=None,
                  seg_kv=None, scale=None):
    """The softmax row ``P[row, :]`` (length Lk, float64) of head ``h`` of batch ``b``.

    Hidden keys carry probability 0.  A row with no visible key is all zeros.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    _, Hq, _, d = q.shape
    Hkv = k.shape[1]
    Lk = k.shape[2]
    g = h // (Hq // Hkv)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    vis = visible([row], Lk, mask_kind=mask_kind, q_pos_offset=q_pos_offset,
                  seg_q=seg_q, seg_kv=seg_kv)[0]
    if not vis.any():
        return np.zeros(Lk)
    s = (k[b, g] @ q[b, h, row]) * scale
    s = np.where(vis, s, -np.inf)
    e = np.exp(s - s.max())
    return e / e.sum()
