"""Gradients of exact grouped-query attention in float64 (test infrastructure).

Test infrastructure (see the package docstring): never imported by the product.

What is computed
----------------
Training with packed long sequences (maxtext PR #4929, description: the splash
kernel runs in training steps over 1,048,576-token packed batches) needs the
gradients of the attention output with respect to its inputs.  For an upstream
gradient ``dout`` of ``out`` (``exact.attention``), per batch entry, query head ``h``
and its key/value head ``g = h // (Hq // Hkv)``, over the visible pairs of
``exact.visible``:

* ``P_ij``   the softmax probabilities of the forward (``exact.probabilities``);
* ``dV_g,j = sum_{h in g} sum_i P_ij dout_h,i``                 (out is linear in v);
* ``dP_ij  = <dout_h,i , v_g,j>``;
* ``D_i    = sum_j P_ij dP_ij = <dout_h,i , out_h,i>``;
* ``dS_ij  = P_ij (dP_ij - D_i)``                  (derivative of the softmax);
* ``dQ_h,i = scale * sum_j dS_ij k_g,j``;
* ``dK_g,j = scale * sum_{h in g} sum_i dS_ij q_h,i``             (scores are linear).

This is the chain rule applied to the definition, written out; a query head's
contribution to its shared key/value head is summed because the forward reads one
key/value head for all query heads of its group.  Rows with no visible key have
``P = 0`` and contribute nothing.

Arithmetic: float64 throughout; scores and probabilities are formed for ``chunk``
query rows at a time (one matrix product per head and chunk, a library primitive),
so memory stays linear in L.
"""

from __future__ import annotations

import math

import numpy as np

from .exact import MASK_CAUSAL, _as_f64, _check_shapes, visible


def attention_backward(q, k, v, dout, *, mask_kind=MASK_CAUSAL, q_pos_offset=0, seg_q=None, seg_kv=None,
                       scale=None, chunk=128):
    """Gradients ``(dq, dk, dv)`` (float64, shapes of q, k, v) of ``sum(out * dout)``."""
    B, Hq, Hkv, Lq, Lk, d = _check_shapes(q, k, v)
    if Lk != q_pos_offset + Lq:
        raise ValueError("Lk must equal q_pos_offset + Lq")
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    if dout.shape != q.shape:
        raise ValueError("dout must have q's shape")
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r0 in range(0, Lq, chunk):
        rows = np.arange(r0, min(Lq, r0 + chunk))
        vis = visible(rows, Lk, mask_kind=mask_kind, q_pos_offset=q_pos_offset, seg_q=seg_q, seg_kv=seg_kv)
        any_vis = vis.any(axis=1)
        for b in range(B):
            for h in range(Hq):
                g = h // G
                s = scale * (q[b, h, rows] @ k[b, g].T)
                s = np.where(vis, s, -np.inf)
                m = np.where(any_vis, s.max(axis=1), 0.0)
                p = np.where(vis, np.exp(s - m[:, None]), 0.0)
                lsum = p.sum(axis=1)
                p = p / np.where(any_vis, lsum, 1.0)[:, None]
                do = dout[b, h, rows]
                dv[b, g] += p.T @ do
                dp = do @ v[b, g].T
                o = p @ v[b, g]
                Dr = np.sum(do * o, axis=1)
                ds = p * (dp - Dr[:, None])
                dq[b, h, rows] = scale * (ds @ k[b, g])
                dk[b, g] += scale * (ds.T @ q[b, h, rows])
    return dq, dk, dv
