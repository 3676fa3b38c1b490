"""Blocks of a sharded sequence and the merge of partial results, in float64 (test
infrastructure).

Test infrastructure (see the package docstring): never imported by the product.

What is computed, and where the pages fix it
--------------------------------------------
The 1,048,576-token training runs of maxtext PR #4929 ("Effect": measured with
context parallelism) shard the sequence across devices, and its code review names
the ring attention path (``use_tokamax_ring``) among the attention paths of that
model.  A ring step attends one device's query rows to another device's key/value
block, and the partial results are combined:

* ``attention_block``: exact causal attention of ``Lq`` query rows against a block of
  ``Lk`` keys that starts ``q_pos_offset`` positions before the first query row (query
  row ``i`` sees key ``j`` iff ``j <= i + q_pos_offset``), for any ``Lk``: the
  definition of ``exact.attention`` without its ``Lk = q_pos_offset + Lq`` contract.
  Reading taken: the pages do not describe the ring schedule; the plainest one gives
  each device a contiguous shard, and a key block wholly after a device's queries is
  skipped, so ``q_pos_offset >= 0`` here.
* ``merge_partials``: two results over disjoint key sets, each normalised over its
  own keys with its log-sum-exp, combine exactly as
  ``lse = log(exp(lse_a) + exp(lse_b))`` and
  ``out = exp(lse_a - lse) out_a + exp(lse_b - lse) out_b``;
  a result with ``lse = -inf`` (no visible key) contributes nothing.
* ``attention_block_backward``: a training step over such a sharded sequence (the
  same page's 1,048,576-token training) also needs the gradients block by block.
  Given the WHOLE sequence's output ``out_i`` and log-sum-exp ``lse_i`` of each query
  row, the softmax probability of a visible key ``j`` of the block is
  ``P_ij = exp(scale <q_i, k_j> - lse_i)`` (the block's share of the row's softmax),
  ``D_i = <dout_i, out_i>`` is the full row's, and with ``dP_ij = <dout_i, v_j>``,
  ``dS_ij = P_ij (dP_ij - D_i)`` the block contributes
  ``dq_i = scale sum_j dS_ij k_j`` (over its keys only),
  ``dk_j = scale sum_{h in group} sum_i dS_ij q_i`` and
  ``dv_j = sum_{h in group} sum_i P_ij dout_i`` (over these query rows only).
  The chain rule of ``backward.attention_backward`` with the softmax normaliser taken
  from the whole row: summed over a partition of the keys into blocks, the
  contributions are the whole sequence's gradients.

Arithmetic: float64; ``attention_block`` uses the same score / softmax code as
``exact.attention`` (one matrix product per head and chunk of rows).
"""

from __future__ import annotations

import math

import numpy as np

from .exact import MASK_CAUSAL, _as_f64, _attention_rows


def attention_block(q, k, v, *, q_pos_offset, rows=None, scale=None, chunk=64):
    """``(out, lse)`` float64 of causal attention against a key block at ``q_pos_offset``."""
    if int(q_pos_offset) < 0:
        raise ValueError("q_pos_offset must be >= 0 (blocks after the queries are skipped)")
    return _attention_rows(q, k, v, mask_kind=MASK_CAUSAL, q_pos_offset=int(q_pos_offset), seg_q=None,
                           seg_kv=None, rows=rows, scale=scale, chunk=chunk)


def attention_block_backward(q, k, v, out, lse, dout, *, q_pos_offset, scale=None, chunk=128):
    """``(dq, dk, dv)`` float64: one key block's contributions to the gradients of
    ``sum(out * dout)``, from the whole sequence's ``out`` and ``lse`` rows."""
    q, k, v, out, lse, dout = (_as_f64(x) for x in (q, k, v, out, lse, dout))
    off = int(q_pos_offset)
    if off < 0:
        raise ValueError("q_pos_offset must be >= 0 (blocks after the queries are skipped)")
    B, Hq, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if Hq % Hkv or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("shapes: q, out, dout [B, Hq, Lq, d]; k, v [B, Hkv, Lk, d]")
    if lse.shape != (B, Hq, Lq):
        raise ValueError("lse must be [B, Hq, Lq]")
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    keys = np.arange(Lk)
    for r0 in range(0, Lq, chunk):
        rows = np.arange(r0, min(Lq, r0 + chunk))
        vis = keys[None, :] <= rows[:, None] + off  # row i sees key j iff j <= i + offset
        for b in range(B):
            for h in range(Hq):
                g = h // G
                l_rows = lse[b, h, rows]
                live = np.isfinite(l_rows)[:, None] & vis
                s = scale * (q[b, h, rows] @ k[b, g].T)
                p = np.where(live, np.exp(np.where(live, s, 0.0) - np.where(np.isfinite(l_rows), l_rows, 0.0)[:, None]),
                             0.0)
                do = dout[b, h, rows]
                dp = do @ v[b, g].T
                D = np.sum(do * out[b, h, rows], axis=1)
                ds = p * (dp - D[:, None])
                dq[b, h, rows] = scale * (ds @ k[b, g])
                dk[b, g] += scale * (ds.T @ q[b, h, rows])
                dv[b, g] += p.T @ do
    return dq, dk, dv


def merge_partials(out_a, lse_a, out_b, lse_b):
    """Exact combination of two partial results over disjoint key sets (float64)."""
    out_a, lse_a, out_b, lse_b = (_as_f64(x) for x in (out_a, lse_a, out_b, lse_b))
    m = np.maximum(lse_a, lse_b)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    wa = np.where(np.isfinite(lse_a), np.exp(lse_a - m_safe), 0.0)
    wb = np.where(np.isfinite(lse_b), np.exp(lse_b - m_safe), 0.0)
    wsum = wa + wb
    has = wsum > 0
    wsum_safe = np.where(has, wsum, 1.0)
    out = (wa[..., None] * out_a + wb[..., None] * out_b) / wsum_safe[..., None]
    out = np.where(has[..., None], out, 0.0)
    lse = np.where(has, m_safe + np.log(wsum_safe), -np.inf)
    return out, lse
