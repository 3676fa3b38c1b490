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

Arithmetic: float64; ``attention_block`` uses the same score / softmax code as
``exact.attention`` (one matrix product per head and chunk of rows).
"""

from __future__ import annotations

import numpy as np

from .exact import MASK_CAUSAL, _as_f64, _attention_rows


def attention_block(q, k, v, *, q_pos_offset, rows=None, scale=None, chunk=64):
    """``(out, lse)`` float64 of causal attention against a key block at ``q_pos_offset``."""
    if int(q_pos_offset) < 0:
        raise ValueError("q_pos_offset must be >= 0 (blocks after the queries are skipped)")
    return _attention_rows(q, k, v, mask_kind=MASK_CAUSAL, q_pos_offset=int(q_pos_offset), seg_q=None,
                           seg_kv=None, rows=rows, scale=scale, chunk=chunk)


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
