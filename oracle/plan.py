"""Tile classes for causal / segment block skipping: the integer definition.

Test infrastructure (see the package docstring): never imported by the product.

Why a plan, and why only per-tile bounds
----------------------------------------
maxtext PR #4929 (description and code review) shows the cost of block-pair
metadata: the segmented splash kernel prefetches per-(query block, key block)
tables into scalar memory, 2,097,152 bytes at 1M tokens against 1 MiB, and the
kernel fails to build.  The plan defined here keeps only O(L / tile) integers:
the [min, max] segment id of every query tile and every key tile.  A (query tile,
key tile) pair is classed from those bounds alone:

* SKIP    -- no pair in the tile is visible; its keys are never read.
* FULL    -- every pair is visible; no per-element mask is applied.
* PARTIAL -- anything else; the per-element rule of ``exact.visible`` applies.

For query rows ``[i0, i1]``, key columns ``[j0, j1]``, offset ``o = q_pos_offset``
and ``P0 = o`` for the shared-prefix branch mask (else 0):

* ``causal_skip = j0 > i1 + o``;  ``causal_full = j1 <= i0 + o``
* ``all_state = j1 < P0``;  ``any_state = j0 < P0``
* with segment ids: ``seg_skip = qmax < kmin or kmax < qmin``,
  ``seg_full = (qmin == qmax == kmin == kmax)``; without: ``False`` / ``True``.
* SKIP iff ``not any_state and (causal_skip or seg_skip)``;
  FULL iff ``all_state or (causal_full and seg_full)``; else PARTIAL.

(State keys ``j < P0`` are visible to every branch row, since every branch row
sits at ``p >= P0``; a tile holding any of them is therefore never skipped.)

Per query tile the key-tile range to visit is ``[first non-SKIP, last non-SKIP + 1)``
or ``(0, 0)`` when every tile is SKIP.  SKIP tiles inside the range are skipped too.
"""

from __future__ import annotations

import numpy as np

SKIP = 0
PARTIAL = 1
FULL = 2


def _ids(x, n):
    if x is None:
        return None
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x).astype(np.int64)
    if x.shape != (n,):
        raise ValueError("segment ids must have one entry per row")
    return x


def tile_plan(Lq, Lk, Br, Bc, *, mask_kind=0, q_pos_offset=0, seg_q=None, seg_kv=None, q_tiles=None):
    """Classes ``[nq, nk]`` (uint8) and key-tile ranges ``[nq, 2]`` (int32).

    ``Br`` is the number of query positions per query tile, ``Bc`` the number of
    keys per key tile; the last tile of each is ragged.  ``mask_kind`` 1 is the
    shared-prefix branch mask.  ``q_tiles`` restricts the evaluation to those query
    tiles (the other rows of the result stay zero).
    """
    seg_q = _ids(seg_q, Lq)
    seg_kv = _ids(seg_kv, Lk)
    if (seg_q is None) != (seg_kv is None):
        raise ValueError("segment ids must be given for both queries and keys, or neither")
    o = int(q_pos_offset)
    P0 = o if mask_kind == 1 else 0
    nq = -(-Lq // Br)
    nk = -(-Lk // Bc)
    classes = np.zeros((nq, nk), dtype=np.uint8)
    ranges = np.zeros((nq, 2), dtype=np.int32)
    for qt in (range(nq) if q_tiles is None else [int(t) for t in q_tiles]):
        i0 = qt * Br
        i1 = min(Lq, i0 + Br) - 1
        if seg_q is not None:
            qmin = int(seg_q[i0:i1 + 1].min())
            qmax = int(seg_q[i0:i1 + 1].max())
        first, last = None, None
        for kt in range(nk):
            j0 = kt * Bc
            j1 = min(Lk, j0 + Bc) - 1
            causal_skip = j0 > i1 + o
            causal_full = j1 <= i0 + o
            all_state = j1 < P0
            any_state = j0 < P0
            if seg_q is not None:
                kmin = int(seg_kv[j0:j1 + 1].min())
                kmax = int(seg_kv[j0:j1 + 1].max())
                seg_skip = qmax < kmin or kmax < qmin
                seg_full = qmin == qmax == kmin == kmax
            else:
                seg_skip, seg_full = False, True
            if not any_state and (causal_skip or seg_skip):
                c = SKIP
            elif all_state or (causal_full and seg_full):
                c = FULL
            else:
                c = PARTIAL
            classes[qt, kt] = c
            if c != SKIP:
                if first is None:
                    first = kt
                last = kt
        if first is not None:
            ranges[qt] = (first, last + 1)
    return classes, ranges
