"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module draws random numbers and lays out index arrays; it holds none of the
attention arithmetic, so the CUDA path and the CPU oracle can both be fed from it
without sharing any of the method.

Recipe (the pages' workloads are long documents and 1M-token packed training runs;
none of their data is available, so these stand in for them at the same shapes):

* Q, K, V ~ N(0, 1) in fp32 from ``torch.randn`` with seeds 1, 2, 3 (one
  generator per tensor).  bf16 inputs are the same fp32 draws rounded to nearest
  even (``tensor.to(torch.bfloat16)``).  With scale 1/16 and d = 256 the scores
  have unit variance: a non-degenerate softmax.
* Segment lengths for packed sequences: seed 4, integers uniform in
  ``[lo, hi]`` drawn until they cover ``L``; the last one is cut to fit.
* Sampled query rows: seed 5, always including row 0, the last row and the first
  and last row of every segment or branch; the rest uniform without replacement.
"""

from __future__ import annotations

import numpy as np
import torch

SEED_Q, SEED_K, SEED_V, SEED_SEGMENTS, SEED_ROWS = 1, 2, 3, 4, 5


def _randn(shape, seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def qkv(B, Hq, Hkv, Lq, Lk, d, *, dtype=torch.float32, device="cpu", seeds=(SEED_Q, SEED_K, SEED_V)):
    """Q ``[B, Hq, Lq, d]``, K and V ``[B, Hkv, Lk, d]``, contiguous, seeded N(0, 1).

    Drawn in fp32 on ``device``'s generator and then cast to ``dtype`` (RNE for bf16).
    The CPU generator and a CUDA generator give different (each reproducible)
    streams; callers that compare against the oracle copy the device tensors to
    the host rather than redrawing.
    """
    q = _randn((B, Hq, Lq, d), seeds[0], device)
    k = _randn((B, Hkv, Lk, d), seeds[1], device)
    v = _randn((B, Hkv, Lk, d), seeds[2], device)
    if dtype != torch.float32:
        q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    return q.contiguous(), k.contiguous(), v.contiguous()


def segment_lengths(L, lo=1024, hi=262144, seed=SEED_SEGMENTS):
    """Seeded segment lengths, uniform integers in ``[lo, hi]`` covering exactly ``L``."""
    rng = np.random.default_rng(seed)
    out = []
    total = 0
    while total < L:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, L - total)
        out.append(n)
        total += n
    return out


def segment_ids(lengths, first_id=0):
    """int32 ids: ``first_id`` repeated ``lengths[0]`` times, then ``first_id+1`` ..."""
    return np.repeat(np.arange(first_id, first_id + len(lengths), dtype=np.int32),
                     np.asarray(lengths, dtype=np.int64)).astype(np.int32)


def branch_ids(state_len, n_branches, branch_len, state_id=-1):
    """Ids for packed branches after a shared state.

    Returns ``(seg_q, seg_kv)``: queries are the ``n_branches * branch_len`` branch
    tokens with ids ``0 .. n_branches-1``; keys are the ``state_len`` state tokens
    (id ``state_id``, which the shared-prefix mask ignores) followed by the branches.
    """
    seg_q = segment_ids([branch_len] * n_branches)
    seg_kv = np.concatenate([np.full(state_len, state_id, dtype=np.int32), seg_q])
    return seg_q, seg_kv


def sample_rows(Lq, n, boundaries=(), seed=SEED_ROWS):
    """Sorted int64 row indices: required rows plus uniform picks, ``n`` in total.

    ``boundaries`` lists segment or branch start rows; the first and last row of
    each segment are always included, as are rows 0 and ``Lq - 1``.
    """
    must = {0, Lq - 1}
    starts = sorted(set(int(b) for b in boundaries) | {0})
    for a, b in zip(starts, starts[1:] + [Lq]):
        if a < Lq:
            must.add(a)
            must.add(min(b, Lq) - 1)
    must = sorted(m for m in must if 0 <= m < Lq)
    if n >= Lq:
        return np.arange(Lq, dtype=np.int64)
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(Lq, dtype=np.int64), np.asarray(must, dtype=np.int64))
    k = max(0, n - len(must))
    pick = rng.choice(rest, size=min(k, rest.size), replace=False) if k else np.empty(0, np.int64)
    return np.sort(np.concatenate([np.asarray(must, dtype=np.int64), pick]))
