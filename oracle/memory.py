"""Closed forms for the memory figures the pages print (test infrastructure).

These are the contrasts of the linear-memory test: what the L x L "math" path and
the per-head key/value repeat would hold, and what block-pair mask metadata
costs.  Each is pinned in ``tests/test_oracle.py`` against the figures printed on
the pages (fixtures in ``tests/golden/memory_figures.txt``).
"""

from __future__ import annotations


def score_matrix_bytes(Hq: int, L: int, elem_bytes: int = 4) -> int:
    """One ``Hq x L x L`` score matrix, as SDPA's math kernel materialises it.

    kev PR #202, "Why fp32 fell to the L x L kernel": 16 x L x L fp32 scores, 69 GB at
    32k and 275 GB at 64k per attention layer; "End to end": a 55.00 GiB allocation
    for one 16 x 30k^2 fp32 score matrix.
    """
    return Hq * L * L * elem_bytes


def repeated_kv_bytes(Hq: int, L: int, d: int, elem_bytes: int = 4) -> int:
    """Keys (or values) repeated to one copy per query head: ``Hq x L x d`` elements.

    kev PR #202, "The change": the repeated K/V cost 1 GiB each at 64k.
    """
    return Hq * L * d * elem_bytes


def block_pair_table_bytes(L: int, block: int, elem_bytes: int = 2) -> int:
    """A per-(query block, key block) table, as splash's mask metadata is shaped.

    maxtext PR #4929, description: 2,097,152 bytes is, among other readings, an
    int16 ``[1, 1024, 1024]`` array at block 1024 and 1M tokens.
    """
    n = -(-L // block)
    return n * n * elem_bytes


def quarter_score_matrix_per_head_bytes(L: int, elem_bytes: int = 4) -> float:
    """The linear-memory bar: a quarter of one fp32 ``L x L`` score matrix per head.

    kev PR #202, "Test plan": the long pass stays under 1/4 of one fp32 L x L score
    matrix per head, and the math pass exceeds it.
    """
    return L * L * elem_bytes / 4.0
