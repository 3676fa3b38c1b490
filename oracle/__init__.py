"""CPU oracle for exact causal grouped-query attention (test infrastructure).

This package is test infrastructure, not part of the product.  Only the tests,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py`` may import it.  It shares no code with the CUDA library under
``long_context_causal_flash_b200/``: it neither imports that package nor is
imported by it.  Inputs reach it as plain arrays produced by the seeded input
generators, never from the CUDA path.

Contents
--------
``exact``      the attention definition in float64 (scores, mask, softmax, LSE).
``plan``       the tile-class definition for causal / segment block skipping.
``memory``     closed forms for the memory figures the pages print.
``backward``   the gradients (dq, dk, dv) of the attention definition in float64.
``context``    attention against one key block of a sharded sequence, and the merge
               of partial results by their log-sum-exp.

Sources (the three pages this build follows):

* kev PR #202, "fp32 long-state attention" (github.com/jaredpalmer/kev/pull/202):
  sections "Why fp32 fell to the L x L kernel", "The change", "Measurements",
  "Test plan".
* system1-omni issue #27, "[New Model]: Support Kev (0.5B-9B)": sections "The
  closest planned or implemented model" (shapes) and its item 3 (state once, then
  one branch per question).
* maxtext PR #4929, "Let splash attention exceed 524,288 tokens when packing is
  off": the description (segment ids, constant ids equal the non-segmented
  kernel) and the code review.

Every function here is pinned by tests in ``tests/test_oracle.py``,
``tests/test_oracle_backward.py`` and ``tests/test_oracle_context.py`` against
library routines, closed forms, invariants and the figures the pages print.
"""

from .exact import (  # noqa: F401
    MASK_CAUSAL,
    MASK_PREFIX_BRANCH,
    attention,
    probabilities,
    visible,
)
from .plan import SKIP, PARTIAL, FULL, tile_plan  # noqa: F401
from .backward import attention_backward  # noqa: F401
from .context import attention_block, attention_block_backward, merge_partials  # noqa: F401
from . import memory  # noqa: F401
