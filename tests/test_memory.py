"""Memory linear in L (the pages' failure: the L x L math kernel's 69-275 GB score
matrices, kev PR #202, "Why fp32 fell to the L x L kernel"; the test plan there asks
the long pass to stay under a quarter of one L x L matrix per head).

The library allocates nothing; a call's device memory beyond its inputs and outputs
is the workspace the binding allocates: 256 bytes without segment ids and O(L / tile)
with them.  Checked from 512 tokens to 262,144 causal tokens and at the 1M-token
packed configuration.
"""

import pytest
import torch

import bench
from long_context_causal_flash_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L", [512, 4096, 15_231, 60_926, 262_144])
def test_causal_memory_over_inputs_is_the_workspace(cuda_device, L):
    dtype = torch.float32 if L <= 60_926 else torch.bfloat16
    peak, delta = bench.memory_point(workloads.causal(L, dtype), torch.device("cuda"))
    assert peak <= 512  # the 256-byte status workspace (allocator granularity: 512)
    assert delta == 0   # nothing else is allocated by the library
    assert peak < (L * L * 4) // 4  # under a quarter of one fp32 L x L matrix


def test_segmented_1m_memory_is_linear(cuda_device):
    w = workloads.by_name("segmented_1M_bf16")
    peak, delta = bench.memory_point(w, torch.device("cuda"))
    # per-tile [min, max] ids and key-tile ranges: 16 bytes per query tile and 8 per key tile
    assert peak <= 256 + 4 * 16 * (w.Lq // 32 + 1) + 8 * (w.Lk // 128 + 1) + 4 * 256 + 4096
    assert delta == 0
