"""The device block-skip plan equals the oracle's tile classes, bit for bit."""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
import oracle
from long_context_causal_flash_b200 import inputs

pytestmark = pytest.mark.gpu


def _cases():
    rng = np.random.default_rng(3)
    out = []
    for dtype in (gqa.GQA_F32, gqa.GQA_BF16):
        for Lq, off in [(1, 0), (63, 0), (64, 0), (65, 0), (1000, 0), (300, 77), (1, 5000), (2048, 30468)]:
            out.append((dtype, Lq, off, "none"))
            out.append((dtype, Lq, off, "packed"))
            out.append((dtype, Lq, off, "random"))
            if off:
                out.append((dtype, Lq, off, "branch"))
    return out


def _ids(kind, Lq, off, rng):
    L = Lq + off
    if kind == "none":
        return None, None, "causal"
    if kind == "packed":
        lens = []
        while sum(lens) < L:
            lens.append(int(rng.integers(1, 300)))
        ids = np.repeat(np.arange(len(lens)), lens)[:L].astype(np.int32)
        return ids[off:], ids, "causal"
    if kind == "random":
        ids = rng.integers(-3, 4, L).astype(np.int32)
        return ids[off:], ids, "causal"
    nb = 4
    bl = -(-Lq // nb)
    sq = np.repeat(np.arange(nb), bl)[:Lq].astype(np.int32)
    skv = np.concatenate([rng.integers(-9, 9, off).astype(np.int32), sq])
    return sq, skv, "prefix_branch"


@pytest.mark.parametrize("case", _cases(), ids=lambda c: f"{c[0]}-{c[1]}-{c[2]}-{c[3]}")
def test_device_plan_is_bit_exact(cuda_device, case):
    dtype, Lq, off, kind = case
    rng = np.random.default_rng(Lq * 31 + off)
    sq, skv, mask = _ids(kind, Lq, off, rng)
    dev = torch.device("cuda")
    tq = None if sq is None else torch.as_tensor(sq, device=dev)
    tkv = None if skv is None else torch.as_tensor(skv, device=dev)
    classes, ranges = gqa.tile_plan(16, 4, Lq, Lq + off, dtype=dtype, mask_kind=mask, q_pos_offset=off,
                                    seg_q=tq, seg_kv=tkv)
    br, bc = gqa.tile_sizes(dtype, 16, 4)
    ref_c, ref_r = oracle.tile_plan(Lq, Lq + off, br, bc, mask_kind=0 if mask == "causal" else 1,
                                    q_pos_offset=off, seg_q=sq, seg_kv=skv)
    np.testing.assert_array_equal(classes, ref_c)
    np.testing.assert_array_equal(ranges, ref_r)


def test_plan_for_the_1m_segmented_workload(cuda_device):
    L = 1_048_576
    lengths = inputs.segment_lengths(L)
    ids = inputs.segment_ids(lengths)
    dev = torch.device("cuda")
    t = torch.as_tensor(ids, device=dev)
    classes, ranges = gqa.tile_plan(16, 4, L, L, dtype=gqa.GQA_BF16, seg_q=t, seg_kv=t)
    br, bc = gqa.tile_sizes(gqa.GQA_BF16, 16, 4)
    # Sampled query tiles against the oracle's definition.
    rng = np.random.default_rng(9)
    pick = rng.choice(classes.shape[0], 24, replace=False)
    ref_c, ref_r = oracle.tile_plan(L, L, br, bc, seg_q=ids, seg_kv=ids, q_tiles=pick)
    np.testing.assert_array_equal(classes[pick], ref_c[pick])
    np.testing.assert_array_equal(ranges[pick], ref_r[pick])
    # O(L / tile) metadata: the workspace is far below the 2 MiB block-pair table
    assert gqa.workspace_bytes(1, 16, 4, L, L, dtype=torch.bfloat16, has_segments=True) < (1 << 20)
