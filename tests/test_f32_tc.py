"""GPU parity of the fp32 path on the tensor cores (GQA_F32_TC, ``fp32_path="tc"``):
fp32 inputs and outputs, both contractions on tcgen05 with split fp16 operands.

The bar is the fp32 one (out 2e-5, LSE 1e-5 against the fp64 oracle).  The cases
mirror test_parity.py (all rows of small shapes across tile edges, group sizes,
offsets, branch and segment masks, empty rows, split-KV, the benchmark's L = 60,926
on sampled rows) and add what the splitting makes new: per-head scales over many
orders of magnitude, and agreement with the FFMA kernel.
"""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
import oracle
from long_context_causal_flash_b200 import inputs
from tests._helpers import TOL, assert_close, to64

pytestmark = pytest.mark.gpu

F32 = torch.float32


def _ids(x, dev):
    return None if x is None else torch.as_tensor(np.asarray(x), dtype=torch.int32, device=dev)


def _run(q, k, v, **kw):
    out, lse = gqa.fwd(q, k, v, fp32_path="tc", **kw)
    torch.cuda.synchronize()
    assert out.dtype == F32
    return out, lse


def _check(q, k, v, rows=None, what="", mask_kind="causal", q_pos_offset=0, seg_q=None, seg_kv=None, splits=1):
    dev = torch.device("cuda")
    out, lse = _run(q.to(dev), k.to(dev), v.to(dev), mask_kind=mask_kind, q_pos_offset=q_pos_offset,
                    seg_q=_ids(seg_q, dev), seg_kv=_ids(seg_kv, dev), splits=splits)
    ref_out, ref_lse = oracle.attention(q, k, v, mask_kind=oracle.MASK_CAUSAL if mask_kind == "causal"
                                        else oracle.MASK_PREFIX_BRANCH, q_pos_offset=q_pos_offset,
                                        seg_q=seg_q, seg_kv=seg_kv, rows=rows)
    sel = slice(None) if rows is None else torch.as_tensor(rows, device=dev)
    return assert_close(out[:, :, sel], lse[:, :, sel], ref_out, ref_lse, F32, what)


@pytest.mark.parametrize("L", [1, 2, 17, 64, 127, 128, 129, 255, 256, 257, 300, 700])
def test_causal_small_all_rows(cuda_device, L):
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256)
    _check(q, k, v, what=f"causal L={L}")


@pytest.mark.parametrize("Hq,Hkv", [(16, 16), (16, 8), (16, 2), (16, 1), (8, 4)])
def test_group_sizes(cuda_device, Hq, Hkv):
    q, k, v = inputs.qkv(1, Hq, Hkv, 150, 150, 256)
    _check(q, k, v, what=f"Hq={Hq} Hkv={Hkv}")


def test_batch_of_two(cuda_device):
    q, k, v = inputs.qkv(2, 16, 4, 200, 200, 256)
    _check(q, k, v, what="B=2")


def test_large_logits(cuda_device):
    """Scores with std 8 (the running-max rescale); bound scaled by 8 as in the FFMA test."""
    q, k, v = inputs.qkv(1, 16, 4, 333, 333, 256)
    q = q * 8
    dev = torch.device("cuda")
    out, lse = _run(q.to(dev), k.to(dev), v.to(dev))
    ref_out, ref_lse = oracle.attention(q, k, v)
    tol_out, tol_lse = TOL[F32]
    assert float(np.max(np.abs(to64(out) - ref_out))) <= 8 * tol_out
    assert float(np.max(np.abs(to64(lse) - ref_lse))) <= 8 * tol_lse


def test_per_head_scales(cuda_device):
    """Heads whose magnitudes differ by up to 10^9: each head's power-of-two scale must
    come back out exactly.  Errors are relative to a head's own magnitude, so the bound
    on out is the fp32 one times that kv head's value scale."""
    q, k, v = inputs.qkv(1, 16, 4, 300, 300, 256)
    q[:, 0] *= 1e-4          # tiny logits: LSE ~ ln(p + 1)
    q[:, 5] *= 1e3           # with kv head 1 scaled by 1e-3: logits unchanged
    k[:, 1] *= 1e-3
    v[:, 2] *= 1e4
    v[:, 3] *= 1e-5
    dev = torch.device("cuda")
    out, lse = _run(q.to(dev), k.to(dev), v.to(dev))
    ref_out, ref_lse = oracle.attention(q, k, v)
    tol_out, tol_lse = TOL[F32]
    vs = [1.0, 1.0, 1e4, 1e-5]
    for g in range(4):
        hs = slice(4 * g, 4 * g + 4)
        d = float(np.max(np.abs(to64(out[:, hs]) - ref_out[:, hs])))
        assert d <= tol_out * max(vs[g], 1e-3), (g, d)
    assert float(np.max(np.abs(to64(lse) - ref_lse))) <= tol_lse


@pytest.mark.parametrize("S,Lq", [(200, 100), (1, 70), (1000, 1), (300, 257)])
def test_query_rows_after_a_state(cuda_device, S, Lq):
    q, k, v = inputs.qkv(1, 16, 4, Lq, S + Lq, 256)
    _check(q, k, v, q_pos_offset=S, what=f"offset {S}")


def test_prefix_branch_small(cuda_device):
    S, nb, bl = 300, 3, 40
    q, k, v = inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    _check(q, k, v, mask_kind="prefix_branch", q_pos_offset=S, seg_q=seg_q, seg_kv=seg_kv, what="prefix branch")


@pytest.mark.parametrize("splits", [2, 3, 5])
def test_split_kv(cuda_device, splits):
    S, nb, bl = 700, 2, 64
    q, k, v = inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    _check(q, k, v, mask_kind="prefix_branch", q_pos_offset=S, seg_q=seg_q, seg_kv=seg_kv, splits=splits,
           what=f"{splits} splits")


def test_segments_and_empty_rows(cuda_device):
    lengths = [1, 70, 5, 200, 64, 33]
    L = sum(lengths)
    ids = inputs.segment_ids(lengths)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256)
    _check(q, k, v, seg_q=ids, seg_kv=ids, what="segments")
    L = 160
    seg_q = np.array([7] * 80 + [1] * 80, dtype=np.int32)
    seg_kv = np.array([1] * 80 + [7] * 80, dtype=np.int32)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256)
    _check(q, k, v, seg_q=seg_q, seg_kv=seg_kv, what="empty rows")
    rng = np.random.default_rng(11)
    ids = rng.integers(0, 3, 257).astype(np.int32)
    q, k, v = inputs.qkv(1, 16, 4, 257, 257, 256)
    _check(q, k, v, seg_q=ids, seg_kv=ids, what="unsorted ids")


def test_constant_ids_equal_no_ids_bitwise(cuda_device):
    L = 777
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256))
    ids = torch.full((L,), 3, dtype=torch.int32, device=dev)
    o1, l1 = _run(q, k, v)
    o2, l2 = _run(q, k, v, seg_q=ids, seg_kv=ids)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_agrees_with_the_ffma_kernel(cuda_device):
    L = 2000
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256))
    o1, l1 = _run(q, k, v)
    o2, l2 = gqa.fwd(q, k, v)
    torch.cuda.synchronize()
    assert float((o1 - o2).abs().max()) <= 2 * TOL[F32][0]
    assert float((l1 - l2).abs().max()) <= 2 * TOL[F32][1]


def test_fwd_host(cuda_device):
    q, k, v = inputs.qkv(1, 16, 4, 300, 300, 256)
    out, lse = gqa.fwd_host(q, k, v, fp32_path="tc")
    ref_out, ref_lse = oracle.attention(q, k, v)
    assert_close(out, lse, ref_out, ref_lse, F32, "fwd_host")


def test_config_branches_after_state(cuda_device):
    S, nb, bl = 30_468, 8, 256
    q, k, v = inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    rows = inputs.sample_rows(nb * bl, 256, boundaries=range(0, nb * bl, bl))
    _check(q, k, v, rows=rows, mask_kind="prefix_branch", q_pos_offset=S, seg_q=seg_q, seg_kv=seg_kv,
           what="8 branches after 30,468")


def test_config_causal_60926(cuda_device):
    L = 60_926
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256)
    _check(q, k, v, rows=inputs.sample_rows(L, 2048), what="L=60,926 tc")


def test_segmented_1m(cuda_device):
    """1,048,576 fp32 tokens packed from the seeded segments: plane offsets past 2^32
    bytes (64-bit indexing in the split kernels and the tensor maps), the block-skip
    plan at 1M; 512 sampled rows against the oracle on their segment's keys."""
    L = 1_048_576
    lengths = inputs.segment_lengths(L)
    ids = inputs.segment_ids(lengths)
    dev = torch.device("cuda")
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, device=dev)
    tid = torch.as_tensor(ids, device=dev)
    out, lse = _run(q, k, v, seg_q=tid, seg_kv=tid)
    starts = np.concatenate([[0], np.cumsum(lengths)[:-1]])
    rows = inputs.sample_rows(L, 512, boundaries=starts)
    for a, n in zip(starts, lengths):
        rel = rows[(rows >= a) & (rows < a + n)] - a
        if rel.size == 0:
            continue
        sl = slice(int(a), int(a + n))
        ref_out, ref_lse = oracle.attention(q[:, :, sl], k[:, :, sl], v[:, :, sl], rows=rel)
        sel = torch.as_tensor(a + rel, device=dev)
        assert_close(out[:, :, sel], lse[:, :, sel], ref_out, ref_lse, F32, f"segment at {a}")
