"""Pins of oracle.context (attention against a key block, merge of partial results).

CPU only.  The pins come from outside the functions under test: torch's
scaled_dot_product_attention in float64 (a library routine), the already pinned
oracle.attention, and the log-sum-exp identity checked against unsplit results.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_causal_flash_b200 import inputs


def _sdpa(q, k, v, mask=None):
    """Library reference in float64 with K/V repeated per query head."""
    G = q.shape[1] // k.shape[1]
    q64, k64, v64 = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    k64 = k64.repeat_interleave(G, dim=1)
    v64 = v64.repeat_interleave(G, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(q64, k64, v64, attn_mask=mask)
    s = (q64 @ k64.transpose(-1, -2)) / np.sqrt(q.shape[-1])
    if mask is not None:
        s = s.masked_fill(~mask, float("-inf"))
    return out.numpy(), torch.logsumexp(s, dim=-1).numpy()


def test_fully_visible_block_is_plain_softmax():
    q, k, v = inputs.qkv(1, 8, 2, 37, 50, 256, dtype=torch.float32)
    for off in (50, 51, 400):
        out, lse = oracle.attention_block(q, k, v, q_pos_offset=off)
        ref_out, ref_lse = _sdpa(q, k, v)
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Lq,Lk,off", [(40, 70, 0), (40, 70, 13), (64, 20, 5), (33, 33, 0)])
def test_partial_block_matches_masked_library_attention(Lq, Lk, off):
    q, k, v = inputs.qkv(1, 8, 2, Lq, Lk, 256, dtype=torch.float32)
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lk)[None, :]
    mask = (j <= i + off)[None, None]
    out, lse = oracle.attention_block(q, k, v, q_pos_offset=off)
    ref_out, ref_lse = _sdpa(q, k, v, mask)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_block_at_the_contract_offset_is_attention():
    q, k, v = inputs.qkv(1, 16, 4, 30, 75, 256, dtype=torch.float32)
    out, lse = oracle.attention_block(q, k, v, q_pos_offset=45)
    ref_out, ref_lse = oracle.attention(q, k, v, q_pos_offset=45)
    np.testing.assert_array_equal(out, ref_out)
    np.testing.assert_array_equal(lse, ref_lse)


def test_negative_offset_rejected():
    q, k, v = inputs.qkv(1, 4, 4, 8, 8, 256, dtype=torch.float32)
    with pytest.raises(ValueError):
        oracle.attention_block(q, k, v, q_pos_offset=-1)


@pytest.mark.parametrize("a", [1, 17, 40])
def test_merge_of_a_key_split_equals_the_unsplit_block(a):
    Lq, Lk, off = 30, 60, 45
    q, k, v = inputs.qkv(1, 16, 4, Lq, Lk, 256, dtype=torch.float32)
    oa, la = oracle.attention_block(q, k[:, :, :a], v[:, :, :a], q_pos_offset=off)
    ob, lb = oracle.attention_block(q, k[:, :, a:], v[:, :, a:], q_pos_offset=off - a)
    out, lse = oracle.merge_partials(oa, la, ob, lb)
    ref_out, ref_lse = oracle.attention_block(q, k, v, q_pos_offset=off)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
    # order does not matter
    out2, lse2 = oracle.merge_partials(ob, lb, oa, la)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-14)


def test_merge_with_empty_results():
    rng = np.random.default_rng(0)
    o = rng.standard_normal((2, 3, 256))
    lse = rng.standard_normal((2, 3))
    empty_o, empty_lse = np.zeros_like(o), np.full_like(lse, -np.inf)
    out, l2 = oracle.merge_partials(o, lse, empty_o, empty_lse)
    np.testing.assert_array_equal(out, o)
    np.testing.assert_array_equal(l2, lse)
    out, l2 = oracle.merge_partials(empty_o, empty_lse, empty_o, empty_lse)
    assert np.all(out == 0) and np.all(l2 == -np.inf)


@pytest.mark.parametrize("world", [2, 3])
def test_ring_of_blocks_reproduces_full_attention(world):
    # Contiguous shards of Ls positions; shard r's rows merge the blocks of shards s <= r
    # at offsets (r - s) * Ls, the schedule of the ring; the result is the full attention.
    Ls = 23
    L = world * Ls
    q, k, v = inputs.qkv(1, 8, 2, L, L, 256, dtype=torch.float32)
    ref_out, ref_lse = oracle.attention(q, k, v)
    for r in range(world):
        qr = q[:, :, r * Ls:(r + 1) * Ls]
        out = np.zeros((1, 8, Ls, 256))
        lse = np.full((1, 8, Ls), -np.inf)
        for s in range(r + 1):
            ob, lb = oracle.attention_block(qr, k[:, :, s * Ls:(s + 1) * Ls], v[:, :, s * Ls:(s + 1) * Ls],
                                            q_pos_offset=(r - s) * Ls)
            out, lse = oracle.merge_partials(out, lse, ob, lb)
        np.testing.assert_allclose(out, ref_out[:, :, r * Ls:(r + 1) * Ls], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse[:, :, r * Ls:(r + 1) * Ls], rtol=0, atol=1e-12)


# ---- the block backward: pinned to the whole sequence's backward (itself pinned by
# autograd and finite differences in test_oracle_backward.py)

def _block_grads_sum(q, k, v, out, lse, dout, cuts):
    """Sum of attention_block_backward over the key blocks [c0, c1) of a causal
    sequence (query row i at position i): a block is seen by the query rows from
    position c0 on, which start at the block's first key (offset 0)."""
    L = q.shape[2]
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for c0, c1 in zip(cuts[:-1], cuts[1:]):
        # queries that can see any key of the block: positions >= c0
        qs = slice(c0, L)
        g = oracle.attention_block_backward(q[:, :, qs], k[:, :, c0:c1], v[:, :, c0:c1], out[:, :, qs],
                                            lse[:, :, qs], dout[:, :, qs], q_pos_offset=0)
        dq[:, :, qs] += g[0]
        dk[:, :, c0:c1] += g[1]
        dv[:, :, c0:c1] += g[2]
    return dq, dk, dv


@pytest.mark.parametrize("cuts", [[0, 37], [0, 10, 37], [0, 5, 6, 20, 37], [0, 1, 2, 3, 37]])
@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (2, 2), (4, 1)])
def test_block_gradients_sum_to_the_whole_sequence(cuts, Hq, Hkv):
    L = 37
    q, k, v = inputs.qkv(1, Hq, Hkv, L, L, 8, dtype=torch.float64)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(11), dtype=torch.float64)
    out, lse = oracle.attention(q, k, v)
    got = _block_grads_sum(q.numpy(), k.numpy(), v.numpy(), out, lse, dout.numpy(), cuts)
    want = oracle.attention_backward(q, k, v, dout)
    for g, w, name in zip(got, want, ("dq", "dk", "dv")):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12, err_msg=name)


def test_block_backward_of_a_whole_causal_sequence_is_the_backward():
    q, k, v = inputs.qkv(2, 4, 2, 20, 20, 8, dtype=torch.float64)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(12), dtype=torch.float64)
    out, lse = oracle.attention(q, k, v)
    got = oracle.attention_block_backward(q, k, v, out, lse, dout, q_pos_offset=0)
    want = oracle.attention_backward(q, k, v, dout)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12)


def test_block_backward_wholly_before_the_queries():
    """A block of keys entirely before the query rows (offset >= its length): every key
    visible; against the whole sequence's backward restricted to those keys."""
    L, C = 30, 10  # queries are positions 20..29, the block keys 0..9
    q, k, v = inputs.qkv(1, 4, 2, L, L, 8, dtype=torch.float64)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(13), dtype=torch.float64)
    out, lse = oracle.attention(q, k, v)
    # only query rows 20..29 and key block 0..9
    q2, dout2 = q[:, :, 20:], dout[:, :, 20:]
    g = oracle.attention_block_backward(q2, k[:, :, :C], v[:, :, :C], out[:, :, 20:], lse[:, :, 20:], dout2,
                                        q_pos_offset=20)
    # reference: the whole backward with dout zero outside rows 20..29; dk / dv of keys
    # 0..9 and dq's part from keys 0..9 follow from the block formulas of the whole
    dz = np.zeros(dout.shape)
    dz[:, :, 20:] = dout2.numpy()
    _, dk_w, dv_w = oracle.attention_backward(q, k, v, torch.from_numpy(dz))
    np.testing.assert_allclose(g[1], dk_w[:, :, :C], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g[2], dv_w[:, :, :C], rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.attention_block_backward(q2, k[:, :, :C], v[:, :, :C], out[:, :, 20:], lse[:, :, 20:], dout2,
                                        q_pos_offset=-1)
