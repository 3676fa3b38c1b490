"""Pins of the backward oracle (oracle/backward.py) without the CUDA path.

* Library special case: torch.autograd through an explicit float64 forward (scores,
  mask, softmax, P @ V, K/V repeated per query head) on small shapes and every mask.
* Brute force: central finite differences of sum(out * dout) on tiny inputs.
* Invariants: key gradients of each key/value head sum to zero (the softmax's
  derivative sums to zero along each row); value gradients sum to the upstream
  gradient of rows that see a key; grouped heads equal repeated key/value heads
  with the gradients summed per group; rows without visible keys get dq = 0.
"""

import math

import numpy as np
import pytest
import torch

import oracle

MASKS = [
    dict(),
    dict(q_pos_offset=9),
    dict(seg=[0] * 11 + [1] * 17 + [2] * 9),
    dict(prefix=(14, 3)),
]


def _case(seed, B=2, Hq=4, Hkv=2, Lq=37, d=16, q_pos_offset=0, seg=None, prefix=None):
    rng = np.random.default_rng(seed)
    kw = dict(mask_kind=oracle.MASK_CAUSAL, q_pos_offset=q_pos_offset)
    if prefix is not None:
        S, nb = prefix
        bl = Lq // nb
        Lq = nb * bl
        kw = dict(mask_kind=oracle.MASK_PREFIX_BRANCH, q_pos_offset=S,
                  seg_q=np.repeat(np.arange(nb), bl), seg_kv=np.concatenate([-np.ones(S, int), np.repeat(np.arange(nb), bl)]))
    elif seg is not None:
        kw.update(seg_q=np.asarray(seg), seg_kv=np.asarray(seg))
        Lq = len(seg)
    Lk = kw["q_pos_offset"] + Lq
    q = rng.standard_normal((B, Hq, Lq, d))
    k = rng.standard_normal((B, Hkv, Lk, d))
    v = rng.standard_normal((B, Hkv, Lk, d))
    do = rng.standard_normal((B, Hq, Lq, d))
    return q, k, v, do, kw


def _torch_grads(q, k, v, do, kw):
    Hq, Hkv = q.shape[1], k.shape[1]
    Lq, Lk = q.shape[2], k.shape[2]
    vis = torch.as_tensor(oracle.visible(np.arange(Lq), Lk, **{x: kw[x] for x in kw}))
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    kk = tk.repeat_interleave(Hq // Hkv, dim=1)
    vv = tv.repeat_interleave(Hq // Hkv, dim=1)
    s = (tq @ kk.transpose(-1, -2)) / math.sqrt(q.shape[-1])
    s = s.masked_fill(~vis, float("-inf"))
    p = torch.softmax(s, dim=-1).nan_to_num(0.0)  # rows with no visible key: p = 0
    out = p @ vv
    (out * torch.tensor(do)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("mask", MASKS, ids=["causal", "offset", "segments", "prefix_branch"])
def test_matches_autograd(mask):
    q, k, v, do, kw = _case(1, **mask)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, **kw)
    tq, tk, tv = _torch_grads(q, k, v, do, kw)
    for a, b, n in ((dq, tq, "dq"), (dk, tk, "dk"), (dv, tv, "dv")):
        assert np.max(np.abs(a - b)) < 1e-11, n


def test_matches_finite_differences():
    q, k, v, do, kw = _case(2, B=1, Hq=2, Hkv=1, Lq=5, d=4, q_pos_offset=2)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, **kw)

    def f(q, k, v):
        out, _ = oracle.attention(q, k, v, **kw)
        return float(np.sum(out * do))

    h = 1e-6
    for x, g, idx in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[pos] += h
            xm[pos] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[idx], args_m[idx] = xp, xm
            num[pos] = (f(*args_p) - f(*args_m)) / (2 * h)
        assert np.max(np.abs(num - g)) < 1e-7, idx


@pytest.mark.parametrize("mask", MASKS, ids=["causal", "offset", "segments", "prefix_branch"])
def test_key_gradients_sum_to_zero_and_value_gradients_to_dout(mask):
    q, k, v, do, kw = _case(3, **mask)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, **kw)
    B, Hq, Lq, _ = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    seen = oracle.visible(np.arange(Lq), Lk, **kw).any(axis=1)
    assert np.max(np.abs(dk.sum(axis=2))) < 1e-11
    want = np.stack([do[:, g * G:(g + 1) * G][:, :, seen].sum(axis=(1, 2)) for g in range(Hkv)], axis=1)
    assert np.max(np.abs(dv.sum(axis=2) - want)) < 1e-11


def test_grouped_heads_equal_repeated_heads_summed():
    q, k, v, do, kw = _case(4, Hq=6, Hkv=2)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, **kw)
    kr, vr = np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1)
    dq2, dk2, dv2 = oracle.attention_backward(q, kr, vr, do, **kw)
    assert np.max(np.abs(dq - dq2)) < 1e-12
    assert np.max(np.abs(dk - dk2.reshape(2, 2, 3, *dk2.shape[2:]).sum(axis=2))) < 1e-12
    assert np.max(np.abs(dv - dv2.reshape(2, 2, 3, *dv2.shape[2:]).sum(axis=2))) < 1e-12


def test_rows_without_visible_keys_get_zero_gradient():
    seg_q = np.array([5] * 4 + [1] * 8)
    seg_kv = np.array([1] * 12)
    q, k, v, do, _ = _case(5, B=1, Hq=2, Hkv=1, Lq=12, d=8)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, seg_q=seg_q, seg_kv=seg_kv)
    assert np.all(dq[:, :, :4] == 0)
    assert np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))
