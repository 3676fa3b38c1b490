"""Pins for the CPU oracle: library routines, closed forms, invariants, page figures.

Nothing here compares the oracle with itself retyped.  The pins are:

* torch's CPU scaled-dot-product attention in float64 (an independent library
  implementation: ``is_causal``, ``enable_gqa`` and its flash routine's LSE);
* closed forms (row 0, zero queries, identical keys, constant values, key shift);
* invariants the pages imply (GQA equals explicitly repeated K/V; constant
  segment ids equal no segment ids; branch rows equal a causal pass over
  state + branch; appending tokens leaves earlier rows unchanged);
* the memory figures printed on the pages (tests/golden/memory_figures.txt).

Plus planted mistakes: each pin must fail on an oracle with a typical bug.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import exact as oatt
from oracle import memory as omem
from oracle.plan import FULL, PARTIAL, SKIP, tile_plan

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def _sdpa(q, k, v, causal=True, gqa=True):
    """torch CPU float64 SDPA: (out, lse) with K/V repeated per head for the LSE call."""
    out = F.scaled_dot_product_attention(q, k, v, is_causal=causal, enable_gqa=gqa)
    G = q.shape[1] // k.shape[1]
    kr, vr = k.repeat_interleave(G, 1), v.repeat_interleave(G, 1)
    o2, lse = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(q, kr, vr, 0.0, causal)
    assert torch.allclose(o2, out, atol=1e-13, rtol=0)
    return out.numpy(), lse.numpy()


# --------------------------------------------------------------------------- library
@pytest.mark.parametrize("B,Hq,Hkv,L,d", [(1, 16, 4, 37, 16), (2, 8, 2, 64, 32), (1, 4, 4, 9, 8),
                                          (1, 16, 4, 70, 256)])
def test_causal_gqa_matches_torch_sdpa(B, Hq, Hkv, L, d):
    q, k, v = _rand((B, Hq, L, d), 1), _rand((B, Hkv, L, d), 2), _rand((B, Hkv, L, d), 3)
    ref_out, ref_lse = _sdpa(q, k, v)
    out, lse = oracle.attention(q, k, v)
    np.testing.assert_allclose(out, ref_out, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12, rtol=0)


def test_offset_rows_equal_last_rows_of_full_causal_pass():
    """Query rows after ``q_pos_offset`` keys = last rows of a causal pass over all keys."""
    Hq, Hkv, S, Lq, d = 8, 2, 40, 13, 16
    q_all = _rand((1, Hq, S + Lq, d), 4)
    k, v = _rand((1, Hkv, S + Lq, d), 5), _rand((1, Hkv, S + Lq, d), 6)
    ref_out, ref_lse = _sdpa(q_all, k, v)
    out, lse = oracle.attention(q_all[:, :, S:], k, v, q_pos_offset=S)
    np.testing.assert_allclose(out, ref_out[:, :, S:], atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, ref_lse[:, :, S:], atol=1e-12, rtol=0)


def test_prefix_branch_rows_equal_causal_over_state_plus_branch():
    """Packed branches (system1-omni issue #27, item 3) = one causal pass per branch."""
    Hq, Hkv, S, nb, bl, d = 8, 2, 50, 3, 7, 16
    qb = _rand((1, Hq, nb * bl, d), 7)
    ks, vs = _rand((1, Hkv, S, d), 8), _rand((1, Hkv, S, d), 9)
    kb, vb = _rand((1, Hkv, nb * bl, d), 10), _rand((1, Hkv, nb * bl, d), 11)
    seg_q = np.repeat(np.arange(nb), bl)
    seg_kv = np.concatenate([np.full(S, -7), seg_q])
    out, lse = oracle.attention(qb, torch.cat([ks, kb], 2), torch.cat([vs, vb], 2),
                                mask_kind=oracle.MASK_PREFIX_BRANCH, q_pos_offset=S,
                                seg_q=seg_q, seg_kv=seg_kv)
    for b in range(nb):
        sl = slice(b * bl, (b + 1) * bl)
        q_full = torch.cat([torch.zeros(1, Hq, S, d, dtype=torch.float64), qb[:, :, sl]], 2)
        ref_out, ref_lse = _sdpa(q_full, torch.cat([ks, kb[:, :, sl]], 2), torch.cat([vs, vb[:, :, sl]], 2))
        np.testing.assert_allclose(out[:, :, sl], ref_out[:, :, S:], atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[:, :, sl], ref_lse[:, :, S:], atol=1e-12, rtol=0)


def test_segments_equal_standalone_causal_calls():
    """Block-causal packing (maxtext PR #4929): each segment = a causal call on it alone."""
    Hq, Hkv, d = 8, 2, 16
    lengths = [5, 1, 17, 9]
    L = sum(lengths)
    q, k, v = _rand((1, Hq, L, d), 12), _rand((1, Hkv, L, d), 13), _rand((1, Hkv, L, d), 14)
    ids = np.repeat(np.arange(len(lengths)) * 3 + 1, lengths)
    out, lse = oracle.attention(q, k, v, seg_q=ids, seg_kv=ids)
    a = 0
    for n in lengths:
        sl = slice(a, a + n)
        ref_out, ref_lse = _sdpa(q[:, :, sl], k[:, :, sl], v[:, :, sl])
        np.testing.assert_allclose(out[:, :, sl], ref_out, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[:, :, sl], ref_lse, atol=1e-12, rtol=0)
        a += n


# --------------------------------------------------------------------------- closed forms
def test_row_zero_sees_only_key_zero():
    d = 256
    q, k, v = _rand((1, 16, 20, d), 15), _rand((1, 4, 20, d), 16), _rand((1, 4, 20, d), 17)
    out, lse = oracle.attention(q, k, v, rows=[0])
    for h in range(16):
        g = h // 4
        np.testing.assert_array_equal(out[0, h, 0], v[0, g, 0].numpy())
        assert abs(lse[0, h, 0] - float(q[0, h, 0] @ k[0, g, 0]) / 16.0) < 1e-12


def test_zero_queries_give_uniform_weights():
    """Q = 0: every visible key has weight 1/(p+1); LSE = ln(p+1); out = prefix mean of V."""
    L, d = 33, 256
    q = torch.zeros(1, 16, L, d, dtype=torch.float64)
    k, v = _rand((1, 4, L, d), 18), _rand((1, 4, L, d), 19)
    out, lse = oracle.attention(q, k, v)
    n = np.arange(1, L + 1, dtype=np.float64)
    for h in range(16):
        mean = np.cumsum(v[0, h // 4].numpy(), axis=0) / n[:, None]
        np.testing.assert_allclose(out[0, h], mean, atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse[0, h], np.log(n), atol=1e-14, rtol=0)


def test_identical_keys_shift_lse_by_the_common_score():
    """All keys equal to c: uniform weights; LSE = q.c/16 + ln(p+1)."""
    L, d = 21, 256
    q = _rand((1, 16, L, d), 20)
    c = _rand((d,), 21)
    k = c.expand(1, 4, L, d).contiguous()
    v = _rand((1, 4, L, d), 22)
    out, lse = oracle.attention(q, k, v)
    n = np.arange(1, L + 1, dtype=np.float64)
    for h in range(16):
        expect = (q[0, h].numpy() @ c.numpy()) / 16.0 + np.log(n)
        np.testing.assert_allclose(lse[0, h], expect, atol=1e-12, rtol=0)
        mean = np.cumsum(v[0, h // 4].numpy(), axis=0) / n[:, None]
        np.testing.assert_allclose(out[0, h], mean, atol=1e-12, rtol=0)


def test_constant_values_pass_through():
    L, d = 25, 256
    q, k = _rand((1, 16, L, d), 23) * 4, _rand((1, 4, L, d), 24)
    row = _rand((d,), 25)
    v = row.expand(1, 4, L, d).contiguous()
    out, _ = oracle.attention(q, k, v)
    np.testing.assert_allclose(out[0], np.broadcast_to(row.numpy(), out[0].shape), atol=1e-12, rtol=0)


def test_key_shift_moves_lse_and_keeps_out():
    L, d = 19, 256
    q, k, v = _rand((1, 16, L, d), 26), _rand((1, 4, L, d), 27), _rand((1, 4, L, d), 28)
    c = _rand((d,), 29)
    o1, l1 = oracle.attention(q, k, v)
    o2, l2 = oracle.attention(q, k + c, v)
    np.testing.assert_allclose(o2, o1, atol=1e-12, rtol=0)
    for h in range(16):
        np.testing.assert_allclose(l2[0, h] - l1[0, h], q[0, h].numpy() @ c.numpy() / 16.0,
                                   atol=1e-12, rtol=0)


def test_tiny_case_by_explicit_loops():
    """L=5, d=3, one head: the softmax written out with Python floats and math.exp."""
    q = [[0.3, -1.0, 2.0], [1.5, 0.2, -0.7], [0.0, 0.0, 1.0], [-2.0, 1.0, 0.5], [0.9, 0.9, 0.9]]
    k = [[1.0, 0.0, -1.0], [0.5, 2.0, 0.0], [-1.0, -1.0, 1.0], [0.0, 3.0, 1.0], [2.0, -0.5, 0.25]]
    v = [[1.0, 2.0, 3.0], [-1.0, 0.0, 1.0], [0.5, 0.5, -0.5], [4.0, -2.0, 0.0], [0.0, 1.0, 1.0]]
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64)[None, None] for x in (q, k, v))
    out, lse = oracle.attention(qt, kt, vt)
    sc = 1.0 / math.sqrt(3.0)
    for i in range(5):
        w = [math.exp(sc * sum(a * b for a, b in zip(q[i], k[j]))) for j in range(i + 1)]
        z = sum(w)
        for c in range(3):
            assert abs(out[0, 0, i, c] - sum(w[j] * v[j][c] for j in range(i + 1)) / z) < 1e-13
        assert abs(lse[0, 0, i] - math.log(z)) < 1e-13


# --------------------------------------------------------------------------- invariants
def test_gqa_equals_repeated_kv():
    """kev PR #202, "Test plan": repeating K/V per query head gives the same outputs."""
    L, d = 45, 64
    q, k, v = _rand((1, 16, L, d), 30), _rand((1, 4, L, d), 31), _rand((1, 4, L, d), 32)
    o1, l1 = oracle.attention(q, k, v)
    o2, l2 = oracle.attention(q, k.repeat_interleave(4, 1), v.repeat_interleave(4, 1))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_constant_segment_ids_equal_no_segments():
    """maxtext PR #4929: with one segment the ids are constant and change nothing."""
    L, d = 40, 32
    q, k, v = _rand((1, 8, L, d), 33), _rand((1, 2, L, d), 34), _rand((1, 2, L, d), 35)
    ids = np.full(L, 7)
    o1, l1 = oracle.attention(q, k, v)
    o2, l2 = oracle.attention(q, k, v, seg_q=ids, seg_kv=ids)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_appending_tokens_leaves_earlier_rows_unchanged():
    L, extra, d = 30, 11, 32
    q, k, v = _rand((1, 8, L + extra, d), 36), _rand((1, 2, L + extra, d), 37), _rand((1, 2, L + extra, d), 38)
    o1, l1 = oracle.attention(q[:, :, :L], k[:, :, :L], v[:, :, :L])
    o2, l2 = oracle.attention(q, k, v)
    np.testing.assert_allclose(o2[:, :, :L], o1, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l2[:, :, :L], l1, atol=1e-13, rtol=0)


def test_probability_rows_sum_to_one_and_reproduce_out():
    L, d = 50, 32
    q, k, v = _rand((1, 8, L, d), 39) * 3, _rand((1, 2, L, d), 40), _rand((1, 2, L, d), 41)
    ids = np.repeat([0, 1, 2], [10, 25, 15])
    out, _ = oracle.attention(q, k, v, seg_q=ids, seg_kv=ids)
    for h, row in [(0, 0), (3, 17), (7, 49), (5, 10)]:
        p = oracle.probabilities(q, k, b=0, h=h, row=row, seg_q=ids, seg_kv=ids)
        assert abs(p.sum() - 1.0) <= 1e-12
        vis = oracle.visible([row], L, seg_q=ids, seg_kv=ids)[0]
        assert np.all(p[~vis] == 0)
        np.testing.assert_allclose(p @ v[0, h // 4].numpy(), out[0, h, row], atol=1e-12, rtol=0)


def test_rows_without_visible_keys():
    """A query whose segment has no key at or before it: out = 0, LSE = -inf."""
    L, d = 12, 16
    q, k, v = _rand((1, 4, L, d), 42), _rand((1, 1, L, d), 43), _rand((1, 1, L, d), 44)
    seg_q = np.array([5] * 6 + [1] * 6)
    seg_kv = np.array([1] * 6 + [5] * 6)
    out, lse = oracle.attention(q, k, v, seg_q=seg_q, seg_kv=seg_kv)
    assert np.all(out[:, :, :6] == 0) and np.all(np.isneginf(lse[:, :, :6]))
    assert np.all(np.isfinite(lse[:, :, 6:]))


def test_sampled_rows_equal_full_rows():
    L, d = 77, 32
    q, k, v = _rand((1, 8, L, d), 45), _rand((1, 2, L, d), 46), _rand((1, 2, L, d), 47)
    rows = np.array([0, 3, 40, 41, 76])
    of, lf = oracle.attention(q, k, v)
    os_, ls = oracle.attention(q, k, v, rows=rows, chunk=2)
    # BLAS may block a different number of rows differently: equal up to rounding
    np.testing.assert_allclose(os_, of[:, :, rows], atol=1e-13, rtol=0)
    np.testing.assert_allclose(ls, lf[:, :, rows], atol=1e-13, rtol=0)


# --------------------------------------------------------------------------- planted bugs
def test_pins_catch_planted_mistakes(monkeypatch):
    """Each typical oracle bug makes at least one library pin fail."""
    q, k, v = _rand((1, 16, 24, 16), 48), _rand((1, 4, 24, 16), 49), _rand((1, 4, 24, 16), 50)
    ref_out, ref_lse = _sdpa(q, k, v)

    def fails(**kw):
        out, lse = oracle.attention(q, k, v, **kw)
        return not (np.allclose(out, ref_out, atol=1e-9) and np.allclose(lse, ref_lse, atol=1e-9))

    assert not fails()
    assert fails(scale=1.0)                     # missing 1/sqrt(d)
    assert fails(q_pos_offset=0, rows=None, seg_q=None, scale=0.5)
    # wrong causal alignment (one position late): emulate via an extra leading key
    real_visible = oatt.visible

    def late(rows, Lk, **kw):
        kw["q_pos_offset"] = kw.get("q_pos_offset", 0) + 1
        return real_visible(rows, Lk, **kw)

    monkeypatch.setattr(oatt, "visible", late)
    assert fails()
    monkeypatch.setattr(oatt, "visible", real_visible)
    # interleaved head mapping (h % Hkv instead of h // G)
    out_bad = np.stack([oracle.attention(q[:, h:h + 1], k[:, h % 4:h % 4 + 1], v[:, h % 4:h % 4 + 1])[0][:, 0]
                        for h in range(16)], 1)
    assert not np.allclose(out_bad, ref_out, atol=1e-9)


# --------------------------------------------------------------------------- memory figures
def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "memory_figures.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, args, value, unit, rnd, src = line.rstrip("\n").split("\t")
            kw = {a.split("=")[0]: int(a.split("=")[1]) for a in args.split()}
            rows.append((name, kw, float(value), unit, int(rnd), src))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: r[0] + " " + str(r[1]))
def test_memory_closed_forms_match_page_figures(row):
    name, kw, value, unit, rnd, _src = row
    if name == "score_matrix_bytes":
        got = omem.score_matrix_bytes(kw["Hq"], kw["L"], kw["elem"])
    elif name == "repeated_kv_bytes":
        got = omem.repeated_kv_bytes(kw["Hq"], kw["L"], kw["d"], kw["elem"])
    else:
        got = omem.block_pair_table_bytes(kw["L"], kw["block"], kw["elem"])
    div = {"GB": 1e9, "GiB": 2.0 ** 30, "B": 1.0}[unit]
    assert round(got / div, rnd) == value


def test_oom_allocation_is_one_score_matrix_in_the_30k_range():
    """kev PR #202, "End to end": "Tried to allocate 55.00 GiB" = one 16 x 30k^2 fp32 matrix."""
    hits = [L for L in range(30000, 31000) if round(omem.score_matrix_bytes(16, L) / 2 ** 30, 2) == 55.00]
    assert hits and all(30000 <= L < 31000 for L in hits)


def test_linear_memory_bar_is_below_the_math_path():
    for L in (512, 22_500, 60_926, 1_048_576):
        assert omem.quarter_score_matrix_per_head_bytes(L) < omem.score_matrix_bytes(16, L)


# --------------------------------------------------------------------------- tile plan
def _brute_classes(Lq, Lk, Br, Bc, **kw):
    vis = oracle.visible(np.arange(Lq), Lk, **kw)
    nq, nk = -(-Lq // Br), -(-Lk // Bc)
    out = np.zeros((nq, nk), np.uint8)
    for a in range(nq):
        for b in range(nk):
            t = vis[a * Br:(a + 1) * Br, b * Bc:(b + 1) * Bc]
            out[a, b] = FULL if t.all() else (SKIP if not t.any() else PARTIAL)
    return out


def _plan_cases():
    rng = np.random.default_rng(0)
    cases = []
    for Lq, off, Br, Bc in [(37, 0, 4, 8), (64, 0, 16, 16), (50, 13, 8, 4), (129, 0, 32, 64), (1, 0, 16, 16),
                            (63, 1, 16, 32), (200, 56, 8, 16)]:
        cases.append(dict(Lq=Lq, off=off, Br=Br, Bc=Bc, kind=0, seg=None))
        L = Lq + off
        lens = []
        while sum(lens) < L:
            lens.append(int(rng.integers(1, 20)))
        ids = np.repeat(np.arange(len(lens)), lens)[:L]
        cases.append(dict(Lq=Lq, off=off, Br=Br, Bc=Bc, kind=0, seg=("packed", ids)))
        cases.append(dict(Lq=Lq, off=off, Br=Br, Bc=Bc, kind=0, seg=("random", rng.integers(-2, 3, L))))
        if off > 0:
            nb = 3
            bq = np.sort(rng.integers(0, nb, Lq))
            cases.append(dict(Lq=Lq, off=off, Br=Br, Bc=Bc, kind=1,
                              seg=("branch", np.concatenate([rng.integers(-5, 5, off), bq]))))
    return cases


@pytest.mark.parametrize("case", _plan_cases())
def test_plan_is_sound_by_brute_force(case):
    Lq, off, Br, Bc, kind = case["Lq"], case["off"], case["Br"], case["Bc"], case["kind"]
    L = Lq + off
    seg = case["seg"]
    kw = dict(mask_kind=kind, q_pos_offset=off)
    if seg is not None:
        ids = seg[1]
        kw.update(seg_q=ids[off:] if kind == 0 else ids[off:], seg_kv=ids)
    classes, ranges = tile_plan(Lq, L, Br, Bc, **kw)
    truth = _brute_classes(Lq, L, Br, Bc, **kw)
    # SKIP only where nothing is visible; FULL only where everything is visible.
    assert np.all(truth[classes == SKIP] == SKIP)
    assert np.all(truth[classes == FULL] == FULL)
    # every tile holding a visible pair lies inside its row's range
    for a in range(classes.shape[0]):
        nz = np.nonzero(truth[a] != SKIP)[0]
        if nz.size:
            assert ranges[a, 0] <= nz.min() and nz.max() < ranges[a, 1]
        else:
            assert tuple(ranges[a]) == (0, 0)
    if seg is None or seg[0] == "packed":
        # tight for no ids and for packed nondecreasing ids: PARTIAL holds some visible pair
        assert np.all(truth[classes == PARTIAL] != SKIP)
        if seg is None:
            np.testing.assert_array_equal(classes, truth)


def test_plan_causal_square_tiles_is_the_triangle():
    classes, ranges = tile_plan(256, 256, 64, 64)
    expect = np.where(np.tri(4, 4, -1, dtype=bool), FULL, SKIP).astype(np.uint8)
    np.fill_diagonal(expect, PARTIAL)
    np.testing.assert_array_equal(classes, expect)
    np.testing.assert_array_equal(ranges, [[0, 1], [0, 2], [0, 3], [0, 4]])
