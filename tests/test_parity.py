"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes and the fp32 configurations up to the 30,468-token state (with its 8
branches) compare every row; the 60,926- and 1,048,576-token configurations compare
seeded sampled rows (always the first and last row of every segment or branch).
Invariants (GQA = repeated K/V, constant ids = no ids, prefix invariance, each
segment = a standalone call, branches = single-branch calls) run on the GPU too.
"""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
import oracle
from long_context_causal_flash_b200 import inputs
from tests._helpers import TOL, assert_close

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16]


def _run(q, k, v, **kw):
    out, lse = gqa.fwd(q, k, v, **kw)
    torch.cuda.synchronize()
    return out, lse


def _ids(x, dev):
    return None if x is None else torch.as_tensor(np.asarray(x), dtype=torch.int32, device=dev)


def _check(q, k, v, dtype, rows=None, what="", mask_kind="causal", q_pos_offset=0, seg_q=None, seg_kv=None):
    """Run on the GPU, then compare with the oracle on `rows` (all rows by default)."""
    dev = torch.device("cuda")
    out, lse = _run(q.to(dev), k.to(dev), v.to(dev), mask_kind=mask_kind, q_pos_offset=q_pos_offset,
                    seg_q=_ids(seg_q, dev), seg_kv=_ids(seg_kv, dev))
    ref_out, ref_lse = oracle.attention(q, k, v, mask_kind=oracle.MASK_CAUSAL if mask_kind == "causal"
                                        else oracle.MASK_PREFIX_BRANCH, q_pos_offset=q_pos_offset,
                                        seg_q=seg_q, seg_kv=seg_kv, rows=rows)
    sel = slice(None) if rows is None else torch.as_tensor(rows, device=dev)
    return assert_close(out[:, :, sel], lse[:, :, sel], ref_out, ref_lse, dtype, what)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("L", [1, 2, 15, 16, 17, 63, 64, 65, 127, 129, 300, 512])
def test_causal_small_all_rows(cuda_device, dtype, L):
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, what=f"causal L={L}")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("Hq,Hkv", [(16, 16), (16, 8), (16, 2), (16, 1), (8, 4)])
def test_group_sizes(cuda_device, dtype, Hq, Hkv):
    q, k, v = inputs.qkv(1, Hq, Hkv, 150, 150, 256, dtype=dtype)
    _check(q, k, v, dtype, what=f"Hq={Hq} Hkv={Hkv}")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("Hq,Hkv,L", [(16, 1, 700), (16, 16, 600), (16, 4, 1100)])
def test_group_sizes_many_tiles(cuda_device, dtype, Hq, Hkv, L):
    """Several key tiles and query tiles with a ragged end for the smallest and largest
    groups (G = 16: 4 positions per fp32 query tile; G = 1: 64)."""
    q, k, v = inputs.qkv(1, Hq, Hkv, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, what=f"Hq={Hq} Hkv={Hkv} L={L}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_batch_and_gqa_equals_repeated_kv(cuda_device, dtype):
    q, k, v = inputs.qkv(2, 16, 4, 200, 200, 256, dtype=dtype)
    _check(q, k, v, dtype, what="B=2")
    dev = torch.device("cuda")
    o1, l1 = _run(q.to(dev), k.to(dev), v.to(dev))
    o2, l2 = _run(q.to(dev), k.repeat_interleave(4, 1).to(dev), v.repeat_interleave(4, 1).to(dev))
    assert_close(o1, l1, o2.double(), l2.double(), dtype, "GQA vs repeated K/V")


@pytest.mark.parametrize("dtype", DTYPES)
def test_large_logits(cuda_device, dtype):
    """Scores with std 8 exercise the running-max rescale.  The fp32 rounding of a
    256-term dot product grows with the size of its terms, so the bound of the unit-
    variance configurations is scaled by the logit scale (8) here."""
    q, k, v = inputs.qkv(1, 16, 4, 333, 333, 256)
    q = q * 8
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    dev = torch.device("cuda")
    out, lse = _run(q.to(dev), k.to(dev), v.to(dev))
    ref_out, ref_lse = oracle.attention(q, k, v)
    tol_out, tol_lse = TOL[dtype]
    d_out = float((out.double().cpu() - torch.from_numpy(ref_out)).abs().max())
    d_lse = float((lse.double().cpu() - torch.from_numpy(ref_lse)).abs().max())
    assert d_out <= 8 * tol_out and d_lse <= 8 * tol_lse, (d_out, d_lse)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("S,Lq", [(200, 100), (64, 64), (1, 70), (1000, 1)])
def test_query_rows_after_a_state(cuda_device, dtype, S, Lq):
    q, k, v = inputs.qkv(1, 16, 4, Lq, S + Lq, 256, dtype=dtype)
    _check(q, k, v, dtype, q_pos_offset=S, what=f"offset {S}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_prefix_branch_small(cuda_device, dtype):
    S, nb, bl = 300, 3, 40
    q, k, v = inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256, dtype=dtype)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    _check(q, k, v, dtype, mask_kind="prefix_branch", q_pos_offset=S, seg_q=seg_q, seg_kv=seg_kv,
           what="prefix branch")
    # each branch equals a causal call over [state | that branch]
    dev = torch.device("cuda")
    ob, lb = _run(q.to(dev), k.to(dev), v.to(dev), mask_kind="prefix_branch", q_pos_offset=S,
                  seg_q=_ids(seg_q, dev), seg_kv=_ids(seg_kv, dev))
    for b in range(nb):
        sl = slice(b * bl, (b + 1) * bl)
        kk = torch.cat([k[:, :, :S], k[:, :, S + b * bl:S + (b + 1) * bl]], 2).to(dev)
        vv = torch.cat([v[:, :, :S], v[:, :, S + b * bl:S + (b + 1) * bl]], 2).to(dev)
        o1, l1 = _run(q[:, :, sl].contiguous().to(dev), kk, vv, q_pos_offset=S)
        assert_close(ob[:, :, sl], lb[:, :, sl], o1.double(), l1.double(), dtype, f"branch {b}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_segments_small(cuda_device, dtype):
    lengths = [1, 70, 5, 200, 64, 33]
    L = sum(lengths)
    ids = inputs.segment_ids(lengths)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, seg_q=ids, seg_kv=ids, what="segments")


@pytest.mark.parametrize("dtype", DTYPES)
def test_unsorted_segment_ids(cuda_device, dtype):
    rng = np.random.default_rng(11)
    L = 257
    ids = rng.integers(0, 3, L).astype(np.int32)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, seg_q=ids, seg_kv=ids, what="unsorted ids")


@pytest.mark.parametrize("dtype", DTYPES)
def test_rows_without_visible_keys(cuda_device, dtype):
    L = 160
    seg_q = np.array([7] * 80 + [1] * 80, dtype=np.int32)
    seg_kv = np.array([1] * 80 + [7] * 80, dtype=np.int32)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, seg_q=seg_q, seg_kv=seg_kv, what="empty rows")


@pytest.mark.parametrize("dtype", DTYPES)
def test_constant_ids_equal_no_ids_bitwise(cuda_device, dtype):
    L = 777
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    ids = torch.full((L,), 3, dtype=torch.int32, device=dev)
    o1, l1 = _run(q, k, v)
    o2, l2 = _run(q, k, v, seg_q=ids, seg_kv=ids)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("dtype", DTYPES)
def test_appending_tokens_keeps_earlier_rows(cuda_device, dtype):
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, 640, 640, 256, dtype=dtype))
    o1, l1 = _run(q[:, :, :512].contiguous(), k[:, :, :512].contiguous(), v[:, :, :512].contiguous())
    o2, l2 = _run(q, k, v)
    # same tiles for the first 512 rows: identical bits
    assert torch.equal(o1, o2[:, :, :512]) and torch.equal(l1, l2[:, :, :512])


@pytest.mark.parametrize("dtype", DTYPES)
def test_each_segment_equals_a_standalone_call(cuda_device, dtype):
    lengths = [100, 37, 300]
    L = sum(lengths)
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype))
    ids = _ids(inputs.segment_ids(lengths), dev)
    o, l = _run(q, k, v, seg_q=ids, seg_kv=ids)
    a = 0
    for n in lengths:
        sl = slice(a, a + n)
        o1, l1 = _run(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous())
        assert_close(o[:, :, sl], l[:, :, sl], o1.double(), l1.double(), dtype, f"segment at {a}")
        a += n


# ------------------------------------------------------------------ benchmark configurations
def _sampled_check(L, n_rows, dtype, what):
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    rows = inputs.sample_rows(L, n_rows)
    return _check(q, k, v, dtype, rows=rows, what=what)


def test_config_causal_512_f32_all_rows(cuda_device):
    q, k, v = inputs.qkv(1, 16, 4, 512, 512, 256)
    _check(q, k, v, torch.float32, what="L=512")


def test_config_causal_15231_f32_all_rows(cuda_device):
    """Every one of the 15,231 rows (all 952 query tiles) against the oracle."""
    q, k, v = inputs.qkv(1, 16, 4, 15_231, 15_231, 256)
    _check(q, k, v, torch.float32, what="L=15,231 all rows")


def test_config_state_30468_f32_all_rows(cuda_device):
    """The state pass of the shared-prefix configuration, every row."""
    q, k, v = inputs.qkv(1, 16, 4, 30_468, 30_468, 256)
    _check(q, k, v, torch.float32, what="state L=30,468 all rows")


def test_config_branches_after_state_f32_all_rows(cuda_device):
    """8 branches of 256 rows after the 30,468-token state, every branch row."""
    S, nb, bl = 30_468, 8, 256
    q, k, v = inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    _check(q, k, v, torch.float32, mask_kind="prefix_branch", q_pos_offset=S, seg_q=seg_q, seg_kv=seg_kv,
           what="8 branches after 30,468, all rows")


def test_config_causal_60926_f32(cuda_device):
    _sampled_check(60_926, 4096, torch.float32, "L=60,926 fp32")


def test_config_causal_60926_bf16(cuda_device):
    _sampled_check(60_926, 4096, torch.bfloat16, "L=60,926 bf16")


def _big_bf16_inputs(L):
    return inputs.qkv(1, 16, 4, L, L, 256, dtype=torch.bfloat16, device="cuda")


def test_config_segmented_1m_bf16(cuda_device):
    """1,048,576 tokens packed from seeded segments of 1k-256k tokens; 2,048 sampled rows.

    Keys of other segments are invisible by definition, so the oracle runs on each
    segment's window of keys (the same definition, without the exp(-inf) = 0 terms)."""
    L = 1_048_576
    lengths = inputs.segment_lengths(L)
    ids = inputs.segment_ids(lengths)
    q, k, v = _big_bf16_inputs(L)
    tid = torch.as_tensor(ids, device="cuda")
    out, lse = _run(q, k, v, seg_q=tid, seg_kv=tid)
    starts = np.concatenate([[0], np.cumsum(lengths)[:-1]])
    rows = inputs.sample_rows(L, 2048, boundaries=starts)
    worst = (0.0, 0.0)
    for a, n in zip(starts, lengths):
        rel = rows[(rows >= a) & (rows < a + n)] - a
        if rel.size == 0:
            continue
        sl = slice(int(a), int(a + n))
        ref_out, ref_lse = oracle.attention(q[:, :, sl], k[:, :, sl], v[:, :, sl], rows=rel)
        sel = torch.as_tensor(a + rel, device="cuda")
        d = assert_close(out[:, :, sel], lse[:, :, sel], ref_out, ref_lse, torch.bfloat16, f"segment at {a}")
        worst = (max(worst[0], d[0]), max(worst[1], d[1]))
    print("segmented 1M worst |dout|, |dlse|:", worst)


def test_config_constant_ids_1m_bf16(cuda_device):
    """Constant segment ids at 1M equal the non-segmented kernel bit for bit (maxtext
    PR #4929: with one segment the non-segmented kernel gives the same result)."""
    L = 1_048_576
    q, k, v = _big_bf16_inputs(L)
    o1, l1 = _run(q, k, v)
    ids = torch.zeros(L, dtype=torch.int32, device="cuda")
    o2, l2 = _run(q, k, v, seg_q=ids, seg_kv=ids)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    del o2, l2
    rows = inputs.sample_rows(L, 64)
    ref_out, ref_lse = oracle.attention(q, k, v, rows=rows)
    sel = torch.as_tensor(rows, device="cuda")
    assert_close(o1[:, :, sel], l1[:, :, sel], ref_out, ref_lse, torch.bfloat16, "1M causal bf16")


@pytest.mark.parametrize("dtype", DTYPES)
def test_fwd_host_pieces_equal_device_call(cuda_device, dtype):
    """fwd_host cuts the call into (batch entry, key/value head) pieces on three
    streams; the result equals one device call bit for bit, with segment ids too."""
    q, k, v = inputs.qkv(2, 16, 4, 300, 300, 256, dtype=dtype)
    ids = inputs.segment_ids([100, 150, 50])
    dev = torch.device("cuda")
    for kw in ({}, {"seg_q": ids, "seg_kv": ids}):
        hq, hk, hv = (t.pin_memory() for t in (q, k, v))
        out_h, lse_h = gqa.fwd_host(hq, hk, hv, device=dev, **kw)
        dkw = {n: torch.as_tensor(x, device=dev) for n, x in kw.items()}
        out_d, lse_d = gqa.fwd(q.to(dev), k.to(dev), v.to(dev), **dkw)
        torch.cuda.synchronize()
        assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())
