"""GPU parity of the attention backward (gqa_attn_bwd) against the fp64 oracle.

The CUDA forward's out and lse feed the CUDA backward, as in training; dq, dk, dv
are compared with oracle.attention_backward on the same inputs.  Tolerances (the
stated targets cover the forward only; these follow from the arithmetic): fp32 runs
every product and sum in fp32 over at most a few thousand terms, so 5e-5 of the
largest gradient; bf16 reads out as bf16 (D = <dout, out> carries its 2^-9 relative
rounding) and rounds the gradients to bf16, so 2e-2 of the largest gradient.  At
full size, properties that hold at any size: each key/value head's key gradients sum
to zero and its value gradients sum to the upstream gradient of its query heads.
"""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
import oracle
from long_context_causal_flash_b200 import inputs
from tests._helpers import to64

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16]
RTOL = {torch.float32: 5e-5, torch.bfloat16: 2e-2}


def _ids(x, dev):
    return None if x is None else torch.as_tensor(np.asarray(x), dtype=torch.int32, device=dev)


def _dout(shape, dtype, seed=7):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


def _check(q, k, v, dtype, what, mask_kind="causal", q_pos_offset=0, seg_q=None, seg_kv=None):
    dev = torch.device("cuda")
    do = _dout(q.shape, dtype)
    kw = dict(mask_kind=mask_kind, q_pos_offset=q_pos_offset, seg_q=_ids(seg_q, dev), seg_kv=_ids(seg_kv, dev))
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    out, lse = gqa.fwd(qd, kd, vd, **kw)
    dq, dk, dv = gqa.bwd(qd, kd, vd, out, lse, dod, **kw)
    torch.cuda.synchronize()
    mk = oracle.MASK_CAUSAL if mask_kind == "causal" else oracle.MASK_PREFIX_BRANCH
    ref = oracle.attention_backward(q, k, v, do, mask_kind=mk, q_pos_offset=q_pos_offset, seg_q=seg_q,
                                    seg_kv=seg_kv)
    for got, want, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
        got = to64(got)
        assert np.all(np.isfinite(got)), f"{what}: non-finite {name}"
        scale = max(1.0, float(np.max(np.abs(want))))
        err = float(np.max(np.abs(got - want)))
        assert err <= RTOL[dtype] * scale, f"{what}: {name} max|d| = {err:.3e} (scale {scale:.2f})"


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 17, 64, 65, 200])
def test_causal(cuda_device, dtype, L):
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, f"causal L={L}")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (16, 2), (16, 1)])
def test_group_sizes_and_batch(cuda_device, dtype, Hq, Hkv):
    q, k, v = inputs.qkv(2, Hq, Hkv, 90, 90, 256, dtype=dtype)
    _check(q, k, v, dtype, f"Hq={Hq} Hkv={Hkv} B=2")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_rows_after_a_state(cuda_device, dtype):
    S, Lq = 150, 70
    q, k, v = inputs.qkv(1, 16, 4, Lq, S + Lq, 256, dtype=dtype)
    _check(q, k, v, dtype, "offset 150", q_pos_offset=S)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_prefix_branch(cuda_device, dtype):
    S, nb, bl = 100, 3, 40
    q, k, v = inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256, dtype=dtype)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    _check(q, k, v, dtype, "prefix branch", mask_kind="prefix_branch", q_pos_offset=S, seg_q=seg_q, seg_kv=seg_kv)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_segments_unsorted_and_empty_rows(cuda_device, dtype):
    rng = np.random.default_rng(3)
    L = 180
    ids = rng.integers(0, 3, L).astype(np.int32)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, "unsorted ids", seg_q=ids, seg_kv=ids)
    seg_q = np.array([9] * 40 + [1] * 140, dtype=np.int32)
    seg_kv = np.array([1] * 180, dtype=np.int32)
    _check(q, k, v, dtype, "rows without keys", seg_q=seg_q, seg_kv=seg_kv)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_packed_segments(cuda_device, dtype):
    lengths = [33, 300, 1, 150, 64]
    L = sum(lengths)
    ids = inputs.segment_ids(lengths)
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, "packed segments", seg_q=ids, seg_kv=ids)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("L,off", [(1000, 0), (700, 300)])
def test_many_tiles(cuda_device, dtype, L, off):
    # bf16 tiles are 128 query rows (32 positions x 4 heads) by 128 keys: 32 x 8 tiles
    # here with ragged last tiles, pairs of tiles per CTA pair and an odd tile count.
    q, k, v = inputs.qkv(1, 16, 4, L, L + off, 256, dtype=dtype)
    _check(q, k, v, dtype, f"L={L} offset {off}", q_pos_offset=off)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
@pytest.mark.parametrize("Hq,Hkv,L", [(4, 4, 700), (8, 4, 450), (16, 2, 300), (16, 1, 500)])
def test_group_sizes_many_tiles(cuda_device, dtype, Hq, Hkv, L):
    # G = 1, 2, 8: query tiles of 128, 64 and 16 positions, each several tiles with a
    # ragged last one, and (for 700 / 128) an odd tile count at one pair per two tiles.
    q, k, v = inputs.qkv(1, Hq, Hkv, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, f"Hq={Hq} Hkv={Hkv} L={L}")


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_prefix_branch_many_tiles(cuda_device, dtype):
    # A 1,000-token state (8 key tiles, visible to every branch row) and 4 branches of
    # 150 rows: key tiles of state keys see every query tile, branch key tiles only
    # their own branch's rows.
    S, nb, bl = 1000, 4, 150
    q, k, v = inputs.qkv(1, 16, 4, nb * bl, S + nb * bl, 256, dtype=dtype)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    _check(q, k, v, dtype, "prefix branch, many tiles", mask_kind="prefix_branch", q_pos_offset=S, seg_q=seg_q,
           seg_kv=seg_kv)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_packed_segments_many_tiles(cuda_device, dtype):
    lengths = [130, 257, 5, 400, 1, 129, 300]
    L = sum(lengths)
    ids = inputs.segment_ids(lengths)
    q, k, v = inputs.qkv(1, 8, 2, L, L, 256, dtype=dtype)
    _check(q, k, v, dtype, "packed segments, many tiles", seg_q=ids, seg_kv=ids)


@pytest.mark.parametrize("dtype", DTYPES, ids=["f32", "bf16"])
def test_invariants_at_16k(cuda_device, dtype):
    L = 16_384
    dev = torch.device("cuda")
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype, device=dev)
    do = _dout(q.shape, dtype).to(dev)
    out, lse = gqa.fwd(q, k, v)
    dq, dk, dv = gqa.bwd(q, k, v, out, lse, do)
    torch.cuda.synchronize()
    dk64, dv64, do64 = dk.double(), dv.double(), do.double()
    # sum over keys of dK is zero; sum over keys of dV is the sum of the group's dout
    tol = 1e-3 if dtype == torch.float32 else 2e-1
    assert float(dk64.sum(dim=2).abs().max()) <= tol * float(dk64.abs().sum(dim=2).max())
    want = do64.view(1, 4, 4, L, 256).sum(dim=(2, 3))
    assert float((dv64.sum(dim=2) - want).abs().max()) <= tol * float(want.abs().max() + 1)
    assert torch.isfinite(dq).all()
