"""GPU parity of the backward at the benchmark's full size (L = 60,926 causal) on
sampled outputs the fp64 oracle computes one by one.

* dQ of a query row i depends on that row and keys 0..i only: it is the oracle's
  backward of the one-row problem (q row i, keys 0..i, q_pos_offset = i).
* dK and dV of the last 64 keys depend only on the last 64 query rows (no earlier row
  sees them causally): they are the oracle's backward of those rows against all keys
  (q_pos_offset = L - 64), exact for keys L - 64 .. L - 1.
The CUDA forward's out and lse feed the CUDA backward, as in training.  Tolerances as
in test_backward.py: fp32 5e-5 and bf16 2e-2 of the largest reference gradient.
"""

import numpy as np
import pytest
import torch

import long_context_causal_flash_b200 as gqa
import oracle
from long_context_causal_flash_b200 import inputs
from tests._helpers import to64

pytestmark = pytest.mark.gpu

L = 60_926
TAIL = 64
RTOL = {torch.float32: 5e-5, torch.bfloat16: 2e-2}


def _sampled_rows():
    rng = np.random.default_rng(5)
    extra = rng.choice(np.arange(2, L - 1), size=5, replace=False)
    return sorted({0, 1, L - 1, *map(int, extra)})


def _close(got, want, dtype, what):
    got = to64(got)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    scale = max(1.0, float(np.max(np.abs(want))))
    err = float(np.max(np.abs(got - want)))
    assert err <= RTOL[dtype] * scale, f"{what}: max|d| = {err:.3e} (scale {scale:.2f})"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_full_size_sampled(cuda_device, dtype):
    dev = torch.device("cuda")
    q, k, v = inputs.qkv(1, 16, 4, L, L, 256, dtype=dtype)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(dtype)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), dout.to(dev)
    out, lse = gqa.fwd(qd, kd, vd)
    dq, dk, dv = gqa.bwd(qd, kd, vd, out, lse, dod)
    torch.cuda.synchronize()
    del qd, kd, vd, dod, out, lse

    for i in _sampled_rows():
        ref_dq, _, _ = oracle.attention_backward(q[:, :, i:i + 1], k[:, :, :i + 1], v[:, :, :i + 1],
                                                 dout[:, :, i:i + 1], q_pos_offset=i)
        _close(dq[:, :, i:i + 1], ref_dq, dtype, f"dq row {i}")

    i0 = L - TAIL
    _, ref_dk, ref_dv = oracle.attention_backward(q[:, :, i0:], k, v, dout[:, :, i0:], q_pos_offset=i0)
    _close(dk[:, :, i0:], ref_dk[:, :, i0:], dtype, f"dk keys {i0}..{L - 1}")
    _close(dv[:, :, i0:], ref_dv[:, :, i0:], dtype, f"dv keys {i0}..{L - 1}")

    # Properties at every key: per key/value head the key gradients sum to zero and
    # the value gradients sum to the group's summed upstream gradient.
    dk64 = dk.double()
    assert float(dk64.sum(dim=2).abs().max()) <= (1e-3 if dtype == torch.float32 else 2e-1) * \
        float(dk64.abs().sum(dim=2).max())
    want = dout.double().view(1, 4, 4, L, 256).sum(dim=(2, 3))
    tol = 1e-3 if dtype == torch.float32 else 2e-1
    assert float((dv.double().cpu().sum(dim=2) - want).abs().max()) <= tol * float(want.abs().max() + 1)


def test_backward_segmented_1m_bf16(cuda_device):
    """The training workload the backward exists for: 1,048,576 tokens packed from
    seeded segments (bf16).  Keys of other segments are invisible by definition, so
    each check runs the oracle on its segment's window: dQ of sampled rows (the row
    against its segment's keys up to it) and dK / dV of the last 32 keys of the first
    and the last segment (those keys are seen only by the last 32 rows of their
    segment)."""
    Lm = 1_048_576
    lengths = inputs.segment_lengths(Lm)
    ids = inputs.segment_ids(lengths)
    starts = np.concatenate([[0], np.cumsum(lengths)[:-1]])
    dev = torch.device("cuda")
    q, k, v = inputs.qkv(1, 16, 4, Lm, Lm, 256, dtype=torch.bfloat16, device=dev)
    dout = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(7), device=dev).to(torch.bfloat16)
    tid = torch.as_tensor(ids, device=dev)
    out, lse = gqa.fwd(q, k, v, seg_q=tid, seg_kv=tid)
    dq, dk, dv = gqa.bwd(q, k, v, out, lse, dout, seg_q=tid, seg_kv=tid)
    torch.cuda.synchronize()
    del out, lse

    rows = inputs.sample_rows(Lm, 24, boundaries=starts)
    for i in rows:
        a = int(starts[np.searchsorted(starts, i, side="right") - 1])
        ref_dq, _, _ = oracle.attention_backward(q[:, :, i:i + 1], k[:, :, a:i + 1], v[:, :, a:i + 1],
                                                 dout[:, :, i:i + 1], q_pos_offset=int(i - a))
        _close(dq[:, :, i:i + 1], ref_dq, torch.bfloat16, f"dq row {i} (segment at {a})")

    T = 32
    for a, n in ((int(starts[0]), lengths[0]), (int(starts[-1]), lengths[-1])):
        e = a + n
        _, ref_dk, ref_dv = oracle.attention_backward(q[:, :, e - T:e], k[:, :, a:e], v[:, :, a:e], dout[:, :, e - T:e],
                                                      q_pos_offset=n - T)
        _close(dk[:, :, e - T:e], ref_dk[:, :, n - T:], torch.bfloat16, f"dk last keys of segment at {a}")
        _close(dv[:, :, e - T:e], ref_dv[:, :, n - T:], torch.bfloat16, f"dv last keys of segment at {a}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_backward_branches_after_state_sampled(cuda_device, dtype):
    """The branch pass of the pages' state-reuse workload at full size: 8 question
    branches of 256 rows after a 30,468-token state (shared-prefix branch mask).  For a
    row of branch b the branch mask equals the causal mask with segment ids in which
    the state keys carry id b: the row sees the state and its own branch up to itself.
    dQ of sampled rows is the oracle's backward of that one-row problem; dK / dV of the
    keys of branch 3 come from that branch's 256 rows, the only rows that see them."""
    S, nb, bl = 30_468, 8, 256
    Lq = nb * bl
    q, k, v = inputs.qkv(1, 16, 4, Lq, S + Lq, 256, dtype=dtype)
    seg_q, seg_kv = inputs.branch_ids(S, nb, bl)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(dtype)
    dev = torch.device("cuda")
    kw = dict(mask_kind="prefix_branch", q_pos_offset=S, seg_q=torch.as_tensor(seg_q, device=dev),
              seg_kv=torch.as_tensor(seg_kv, device=dev))
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), dout.to(dev)
    out, lse = gqa.fwd(qd, kd, vd, **kw)
    dq, dk, dv = gqa.bwd(qd, kd, vd, out, lse, dod, **kw)
    torch.cuda.synchronize()

    def ids_for(branch, e):
        ids = seg_kv[:e].copy()
        ids[:S] = branch
        return ids

    for i in inputs.sample_rows(Lq, 10, boundaries=range(0, Lq, bl)):
        i = int(i)
        e = S + i + 1
        ref_dq, _, _ = oracle.attention_backward(q[:, :, i:i + 1], k[:, :, :e], v[:, :, :e], dout[:, :, i:i + 1],
                                                 q_pos_offset=S + i, seg_q=seg_q[i:i + 1],
                                                 seg_kv=ids_for(int(seg_q[i]), e))
        _close(dq[:, :, i:i + 1], ref_dq, dtype, f"dq row {i}")

    b = 3
    r0, r1 = b * bl, (b + 1) * bl
    e = S + r1
    _, ref_dk, ref_dv = oracle.attention_backward(q[:, :, r0:r1], k[:, :, :e], v[:, :, :e], dout[:, :, r0:r1],
                                                  q_pos_offset=S + r0, seg_q=seg_q[r0:r1], seg_kv=ids_for(b, e))
    _close(dk[:, :, S + r0:S + r1], ref_dk[:, :, S + r0:], dtype, f"dk of branch {b}")
    _close(dv[:, :, S + r0:S + r1], ref_dv[:, :, S + r0:], dtype, f"dv of branch {b}")
