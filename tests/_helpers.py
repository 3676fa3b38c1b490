"""Comparison helpers for the GPU parity tests (numpy / torch only)."""

import numpy as np
import torch

# Tolerances: fp32 from the stated target (out 2e-5, LSE 1e-5); bf16 out 2e-2 on the
# same bf16 inputs.  The bf16 LSE bound (2e-3) follows from the arithmetic: scores are
# exact products of bf16 values summed in fp32 (error ~1e-6), so the LSE error is
# dominated by the fp32 row sum of bf16-rounded probabilities (relative 2^-9 per
# term, averaging out over many keys) -- far below 2e-3.
TOL = {torch.float32: (2e-5, 1e-5), torch.bfloat16: (2e-2, 2e-3)}


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def assert_close(out_gpu, lse_gpu, out_ref, lse_ref, dtype, what=""):
    """Element-wise check of out and LSE; rows with LSE = -inf must match exactly."""
    tol_out, tol_lse = TOL[dtype]
    out_gpu, lse_gpu = to64(out_gpu), to64(lse_gpu)
    out_ref, lse_ref = to64(out_ref), to64(lse_ref)
    assert out_gpu.shape == out_ref.shape and lse_gpu.shape == lse_ref.shape
    assert np.all(np.isfinite(out_gpu)), f"{what}: non-finite output"
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ninf_ref), f"{what}: empty-row pattern differs"
    d_out = float(np.max(np.abs(out_gpu - out_ref))) if out_ref.size else 0.0
    fin = ~ninf_ref
    d_lse = float(np.max(np.abs(lse_gpu[fin] - lse_ref[fin]))) if fin.any() else 0.0
    assert d_out <= tol_out, f"{what}: max|dout| = {d_out:.3e} > {tol_out}"
    assert d_lse <= tol_lse, f"{what}: max|dlse| = {d_lse:.3e} > {tol_lse}"
    return d_out, d_lse
