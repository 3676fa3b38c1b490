"""The packed-FMA ceiling probe (`gqa_attn_probe_ffma2`), the measurement aid the bench
reports next to the nominal FP32 peak: argument checks on the CPU, a plausible rate on
the GPU."""

import ctypes

import pytest
import torch

from long_context_causal_flash_b200 import _lib
from long_context_causal_flash_b200.build import build


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def test_probe_rejects_bad_arguments_before_any_cuda_call(lib):
    buf = ctypes.create_string_buffer(4096 + 16)
    ok = (ctypes.addressof(buf) + 15) & ~15
    assert lib.gqa_attn_probe_ffma2(None, 1, 1, 0, None) == _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_probe_ffma2(ok, 0, 1, 0, None) == _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_probe_ffma2(ok, 70000, 1, 0, None) == _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_probe_ffma2(ok, 1, 0, 0, None) == _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_probe_ffma2(ok, 1, 1, 4, None) == _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_probe_ffma2(ok, 1, 1, -1, None) == _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_probe_ffma2(ok + 4, 1, 1, 0, None) == _lib.GQA_ERR_MISALIGNED


@pytest.mark.gpu
def test_probe_rate_is_below_the_nominal_peak(cuda_device, lib):
    """148 CTAs x 256 threads x iters x 64 FMAs: finite outputs, and a rate between a
    third of the nominal FP32 peak at the maximum clock and just above it."""
    import bench

    out = torch.empty(148 * 256, dtype=torch.float32, device=cuda_device)
    s = torch.cuda.current_stream(cuda_device).cuda_stream
    for form in range(4):
        out.fill_(float("nan"))
        assert lib.gqa_attn_probe_ffma2(out.data_ptr(), 148, 10, form, s) == _lib.GQA_OK
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), form
    rate = bench._ffma2_ceiling(cuda_device)
    nominal = bench._fp32_peak_tflops(148, 1965.0)
    assert nominal / 3 < rate < 1.05 * nominal, rate
