"""C ABI checks that need no GPU: the library loads, exports every declared symbol,
sizes its workspace linearly in L and rejects bad arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

import long_context_causal_flash_b200 as gqa
from long_context_causal_flash_b200 import _lib
from long_context_causal_flash_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_attn.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_attn_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_strerror_covers_every_status(lib):
    for code in range(0, -8, -1):
        msg = gqa._lib.strerror(code)
        assert msg and msg != "unknown status"
    assert gqa._lib.strerror(-99) == "unknown status"


def test_tile_sizes_per_dtype_and_group(lib):
    assert gqa.tile_sizes(gqa.GQA_F32, 16, 4) == (16, 256)
    assert gqa.tile_sizes(gqa.GQA_F32, 16, 16) == (64, 256)
    assert gqa.tile_sizes(gqa.GQA_BF16, 16, 4) == (32, 128)
    with pytest.raises(gqa.GqaAttnError):
        gqa.tile_sizes(gqa.GQA_F32, 16, 5)
    with pytest.raises(gqa.GqaAttnError):
        gqa.tile_sizes(gqa.GQA_F32, 96, 3)  # group of 32 is not supported


def test_workspace_is_linear_in_length(lib):
    ws = lambda L, seg: lib.gqa_attn_workspace_bytes(1, 16, 4, L, L, 256, 0, 0, seg)
    assert ws(60926, 0) == 256
    sizes = [ws(L, 1) for L in (1 << 16, 1 << 18, 1 << 20)]
    assert sizes[1] / sizes[0] == pytest.approx(4, rel=0.01)
    assert sizes[2] / sizes[1] == pytest.approx(4, rel=0.01)
    assert sizes[2] < 2 << 20  # well under the 2 MiB block-pair table splash needed at 1M
    assert lib.gqa_attn_workspace_bytes(1, 16, 4, 10, 11, 256, 0, 0, 0) == 256  # offset 1
    assert lib.gqa_attn_workspace_bytes(1, 16, 4, 10, 10, 128, 0, 0, 0) == 0  # d unsupported
    assert lib.gqa_attn_workspace_bytes(1, 16, 4, 10, 10, 256, 0, 1, 0) == 0  # branch mask needs ids


def _fwd(lib, **over):
    a = dict(q=16, k=16, v=16, out=16, lse=16, B=1, Hq=16, Hkv=4, Lq=64, Lk=64, d=256, dtype=0, mask=0, off=0,
             sq=None, skv=None, ws=256, wsb=256)
    a.update(over)
    return lib.gqa_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Lq"],
                            a["Lk"], a["d"], a["dtype"], a["mask"], a["off"], a["sq"], a["skv"], a["ws"],
                            a["wsb"], None)


def test_fwd_rejects_bad_arguments_without_launching(lib):
    # Fake (never dereferenced) pointer values: validation fails before any CUDA call.
    assert _fwd(lib, q=None) == _lib.GQA_ERR_INVALID_ARG
    assert _fwd(lib, Hkv=3) == _lib.GQA_ERR_INVALID_ARG
    assert _fwd(lib, Lk=65) == _lib.GQA_ERR_INVALID_ARG            # Lk != offset + Lq
    assert _fwd(lib, Lq=0, Lk=0) == _lib.GQA_ERR_INVALID_ARG
    assert _fwd(lib, off=-1, Lk=63) == _lib.GQA_ERR_INVALID_ARG
    assert _fwd(lib, dtype=7) == _lib.GQA_ERR_INVALID_ARG
    assert _fwd(lib, mask=1) == _lib.GQA_ERR_INVALID_ARG            # branch mask without ids
    assert _fwd(lib, sq=16) == _lib.GQA_ERR_INVALID_ARG             # only one id array
    assert _fwd(lib, d=128) == _lib.GQA_ERR_UNSUPPORTED
    assert _fwd(lib, Hq=12, Hkv=4) == _lib.GQA_ERR_UNSUPPORTED      # group of 3
    assert _fwd(lib, q=17) == _lib.GQA_ERR_MISALIGNED
    assert _fwd(lib, lse=20) == _lib.GQA_ERR_MISALIGNED
    assert _fwd(lib, ws=None) == _lib.GQA_ERR_WORKSPACE
    assert _fwd(lib, sq=16, skv=16, wsb=256) == _lib.GQA_ERR_WORKSPACE  # segments need the plan tables


def test_tile_plan_and_selftest_reject_bad_arguments(lib):
    assert lib.gqa_attn_tile_plan(16, 4, 64, 64, 0, 0, 0, None, None, 16, 256, None, 16, None) == \
        _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_tile_plan(16, 4, 64, 64, 0, 1, 0, None, None, 16, 256, 16, 16, None) == \
        _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_selftest_wait(None, 256, 10**8, None) == _lib.GQA_ERR_WORKSPACE
    assert lib.gqa_attn_selftest_wait(16, 256, 10, None) == _lib.GQA_ERR_INVALID_ARG
    assert lib.gqa_attn_status(None, None) == _lib.GQA_ERR_INVALID_ARG


def test_binding_validates_before_calling(lib):
    import torch

    q = torch.zeros(1, 16, 8, 256)
    with pytest.raises(ValueError):
        gqa.fwd(q, q, q)  # host tensors go through fwd_host
    with pytest.raises(ValueError):
        gqa._mask("sliding")
    with pytest.raises(ValueError):
        gqa._dtype_code(torch.float16)


def test_offset_and_merge_reject_bad_arguments(lib):
    # Validation happens before any CUDA call, so none of these needs a GPU.  Pointers
    # are fake but 16-byte aligned; every call must fail on its arguments first.
    p = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 21)
    fwd = lambda *a: lib.gqa_attn_fwd_offset(p, p, p, p, p, *a)  # noqa: E731
    # B, Hq, Hkv, Lq, Lk, d, dtype, q_pos_offset, workspace, bytes, stream
    assert fwd(1, 16, 4, 100, 300, 256, 1, -1, ws, 256, None) == _lib.GQA_ERR_INVALID_ARG  # offset < 0
    assert fwd(1, 16, 5, 100, 300, 256, 1, 0, ws, 256, None) == _lib.GQA_ERR_INVALID_ARG   # Hq % Hkv
    assert fwd(1, 16, 4, 100, 300, 128, 1, 0, ws, 256, None) == _lib.GQA_ERR_UNSUPPORTED   # d
    assert fwd(1, 16, 4, 100, 300, 256, 1, 0, ws, 255, None) == _lib.GQA_ERR_WORKSPACE     # too small
    assert fwd(1, 16, 4, 0, 300, 256, 1, 0, ws, 256, None) == _lib.GQA_ERR_INVALID_ARG     # Lq < 1
    mrg = lib.gqa_attn_merge
    # o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d, dtype_b, dtype_out, stream
    assert mrg(p, p, p, p, None, p, 10, 256, 0, 0, None) == _lib.GQA_ERR_INVALID_ARG       # no output
    assert mrg(p, None, p, p, p, p, 10, 256, 0, 0, None) == _lib.GQA_ERR_INVALID_ARG       # half a pair
    assert mrg(p, p, p, p, p, p, 0, 256, 0, 0, None) == _lib.GQA_ERR_INVALID_ARG           # rows < 1
    assert mrg(p, p, p, p, p, p, 10, 256, 2, 0, None) == _lib.GQA_ERR_INVALID_ARG          # dtype
    assert mrg(p, p, p, p, p, p, 10, 128, 0, 0, None) == _lib.GQA_ERR_UNSUPPORTED          # d
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert mrg(odd, p, p, p, p, p, 10, 256, 0, 0, None) == _lib.GQA_ERR_MISALIGNED


def test_split_operand_dtype_sizes_and_rejections(lib):
    # GQA_F32_TC uses the bf16 kernel's tiles and adds the hi / lo fp16 planes of q, k
    # and v (4 bytes per element, like the fp32 inputs) and the per-head maxima.
    assert gqa.tile_sizes(gqa.GQA_F32_TC, 16, 4) == gqa.tile_sizes(gqa.GQA_BF16, 16, 4)
    L = 60_926
    tc = lib.gqa_attn_workspace_bytes(1, 16, 4, L, L, 256, gqa.GQA_F32_TC, 0, 0)
    planes = 4 * 256 * L * (16 + 4 + 4)
    assert planes <= tc - 256 <= planes + 4 * 256
    base = lib.gqa_attn_split_workspace_bytes(1, 16, 4, 100, 300, 256, 0, 0, 0, 3)
    assert lib.gqa_attn_split_workspace_bytes(1, 16, 4, 100, 300, 256, gqa.GQA_F32_TC, 0, 0, 3) > base
    assert lib.gqa_attn_bwd_workspace_bytes(1, 16, 4, 64, 64, 256, gqa.GQA_F32_TC, 0, 0) == 0
    # the workspace must hold the planes
    assert _fwd(lib, dtype=gqa.GQA_F32_TC, wsb=4096) == _lib.GQA_ERR_WORKSPACE
    # key blocks at an offset and the backward take dtype 0 or 1 only
    p = ctypes.c_void_p(1 << 20)
    assert lib.gqa_attn_fwd_offset(p, p, p, p, p, 1, 16, 4, 100, 300, 256, gqa.GQA_F32_TC, 0, p, 1 << 30,
                                   None) == _lib.GQA_ERR_UNSUPPORTED
    assert lib.gqa_attn_bwd(*([p] * 9), 1, 16, 4, 64, 64, 256, gqa.GQA_F32_TC, 0, 0, None, None, p, 1 << 30,
                            None) == _lib.GQA_ERR_UNSUPPORTED


def test_fp32_path_option(lib):
    import torch

    assert gqa._call_dtype(torch.float32, "ffma") == gqa.GQA_F32
    assert gqa._call_dtype(torch.float32, "tc") == gqa.GQA_F32_TC
    assert gqa._call_dtype(torch.bfloat16, "ffma") == gqa.GQA_BF16
    with pytest.raises(ValueError):
        gqa._call_dtype(torch.bfloat16, "tc")
    with pytest.raises(ValueError):
        gqa._call_dtype(torch.float32, "tf32")


def test_static_scratch_limit_depends_on_the_group_size(lib):
    """The no-allocation entry point's fixed 2 MiB scratch holds the block-skip tables of
    1,048,576-token segmented calls only up to a group size: the tables grow with the
    number of query tiles, Lq * G / 64 (fp32) or Lq * G / 128 (bf16).  Calls beyond it are
    rejected on the host before any pointer is used (the pointer values are never read)."""
    static_bytes = 2 << 20
    L = 1 << 20
    need = lambda Hq, Hkv, dtype: lib.gqa_attn_workspace_bytes(1, Hq, Hkv, L, L, 256, dtype, 0, 1)
    assert need(16, 4, gqa.GQA_F32) <= static_bytes   # G = 4
    assert need(16, 2, gqa.GQA_F32) > static_bytes    # G = 8
    assert need(16, 2, gqa.GQA_BF16) <= static_bytes  # G = 8
    assert need(16, 1, gqa.GQA_BF16) > static_bytes   # G = 16
    assert need(16, 4, gqa.GQA_F32_TC) > static_bytes  # split operand planes
    assert lib.gqa_attn_workspace_bytes(1, 16, 1, L, L, 256, gqa.GQA_F32, 0, 0) <= static_bytes  # no ids
    for Hkv, dtype in ((1, gqa.GQA_BF16), (2, gqa.GQA_F32), (4, gqa.GQA_F32_TC)):
        rc = lib.gqa_attn_fwd_static_ws(16, 16, 16, 16, 16, 1, 16, Hkv, L, L, 256, dtype, 0, 0, 16, 16, None)
        assert rc == _lib.GQA_ERR_WORKSPACE
