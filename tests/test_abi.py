"""The C-ABI library loads, exports every symbol include/fa.h declares, and
rejects bad arguments on the host before anything is launched.

Only calls that return before any device work are made here (null pointers,
bad sizes, misaligned addresses), so these tests are safe with or without a
GPU.
"""

import os
import re

import pytest

import exact_io_aware_84_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    return fa.load_library()


def test_library_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert "fa_fwd" in declared and "fa_bwd" in declared
    for name in declared:
        assert hasattr(lib, name), name
    # the binding wraps exactly the declared entry points
    assert set(fa.EXPORTED_SYMBOLS) == set(declared)


def test_status_strings(lib):
    for code, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID_ARG"), (2, "FA_ERR_UNSUPPORTED"),
                       (3, "FA_ERR_MISALIGNED"), (4, "FA_ERR_CUDA"), (5, "FA_ERR_TIMEOUT"),
                       (6, "FA_ERR_WORKSPACE"), (7, "FA_ERR_NO_DEVICE")]:
        assert fa.fa_status_string(code) == name
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"
    assert fa.fa_version().startswith("fa-sm100")


def test_debug_setters_validate(lib):
    assert fa.fa_debug_set_wait_limit_ms(0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_set_flags(-1) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_set_wait_limit_ms(1000) == fa.FA_OK
    assert fa.fa_debug_set_flags(0) == fa.FA_OK


def _fwd(lib, q=0x1000, k=0x1000, v=0x1000, o=0x1000, lse=0x1000, B=1, H=1, N=128, d=64,
         scale=0.125, causal=0, dtype=0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, None)


def test_fwd_argument_errors(lib):
    assert _fwd(lib, q=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, lse=None) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, N=0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=-1) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == fa.FA_ERR_INVALID_ARG
    assert _fwd(lib, d=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(lib, d=256) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=7) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=4) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(lib, B=1 << 14, H=1 << 10, N=1 << 10) == fa.FA_ERR_INVALID_ARG  # > 2^31 elements
    assert _fwd(lib, k=0x1008) == fa.FA_ERR_MISALIGNED
    assert _fwd(lib, lse=0x1004) == fa.FA_ERR_MISALIGNED


def test_bwd_workspace_size(lib):
    # fp32 dQ accumulator over ceil(N/128)*128 rows + two fp32 row vectors, 256-B sections
    up = lambda x: (x + 255) // 256 * 256
    for B, H, N, d in [(1, 1, 1, 64), (8, 12, 1024, 64), (1, 12, 23400, 64), (2, 16, 2048, 128)]:
        npad = (N + 127) // 128 * 128
        want = up(B * H * npad * d * 4) + 2 * up(B * H * npad * 4)
        assert fa.fa_bwd_workspace_size(B, H, N, d) == want
    assert fa.fa_bwd_workspace_size(1, 1, 0, 64) == 0
    assert fa.fa_bwd_workspace_size(1, 1, 128, 80) == 0


def _bwd(lib, ws=0x10000, ws_bytes=1 << 30, N=128, d=64, **kw):
    p = 0x1000
    args = dict(q=p, k=p, v=p, o=p, do=p, lse=p, dq=p, dk=p, dv=p)
    args.update(kw)
    return lib.fa_bwd(args["q"], args["k"], args["v"], args["o"], args["do"], args["lse"], args["dq"],
                      args["dk"], args["dv"], ws, ws_bytes, 1, 1, N, d, 0.125, 0, 0, None)


def test_bwd_argument_errors(lib):
    assert _bwd(lib, do=None) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, dk=None) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, d=72) == fa.FA_ERR_UNSUPPORTED
    assert _bwd(lib, N=-5) == fa.FA_ERR_INVALID_ARG
    assert _bwd(lib, dv=0x1002) == fa.FA_ERR_MISALIGNED
    assert _bwd(lib, ws=None) == fa.FA_ERR_WORKSPACE
    assert _bwd(lib, ws_bytes=16) == fa.FA_ERR_WORKSPACE
    assert _bwd(lib, ws=0x10010) == fa.FA_ERR_MISALIGNED


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_device_reports_no_device(lib):
    assert _fwd(lib) == fa.FA_ERR_NO_DEVICE


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fa_fwd(q, q, q)


def test_gqa_argument_errors(lib):
    p = 0x1000
    assert lib.fa_fwd_gqa(p, p, p, p, p, 1, 6, 4, 128, 64, 0.125, 0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_gqa(p, p, p, p, p, 1, 6, 0, 128, 64, 0.125, 0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_gqa(p, p, p, p, p, p, p, p, p, 0x10000, 1 << 30, 1, 8, 3, 128, 64, 0.125, 0, 0,
                          None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_gqa(p, p, p, p, p, 1, 8, 2, 128, 96, 0.125, 0, 0, None) == fa.FA_ERR_UNSUPPORTED


def test_blocksparse_rejects_null_mask_and_negative_stride():
    lib = fa.load_library()
    p = 0x1000
    assert lib.fa_fwd_blocksparse(p, p, p, p, p, None, 0, 1, 1, 128, 64, 0.125, 0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_blocksparse(p, p, p, p, p, p, -1, 1, 1, 128, 64, 0.125, 0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_blocksparse(p, p, p, p, p, p, None, 0, p, p, p, p, 1 << 20, 1, 1, 128, 64, 0.125, 0, 0,
                                  None) == fa.FA_ERR_INVALID_ARG


def test_ring_helpers_argument_errors():
    lib = fa.load_library()
    p = 0x1000
    # d, out type, sizes, pointers and alignment are checked before any launch
    assert lib.fa_merge(p, p, p, p, None, -1, 10, 96, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_merge(p, p, p, p, None, 2, 10, 64, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_merge(p, p, p, p, None, -1, -1, 64, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_merge(p, p, p, p, None, -1, 0, 64, None) == fa.FA_OK
    assert lib.fa_merge(p, p, None, p, None, -1, 4, 64, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_merge(p, p, p, p, None, 0, 4, 64, None) == fa.FA_ERR_INVALID_ARG      # out missing
    assert lib.fa_merge(p + 4, p, p, p, None, -1, 4, 64, None) == fa.FA_ERR_MISALIGNED
    assert lib.fa_merge(p, p, p, p, p + 2, 0, 4, 64, None) == fa.FA_ERR_MISALIGNED
    assert lib.fa_grad_accumulate(p, p, 0, 0, None) == fa.FA_OK
    assert lib.fa_grad_accumulate(p, p, 8, 2, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_grad_accumulate(p, p, -1, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_grad_accumulate(p, p + 8, 8, 0, None) == fa.FA_ERR_MISALIGNED
    assert lib.fa_convert(p, p, 0, 1, None) == fa.FA_OK
    assert lib.fa_convert(p, p, 8, 3, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_convert(p + 4, p, 8, 0, None) == fa.FA_ERR_MISALIGNED
    assert lib.fa_convert(None, p, 8, 0, None) == fa.FA_ERR_INVALID_ARG


def test_fp8_argument_errors():
    lib = fa.load_library()
    p = 0x1000
    assert lib.fa_fwd_fp8_workspace_size(1, 1, 128, 64) == 0
    assert lib.fa_fwd_fp8_workspace_size(1, 1, 128, 128) > 3 * 128 * 128
    assert lib.fa_fwd_fp8(p, p, p, p, p, None, p, 1 << 30, 1, 1, 128, 64, 0.1, 0, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_fp8(p, p, p, p, p, None, None, 0, 1, 1, 128, 128, 0.1, 0, 0, None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_fwd_fp8(p, p, p, p, p, None, p, 16, 1, 1, 128, 128, 0.1, 0, 0, None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_fwd_fp8(p, p, p, None, p, None, p, 1 << 30, 1, 1, 128, 128, 0.1, 0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fp8_quantize(None, p, p, None, p, 1 << 30, 1, 1, 128, 128, 0, None) == fa.FA_ERR_INVALID_ARG


def test_environment_settings_are_applied_and_checked(monkeypatch):
    # FA_WAIT_LIMIT / FA_DEBUG are read when the library is loaded
    monkeypatch.setenv("FA_WAIT_LIMIT", "250")
    monkeypatch.setenv("FA_DEBUG", "0")
    saved = fa._LIB
    try:
        fa._LIB = None
        fa.load_library()
        monkeypatch.setenv("FA_WAIT_LIMIT", "0")      # the library rejects ms < 1
        fa._LIB = None
        with pytest.raises(ValueError):
            fa.load_library()
        monkeypatch.setenv("FA_WAIT_LIMIT", "soon")
        fa._LIB = None
        with pytest.raises(ValueError):
            fa.load_library()
    finally:
        monkeypatch.delenv("FA_WAIT_LIMIT")
        monkeypatch.delenv("FA_DEBUG")
        fa._LIB = None
        fa.load_library()
        fa.load_library().fa_debug_set_wait_limit_ms(1000)
        fa._LIB = saved if saved is not None else fa._LIB
