"""Exact IO-aware attention for B200 (sm_100a): Python binding of libfa.so.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libfa.so`` (see ``include/fa.h``).  PyTorch provides device
memory and streams.  There is no fallback: if the library is missing or no
sm_100 device is present, the calls raise.

    o, lse = fa_fwd(q, k, v, causal=True)              # q,k,v: [B,H,N,d] cuda bf16/fp16
    dq, dk, dv = fa_bwd(q, k, v, o, do, lse, causal=True)
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "FAError",
    "library_path",
    "load_library",
    "fa_fwd",
    "fa_bwd",
    "fa_bwd_workspace_size",
    "fa_bwd_noalloc",
    "fa_fwd_gqa",
    "fa_bwd_gqa",
    "fa_fwd_blocksparse",
    "fa_bwd_blocksparse",
    "fa_fwd_fp8_workspace_size",
    "fa_fp8_quantize",
    "fa_fwd_fp8",
    "fa_merge",
    "fa_grad_accumulate",
    "fa_convert",
    "fa_status_string",
    "fa_last_device_status",
    "fa_debug_set_wait_limit_ms",
    "fa_debug_set_flags",
    "fa_debug_set_timing_events",
    "fa_version",
    "FA_OK",
    "FA_ERR_INVALID_ARG",
    "FA_ERR_UNSUPPORTED",
    "FA_ERR_MISALIGNED",
    "FA_ERR_CUDA",
    "FA_ERR_TIMEOUT",
    "FA_ERR_WORKSPACE",
    "FA_ERR_NO_DEVICE",
    "EXPORTED_SYMBOLS",
]

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5
FA_ERR_WORKSPACE = 6
FA_ERR_NO_DEVICE = 7

FA_BF16 = 0
FA_FP16 = 1
FA_BF16_O_F32 = 2  # 16-bit q, k, v, dO and gradients; O stored in float32
FA_FP16_O_F32 = 3

_c_int, _c_float, _vp, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/fa.h
_SIGNATURES = {
    "fa_fwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _vp]),
    "fa_bwd_workspace_size": (_sz, [_c_int, _c_int, _c_int, _c_int]),
    "fa_bwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                        _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _vp]),
    "fa_fwd_gqa": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int,
                            _c_int, _vp]),
    "fa_bwd_gqa": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                            _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _vp]),
    "fa_fwd_blocksparse": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_longlong, _c_int, _c_int, _c_int,
                                    _c_int, _c_float, _c_int, _c_int, _vp]),
    "fa_bwd_blocksparse": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_longlong, _vp, _vp, _vp, _vp,
                                    _sz, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _vp]),
    "fa_fwd_fp8_workspace_size": (_sz, [_c_int, _c_int, _c_int, _c_int]),
    "fa_fp8_quantize": (_c_int, [_vp, _vp, _vp, _vp, _vp, _sz, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "fa_fwd_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _c_int, _c_int, _c_int, _c_int, _c_float,
                            _c_int, _c_int, _vp]),
    "fa_merge": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, ctypes.c_longlong, _c_int, _vp]),
    "fa_grad_accumulate": (_c_int, [_vp, _vp, ctypes.c_longlong, _c_int, _vp]),
    "fa_convert": (_c_int, [_vp, _vp, ctypes.c_longlong, _c_int, _vp]),
    "fa_bwd_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _vp]),
    "fa_status_string": (ctypes.c_char_p, [_c_int]),
    "fa_last_device_status": (_c_int, [_vp]),
    "fa_debug_set_wait_limit_ms": (_c_int, [_c_int]),
    "fa_debug_set_flags": (_c_int, [_c_int]),
    "fa_debug_set_timing_events": (_c_int, [_vp, _vp]),
    "fa_version": (ctypes.c_char_p, []),
}
EXPORTED_SYMBOLS = tuple(_SIGNATURES)

_LIB = None


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_status_name(status)} ({status})")


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")


def load_library():
    """Load libfa.so (built in-tree by ``python -m exact_io_aware_84_b200.build``)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise FileNotFoundError(
                f"{path} is missing: build it with `python -m exact_io_aware_84_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _apply_env(lib)
        _LIB = lib
    return _LIB


def _apply_env(lib) -> None:
    """Process-wide settings from the environment, applied once at load:
    FA_WAIT_LIMIT (milliseconds, the bound on every pipeline wait inside a
    kernel; default 1000) and FA_DEBUG (the debug flags of
    fa_debug_set_flags; default 0)."""
    for var, fn in (("FA_WAIT_LIMIT", lib.fa_debug_set_wait_limit_ms), ("FA_DEBUG", lib.fa_debug_set_flags)):
        val = os.environ.get(var)
        if val is None or val == "":
            continue
        try:
            num = int(val, 0)
        except ValueError as e:
            raise ValueError(f"{var}={val!r} is not an integer") from e
        st = fn(num)
        if st != 0:
            raise ValueError(f"{var}={val!r} rejected by the library (status {st})")


def _status_name(status: int) -> str:
    try:
        return load_library().fa_status_string(int(status)).decode()
    except Exception:  # the library itself may be what is missing
        return f"status {status}"


def fa_status_string(status: int) -> str:
    return load_library().fa_status_string(int(status)).decode()


def fa_version() -> str:
    return load_library().fa_version().decode()


def fa_debug_set_wait_limit_ms(ms: int) -> int:
    return load_library().fa_debug_set_wait_limit_ms(int(ms))


def fa_debug_set_flags(flags: int) -> int:
    return load_library().fa_debug_set_flags(int(flags))


def fa_debug_set_timing_events(before_main=None, after_main=None) -> int:
    """Have every backward call record these torch.cuda.Event objects (timing
    enabled, already recorded once so that they exist) around the launch of
    its main kernel; None, None clears the setting."""
    h = lambda e: None if e is None else e.cuda_event
    return load_library().fa_debug_set_timing_events(h(before_main), h(after_main))


def _torch():
    import torch
    return torch


def _stream_handle(stream, device=None) -> Optional[int]:
    """Raw cudaStream_t of ``stream``; None means the current stream of
    ``device`` (the device the call's tensors live on)."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _on(t):
    """Context that makes the device of tensor ``t`` current for a library
    call: the library launches on the current device, resolves its status word
    (and the fixed scratch of fa_bwd_noalloc) there, and every pointer it is
    given must belong to that device."""
    return _torch().cuda.device(t.device)


def _check_workspace(ws, q):
    if not getattr(ws, "is_cuda", False) or ws.device != q.device or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor on q's device")


def _check_lse(lse, q):
    """lse must be a contiguous float32 [B, H, N] CUDA tensor on q's device."""
    B, H, N = q.shape[0], q.shape[1], q.shape[2]
    if not getattr(lse, "is_cuda", False):
        raise ValueError("lse must be a CUDA tensor (a host pointer would reach the kernels)")
    if lse.device != q.device:
        raise ValueError(f"lse is on {lse.device}, q on {q.device}: they must share a device")
    if tuple(lse.shape) != (B, H, N) or lse.dtype != _torch().float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, N] tensor")


def fa_last_device_status(stream=None) -> int:
    return load_library().fa_last_device_status(_stream_handle(stream))


def _dtype_code(t, o=None) -> int:
    """Storage code for 16-bit tensor ``t``; O in float32 selects the *_O_F32 codes."""
    torch = _torch()
    o32 = o is not None and o.dtype == torch.float32
    if t.dtype == torch.bfloat16:
        return FA_BF16_O_F32 if o32 else FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16_O_F32 if o32 else FA_FP16
    raise TypeError(f"unsupported dtype {t.dtype}: expected bfloat16 or float16")


def _check_bhnd(name, t, ref=None, allow_f32=False):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 4:
        raise ValueError(f"{name} must be [B, H, N, d], got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ref is not None:
        same_type = t.dtype == ref.dtype or (allow_f32 and t.dtype == _torch().float32)
        if t.shape != ref.shape or not same_type or t.device != ref.device:
            raise ValueError(f"{name} must match q in shape, dtype and device")


def fa_fwd(q, k, v, o=None, lse=None, scale: Optional[float] = None, causal: bool = False, stream=None,
           o_fp32: bool = False):
    """O = softmax(scale Q K^T [causal]) V and LSE (float32, natural log).

    q, k, v: [B, H, N, d] contiguous CUDA tensors (bf16 or fp16).  ``o`` and
    ``lse`` may be preallocated ([B,H,N,d]; [B,H,N] float32).  O has q's
    dtype unless ``o`` is a float32 tensor or ``o_fp32`` is set, in which case
    it is stored in float32 (see the storage codes in include/fa.h).
    """
    torch = _torch()
    _check_bhnd("q", q)
    _check_bhnd("k", k, q)
    _check_bhnd("v", v, q)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty(q.shape, dtype=torch.float32 if o_fp32 else q.dtype, device=q.device)
    else:
        _check_bhnd("o", o, q, allow_f32=True)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    else:
        _check_lse(lse, q)
    with _on(q):
        st = load_library().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   B, H, N, d, float(scale), int(bool(causal)), _dtype_code(q, o),
                                   _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_fwd")
    return o, lse


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_bwd_workspace_size(int(B), int(H), int(N), int(d)))


def fa_bwd(q, k, v, o, do, lse, dq=None, dk=None, dv=None, workspace=None,
           scale: Optional[float] = None, causal: bool = False, stream=None):
    """dQ, dK, dV of L with dL/dO = ``do``, recomputing P from Q, K and LSE."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _check_bhnd(name, t, None if name == "q" else q, allow_f32=(name == "o"))
    B, H, N, d = q.shape
    _check_lse(lse, q)
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_bhnd(name, t, q)
    need = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q)
    with _on(q):
        st = load_library().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                   lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                   workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                   B, H, N, d, float(scale), int(bool(causal)), _dtype_code(q, o),
                                   _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_bwd")
    return dq, dk, dv


def fa_bwd_noalloc(q, k, v, o, do, lse, dq=None, dk=None, dv=None, scale: Optional[float] = None,
                   causal: bool = False, stream=None):
    """fa_bwd without a workspace argument: the library's fixed 32 MiB scratch
    is used instead (for callers that cannot allocate device memory).  Calls
    on one device share that scratch and must not overlap on the GPU."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _check_bhnd(name, t, None if name == "q" else q, allow_f32=(name == "o"))
    B, H, N, d = q.shape
    _check_lse(lse, q)
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_bhnd(name, t, q)
    with _on(q):
        st = load_library().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                           lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                           B, H, N, d, float(scale), int(bool(causal)), _dtype_code(q, o),
                                           _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_noalloc")
    return dq, dk, dv


def _check_kv(name, t, q):
    _check_bhnd(name, t)
    if t.dtype != q.dtype or t.device != q.device or t.shape[0] != q.shape[0] or t.shape[2:] != q.shape[2:]:
        raise ValueError(f"{name} must be [B, Hkv, N, d] with q's B, N, d, dtype and device")
    if q.shape[1] % t.shape[1] != 0:
        raise ValueError(f"q's {q.shape[1]} heads are not a multiple of {name}'s {t.shape[1]}")


def fa_fwd_gqa(q, k, v, o=None, lse=None, scale: Optional[float] = None, causal: bool = False, stream=None,
               o_fp32: bool = False):
    """Grouped-query forward: q [B, H, N, d]; k, v [B, Hkv, N, d] with H % Hkv == 0."""
    torch = _torch()
    _check_bhnd("q", q)
    _check_kv("k", k, q)
    _check_kv("v", v, q)
    if v.shape != k.shape:
        raise ValueError("k and v must have the same shape")
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty(q.shape, dtype=torch.float32 if o_fp32 else q.dtype, device=q.device)
    else:
        _check_bhnd("o", o, q, allow_f32=True)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    else:
        _check_lse(lse, q)
    with _on(q):
        st = load_library().fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                       B, H, Hkv, N, d, float(scale), int(bool(causal)), _dtype_code(q, o),
                                       _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_gqa")
    return o, lse


def fa_bwd_gqa(q, k, v, o, do, lse, dq=None, dk=None, dv=None, workspace=None,
               scale: Optional[float] = None, causal: bool = False, stream=None):
    """Grouped-query backward: dQ per query head; dK, dV summed over each group."""
    torch = _torch()
    _check_bhnd("q", q)
    _check_kv("k", k, q)
    _check_kv("v", v, q)
    _check_bhnd("o", o, q, allow_f32=True)
    _check_bhnd("do", do, q)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    _check_lse(lse, q)
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_bhnd("dq", dq, q)
    _check_kv("dk", dk, q)
    _check_kv("dv", dv, q)
    need = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q)
    with _on(q):
        st = load_library().fa_bwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                       lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                       workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                       B, H, Hkv, N, d, float(scale), int(bool(causal)), _dtype_code(q, o),
                                       _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_gqa")
    return dq, dk, dv


def _check_mask(block_mask, q):
    torch = _torch()
    B, H, N, _ = q.shape
    nb = (N + 127) // 128
    if not block_mask.is_cuda or block_mask.dtype != torch.uint8 or not block_mask.is_contiguous():
        raise ValueError("block_mask must be a contiguous CUDA uint8 tensor")
    if block_mask.device != q.device:
        raise ValueError("block_mask must be on q's device")
    if tuple(block_mask.shape[-2:]) != (nb, nb):
        raise ValueError(f"block_mask must end in ({nb}, {nb}) for N = {N}")
    if block_mask.dim() == 2:
        return 0
    if tuple(block_mask.shape) != (B, H, nb, nb):
        raise ValueError("block_mask must be [nb, nb] (shared) or [B, H, nb, nb]")
    return nb * nb


def fa_fwd_blocksparse(q, k, v, block_mask, o=None, lse=None, scale: Optional[float] = None,
                       causal: bool = False, stream=None, o_fp32: bool = False):
    """Forward that skips the 128 x 128 tiles where ``block_mask`` (uint8,
    [nb, nb] shared or [B, H, nb, nb], nb = ceil(N/128)) is 0."""
    torch = _torch()
    _check_bhnd("q", q)
    _check_bhnd("k", k, q)
    _check_bhnd("v", v, q)
    stride = _check_mask(block_mask, q)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty(q.shape, dtype=torch.float32 if o_fp32 else q.dtype, device=q.device)
    else:
        _check_bhnd("o", o, q, allow_f32=True)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    else:
        _check_lse(lse, q)
    with _on(q):
        st = load_library().fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                           block_mask.data_ptr(), stride, B, H, N, d, float(scale),
                                           int(bool(causal)), _dtype_code(q, o), _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_blocksparse")
    return o, lse


def fa_bwd_blocksparse(q, k, v, o, do, lse, block_mask, dq=None, dk=None, dv=None, workspace=None,
                       scale: Optional[float] = None, causal: bool = False, stream=None):
    """Backward of fa_fwd_blocksparse (the same mask)."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _check_bhnd(name, t, None if name == "q" else q, allow_f32=(name == "o"))
    stride = _check_mask(block_mask, q)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    need = fa_bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    else:
        _check_workspace(workspace, q)
    with _on(q):
        st = load_library().fa_bwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                               lse.data_ptr(), block_mask.data_ptr(), stride, dq.data_ptr(),
                                               dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                               workspace.numel() * workspace.element_size(), B, H, N, d, float(scale),
                                               int(bool(causal)), _dtype_code(q, o), _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_blocksparse")
    return dq, dk, dv


def _dense_cuda(name, t, dtypes, ref=None):
    if not t.is_cuda or not t.is_contiguous() or t.dtype not in dtypes:
        raise ValueError(f"{name} must be a contiguous CUDA tensor of type {dtypes}")
    if ref is not None and t.device != ref.device:
        raise ValueError(f"{name} must be on the same device as the other arguments")


def fa_merge(o, lse, o_part, lse_part, out=None, stream=None):
    """In place: (o, lse) <- merge of two partial results over disjoint key
    sets.  o, o_part fp32 [..., n, d]; lse, lse_part fp32 [..., n]; ``out``
    (optional, bf16/fp16, shape of o) receives the merged O as well."""
    torch = _torch()
    for name, t in (("o", o), ("o_part", o_part)):
        _dense_cuda(name, t, (torch.float32,), o)
    for name, t in (("lse", lse), ("lse_part", lse_part)):
        _dense_cuda(name, t, (torch.float32,), o)
    if o_part.shape != o.shape or lse.shape != o.shape[:-1] or lse_part.shape != lse.shape:
        raise ValueError("fa_merge: shapes of o, o_part, lse, lse_part disagree")
    code = -1
    if out is not None:
        _dense_cuda("out", out, (torch.bfloat16, torch.float16), o)
        if out.shape != o.shape:
            raise ValueError("fa_merge: out must have the shape of o")
        code = FA_BF16 if out.dtype == torch.bfloat16 else FA_FP16
    d = o.shape[-1]
    with _on(o):
        st = load_library().fa_merge(o.data_ptr(), lse.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
                                     out.data_ptr() if out is not None else None, code, lse.numel(), d,
                                     _stream_handle(stream, o.device))
    if st != FA_OK:
        raise FAError(st, "fa_merge")
    return o, lse


def fa_grad_accumulate(acc, src, stream=None):
    """In place: acc (fp32) += src (bf16/fp16), elementwise, same shape."""
    torch = _torch()
    _dense_cuda("acc", acc, (torch.float32,))
    _dense_cuda("src", src, (torch.bfloat16, torch.float16), acc)
    if acc.shape != src.shape:
        raise ValueError("fa_grad_accumulate: shapes differ")
    with _on(acc):
        st = load_library().fa_grad_accumulate(acc.data_ptr(), src.data_ptr(), acc.numel(),
                                               FA_BF16 if src.dtype == torch.bfloat16 else FA_FP16,
                                               _stream_handle(stream, acc.device))
    if st != FA_OK:
        raise FAError(st, "fa_grad_accumulate")
    return acc


def fa_convert(src, dtype=None, out=None, stream=None):
    """fp32 -> bf16/fp16 (round to nearest even) on the device."""
    torch = _torch()
    _dense_cuda("src", src, (torch.float32,))
    if out is None:
        out = torch.empty(src.shape, dtype=dtype or torch.bfloat16, device=src.device)
    _dense_cuda("out", out, (torch.bfloat16, torch.float16), src)
    if out.shape != src.shape:
        raise ValueError("fa_convert: shapes differ")
    with _on(src):
        st = load_library().fa_convert(out.data_ptr(), src.data_ptr(), src.numel(),
                                       FA_BF16 if out.dtype == torch.bfloat16 else FA_FP16, _stream_handle(stream, src.device))
    if st != FA_OK:
        raise FAError(st, "fa_convert")
    return out


def fa_fwd_fp8_workspace_size(B: int, H: int, N: int, d: int = 128) -> int:
    return int(load_library().fa_fwd_fp8_workspace_size(B, H, N, d))


def _fp8_views(ws, B, H, N):
    """Views of the FP8 workspace's parts (layout of fa_fwd_fp8_workspace_size)."""
    torch = _torch()
    bh, nb = B * H, (N + 127) // 128
    n_pad = nb * 128
    up = lambda x: (x + 255) // 256 * 256
    off, out = 0, {}
    for name, n, dt, shape in (("q8", bh * n_pad * 128, torch.uint8, (B, H, n_pad, 128)),
                               ("k8", bh * n_pad * 128, torch.uint8, (B, H, n_pad, 128)),
                               ("v8t", bh * n_pad * 128, torch.uint8, (B, H, 128, n_pad)),
                               ("sq", bh * nb * 4, torch.float32, (B, H, nb)),
                               ("sk", bh * nb * 4, torch.float32, (B, H, nb)),
                               ("sv", bh * 128 * 4, torch.float32, (B, H, 128))):
        out[name] = ws[off:off + n].view(dt).view(shape)
        off += up(n)
    return out


def fa_fp8_quantize(q, k, v, signs=None, workspace=None, stream=None):
    """Rotation (when ``signs`` is given), scales and e4m3 codes of the FP8
    forward.  Returns a dict of views into the workspace: q8, k8 [B,H,n_pad,128]
    and v8t [B,H,128,n_pad] (uint8 e4m3 bits), sq, sk [B,H,nb], sv [B,H,128]."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bhnd(name, t, None if name == "q" else q)
    B, H, N, d = q.shape
    if workspace is None:
        workspace = torch.empty(fa_fwd_fp8_workspace_size(B, H, N, d), dtype=torch.uint8, device=q.device)
    with _on(q):
        st = load_library().fa_fp8_quantize(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            signs.data_ptr() if signs is not None else None, workspace.data_ptr(),
                                            workspace.numel(), B, H, N, d, _dtype_code(q, q), _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_fp8_quantize")
    return _fp8_views(workspace, B, H, N)


def fa_fwd_fp8(q, k, v, signs=None, o=None, lse=None, workspace=None, scale: Optional[float] = None,
               causal: bool = False, stream=None, o_fp32: bool = False):
    """FP8 forward (head dim 128) with incoherent processing when ``signs``
    (CUDA float32 [128] of +-1) is given.  Returns (O, LSE)."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bhnd(name, t, None if name == "q" else q)
    B, H, N, d = q.shape
    if signs is not None and (not signs.is_cuda or signs.dtype != torch.float32 or signs.numel() != d
                              or signs.device != q.device or not signs.is_contiguous()):
        raise ValueError("signs must be a contiguous CUDA float32 tensor of d entries on q's device")
    if scale is None:
        scale = 1.0 / float(d) ** 0.5
    if o is None:
        o = torch.empty(q.shape, dtype=torch.float32 if o_fp32 else q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(1, fa_fwd_fp8_workspace_size(B, H, N, d)), dtype=torch.uint8, device=q.device)
    with _on(q):
        st = load_library().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                       signs.data_ptr() if signs is not None else None, workspace.data_ptr(),
                                       workspace.numel(), B, H, N, d, float(scale), int(bool(causal)),
                                       _dtype_code(q, o), _stream_handle(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_fp8")
    return o, lse
