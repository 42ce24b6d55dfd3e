"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic: it only draws random tensors.  It
is the one module that both the CUDA path's callers (tests, bench) and the
fp64 oracle's callers use, so that both sides see bit-identical inputs.

Recipe (every workload): a fresh CPU ``torch.Generator`` seeded with ``seed``
(default 0) draws float32 standard normals in the order q, k, v, dO, each of
shape [B, H, N, d]; the draws are then rounded to the storage dtype
(bf16 or fp16, round-to-nearest-even via ``Tensor.to``).  The rounded values,
widened to float64, are what the oracle sees.

Two workloads modify the draws before rounding:

* ``scale_inputs`` (the 4K single-sequence fp16 workload): q, k and v are
  multiplied by 0.5 in float32.
* ``low_rank`` (the 23,400-step trading-day workload): per (b, h),
  U in R^{N x 4} ~ N(0, 1) and A in R^{4 x d} ~ N(0, 1/4) (so U A has unit
  variance per coordinate); q = z_q + 2 U A and k = z_k + 2 U A with z ~ N(0,1).
  Draw order z_q, z_k, U, A, v, dO.  This gives peaked softmax rows.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "workload"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str           # "bf16" | "fp16"
    causal: bool
    scale: float
    backward: bool
    scale_inputs: float = 1.0
    low_rank: bool = False
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    def with_(self, **kw):
        return dataclasses.replace(self, **kw)


def _w(name, B, H, N, d, dtype, causal, backward, **kw):
    scale = kw.pop("scale", 1.0 / (d ** 0.5))
    return Workload(name, B, H, N, d, dtype, causal, scale, backward, **kw)


# The five workloads: tiny forward; GPT-2-small-like batch; a single 4K fp16
# sequence; one trading day at 1 s (ragged N); the d=128 sweep.
WORKLOADS = {
    "tiny_fwd": _w("tiny_fwd", 1, 1, 256, 64, "bf16", False, False, scale=1.0 / 8),
    "gpt2_batch": _w("gpt2_batch", 8, 12, 1024, 64, "bf16", True, True),
    "seq4k_fp16": _w("seq4k_fp16", 1, 32, 4096, 64, "fp16", False, False, scale_inputs=0.5),
    "trading_day": _w("trading_day", 1, 12, 23400, 64, "bf16", True, True, low_rank=True),
}
for _n in (2048, 8192, 16384):
    for _c in (False, True):
        _k = f"d128_n{_n}_{'causal' if _c else 'nc'}"
        WORKLOADS[_k] = _w(_k, 2, 16, _n, 128, "bf16", _c, True)


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def make_inputs(w: Workload, with_grad: Optional[bool] = None):
    """Return dict(q, k, v[, do]) of CPU tensors in ``w``'s storage dtype."""
    if with_grad is None:
        with_grad = w.backward
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)

    def randn(*s):
        return torch.randn(*s, generator=g, dtype=torch.float32)

    if w.low_rank:
        zq = randn(*shape)
        zk = randn(*shape)
        u = randn(w.B, w.H, w.N, 4)
        a = randn(w.B, w.H, 4, w.d) * 0.5
        shared = 2.0 * torch.matmul(u, a)
        q = zq + shared
        k = zk + shared
        del zq, zk, u, a, shared
    else:
        q = randn(*shape)
        k = randn(*shape)
    v = randn(*shape)
    if w.scale_inputs != 1.0:
        q = q * w.scale_inputs
        k = k * w.scale_inputs
        v = v * w.scale_inputs
    out = {}
    for name, t in (("q", q), ("k", k), ("v", v)):
        out[name] = t.to(w.torch_dtype)
    if with_grad:
        out["do"] = randn(*shape).to(w.torch_dtype)
    return out
