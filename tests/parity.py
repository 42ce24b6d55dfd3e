"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used by every parity test):
  O    : max |GPU - oracle| <= 2e-2 and mean |GPU - oracle| <= 2e-3
  LSE  : max |GPU - oracle| <= 1e-3
  dQ, dK, dV : ||GPU - oracle||_F / ||oracle||_F <= 1e-2 (per tensor); where
               the oracle's gradient is exactly zero (N = 1: P = 1, so dS = 0
               and dQ = dK = 0) the ratio is undefined and max |GPU| <= 1e-4
               applies instead.
The oracle runs in float64 on the same bf16/fp16-rounded inputs the GPU sees.
"""

import numpy as np
import torch

TOL_O_MAX = 2e-2
TOL_O_MEAN = 2e-3
TOL_LSE = 1e-3
TOL_GRAD_REL = 1e-2
TOL_GRAD_ABS_ZERO = 1e-4


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def sample_rows(N, rng, n_random=512, block=128):
    """Rows the oracle checks on long sequences: the first and last query
    tiles, every tile boundary +-1, the ragged tail, and random rows."""
    rows = set(range(min(N, block)))
    rows |= set(range(max(0, (N - 1) // block * block), N))
    for b in range(block, N, block):
        rows |= {b - 1, b, b + 1}
    rows |= set(rng.integers(0, N, size=min(n_random, N)).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N))


def check_o_lse(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite O"
    assert np.isfinite(lse_gpu).all(), f"{what}: non-finite LSE"
    d = np.abs(o_gpu - o_ref)
    dl = np.abs(lse_gpu - lse_ref)
    msg = (f"{what}: O max {d.max():.3e} mean {d.mean():.3e}; LSE max {dl.max():.3e}"
           f" (worst O at {np.unravel_index(d.argmax(), d.shape)}, LSE at {np.unravel_index(dl.argmax(), dl.shape)})")
    assert d.max() <= TOL_O_MAX and d.mean() <= TOL_O_MEAN and dl.max() <= TOL_LSE, msg
    return d.max(), d.mean(), dl.max()


def rel_fro(a, ref):
    a = np.asarray(a, dtype=np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))


def check_grads(gpu, ref, what=""):
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), gpu, ref):
        g = np.asarray(g, dtype=np.float64)
        assert np.isfinite(g).all(), f"{what}: non-finite {name}"
        if not np.any(r):
            assert np.abs(g).max() <= TOL_GRAD_ABS_ZERO, f"{what}: {name} should be 0, max {np.abs(g).max():.3e}"
            out[name] = 0.0
            continue
        e = rel_fro(g, r)
        out[name] = e
    assert all(e <= TOL_GRAD_REL for e in out.values()), f"{what}: rel Frobenius {out}"
    return out
