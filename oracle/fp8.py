"""CPU oracle for the FP8 forward with incoherent processing.

TEST INFRASTRUCTURE ONLY, like ``oracle.attention``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it, and it
shares nothing with the CUDA library.

The method (marketmaker.cc "Flash Attention and the sequence-length problem",
section "FA3: Hopper mechanics", item 3): FP8 attention is hurt by outliers,
so the vectors are multiplied by a random orthogonal matrix before they are
quantised block by block, which spreads an outlier over all coordinates; the
page reports 2.6x lower numerical error than plain FP8.  The page fixes
neither the rotation, the format nor the block shape; the readings taken here
(each a plain choice, listed with the others in the design notes):

* rotation: R = diag(s) H / sqrt(d), H the Sylvester Hadamard matrix of order
  d (d a power of two), s a vector of random signs drawn by the caller.
  R is orthogonal, so (Q R)(K R)^T = Q K^T and only Q and K are rotated.
  It is applied by the fast Walsh-Hadamard transform in float32: signs, then
  butterfly stages of span 1, 2, 4, ..., d/2 (a, b) -> (a + b, a - b), then
  the factor 1/sqrt(d) rounded to float32.
* format: float8 e4m3 (4 exponent bits, bias 7, 3 mantissa bits, subnormals,
  largest finite 448), round to nearest even, saturating at +-448.
* block scales: Q and K one scale per head and 128-row block, V one scale per
  head and channel; scale = amax / 448 in float32 (1 when amax = 0), code =
  e4m3(x / scale) with the division in float32.
* attention on the dequantised values (code * scale, exact in float64) is the
  plain two-pass definition; the kernel additionally rounds P to e4m3 before
  the P V product, which the parity tolerance covers.

Pins (tests/test_oracle_pins.py): e4m3 rounding against exhaustive search over
all 256 codes and against torch's float8_e4m3fn cast; the Hadamard matrix
against scipy.linalg.hadamard and H H^T = d I; the float32 transform against
the float64 product with the matrix; the scales and codes against their
definitions; the rotation leaving Q K^T unchanged.
"""

from __future__ import annotations

import numpy as np

from .attention import attn_fwd_ref

__all__ = [
    "E4M3_MAX",
    "e4m3_round_ref",
    "hadamard_ref",
    "rotate_ref",
    "quantize_rows_ref",
    "quantize_cols_ref",
    "fp8_inputs_ref",
    "fp8_attn_fwd_ref",
]

E4M3_MAX = 448.0


def e4m3_round_ref(x):
    """Round to the nearest float8 e4m3 value (ties to even), saturating at
    +-448.  Input and output are float64 arrays of values."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # spacing of representable values: 2^(e-3) in the binade [2^e, 2^(e+1))
    # for normals (e >= -6), 2^-9 for subnormals
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    q = np.exp2(np.maximum(e, -6.0) - 3.0)
    r = np.round(a / q) * q          # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def hadamard_ref(d):
    """Sylvester Hadamard matrix of order d (a power of two), entries +-1."""
    if d < 1 or d & (d - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def rotate_ref(x, signs):
    """x R with R = diag(signs) H / sqrt(d), by the float32 fast transform
    (signs, butterflies of span 1, 2, ..., d/2, then 1/sqrt(d)).  x: [..., d]."""
    y = np.asarray(x, dtype=np.float32) * np.asarray(signs, dtype=np.float32)
    d = y.shape[-1]
    h = 1
    while h < d:
        y = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a = y[..., 0, :].copy()
        b = y[..., 1, :].copy()
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        y = y.reshape(y.shape[:-3] + (d,))
        h *= 2
    return y * np.float32(1.0 / np.sqrt(d))


def _scale_of(amax):
    amax = np.asarray(amax, dtype=np.float32)
    s = amax / np.float32(E4M3_MAX)
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows_ref(x, block=128):
    """Per 128-row block of each head: scale = amax / 448, values e4m3(x /
    scale).  x: [..., N, d] float32; returns (code values [..., N, d] float64,
    scales [..., ceil(N/block)] float32)."""
    x = np.asarray(x, dtype=np.float32)
    n = x.shape[-2]
    nb = -(-n // block)
    scales = np.empty(x.shape[:-2] + (nb,), dtype=np.float32)
    vals = np.empty(x.shape, dtype=np.float64)
    for b in range(nb):
        blk = x[..., b * block:(b + 1) * block, :]
        s = _scale_of(np.abs(blk).max(axis=(-2, -1)))
        scales[..., b] = s
        vals[..., b * block:(b + 1) * block, :] = e4m3_round_ref(blk / s[..., None, None])
    return vals, scales


def quantize_cols_ref(x):
    """Per head and channel: scale = amax over the rows / 448.  Returns (code
    values [..., N, d] float64, scales [..., d] float32)."""
    x = np.asarray(x, dtype=np.float32)
    s = _scale_of(np.abs(x).max(axis=-2))
    return e4m3_round_ref(x / s[..., None, :]), s


def fp8_inputs_ref(q, k, v, signs=None, block=128):
    """The quantised operands: Q and K rotated (when ``signs`` is given) and
    quantised per row block, V per channel.  Returns a dict of code values
    and scales."""
    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    if signs is not None:
        q = rotate_ref(q, signs)
        k = rotate_ref(k, signs)
    qv, sq = quantize_rows_ref(q, block)
    kv, sk = quantize_rows_ref(k, block)
    vv, sv = quantize_cols_ref(v)
    return {"q": qv, "sq": sq, "k": kv, "sk": sk, "v": vv, "sv": sv}


def fp8_attn_fwd_ref(q, k, v, scale, causal=False, signs=None, block=128):
    """Attention of the dequantised operands (float64, two-pass).  Returns
    (O, LSE) like ``attn_fwd_ref``."""
    z = fp8_inputs_ref(q, k, v, signs, block)
    rep = lambda s, n: np.repeat(s.astype(np.float64), block, axis=-1)[..., :n]
    n = z["q"].shape[-2]
    qd = z["q"] * rep(z["sq"], n)[..., None]
    kd = z["k"] * rep(z["sk"], n)[..., None]
    vd = z["v"] * z["sv"].astype(np.float64)[..., None, :]
    return attn_fwd_ref(qd, kd, vd, scale, causal)
