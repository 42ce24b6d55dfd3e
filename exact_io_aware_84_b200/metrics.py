"""Measurement conventions: FLOP counts, algorithmic bytes, avoided bytes.

No attention arithmetic happens here; these are the counting rules that the
benchmark and the roofline report use.
"""

from __future__ import annotations

__all__ = [
    "attn_fwd_flops",
    "attn_bwd_flops",
    "score_matrix_bytes",
    "fwd_algorithmic_bytes",
    "bwd_algorithmic_bytes",
]


def attn_fwd_flops(B, H, N, d, causal):
    """Forward FLOPs: two N x N x d matmuls per (b, h) = 4 B H N^2 d.

    Causal halves it exactly by convention (tiles entirely in the future are
    skipped: marketmaker.cc "Flash Attention and the sequence-length problem",
    section on causal masking), ragged N included.
    """
    f = 4.0 * B * H * N * N * d
    return f / 2.0 if causal else f


def attn_bwd_flops(B, H, N, d, causal):
    """Backward FLOPs: 2.5 x the forward (five N x N x d matmuls vs two)."""
    return 2.5 * attn_fwd_flops(B, H, N, d, causal)


def score_matrix_bytes(B, H, N, elem_bytes):
    """A_bytes = B H N^2 e: the score matrix standard attention materialises.

    Source: onecalc.app "Attention memory calculator", section "Formula".
    """
    return int(B) * int(H) * int(N) * int(N) * int(elem_bytes)


def fwd_algorithmic_bytes(B, H, N, d, elem_bytes=2):
    """Compulsory HBM bytes of the forward: read Q, K, V; write O (each
    B H N d elements) and the fp32 LSE (B H N)."""
    return 4 * B * H * N * d * elem_bytes + 4 * B * H * N


def bwd_algorithmic_bytes(B, H, N, d, elem_bytes=2):
    """Compulsory HBM bytes of the backward: read Q, K, V, O, dO and the LSE;
    write dQ, dK, dV.  The fp32 dQ accumulator is implementation overhead and
    is not counted."""
    return 8 * B * H * N * d * elem_bytes + 4 * B * H * N
