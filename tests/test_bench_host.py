"""Host-side pieces of bench.py that need no GPU: the pair count behind the
block-sparse FLOPs, the FLOP convention, the comment-blind hash of the
kernel sources and the rule that a committed DRAM-traffic figure is used
only while the kernels it was measured on are unchanged."""

import numpy as np
import pytest

import bench
from exact_io_aware_84_b200.metrics import attn_fwd_flops


def _pairs_brute(mask, N, causal):
    q = np.arange(N)[:, None]
    k = np.arange(N)[None, :]
    keep = np.ones((N, N), dtype=bool) if not causal else (k <= q)
    total = 0
    for b in range(mask.shape[0]):
        for h in range(mask.shape[1]):
            m = mask[b, h][q // 128, k // 128].astype(bool)
            total += int((m & keep).sum())
    return total


@pytest.mark.parametrize("N", [1, 128, 300, 640])
@pytest.mark.parametrize("causal", [False, True])
def test_attended_pairs_matches_brute_force(N, causal):
    nb = (N + 127) // 128
    mask = (np.random.default_rng(N + causal).random((2, 3, nb, nb)) < 0.6).astype(np.uint8)
    assert bench._attended_pairs(mask, N, causal) == _pairs_brute(mask, N, causal)


def test_dense_mask_gives_the_flop_convention():
    # all tiles kept: 4 d x pairs is the dense forward count.  Causal keeps
    # N (N + 1) / 2 pairs per head, while the FLOP convention counts exactly
    # half of the dense N^2: the two differ by the diagonal's N / 2.
    B, H, N, d = 1, 2, 384, 64
    full = np.ones((B, H, 3, 3), dtype=np.uint8)
    assert 4 * d * bench._attended_pairs(full, N, False) == attn_fwd_flops(B, H, N, d, False)
    causal_pairs = bench._attended_pairs(full, N, True)
    assert causal_pairs == B * H * N * (N + 1) / 2
    assert 4 * d * (causal_pairs - B * H * N / 2) == attn_fwd_flops(B, H, N, d, True)


def test_code_only_drops_comments_and_keeps_strings():
    src = 'int a; // note\n/* block\n comment */ const char* s = "x // y /* z */";\n\n  b += 1; /* t */\n'
    assert bench._code_only(src) == 'int a;\n const char* s = "x // y /* z */";\n  b += 1;'


def test_kernel_hash_ignores_comment_edits(tmp_path, monkeypatch):
    csrc = tmp_path / "exact_io_aware_84_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k() {}  // first\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h1 = bench.kernel_sources_hash()
    (csrc / "k.cu").write_text("// a new comment\n__global__ void k() {}\n")
    assert bench.kernel_sources_hash() == h1
    (csrc / "k.cu").write_text("__global__ void k() { int x = 1; }\n")
    assert bench.kernel_sources_hash() != h1


def test_traffic_key_only_while_kernels_unchanged(tmp_path, monkeypatch):
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"kernel_sources": "0123456789abcdef", "per_launch_bytes": {"w": {"fa_bwd_main": 4096}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda: "0123456789abcdef")
    assert bench._ncu_traffic("w", "fa_bwd_main") == 4096
    assert bench._ncu_traffic("w", "fa_fwd_kernel") is None
    assert bench._ncu_traffic("other", "fa_bwd_main") is None
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda: "fedcba9876543210")
    assert bench._ncu_traffic("w", "fa_bwd_main") is None


def test_oracle_unit_is_bounded():
    from exact_io_aware_84_b200.inputs import workload
    for name in ("gpt2_batch", "trading_day", "d128_n8192_nc", "d128_n16384_causal", "tiny_fwd"):
        w = workload(name)
        n, flops = bench._oracle_unit(w)
        assert n % 128 == 0 or n == w.N
        assert n <= w.N and flops <= bench.ORACLE_HEAD_FLOP_CAP
    assert bench._oracle_unit(workload("gpt2_batch"))[0] == 1024   # small heads stay whole
