"""Pins for the fp64 oracle, each against something other than the oracle.

* brute force: pure-Python loops over math.exp on tiny inputs;
* a library routine: scipy.special.softmax / logsumexp for the special case
  of one query row;
* closed forms and invariants of softmax attention;
* finite differences of an independent (pure-Python) forward for the
  gradient;
* the pages' own worked numbers (tests/golden/).

Each is chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand, a wrong mask direction) fails at least
one of them.
"""

import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import (attn_bwd_ref, attn_fwd_ref, attn_fwd_rows_ref,
                    attn_probs_ref, attn_scores_ref, fa1_fwd_ref,
                    blocksparse_bwd_ref, blocksparse_fwd_ref,
                    gqa_bwd_ref, gqa_fwd_ref, online_fwd_ref,
                    attn_bwd_partial_ref, attn_dq_rows_ref, merge_partials_ref,
                    ring_bwd_ref, ring_fwd_ref)
from exact_io_aware_84_b200.metrics import score_matrix_bytes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _brute_fwd(q, k, v, scale, causal):
    """Explicit loops: for every query row, every key, every channel."""
    n, d = len(q), len(q[0])
    nk, dv = len(k), len(v[0])
    o = [[0.0] * dv for _ in range(n)]
    lse = [0.0] * n
    for i in range(n):
        s = []
        for j in range(nk):
            if causal and j > i:
                continue
            dot = 0.0
            for c in range(d):
                dot += float(q[i][c]) * float(k[j][c])
            s.append((j, scale * dot))
        mx = max(x for _, x in s)
        tot = sum(math.exp(x - mx) for _, x in s)
        lse[i] = mx + math.log(tot)
        for j, x in s:
            w = math.exp(x - mx) / tot
            for c in range(dv):
                o[i][c] += w * float(v[j][c])
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 1), (2, 3), (5, 4), (8, 2), (8, 4)])
def test_forward_matches_brute_force(n, d, causal):
    r = _rng(100 * n + d + causal)
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    scale = 0.7
    o_b, lse_b = _brute_fwd(q, k, v, scale, causal)
    o, lse = attn_fwd_ref(q, k, v, scale, causal)
    np.testing.assert_allclose(o, o_b, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, lse_b, rtol=0, atol=1e-14)


def test_forward_matches_brute_force_rectangular_keys():
    # more keys than queries, non-causal: a transposed q/k operand would fail
    r = _rng(7)
    q = r.standard_normal((3, 4))
    k = r.standard_normal((6, 4))
    v = r.standard_normal((6, 2))
    o_b, lse_b = _brute_fwd(q, k, v, 0.3, False)
    o, lse = attn_fwd_rows_ref(q, k, v, 0.3, False)
    np.testing.assert_allclose(o, o_b, atol=1e-14)
    np.testing.assert_allclose(lse, lse_b, atol=1e-14)


def test_batched_leading_dims_match_per_head():
    r = _rng(11)
    q, k, v = (r.standard_normal((2, 3, 9, 5)) for _ in range(3))
    o, lse = attn_fwd_ref(q, k, v, 0.5, True)
    for b in range(2):
        for h in range(3):
            ob, lb = _brute_fwd(q[b, h], k[b, h], v[b, h], 0.5, True)
            np.testing.assert_allclose(o[b, h], ob, atol=1e-14)
            np.testing.assert_allclose(lse[b, h], lb, atol=1e-14)


def test_single_row_is_library_softmax():
    # one query row: P is scipy's softmax of the scaled scores, LSE its logsumexp
    r = _rng(3)
    q = r.standard_normal((1, 16))
    k = r.standard_normal((40, 16))
    v = r.standard_normal((40, 8))
    scale = 1 / 4
    s = scale * (k @ q[0])
    p_lib = scipy.special.softmax(s)
    o, lse = attn_fwd_ref(q, k, v, scale, False)
    np.testing.assert_allclose(lse[0], scipy.special.logsumexp(s), atol=1e-13)
    np.testing.assert_allclose(o[0], p_lib @ v, atol=1e-13)
    np.testing.assert_allclose(attn_probs_ref(q, k, scale)[0], p_lib, atol=1e-15)


def test_row_chunking_does_not_change_results():
    r = _rng(5)
    q, k, v, do = (r.standard_normal((2, 37, 6)) for _ in range(4))
    o1, l1 = attn_fwd_ref(q, k, v, 0.4, True, row_chunk=1000)
    o2, l2 = attn_fwd_ref(q, k, v, 0.4, True, row_chunk=5)
    np.testing.assert_allclose(o1, o2, atol=1e-15)
    np.testing.assert_allclose(l1, l2, atol=1e-15)
    g1 = attn_bwd_ref(q, k, v, do, 0.4, True, row_chunk=1000)
    g2 = attn_bwd_ref(q, k, v, do, 0.4, True, row_chunk=4)
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, atol=1e-13)


def test_sampled_rows_match_full():
    r = _rng(6)
    q, k, v = (r.standard_normal((50, 8)) for _ in range(3))
    rows = np.array([0, 1, 17, 31, 49])
    o, lse = attn_fwd_ref(q, k, v, 0.3, True)
    os_, ls = attn_fwd_rows_ref(q, k, v, 0.3, True, rows=rows, row_chunk=2)
    np.testing.assert_allclose(os_, o[rows], atol=1e-15)
    np.testing.assert_allclose(ls, lse[rows], atol=1e-15)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    r = _rng(8)
    q, k = r.standard_normal((33, 7)), r.standard_normal((33, 7))
    p = attn_probs_ref(q, k, 0.9, causal)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)
    assert (p >= 0).all()
    if causal:
        assert np.all(np.triu(p, 1) == 0)
        assert np.all(np.diag(p) > 0)


def test_zero_query_gives_column_means():
    r = _rng(9)
    n = 21
    q = np.zeros((n, 5))
    k, v = r.standard_normal((n, 5)), r.standard_normal((n, 3))
    o, lse = attn_fwd_ref(q, k, v, 0.5, False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(n), atol=1e-14)
    o, lse = attn_fwd_ref(q, k, v, 0.5, True)
    cum = np.cumsum(v, 0) / np.arange(1, n + 1)[:, None]
    np.testing.assert_allclose(o, cum, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.arange(1, n + 1)), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_value_rows(causal):
    r = _rng(10)
    q, k = r.standard_normal((19, 4)), r.standard_normal((19, 4))
    c = r.standard_normal(6)
    v = np.broadcast_to(c, (19, 6)).copy()
    o, _ = attn_fwd_ref(q, k, v, 1.3, causal)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-14)


def test_causal_first_row():
    r = _rng(12)
    q, k, v = (r.standard_normal((10, 4)) for _ in range(3))
    o, lse = attn_fwd_ref(q, k, v, 0.6, True)
    np.testing.assert_allclose(o[0], v[0], atol=1e-15)
    np.testing.assert_allclose(lse[0], 0.6 * q[0] @ k[0], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    # adding the same vector u to every key adds scale*q_i.u to row i's scores
    r = _rng(13)
    q, k, v = (r.standard_normal((15, 4)) for _ in range(3))
    u = r.standard_normal(4)
    o1, l1 = attn_fwd_ref(q, k, v, 0.8, causal)
    o2, l2 = attn_fwd_ref(q, k + u, v, 0.8, causal)
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + 0.8 * (q @ u), atol=1e-13)


def test_joint_key_value_permutation_invariance():
    r = _rng(14)
    q, k, v = (r.standard_normal((12, 4)) for _ in range(3))
    perm = r.permutation(12)
    o1, l1 = attn_fwd_ref(q, k, v, 0.8, False)
    o2, l2 = attn_fwd_ref(q, k[perm], v[perm], 0.8, False)
    np.testing.assert_allclose(o2, o1, atol=1e-14)
    np.testing.assert_allclose(l2, l1, atol=1e-14)


def test_two_keys_is_logistic():
    # one query, two keys: weight on key 0 is sigmoid(s0 - s1)
    q = np.array([[0.3, -1.2]])
    k = np.array([[1.0, 0.5], [-0.4, 2.0]])
    v = np.array([[2.0], [-3.0]])
    s0, s1 = 0.5 * q[0] @ k[0], 0.5 * q[0] @ k[1]
    w0 = 1 / (1 + math.exp(-(s0 - s1)))
    o, lse = attn_fwd_ref(q, k, v, 0.5, False)
    np.testing.assert_allclose(o[0, 0], w0 * 2.0 + (1 - w0) * -3.0, atol=1e-15)
    np.testing.assert_allclose(lse[0], math.log(math.exp(s0) + math.exp(s1)), atol=1e-15)


# ------------------------------------------------------ online / tiled forms

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 3, 64, 128, 300])
def test_online_matches_two_pass(block, causal):
    r = _rng(15)
    q, k, v = (r.standard_normal((300, 16)) for _ in range(3))
    o, lse = attn_fwd_ref(q, k, v, 0.25, causal)
    o2, lse2 = online_fwd_ref(q, k, v, 0.25, causal, block=block)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("br,bc", [(1, 1), (3, 5), (128, 128), (64, 256)])
def test_per_step_normalised_loop_matches_two_pass(br, bc, causal):
    r = _rng(16)
    q, k, v = (r.standard_normal((203, 8)) for _ in range(3))
    o, lse = attn_fwd_ref(q, k, v, 0.35, causal)
    o2, lse2 = fa1_fwd_ref(q, k, v, 0.35, causal, block_r=br, block_c=bc)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


def test_online_handles_large_scores():
    # scores of order 1e3 would overflow a naive exp; the recurrence must not
    r = _rng(17)
    q, k, v = (r.standard_normal((40, 8)) * 12 for _ in range(3))
    o, lse = attn_fwd_ref(q, k, v, 1.0, True)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    o2, lse2 = online_fwd_ref(q, k, v, 1.0, True, block=7)
    np.testing.assert_allclose(o2, o, atol=1e-11)
    np.testing.assert_allclose(lse2, lse, rtol=1e-14, atol=1e-11)


def test_glossary_fp32_loop_error_magnitude():
    """The glossary's float32 online loop differs from float32 full-matrix
    attention by rounding only (tests/golden/online_loop_fp32_error.txt)."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "online_loop_fp32_error.txt"))
            if l.strip() and not l.startswith("#")]
    n, d, block, seed, page, factor = rows[0]
    n, d, block, seed, page, factor = int(n), int(d), int(block), int(seed), float(page), float(factor)
    torch.manual_seed(seed)
    q, k, v = torch.randn(3, n, d).unbind(0)
    full = (torch.softmax(q @ k.T / d ** 0.5, dim=-1) @ v).numpy()
    o32, _ = online_fwd_ref(q.numpy(), k.numpy(), v.numpy(), 1.0 / d ** 0.5,
                            block=block, dtype=np.float32)
    err = float(np.abs(o32.astype(np.float64) - full).max())
    assert page / factor <= err <= page * factor, err


# ----------------------------------------------------------------- gradient

def _fd_grads(q, k, v, do, scale, causal, h=1e-6):
    """Central differences of L = sum(dO * O) using the brute-force forward."""
    grads = []
    for x in (q, k, v):
        g = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            op, _ = _brute_fwd(q, k, v, scale, causal)
            x[idx] = old - h
            om, _ = _brute_fwd(q, k, v, scale, causal)
            x[idx] = old
            g[idx] = np.sum(do * (op - om)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(4, 3), (7, 2), (16, 4)])
def test_gradient_matches_finite_differences(n, d, causal):
    r = _rng(200 + n + causal)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    scale = 0.6
    dq, dk, dv = attn_bwd_ref(q, k, v, do, scale, causal)
    for name, ana, num in zip("qkv", (dq, dk, dv), _fd_grads(q, k, v, do, scale, causal)):
        rel = np.linalg.norm(ana - num) / max(np.linalg.norm(num), 1e-30)
        assert rel <= 1e-6, (name, rel)
        np.testing.assert_allclose(ana, num, rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("causal", [False, True])
def test_row_dq_matches_finite_differences(causal):
    # dQ of a subset of rows, straight from the finite differences of the
    # brute-force forward (row i of dQ only moves O_i)
    r = _rng(210 + causal)
    n, d = 9, 3
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    rows = np.array([0, 4, 8])
    dq_rows = attn_dq_rows_ref(q, k, v, do, 0.7, causal, rows=rows)
    num = _fd_grads(q, k, v, do, 0.7, causal)[0]
    np.testing.assert_allclose(dq_rows, num[rows], rtol=1e-5, atol=1e-7)


def test_row_dq_with_stored_o():
    # an identity "storage" gives the exact gradient; a perturbed O changes dQ
    # by exactly -scale * dD_i * (P K)_i, the only term in which D appears
    r = _rng(212)
    n, d = 11, 4
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    rows = np.arange(n)
    exact, same, shifted = attn_dq_rows_ref(q, k, v, do, 0.5, True, rows=rows,
                                            o_for_d=[None, lambda o: o, lambda o: o + 0.01])
    np.testing.assert_array_equal(same, exact)
    p = attn_probs_ref(q, k, 0.5, True)
    d_d = (do * 0.01).sum(-1, keepdims=True)
    np.testing.assert_allclose(shifted - exact, -0.5 * d_d * (p @ k), rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    r = _rng(18)
    q, k, v, do = (r.standard_normal((2, 3, 29, 8)) for _ in range(4))
    dq, dk, dv = attn_bwd_ref(q, k, v, do, 0.4, causal)
    # rows of dS sum to zero, so the key gradients sum to zero over keys
    np.testing.assert_allclose(dk.sum(-2), 0.0, atol=1e-12)
    # every row of P sums to one, so dV summed over keys is dO summed over rows
    np.testing.assert_allclose(dv.sum(-2), do.sum(-2), atol=1e-12)


def test_constant_value_has_no_score_gradient():
    r = _rng(19)
    q, k = r.standard_normal((17, 4)), r.standard_normal((17, 4))
    do = r.standard_normal((17, 5))
    v = np.broadcast_to(r.standard_normal(5), (17, 5)).copy()
    dq, dk, _ = attn_bwd_ref(q, k, v, do, 0.9, True)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dk, 0.0, atol=1e-13)


def test_causal_mask_direction():
    # with causal masking, row i never depends on keys/values after i
    r = _rng(20)
    q, k, v = (r.standard_normal((9, 3)) for _ in range(3))
    o1, l1 = attn_fwd_ref(q, k, v, 1.0, True)
    k2, v2 = k.copy(), v.copy()
    k2[5:] += 3.0
    v2[5:] -= 2.0
    o2, l2 = attn_fwd_ref(q, k2, v2, 1.0, True)
    np.testing.assert_allclose(o2[:5], o1[:5], atol=0)
    np.testing.assert_allclose(l2[:5], l1[:5], atol=0)
    assert np.abs(o2[5:] - o1[5:]).max() > 1e-3
    s, _ = attn_scores_ref(q, k, 1.0, True)
    assert np.isneginf(s[0, 1]) and np.isfinite(s[1, 0])


# ---------------------------------------------------------- pages' figures

def test_score_matrix_memory_worked_examples():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "score_matrix_memory.txt"))
            if l.strip() and not l.startswith("#")]
    for B, H, s, e, expect, page_gb, tol in rows:
        got = score_matrix_bytes(int(B), int(H), int(s), int(e))
        assert got == int(expect)
        assert abs(got / 1e9 - float(page_gb)) <= float(tol) * float(page_gb)


# ------------------------------------------------------- grouped-query heads

@pytest.mark.parametrize("causal", [False, True])
def test_gqa_forward_brute_force(causal):
    # 4 query heads over 2 key/value heads: query head h reads kv head h // 2
    r = _rng(40 + causal)
    q = r.standard_normal((1, 4, 6, 3))
    k = r.standard_normal((1, 2, 6, 3))
    v = r.standard_normal((1, 2, 6, 2))
    o, lse = gqa_fwd_ref(q, k, v, 0.7, causal)
    for h in range(4):
        ob, lb = _brute_fwd(q[0, h], k[0, h // 2], v[0, h // 2], 0.7, causal)
        np.testing.assert_allclose(o[0, h], ob, atol=1e-14)
        np.testing.assert_allclose(lse[0, h], lb, atol=1e-14)


def test_gqa_group_of_one_is_multi_head():
    r = _rng(42)
    q, k, v, do = (r.standard_normal((2, 3, 9, 4)) for _ in range(4))
    for a, b in zip(gqa_fwd_ref(q, k, v, 0.5, True), attn_fwd_ref(q, k, v, 0.5, True)):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(gqa_bwd_ref(q, k, v, do, 0.5, True), attn_bwd_ref(q, k, v, do, 0.5, True)):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_gradient_matches_finite_differences(causal):
    # the shared key/value heads receive gradient from every query head of
    # their group: central differences of L = sum(dO * O) over all heads
    r = _rng(43 + causal)
    H, Hkv, n, d = 4, 2, 5, 3
    q = r.standard_normal((1, H, n, d))
    k = r.standard_normal((1, Hkv, n, d))
    v = r.standard_normal((1, Hkv, n, d))
    do = r.standard_normal((1, H, n, d))
    scale, h_step = 0.6, 1e-6

    def loss():
        tot = 0.0
        for hh in range(H):
            o, _ = _brute_fwd(q[0, hh], k[0, hh // 2], v[0, hh // 2], scale, causal)
            tot += float(np.sum(do[0, hh] * o))
        return tot

    dq, dk, dv = gqa_bwd_ref(q, k, v, do, scale, causal)
    for x, ana in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h_step
            lp = loss()
            x[idx] = old - h_step
            lm = loss()
            x[idx] = old
            num[idx] = (lp - lm) / (2 * h_step)
        np.testing.assert_allclose(ana, num, rtol=1e-5, atol=1e-7)


# ------------------------------------------------------------ block sparsity

def _brute_masked(q, k, v, scale, keep):
    """Explicit loops over the kept (query, key) pairs; empty rows give O = 0
    and LSE = -inf."""
    n, dv = len(q), len(v[0])
    o = np.zeros((n, dv))
    lse = np.full(n, -np.inf)
    for i in range(n):
        s = [(j, scale * sum(float(q[i][c]) * float(k[j][c]) for c in range(len(q[0]))))
             for j in range(len(k)) if keep[i][j]]
        if not s:
            continue
        mx = max(x for _, x in s)
        tot = sum(math.exp(x - mx) for _, x in s)
        lse[i] = mx + math.log(tot)
        for j, x in s:
            o[i] += math.exp(x - mx) / tot * np.asarray(v[j], dtype=float)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_forward_brute_force(causal):
    # blocks of 2 over 7 rows (4 blocks, the last one ragged); query block 1
    # sees no key block at all, so its rows are empty
    r = _rng(50 + causal)
    n = 7
    q, k, v = (r.standard_normal((n, 3)) for _ in range(3))
    bm = np.array([[1, 0, 1, 1], [0, 0, 0, 0], [1, 1, 0, 1], [0, 1, 1, 1]], dtype=bool)
    keep = [[bool(bm[i // 2, j // 2]) and (not causal or j <= i) for j in range(n)] for i in range(n)]
    o, lse = blocksparse_fwd_ref(q, k, v, 0.8, causal, bm, block=2)
    ob, lb = _brute_masked(q, k, v, 0.8, keep)
    np.testing.assert_allclose(o, ob, atol=1e-14)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], atol=1e-14)
    assert np.all(o[2:4] == 0) and np.all(np.isneginf(lse[2:4]))


def test_blocksparse_dense_mask_is_full_attention():
    r = _rng(52)
    q, k, v, do = (r.standard_normal((2, 2, 9, 4)) for _ in range(4))
    bm = np.ones((5, 5), dtype=bool)
    for a, b in zip(blocksparse_fwd_ref(q, k, v, 0.5, True, bm, block=2), attn_fwd_ref(q, k, v, 0.5, True)):
        np.testing.assert_allclose(a, b, atol=1e-15)
    for a, b in zip(blocksparse_bwd_ref(q, k, v, do, 0.5, True, bm, block=2), attn_bwd_ref(q, k, v, do, 0.5, True)):
        np.testing.assert_allclose(a, b, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_gradient_matches_finite_differences(causal):
    r = _rng(53 + causal)
    n, d = 6, 3
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    bm = np.array([[1, 0, 1], [1, 1, 0], [0, 0, 0]], dtype=bool)  # last query block empty
    keep = [[bool(bm[i // 2, j // 2]) and (not causal or j <= i) for j in range(n)] for i in range(n)]
    scale, h = 0.7, 1e-6
    dq, dk, dv = blocksparse_bwd_ref(q, k, v, do, scale, causal, bm, block=2)
    for x, ana in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = float(np.sum(do * _brute_masked(q, k, v, scale, keep)[0]))
            x[idx] = old - h
            lm = float(np.sum(do * _brute_masked(q, k, v, scale, keep)[0]))
            x[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(ana, num, rtol=1e-5, atol=1e-7)
    assert np.all(dq[4:] == 0)  # empty rows: no gradient



# ---------------------------------------------------------------- ring attention

def test_merge_of_disjoint_key_sets_is_brute_force_of_their_union():
    r = _rng(61)
    n, m, d = 5, 9, 3
    q, k, v = r.standard_normal((n, d)), r.standard_normal((m, d)), r.standard_normal((m, d))
    # interleaved, uneven split of the keys; row 4 sees keys of one set only
    in_a = [[j % 3 == 0 for j in range(m)] for _ in range(n)]
    in_b = [[j % 3 != 0 for j in range(m)] for _ in range(n)]
    in_b[4] = [False] * m
    both = [[a or b for a, b in zip(ra, rb)] for ra, rb in zip(in_a, in_b)]
    oa, la = _brute_masked(q, k, v, 0.6, in_a)
    ob, lb = _brute_masked(q, k, v, 0.6, in_b)
    o, lse = merge_partials_ref(oa, la, ob, lb)
    o_ref, l_ref = _brute_masked(q, k, v, 0.6, both)
    np.testing.assert_allclose(o, o_ref, atol=1e-14)
    np.testing.assert_allclose(lse, l_ref, atol=1e-14)


def test_merge_special_cases():
    r = _rng(62)
    o1, l1 = r.standard_normal((4, 3)), r.standard_normal(4)
    empty_o, empty_l = np.zeros((4, 3)), np.full(4, -np.inf)
    for o, lse in (merge_partials_ref(o1, l1, empty_o, empty_l), merge_partials_ref(empty_o, empty_l, o1, l1)):
        np.testing.assert_array_equal(o, o1)
        np.testing.assert_array_equal(lse, l1)
    o, lse = merge_partials_ref(empty_o, empty_l, empty_o, empty_l)
    assert not o.any() and np.all(np.isneginf(lse))
    # two copies of one partial: same O, LSE + ln 2
    o, lse = merge_partials_ref(o1, l1, o1, l1)
    np.testing.assert_allclose(o, o1, atol=1e-15)
    np.testing.assert_allclose(lse, l1 + math.log(2.0), atol=1e-15)
    # the heavier partial dominates: LSE_b = LSE_a + ln 3 gives weights 1/4, 3/4
    o2 = r.standard_normal((4, 3))
    o, lse = merge_partials_ref(o1, l1, o2, l1 + math.log(3.0))
    np.testing.assert_allclose(o, 0.25 * o1 + 0.75 * o2, atol=1e-14)
    np.testing.assert_allclose(lse, l1 + math.log(4.0), atol=1e-14)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_forward_is_brute_force(world, causal):
    r = _rng(63 + world)
    n, d = 12, 3
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    o, lse = ring_fwd_ref(q, k, v, 0.9, causal, world)
    ob, lb = _brute_fwd(q.tolist(), k.tolist(), v.tolist(), 0.9, causal)
    np.testing.assert_allclose(o, np.array(ob), atol=1e-14)
    np.testing.assert_allclose(lse, np.array(lb), atol=1e-14)


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_gradient_matches_finite_differences(world, causal):
    r = _rng(71 + world + 2 * causal)
    n, d = 6, 2
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    scale, h = 0.8, 1e-6
    dq, dk, dv = ring_bwd_ref(q, k, v, do, scale, causal, world)
    loss = lambda: sum(float(a) * float(b) for ra, rb in zip(do.tolist(), _brute_fwd(q.tolist(), k.tolist(), v.tolist(), scale, causal)[0]) for a, b in zip(ra, rb))
    for x, ana in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = loss()
            x[idx] = old - h
            lm = loss()
            x[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(ana, num, rtol=1e-5, atol=1e-7)


def test_partial_gradient_over_all_keys_is_the_full_gradient():
    r = _rng(81)
    q, k, v, do = (r.standard_normal((2, 7, 4)) for _ in range(4))
    o, lse = attn_fwd_ref(q, k, v, 0.5, True)
    for a, b in zip(attn_bwd_partial_ref(q, k, v, o, do, lse, 0.5, True), attn_bwd_ref(q, k, v, do, 0.5, True)):
        np.testing.assert_allclose(a, b, atol=1e-13)


def test_partial_gradient_needs_the_full_row_statistics():
    # with the chunk's own (O, LSE) instead of the full rows' the partial
    # gradients do not add up: the sum over chunks is right only with the
    # merged statistics
    r = _rng(82)
    q, k, v, do = (r.standard_normal((6, 3)) for _ in range(4))
    o, lse = attn_fwd_ref(q, k, v, 0.7)
    full = attn_bwd_ref(q, k, v, do, 0.7)
    parts = [attn_bwd_partial_ref(q, k[c], v[c], o, do, lse, 0.7) for c in (slice(0, 2), slice(2, 6))]
    np.testing.assert_allclose(parts[0][0] + parts[1][0], full[0], atol=1e-13)
    np.testing.assert_allclose(np.concatenate([parts[0][1], parts[1][1]]), full[1], atol=1e-13)
    np.testing.assert_allclose(np.concatenate([parts[0][2], parts[1][2]]), full[2], atol=1e-13)
    o0, l0 = attn_fwd_ref(q, k[:2], v[:2], 0.7)
    wrong = attn_bwd_partial_ref(q, k[:2], v[:2], o0, do, l0, 0.7)
    assert np.abs(wrong[2] - parts[0][2]).max() > 1e-3


# ---------------------------------------------------------------- FP8 forward

from oracle import (E4M3_MAX, e4m3_round_ref, fp8_attn_fwd_ref, fp8_inputs_ref,  # noqa: E402
                    hadamard_ref, quantize_cols_ref, quantize_rows_ref, rotate_ref)


def _e4m3_table():
    """Every non-negative finite e4m3 value with its code (exponent bias 7,
    3 mantissa bits; exponent 0 = subnormal; code 0x7f is NaN)."""
    out = []
    for code in range(0x7f):
        e, m = code >> 3, code & 7
        val = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        out.append((val, code))
    return out


def test_e4m3_rounding_is_exhaustive_nearest_ties_to_even():
    table = _e4m3_table()
    vals = np.array([v for v, _ in table])
    codes = np.array([c for _, c in table])
    assert vals.max() == E4M3_MAX == 448.0
    r = _rng(91)
    x = np.concatenate([r.uniform(0, 448, 3000), np.exp2(r.uniform(-12, 8.8, 3000)),
                        (vals[:-1] + vals[1:]) / 2,           # every midpoint: a tie
                        vals])
    x = x[x <= 448.0]
    got = e4m3_round_ref(x)
    for xi, gi in zip(x, got):
        dist = np.abs(vals - xi)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:                                      # tie: even mantissa code
            best = [b for b in best if codes[b] % 2 == 0]
        assert gi == vals[best[0]], (xi, gi, vals[best[0]])
    np.testing.assert_array_equal(e4m3_round_ref(-x), -got)


def test_e4m3_rounding_matches_torch_float8_cast_and_saturates():
    r = _rng(92)
    x = np.concatenate([r.standard_normal(5000) * 50, r.standard_normal(5000) * 0.01]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(e4m3_round_ref(x), want)
    # beyond the largest finite value the oracle saturates (satfinite)
    np.testing.assert_array_equal(e4m3_round_ref([464.0, 500.0, 1e6, -1e6]), [448.0, 448.0, 448.0, -448.0])


def test_hadamard_is_sylvester_and_orthogonal():
    import scipy.linalg
    for d in (1, 2, 8, 64, 128):
        h = hadamard_ref(d)
        np.testing.assert_array_equal(h, scipy.linalg.hadamard(d))
        np.testing.assert_array_equal(h @ h.T, d * np.eye(d))
    with pytest.raises(ValueError):
        hadamard_ref(96)


@pytest.mark.parametrize("d", [64, 128])
def test_fast_rotation_equals_the_matrix_product(d):
    r = _rng(93 + d)
    x = r.standard_normal((3, 50, d)).astype(np.float32)
    s = r.choice([-1.0, 1.0], d)
    y = rotate_ref(x, s)
    assert y.dtype == np.float32
    want = x.astype(np.float64) @ (np.diag(s) @ hadamard_ref(d)) / np.sqrt(d)
    np.testing.assert_allclose(y, want, rtol=0, atol=2e-6 * np.abs(x).max() * np.sqrt(d))
    # orthogonal: norms and inner products are kept
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-5)
    k = r.standard_normal((3, 40, d)).astype(np.float32)
    np.testing.assert_allclose(y @ np.swapaxes(rotate_ref(k, s), -1, -2), x @ np.swapaxes(k, -1, -2),
                               atol=1e-3)


def test_row_block_and_channel_quantisation():
    r = _rng(94)
    x = (r.standard_normal((2, 300, 16)) * np.array([1.0, 10.0])[:, None, None]).astype(np.float32)
    x[1, 128:256] = 0.0                                        # an all-zero block
    vals, sc = quantize_rows_ref(x)
    assert sc.shape == (2, 3) and sc.dtype == np.float32
    for h in range(2):
        for b in range(3):
            blk = x[h, 128 * b:128 * (b + 1)]
            amax = np.float32(np.abs(blk).max())
            if amax == 0:
                assert sc[h, b] == 1.0 and not vals[h, 128 * b:128 * (b + 1)].any()
                continue
            assert sc[h, b] == amax / np.float32(448.0)
            v = vals[h, 128 * b:128 * (b + 1)]
            assert np.abs(v).max() == 448.0                    # the largest element maps to the top code
            np.testing.assert_array_equal(v, e4m3_round_ref(blk / sc[h, b]))
            # dequantised values within half an e4m3 step (2^-4 relative) or a subnormal step
            err = np.abs(v * np.float64(sc[h, b]) - blk)
            assert np.all(err <= np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * float(sc[h, b])) * (1 + 1e-6))
    cv, cs = quantize_cols_ref(x)
    assert cs.shape == (2, 16)
    np.testing.assert_array_equal(cs, np.where(np.abs(x).max(axis=1) > 0, np.abs(x).max(axis=1) / np.float32(448), 1))
    assert np.all(np.abs(cv).max(axis=1)[np.abs(x).max(axis=1) > 0] == 448.0)


def test_fp8_attention_of_exactly_representable_inputs_is_attention():
    # entries in {0, +-1, +-2, +-4}, each block and channel holding a 4: every
    # value is a code (112, 224 or 448) times the scale 4/448, so only the
    # float32 rounding of the scale separates the result from exact attention
    r = _rng(95)
    q, k, v = (r.choice([0.0, 1.0, -1.0, 2.0, -2.0, 4.0, -4.0], (2, 256, 8)) for _ in range(3))
    for x in (q, k, v):
        x[:, ::128, :] = 4.0
        x[:, :, 0] = np.where(np.arange(256) == 5, 4.0, x[:, :, 0])
    o, lse = fp8_attn_fwd_ref(q, k, v, 0.3, True)
    o2, lse2 = attn_fwd_ref(q, k, v, 0.3, True)
    np.testing.assert_allclose(o, o2, atol=1e-5)
    np.testing.assert_allclose(lse, lse2, atol=1e-5)


def test_rotation_lowers_fp8_error_on_outlier_channels():
    # the pages' claim (lower error than plain FP8 when a few channels carry
    # outliers), on the oracle's own quantised attention
    r = _rng(96)
    d = 64
    q, k, v = (r.standard_normal((1, 512, d)) for _ in range(3))
    q[..., :2] *= 30.0
    k[..., :2] *= 30.0
    s = r.choice([-1.0, 1.0], d)
    exact, _ = attn_fwd_ref(q, k, v, d ** -0.5)
    plain, _ = fp8_attn_fwd_ref(q, k, v, d ** -0.5)
    rot, _ = fp8_attn_fwd_ref(q, k, v, d ** -0.5, signs=s)
    e_plain = np.sqrt(np.mean((plain - exact) ** 2))
    e_rot = np.sqrt(np.mean((rot - exact) ** 2))
    assert e_rot < e_plain / 1.5, (e_rot, e_plain)
