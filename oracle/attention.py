"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, constant or helper with the CUDA library and imports nothing from it.

What it computes (all in float64, on whatever arrays it is handed):

* ``attn_fwd_ref``  -- the plain definition: S = scale * Q K^T, causal entries
  (key j > query i) set to -inf, two-pass softmax (row max, then the sum of
  exponentials), P = exp(S - LSE), O = P V, LSE = m + ln(sum exp(S - m)).
  Source: marketmaker.cc "Flash Attention and the sequence-length problem",
  section "Why attention is memory-bound" (the softmax(QK^T/sqrt(d_k))V
  definition) and the explicit-score PyTorch snippet of section "Integration
  is eight lines"; ultralytics.com glossary "Flash Attention", the
  full-matrix reference line of its code listing.  The log-sum-exp is the
  natural log of the row sum of exp(scaled scores): the pages keep a running
  max m and running sum l per row and write back only those two numbers per
  row (ultralytics glossary, "How Flash Attention works"); storing them as
  m + ln l is the reading used here.
* ``attn_bwd_ref`` -- the analytic gradient of that definition (the pages do
  not print it; it follows from the softmax Jacobian): dV = P^T dO,
  dP = dO V^T, D_i = sum_c dO_ic O_ic, dS = P * (dP - D), dQ = scale dS K,
  dK = scale dS^T Q.  The recomputation of P from Q, K and the stored LSE is
  the marketmaker.cc section "Backward pass: recompute instead of store".
* ``online_fwd_ref`` -- the online-softmax re-association, one key/value block
  at a time: running row max m, running sum l, unnormalised accumulator O~;
  when the max grows, O~ and l are rescaled by exp(m_old - m_new); O = O~ / l
  at the end.  Source: ultralytics.com glossary "Flash Attention", section
  "How Flash Attention works" (streaming blocks with a running max and
  sum), and marketmaker.cc section "Online
  softmax recurrence" (whose displayed equations were lost in extraction; they
  are reconstructed from its prose, which says that whenever a block raises
  the running maximum the output accumulated so far is multiplied by
  e^{m^(j-1) - m^(j)}).
* ``gqa_fwd_ref`` / ``gqa_bwd_ref`` -- grouped-query attention: H query heads
  share Hkv key/value heads, query head h reading key/value head
  h // (H / Hkv).  The forward is the definition above with K and V repeated
  per group; the gradient of K and V is the chain rule of that repetition
  (the per-query-head gradients summed over the group).  The delect.ru
  glossary ("What is confirmed") notes that the attention computation does
  not change the number of key/value heads: grouping is orthogonal to it.
* ``blocksparse_fwd_ref`` / ``blocksparse_bwd_ref`` -- block-sparse attention:
  a boolean mask over 128 x 128 (query block, key block) tiles; scores in
  inactive tiles are excluded (-inf) on top of the causal mask.  It is an
  approximation of full attention (ultralytics glossary, "Flash Attention and
  related terms": the block-sparse variant skips empty tiles; delect.ru
  glossary, "What is confirmed": it is described separately as an
  approximation).  A row whose keys are all excluded has O = 0 and
  LSE = -inf, and contributes no gradient.
* ``merge_partials_ref`` / ``attn_bwd_partial_ref`` / ``ring_fwd_ref`` /
  ``ring_bwd_ref`` -- ring attention: the sequence is split into equal chunks,
  one per device; each device keeps its query chunk and computes attention
  block by block against the key/value chunks as they pass around a ring
  (ultralytics glossary, "Flash Attention and related terms", ring
  attention).  A chunk's result is a partial (O, LSE) over that chunk's keys;
  two partials over disjoint key sets combine as
  LSE = ln(e^{LSE_a} + e^{LSE_b}), O = e^{LSE_a - LSE} O_a + e^{LSE_b - LSE} O_b,
  which is the online-softmax recurrence of marketmaker.cc "Online softmax
  recurrence" taken one whole chunk at a time.  With causal masking and chunks
  aligned to the sequence, a key chunk before the query chunk is attended in
  full, the same chunk with the causal mask, and a later chunk not at all.
  The gradient of a chunk pair uses the full row statistics (the merged LSE
  and O): P = exp(S - LSE), D = rowsum(dO o O), and the per-pair dQ, dK, dV
  sum to the full gradient.
* ``attn_dq_rows_ref`` -- dQ of selected query rows only (each row's dQ
  needs only that row's P, dP and D), with an optional stored O standing in
  for the exact O inside D = rowsum(dO o O): the tool that measures how much
  of the gradient error comes from the storage precision of O alone.
* ``fa1_fwd_ref`` -- the per-step-normalised loop of the marketmaker.cc
  section "The Flash Attention algorithm" (query blocks outer, key/value blocks
  inner, O normalised by the running sum after every block).

Row chunking: ``attn_fwd_ref`` and ``attn_bwd_ref`` may process the query rows
in chunks (``row_chunk``) so that an N x N fp64 matrix never has to exist for
the long configurations.  Every chunk holds complete rows, so each row is
still computed with the plain two-pass definition; the gradient sums over rows
(dK, dV) are just added chunk by chunk.

Parity pins for every function live in ``tests/test_oracle_pins.py`` (brute
force, closed forms, invariants, finite differences, the pages' worked
numbers).  No function here is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "attn_scores_ref",
    "attn_probs_ref",
    "attn_fwd_ref",
    "attn_fwd_rows_ref",
    "attn_bwd_ref",
    "online_fwd_ref",
    "fa1_fwd_ref",
    "gqa_fwd_ref",
    "gqa_bwd_ref",
    "blocksparse_fwd_ref",
    "merge_partials_ref",
    "attn_bwd_partial_ref",
    "attn_dq_rows_ref",
    "ring_fwd_ref",
    "ring_bwd_ref",
    "blocksparse_bwd_ref",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _causal_mask(rows, n_k):
    """True where key j is in the future of query row i (j > i)."""
    rows = np.asarray(rows)
    return np.arange(n_k)[None, :] > rows[:, None]


def attn_scores_ref(q, k, scale, causal=False, rows=None):
    """S = scale * Q K^T for one head; masked entries are -inf.

    q: [Nq, d], k: [Nk, d].  ``rows`` selects query rows (their absolute
    indices are used for the causal mask).
    """
    q = _f64(q)
    k = _f64(k)
    if rows is None:
        rows = np.arange(q.shape[0])
    else:
        rows = np.asarray(rows)
        q = q[rows]
    s = float(scale) * (q @ k.T)
    if causal:
        s = np.where(_causal_mask(rows, k.shape[0]), -np.inf, s)
    return s, rows


def _two_pass(s):
    """Row max, then log of the row sum of exp(s - max).  Returns (lse, p)."""
    m = s.max(axis=-1, keepdims=True)
    # A fully masked row (never produced by square causal inputs) has m = -inf;
    # its probabilities are 0 and its LSE is -inf.
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    l = e.sum(axis=-1, keepdims=True)
    with np.errstate(divide="ignore"):
        lse = np.where(l > 0, m_safe + np.log(l), -np.inf)
    p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
    return lse[..., 0], p


def attn_probs_ref(q, k, scale, causal=False):
    """P = softmax(S) for one head (two-pass)."""
    s, _ = attn_scores_ref(q, k, scale, causal)
    _, p = _two_pass(s)
    return p


def attn_fwd_rows_ref(q, k, v, scale, causal=False, rows=None, row_chunk=1024):
    """O and LSE for the selected query rows of one head.

    q, k, v: [N, d].  Returns (o [len(rows), d], lse [len(rows)]).
    """
    v = _f64(v)
    if rows is None:
        rows = np.arange(np.asarray(q).shape[0])
    rows = np.asarray(rows)
    o = np.empty((rows.shape[0], v.shape[1]), dtype=np.float64)
    lse = np.empty((rows.shape[0],), dtype=np.float64)
    for c0 in range(0, rows.shape[0], row_chunk):
        r = rows[c0:c0 + row_chunk]
        s, _ = attn_scores_ref(q, k, scale, causal, rows=r)
        lse_c, p = _two_pass(s)
        o[c0:c0 + r.shape[0]] = p @ v
        lse[c0:c0 + r.shape[0]] = lse_c
    return o, lse


def attn_fwd_ref(q, k, v, scale, causal=False, row_chunk=1024):
    """Forward for [..., N, d] inputs (any number of leading batch/head dims).

    Returns (O [..., N, d], LSE [..., N]) in float64.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    qf = q.reshape((-1, n, d))
    kf = k.reshape((-1,) + k.shape[-2:])
    vf = v.reshape((-1,) + v.shape[-2:])
    o = np.empty((qf.shape[0], n, vf.shape[-1]))
    lse = np.empty((qf.shape[0], n))
    for h in range(qf.shape[0]):
        o[h], lse[h] = attn_fwd_rows_ref(qf[h], kf[h], vf[h], scale, causal,
                                         row_chunk=row_chunk)
    return o.reshape(lead + (n, vf.shape[-1])), lse.reshape(lead + (n,))


def attn_bwd_ref(q, k, v, do, scale, causal=False, row_chunk=1024):
    """Analytic gradient of O = softmax(scale Q K^T [+ causal mask]) V.

    Inputs [..., N, d]; returns (dQ, dK, dV) in float64.  O and P are the
    oracle's own fp64 values (not a GPU's).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    nk = k.shape[-2]
    qf, kf, vf, dof = (x.reshape((-1,) + x.shape[-2:]) for x in (q, k, v, do))
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    for h in range(qf.shape[0]):
        for c0 in range(0, n, row_chunk):
            rows = np.arange(c0, min(n, c0 + row_chunk))
            s, _ = attn_scores_ref(qf[h], kf[h], scale, causal, rows=rows)
            _, p = _two_pass(s)                     # [r, Nk]
            o = p @ vf[h]                           # [r, d]
            dO = dof[h, rows]                       # [r, d]
            dv[h] += p.T @ dO                       # dV = P^T dO
            dp = dO @ vf[h].T                       # dP = dO V^T
            D = np.sum(dO * o, axis=-1, keepdims=True)  # D_i = sum_c dO_ic O_ic
            ds = p * (dp - D)                       # dS = P o (dP - D)
            dq[h, rows] = float(scale) * (ds @ kf[h])   # dQ = scale dS K
            dk[h] += float(scale) * (ds.T @ qf[h, rows])  # dK = scale dS^T Q
    shp = lambda x, ref: x.reshape(lead + ref.shape[-2:])
    return shp(dq, q), shp(dk, k), shp(dv, v)


def online_fwd_ref(q, k, v, scale, causal=False, block=128, dtype=np.float64):
    """Online-softmax forward for one head: the key/value sequence is consumed
    one block at a time and never seen again.

    State per query row i, after the first j key blocks: the largest scaled
    score seen so far (mu), the sum of exp(score - mu) over those keys (ell),
    and the matching unnormalised output, sum of exp(score - mu) v_key (acc).
    Block j+1 moves the reference point to mu' = max(mu, its own row max);
    the old state is carried over by the factor exp(mu - mu') (zero while mu
    is still -inf), and the block adds its own exp(score - mu') terms.  At the
    end O = acc / ell and LSE = mu + ln ell.  ``dtype`` selects the working
    precision (float32 reproduces the glossary's worked error figure).
    """
    dt = np.dtype(dtype).type
    Q = np.asarray(q, dtype=dt)
    K = np.asarray(k, dtype=dt)
    V = np.asarray(v, dtype=dt)
    n_q, n_k = Q.shape[0], K.shape[0]
    query_pos = np.arange(n_q)[:, None]
    mu = np.full((n_q, 1), -np.inf, dtype=dt)
    ell = np.zeros((n_q, 1), dtype=dt)
    acc = np.zeros((n_q, V.shape[1]), dtype=dt)
    for j0 in range(0, n_k, block):
        j1 = min(n_k, j0 + block)
        sc = (Q @ K[j0:j1].T) * dt(scale)
        if causal:
            sc = np.where(np.arange(j0, j1)[None, :] > query_pos, -np.inf, sc)
        mu_new = np.maximum(mu, sc.max(axis=1, keepdims=True))
        seen = np.isfinite(mu_new)                # at least one unmasked key so far
        ref = np.where(seen, mu_new, 0.0).astype(dt)
        with np.errstate(invalid="ignore"):
            carry = np.where(seen, np.exp(mu - ref), 0.0).astype(dt)
        w = np.exp(sc - ref)                      # masked entries give exp(-inf) = 0
        ell = carry * ell + w.sum(axis=1, keepdims=True)
        acc = carry * acc + w @ V[j0:j1]
        mu = mu_new
    live = ell > 0
    ell_safe = np.where(live, ell, 1)
    o = np.where(live, acc / ell_safe, 0.0)
    with np.errstate(divide="ignore"):
        lse = np.where(live, mu + np.log(ell_safe), -np.inf)
    return o.astype(dt), lse[:, 0].astype(dt)


def fa1_fwd_ref(q, k, v, scale, causal=False, block_r=128, block_c=128):
    """The tiled loop with per-step normalisation, for one head.

    For each query block: O = 0, m = -inf, l = 0.  For each key/value block:
    S = scale Q_i K_j^T, m_ij = rowmax S, P = exp(S - m_ij), l_ij = rowsum P,
    m_new = max(m, m_ij), l_new = e^{m - m_new} l + e^{m_ij - m_new} l_ij,
    O = O (l e^{m - m_new} / l_new) + (P V_j) (e^{m_ij - m_new} / l_new),
    then m = m_new, l = l_new.  Returns (O, LSE = m + ln l).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    n, nk = q.shape[0], k.shape[0]
    o_all = np.zeros((n, v.shape[1]))
    lse_all = np.zeros((n,))
    for r0 in range(0, n, block_r):
        rows = np.arange(r0, min(n, r0 + block_r))
        o = np.zeros((rows.shape[0], v.shape[1]))
        m = np.full((rows.shape[0], 1), -np.inf)
        l = np.zeros((rows.shape[0], 1))
        for c0 in range(0, nk, block_c):
            cols = np.arange(c0, min(nk, c0 + block_c))
            s = float(scale) * (q[rows] @ k[cols].T)
            if causal:
                s = np.where(cols[None, :] > rows[:, None], -np.inf, s)
            m_ij = s.max(axis=-1, keepdims=True)
            fin_ij = np.isfinite(m_ij)
            p = np.where(fin_ij, np.exp(s - np.where(fin_ij, m_ij, 0.0)), 0.0)
            l_ij = p.sum(axis=-1, keepdims=True)
            m_new = np.maximum(m, m_ij)
            fin_new = np.isfinite(m_new)
            mn = np.where(fin_new, m_new, 0.0)
            a_old = np.where(np.isfinite(m), np.exp(m - mn), 0.0)
            a_blk = np.where(fin_ij, np.exp(np.where(fin_ij, m_ij, 0.0) - mn), 0.0)
            l_new = a_old * l + a_blk * l_ij
            safe_l = np.where(l_new > 0, l_new, 1.0)
            o = o * (l * a_old / safe_l) + (p @ v[cols]) * (a_blk / safe_l)
            m, l = m_new, l_new
        o_all[rows] = o
        lse_all[rows] = (m + np.log(np.where(l > 0, l, 1.0)))[:, 0]
    return o_all, lse_all



def _repeat_kv(x, group):
    """[B, Hkv, N, d] -> [B, Hkv*group, N, d], each key/value head repeated
    for the `group` consecutive query heads that read it."""
    return np.repeat(_f64(x), group, axis=1)


def gqa_fwd_ref(q, k, v, scale, causal=False, row_chunk=1024):
    """Grouped-query forward: q [B, H, N, d]; k, v [B, Hkv, N, d]."""
    H, Hkv = np.asarray(q).shape[1], np.asarray(k).shape[1]
    assert H % Hkv == 0
    g = H // Hkv
    return attn_fwd_ref(q, _repeat_kv(k, g), _repeat_kv(v, g), scale, causal, row_chunk)


def gqa_bwd_ref(q, k, v, do, scale, causal=False, row_chunk=1024):
    """Grouped-query gradient: dQ per query head; dK, dV summed over the
    query heads of each group."""
    q = _f64(q)
    B, H = q.shape[:2]
    Hkv = np.asarray(k).shape[1]
    assert H % Hkv == 0
    g = H // Hkv
    dq, dk, dv = attn_bwd_ref(q, _repeat_kv(k, g), _repeat_kv(v, g), do, scale, causal, row_chunk)
    n, d = dk.shape[-2:]
    return dq, dk.reshape(B, Hkv, g, n, d).sum(2), dv.reshape(B, Hkv, g, n, d).sum(2)


def _element_mask(n, block_mask, block):
    """Expand a [n_qb, n_kb] tile mask to an [n, n] element mask (True = kept)."""
    bm = np.asarray(block_mask, dtype=bool)
    idx = np.arange(n) // block
    return bm[idx[:, None], idx[None, :]]


def _masked_scores(q, k, scale, causal, keep):
    s = float(scale) * (_f64(q) @ _f64(k).T)
    if causal:
        s = np.where(_causal_mask(np.arange(s.shape[0]), s.shape[1]), -np.inf, s)
    return np.where(keep, s, -np.inf)


def blocksparse_fwd_ref(q, k, v, scale, causal, block_mask, block=128):
    """Block-sparse forward for [..., N, d] inputs.  ``block_mask`` is
    [..., n_qb, n_kb] (leading dims broadcast against the heads)."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    bm = np.broadcast_to(np.asarray(block_mask, dtype=bool), lead + np.asarray(block_mask).shape[-2:])
    qf, kf, vf = (x.reshape((-1,) + x.shape[-2:]) for x in (q, k, v))
    bmf = bm.reshape((-1,) + bm.shape[-2:])
    o = np.empty((qf.shape[0], n, vf.shape[-1]))
    lse = np.empty((qf.shape[0], n))
    for h in range(qf.shape[0]):
        s = _masked_scores(qf[h], kf[h], scale, causal, _element_mask(n, bmf[h], block))
        lse[h], p = _two_pass(s)
        o[h] = p @ vf[h]
    return o.reshape(lead + (n, vf.shape[-1])), lse.reshape(lead + (n,))


def blocksparse_bwd_ref(q, k, v, do, scale, causal, block_mask, block=128):
    """Gradient of the block-sparse forward (excluded scores carry none)."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    lead = q.shape[:-2]
    n = q.shape[-2]
    bm = np.broadcast_to(np.asarray(block_mask, dtype=bool), lead + np.asarray(block_mask).shape[-2:])
    qf, kf, vf, dof = (x.reshape((-1,) + x.shape[-2:]) for x in (q, k, v, do))
    bmf = bm.reshape((-1,) + bm.shape[-2:])
    dq, dk, dv = np.zeros_like(qf), np.zeros_like(kf), np.zeros_like(vf)
    for h in range(qf.shape[0]):
        s = _masked_scores(qf[h], kf[h], scale, causal, _element_mask(n, bmf[h], block))
        _, p = _two_pass(s)
        o = p @ vf[h]
        dv[h] = p.T @ dof[h]
        dp = dof[h] @ vf[h].T
        D = np.sum(dof[h] * o, axis=-1, keepdims=True)
        ds = p * (dp - D)
        dq[h] = float(scale) * (ds @ kf[h])
        dk[h] = float(scale) * (ds.T @ qf[h])
    shp = lambda x, ref: x.reshape(lead + ref.shape[-2:])
    return shp(dq, q), shp(dk, k), shp(dv, v)


def attn_dq_rows_ref(q, k, v, do, scale, causal=False, rows=None, o_for_d=None):
    """dQ of the selected query rows of one head (q, k, v, do: [N, d]).

    dQ_i depends on row i alone: P_i = softmax(S_i) (two-pass), O_i = P_i V,
    dP_i = dO_i V^T, D_i = sum_c dO_ic O_ic, dS_i = P_i o (dP_i - D_i),
    dQ_i = scale dS_i K.  ``o_for_d``, when given, replaces the exact O_i in
    D_i only -- the O a backward reads back from storage -- so that the effect
    of storing O at a lower precision can be isolated with every other step
    exact.  It is a function applied to the exact fp64 O of the rows (the
    storage rounding), or a list of such functions and None (one dQ per
    entry, all from the same scores).  Returns [len(rows), d] float64, or a
    list of them.
    """
    k, v = _f64(k), _f64(v)
    do = _f64(do)
    s, rows = attn_scores_ref(q, k, scale, causal, rows=rows)
    _, p = _two_pass(s)
    o = p @ v
    d_o = do[rows]
    dp = d_o @ v.T
    many = isinstance(o_for_d, (list, tuple))
    outs = []
    for store in (o_for_d if many else [o_for_d]):
        o_d = o if store is None else _f64(store(o))
        D = np.sum(d_o * o_d, axis=-1, keepdims=True)
        outs.append(float(scale) * ((p * (dp - D)) @ k))
    return outs if many else outs[0]


def merge_partials_ref(o_a, lse_a, o_b, lse_b):
    """Combine two partial attention results of the same queries over
    disjoint key sets.  o_*: [..., n, d]; lse_*: [..., n].  Rows where both
    LSEs are -inf (no key seen yet) stay O = 0, LSE = -inf."""
    o_a, lse_a, o_b, lse_b = (_f64(x) for x in (o_a, lse_a, o_b, lse_b))
    m = np.maximum(lse_a, lse_b)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w_a = np.exp(lse_a - m_safe)      # e^{LSE_a - m}; 0 where LSE_a = -inf
    w_b = np.exp(lse_b - m_safe)
    tot = w_a + w_b
    with np.errstate(divide="ignore"):
        lse = np.where(tot > 0, m_safe + np.log(tot), -np.inf)
    den = np.where(tot > 0, tot, 1.0)[..., None]
    o = (w_a[..., None] * o_a + w_b[..., None] * o_b) / den
    return o, lse


def attn_bwd_partial_ref(q, k, v, o, do, lse, scale, causal=False):
    """Gradient contributions of one key/value chunk to rows whose full
    output O and log-sum-exp LSE are given (computed over all keys):
    P = exp(S - LSE), dV = P^T dO, dP = dO V^T, D = rowsum(dO o O),
    dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q.  Inputs
    [..., n, d] (q, o, do), [..., m, d] (k, v), [..., n] (lse)."""
    q, k, v, o, do, lse = (_f64(x) for x in (q, k, v, o, do, lse))
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    qf, of, dof = (x.reshape((-1, n, x.shape[-1])) for x in (q, o, do))
    kf, vf = (x.reshape((-1,) + x.shape[-2:]) for x in (k, v))
    lf = lse.reshape((-1, n))
    dq, dk, dv = np.zeros_like(qf), np.zeros_like(kf), np.zeros_like(vf)
    for h in range(qf.shape[0]):
        s, _ = attn_scores_ref(qf[h], kf[h], scale, causal)
        with np.errstate(invalid="ignore"):
            p = np.where(np.isfinite(lf[h])[:, None], np.exp(s - lf[h][:, None]), 0.0)
        dv[h] = p.T @ dof[h]
        dp = dof[h] @ vf[h].T
        D = np.sum(dof[h] * of[h], axis=-1, keepdims=True)
        ds = p * (dp - D)
        dq[h] = float(scale) * (ds @ kf[h])
        dk[h] = float(scale) * (ds.T @ qf[h])
    return dq.reshape(lead + (n, d)), dk.reshape(k.shape), dv.reshape(v.shape)


def _ring_pairs(world, causal):
    """(rank, step, source chunk, chunk-causal) in ring order: at step s rank
    r holds the key/value chunk that started on rank (r - s) mod world."""
    for r in range(world):
        for step in range(world):
            src = (r - step) % world
            if causal and src > r:
                continue            # every key of that chunk is in the future
            yield r, step, src, causal and src == r


def _chunks(x, world):
    n = x.shape[-2]
    if n % world:
        raise ValueError("sequence length must be a multiple of the ring size")
    c = n // world
    return [x[..., i * c:(i + 1) * c, :] for i in range(world)]


def ring_fwd_ref(q, k, v, scale, causal=False, world=2):
    """Forward by the ring schedule: per rank, merge the partial results of
    its query chunk against each key/value chunk in the order they arrive.
    Inputs [..., N, d] with N a multiple of ``world``; returns (O, LSE)."""
    q, k, v = (_f64(x) for x in (q, k, v))
    qs, ks, vs = (_chunks(x, world) for x in (q, k, v))
    o = [None] * world
    lse = [None] * world
    for r, _, src, diag in _ring_pairs(world, causal):
        o_p, l_p = attn_fwd_ref(qs[r], ks[src], vs[src], scale, diag)
        if o[r] is None:
            o[r], lse[r] = o_p, l_p
        else:
            o[r], lse[r] = merge_partials_ref(o[r], lse[r], o_p, l_p)
    return np.concatenate(o, axis=-2), np.concatenate(lse, axis=-1)


def ring_bwd_ref(q, k, v, do, scale, causal=False, world=2):
    """Gradient by the ring schedule: O and LSE from ``ring_fwd_ref``, then
    per (rank, chunk) pair the partial gradients, dQ summed on the query's
    rank and dK, dV summed for the chunk's owner."""
    q, k, v, do = (_f64(x) for x in (q, k, v, do))
    o, lse = ring_fwd_ref(q, k, v, scale, causal, world)
    qs, ks, vs, os_, dos = (_chunks(x, world) for x in (q, k, v, o, do))
    ls = [lse[..., i * (q.shape[-2] // world):(i + 1) * (q.shape[-2] // world)] for i in range(world)]
    dq = [np.zeros_like(x) for x in qs]
    dk = [np.zeros_like(x) for x in ks]
    dv = [np.zeros_like(x) for x in vs]
    for r, _, src, diag in _ring_pairs(world, causal):
        gq, gk, gv = attn_bwd_partial_ref(qs[r], ks[src], vs[src], os_[r], dos[r], ls[r], scale, diag)
        dq[r] += gq
        dk[src] += gk
        dv[src] += gv
    cat = lambda xs: np.concatenate(xs, axis=-2)
    return cat(dq), cat(dk), cat(dv)
