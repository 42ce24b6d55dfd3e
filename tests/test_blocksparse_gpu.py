"""Block-sparse attention through the C ABI (fa_fwd_blocksparse /
fa_bwd_blocksparse) against the fp64 oracle: 128 x 128 (query block, key
block) tiles whose mask entry is 0 are skipped.  Rows with no kept key must
come back with O = 0, LSE = -inf and zero gradients; keys that no query
attends must get dK = dV = 0, exactly."""

import numpy as np
import pytest
import torch

import exact_io_aware_84_b200 as fa
from oracle import blocksparse_bwd_ref, blocksparse_fwd_ref
from parity import check_grads, check_o_lse, to64

pytestmark = pytest.mark.gpu

BLOCK = 128


def _inputs(B, H, N, d, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return tuple(torch.randn(B, H, N, d, generator=g).to(dtype) for _ in range(4))


def _random_mask(B, H, nb, density, seed, per_head=True):
    rng = np.random.default_rng(seed)
    shape = (B, H, nb, nb) if per_head else (nb, nb)
    return (rng.random(shape) < density).astype(np.uint8)


def _check(q, k, v, do, mask, causal, what):
    B, H, N, d = q.shape
    scale = d ** -0.5
    gq, gk, gv, gdo = (x.cuda() for x in (q, k, v, do))
    gm = torch.from_numpy(mask).cuda()
    o, lse = fa.fa_fwd_blocksparse(gq, gk, gv, gm, scale=scale, causal=causal)
    dq, dk, dv = fa.fa_bwd_blocksparse(gq, gk, gv, o, gdo, lse, gm, scale=scale, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK

    bm = np.broadcast_to(mask, (B, H) + mask.shape[-2:]).astype(bool)
    o_ref, lse_ref = blocksparse_fwd_ref(to64(q), to64(k), to64(v), scale, causal, bm)
    o64, lse64 = to64(o), to64(lse)
    empty = np.isneginf(lse_ref)
    # rows with no kept key: O exactly zero, LSE exactly -inf
    assert np.array_equal(np.isneginf(lse64), empty), f"{what}: empty-row pattern differs"
    assert not np.any(o64[empty]), f"{what}: O of empty rows is not zero"
    live = ~empty
    if live.any():
        check_o_lse(o64[live], lse64[live], o_ref[live], lse_ref[live], f"{what} fwd")

    ref = blocksparse_bwd_ref(to64(q), to64(k), to64(v), to64(do), scale, causal, bm)
    got = [to64(dq), to64(dk), to64(dv)]
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        zero_rows = ~np.any(r, axis=-1)
        # rows the oracle leaves exactly zero because nothing reaches them
        # structurally (empty query rows, keys no query attends)
        struct = empty if name == "dq" else _unattended_keys(bm, N, causal)
        assert not np.any(g[struct]), f"{what}: {name} of unreached rows is not zero"
        assert np.all(zero_rows[struct])
    check_grads(got, ref, f"{what} bwd")


def _unattended_keys(bm, N, causal):
    """[B, H, N] True where no query attends key j under the mask."""
    nb = bm.shape[-1]
    out = np.zeros(bm.shape[:2] + (N,), dtype=bool)
    for j in range(N):
        jb = j // BLOCK
        col = bm[..., :, jb].copy()  # [B, H, n_qb]
        if causal:
            # query block ib holds a query >= j only if its last row >= j
            last = np.minimum((np.arange(nb) + 1) * BLOCK, N) - 1
            col &= (last >= j)[None, None, :]
        out[..., j] = ~col.any(-1)
    return out


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,density", [(600, 0.5), (1024, 0.3), (777, 0.8)])
def test_blocksparse_random_masks(N, density, d, causal):
    q, k, v, do = _inputs(2, 3, N, d, seed=N + d + int(causal))
    nb = (N + BLOCK - 1) // BLOCK
    mask = _random_mask(2, 3, nb, density, seed=N * 7 + d)
    _check(q, k, v, do, mask, causal, f"N={N} d={d} density={density} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse_shared_mask_with_empty_rows_and_columns(d):
    N = 700
    nb = 6
    mask = np.zeros((nb, nb), dtype=np.uint8)
    mask[0, 0] = 1          # first query block sees only the first key block
    mask[2, [1, 4, 5]] = 1  # query block 1 attends nothing; key blocks 2, 3 unattended
    mask[3, 5] = 1          # the ragged last key block alone
    mask[5, :] = 1          # ragged last query block sees everything
    q, k, v, do = _inputs(1, 2, N, d, seed=11 + d)
    _check(q, k, v, do, mask, False, f"shared mask d={d}")


@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse_causal_upper_only_mask_gives_empty_rows(d):
    # tiles kept only above the diagonal: causal removes them all except the
    # diagonal ones, so even query blocks attend only their own block
    N = 512
    nb = 4
    mask = np.triu(np.ones((nb, nb), dtype=np.uint8), 1)
    mask[np.arange(0, nb, 2), np.arange(0, nb, 2)] = 1
    q, k, v, do = _inputs(1, 2, N, d, seed=3 + d)
    _check(q, k, v, do, mask, True, f"causal upper mask d={d}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse_full_mask_matches_dense(d, causal):
    # every tile kept: block-sparse attention is full attention.  Both the
    # sparse and the dense kernels are checked against the dense fp64 oracle
    # (the plain two-pass definition, not the block-sparse one), and against
    # each other.
    from oracle import attn_bwd_ref, attn_fwd_ref
    N = 1000
    nb = 8
    q, k, v, do = (x.cuda() for x in _inputs(2, 2, N, d, seed=21 + d))
    mask = torch.ones(nb, nb, dtype=torch.uint8, device="cuda")
    scale = 1.0 / d ** 0.5
    o1, l1 = fa.fa_fwd_blocksparse(q, k, v, mask, causal=causal)
    o2, l2 = fa.fa_fwd(q, k, v, causal=causal)
    g1 = fa.fa_bwd_blocksparse(q, k, v, o1, do, l1, mask, causal=causal)
    g2 = fa.fa_bwd(q, k, v, o2, do, l2, causal=causal)
    torch.cuda.synchronize()
    for b in range(2):
        for h in range(2):
            args = [to64(t[b, h]) for t in (q, k, v)]
            o_ref, l_ref = attn_fwd_ref(*args, scale, causal)
            g_ref = attn_bwd_ref(*args, to64(do[b, h]), scale, causal)
            for o, l, g, name in ((o1, l1, g1, "sparse"), (o2, l2, g2, "dense")):
                check_o_lse(to64(o[b, h]), to64(l[b, h]), o_ref, l_ref, f"{name} b={b} h={h}")
                check_grads([to64(t[b, h]) for t in g], g_ref, f"{name} b={b} h={h}")
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_blocksparse_all_zero_mask():
    N, d = 300, 64
    q, k, v, do = (x.cuda() for x in _inputs(1, 2, N, d, seed=9))
    mask = torch.zeros(3, 3, dtype=torch.uint8, device="cuda")
    o, lse = fa.fa_fwd_blocksparse(q, k, v, mask)
    dq, dk, dv = fa.fa_bwd_blocksparse(q, k, v, o, do, lse, mask)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    assert not o.any() and torch.isneginf(lse).all()
    assert not dq.any() and not dk.any() and not dv.any()


def test_blocksparse_fp16_per_head_masks():
    N, d = 640, 128
    q, k, v, do = _inputs(1, 4, N, d, seed=17, dtype=torch.float16)
    mask = _random_mask(1, 4, 5, 0.6, seed=17)
    _check(q, k, v, do, mask, False, "fp16 per-head")

