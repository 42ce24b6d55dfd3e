"""Grouped-query attention through the C ABI (fa_fwd_gqa / fa_bwd_gqa)
against the fp64 oracle: H query heads over Hkv key/value heads."""

import pytest
import torch

import exact_io_aware_84_b200 as fa
from oracle import gqa_bwd_ref, gqa_fwd_ref
from parity import check_grads, check_o_lse, to64

pytestmark = pytest.mark.gpu


def _inputs(B, H, Hkv, N, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    t = torch.bfloat16 if dtype == "bf16" else torch.float16
    q = torch.randn(B, H, N, d, generator=g).to(t)
    k = torch.randn(B, Hkv, N, d, generator=g).to(t)
    v = torch.randn(B, Hkv, N, d, generator=g).to(t)
    do = torch.randn(B, H, N, d, generator=g).to(t)
    return q, k, v, do


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv", [(4, 2), (8, 2), (6, 1), (3, 3)])
@pytest.mark.parametrize("N", [200, 513])
def test_gqa_forward_backward(N, H, Hkv, d, causal):
    q, k, v, do = _inputs(2, H, Hkv, N, d, "bf16", seed=N + H + Hkv + d)
    scale = d ** -0.5
    gq, gk, gv, gdo = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.fa_fwd_gqa(gq, gk, gv, scale=scale, causal=causal)
    dq, dk, dv = fa.fa_bwd_gqa(gq, gk, gv, o, gdo, lse, scale=scale, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    o_ref, lse_ref = gqa_fwd_ref(to64(q), to64(k), to64(v), scale, causal)
    check_o_lse(to64(o), to64(lse), o_ref, lse_ref, f"gqa fwd H={H} Hkv={Hkv}")
    ref = gqa_bwd_ref(to64(q), to64(k), to64(v), to64(do), scale, causal)
    assert dk.shape == k.shape and dv.shape == v.shape
    check_grads([to64(dq), to64(dk), to64(dv)], ref, f"gqa bwd H={H} Hkv={Hkv}")


def test_gqa_with_one_group_equals_multi_head():
    q, k, v, do = _inputs(1, 4, 4, 300, 64, "bf16", seed=5)
    gq, gk, gv, gdo = (x.cuda() for x in (q, k, v, do))
    o1, l1 = fa.fa_fwd_gqa(gq, gk, gv, causal=True)
    o2, l2 = fa.fa_fwd(gq, gk, gv, causal=True)
    g1 = fa.fa_bwd_gqa(gq, gk, gv, o1, gdo, l1, causal=True)
    g2 = fa.fa_bwd(gq, gk, gv, o2, gdo, l2, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        # dQ accumulates through floating-point reduce-adds in any order
        assert (a.float() - b.float()).abs().max().item() < 1e-2


def test_gqa_rejects_bad_grouping():
    lib = fa.load_library()
    p = 0x1000
    assert lib.fa_fwd_gqa(p, p, p, p, p, 1, 6, 4, 128, 64, 0.125, 0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_gqa(p, p, p, p, p, 1, 6, 0, 128, 64, 0.125, 0, 0, None) == fa.FA_ERR_INVALID_ARG
