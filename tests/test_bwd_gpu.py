"""Backward parity: dQ, dK, dV from the CUDA path (through the C ABI) against
the fp64 oracle's analytic gradient on the same rounded inputs.

The GPU side always computes every head in full; the oracle checks all heads
on the small and medium shapes and a subset of heads on the long ones.  The
full-size gradient invariants (sum_j dK_j = 0, sum_j dV_j = sum_i dO_i) need
no oracle and are checked on every head.
"""

import numpy as np
import pytest
import torch

import exact_io_aware_84_b200 as fa
from exact_io_aware_84_b200.inputs import Workload, make_inputs, workload
from oracle import attn_bwd_ref
from parity import TOL_GRAD_REL, check_grads, rel_fro, to64

pytestmark = pytest.mark.gpu


def _run(w, x=None, o_fp32=False):
    x = make_inputs(w, with_grad=True) if x is None else x
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fa_fwd(g["q"], g["k"], g["v"], scale=w.scale, causal=w.causal, o_fp32=o_fp32)
    dq, dk, dv = fa.fa_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    return x, g, (dq, dk, dv)


def _check_heads(w, x, grads, pairs=None):
    pairs = pairs or [(b, h) for b in range(w.B) for h in range(w.H)]
    out = []
    for b, h in pairs:
        ref = attn_bwd_ref(to64(x["q"][b, h]), to64(x["k"][b, h]), to64(x["v"][b, h]),
                           to64(x["do"][b, h]), w.scale, w.causal)
        got = [to64(t[b, h]) for t in grads]
        out.append(check_grads(got, ref, f"{w.name} b={b} h={h}"))
    return out


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 17, 64, 128, 129, 200, 256, 383, 520])
def test_small_shapes(N, d, causal):
    w = Workload("small", 2, 2, N, d, "bf16", causal, 1.0 / d ** 0.5, True, seed=N * 3 + d)
    x, g, grads = _run(w)
    _check_heads(w, x, grads)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_small_shapes_fp16(d, causal):
    w = Workload("small16", 1, 3, 300, d, "fp16", causal, 1.0 / d ** 0.5, True, seed=11)
    x, g, grads = _run(w)
    _check_heads(w, x, grads)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_many_units_per_cta(d, causal):
    # several units per CTA: the barrier phases carried across units (and at
    # d = 128 the issuer's waits folded into the P and dS barriers)
    w = Workload("many", 3, 64, 384, d, "bf16", causal, 1.0 / d ** 0.5, True, seed=5 + d)
    x, g, grads = _run(w)
    _check_heads(w, x, grads, pairs=[(0, 0), (1, 31), (2, 63)])


def test_gpt2_batch_backward():
    w = workload("gpt2_batch")
    x, g, grads = _run(w)
    _check_heads(w, x, grads, pairs=[(b, h) for b in range(w.B) for h in range(0, w.H, 3)])
    _full_size_invariants(g, grads)


def _full_size_invariants(g, grads):
    dq, dk, dv = grads
    # rows of dS sum to zero => sum over keys of dK is zero (relative to |dK|)
    s = dk.float().sum(dim=2)
    scale = dk.float().abs().sum(dim=2).clamp_min(1e-6)
    assert (s.abs() / scale).max().item() < 2e-2
    # P rows sum to one => sum over keys of dV equals sum over queries of dO
    lhs = dv.float().sum(dim=2)
    rhs = g["do"].float().sum(dim=2)
    assert rel_fro(to64(lhs), to64(rhs)) < TOL_GRAD_REL


def test_trading_day_backward():
    # The training path: O stored in float32 by the forward and read back by
    # the backward for D = rowsum(dO o O).  With O in bf16, that rounding alone
    # puts dQ at 1.03e-2 / 1.16e-2 on these two heads with every other step
    # exact (tests/test_storage_floor.py, oracle only), so the 1e-2 tolerance
    # can only be met through float32 O.
    w = workload("trading_day")
    x, g, grads = _run(w, o_fp32=True)
    _check_heads(w, x, grads, pairs=[(0, 0), (0, 11)])
    _full_size_invariants(g, grads)


def test_trading_day_backward_bf16_o_documented_bound():
    # bf16 storage of O (inference-style callers that keep only a bf16 O):
    # dK and dV within tolerance; dQ is bounded by 2e-2 because the storage
    # rounding of O alone contributes 1.03e-2 on this head (the floor pinned
    # by tests/test_storage_floor.py); this is not the training path.
    w = workload("trading_day")
    x, g, grads = _run(w)
    ref = attn_bwd_ref(to64(x["q"][0, 0]), to64(x["k"][0, 0]), to64(x["v"][0, 0]), to64(x["do"][0, 0]),
                       w.scale, w.causal)
    errs = [rel_fro(to64(t[0, 0]), r) for t, r in zip(grads, ref)]
    assert errs[0] <= 2e-2 and errs[1] <= TOL_GRAD_REL and errs[2] <= TOL_GRAD_REL, errs


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_fp32_o_storage(d, causal, dtype):
    w = Workload("o32", 2, 2, 333, d, dtype, causal, 1.0 / d ** 0.5, True, seed=31)
    x, g, grads = _run(w, o_fp32=True)
    _check_heads(w, x, grads)


@pytest.mark.parametrize("name", ["d128_n2048_nc", "d128_n2048_causal", "d128_n8192_nc",
                                  "d128_n8192_causal", "d128_n16384_causal", "d128_n16384_nc"])
def test_d128_sweep_backward(name):
    w = workload(name)
    x, g, grads = _run(w)
    _check_heads(w, x, grads, pairs=[(0, 0), (1, 15)])
    _full_size_invariants(g, grads)


def test_constant_value_gives_zero_score_gradient():
    w = Workload("constv", 1, 2, 700, 128, "bf16", True, 128 ** -0.5, True, seed=2)
    x = make_inputs(w)
    c = torch.randn(w.d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    x["v"] = c.view(1, 1, 1, -1).expand_as(x["v"]).contiguous()
    _, g, (dq, dk, dv) = _run(w, x)
    # with constant V, dP - D = 0 exactly in exact arithmetic; what remains is
    # rounding, tiny next to the magnitude of dV
    assert dq.float().abs().max().item() < 2e-2
    assert dk.float().abs().max().item() < 2e-2
