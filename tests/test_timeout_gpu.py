"""Bounded pipeline waits: a kernel whose barrier never completes ends with
FA_ERR_TIMEOUT instead of hanging, and the context stays usable.

The debug flag makes the forward kernel withhold one arrival on its first
tile (a barrier that nothing else completes); every wait in the kernel is
bounded, so all roles give up after the wait limit, drain their in-flight
copies and MMAs, free tensor memory and return.
"""

import pytest
import torch

import exact_io_aware_84_b200 as fa
from exact_io_aware_84_b200.inputs import Workload, make_inputs
from oracle import attn_fwd_ref
from parity import check_o_lse, to64

pytestmark = pytest.mark.gpu


def test_withheld_arrival_times_out_and_recovers():
    w = Workload("one_tile", 1, 1, 128, 64, "bf16", False, 0.125, False, seed=1)
    x = {k: v.cuda() for k, v in make_inputs(w, with_grad=False).items()}
    assert fa.fa_last_device_status() == fa.FA_OK
    assert fa.fa_debug_set_wait_limit_ms(100) == fa.FA_OK
    assert fa.fa_debug_set_flags(1) == fa.FA_OK
    try:
        fa.fa_fwd(x["q"], x["k"], x["v"], scale=w.scale)
        assert fa.fa_last_device_status() == fa.FA_ERR_TIMEOUT
        assert fa.fa_last_device_status() == fa.FA_OK  # the record is cleared
    finally:
        fa.fa_debug_set_flags(0)
        fa.fa_debug_set_wait_limit_ms(1000)
    # the context is still healthy: a normal launch is correct
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    o_ref, lse_ref = attn_fwd_ref(to64(x["q"]), to64(x["k"]), to64(x["v"]), w.scale)
    check_o_lse(to64(o), to64(lse), o_ref, lse_ref, "after timeout")


def test_backward_withheld_arrival_times_out_and_recovers():
    # the backward's compute warpgroups withhold one P arrival on their first
    # tile: the MMA issuer's wait runs out, every role aborts, drains its
    # in-flight copies and MMAs and returns; the context stays usable
    from oracle import attn_bwd_ref
    from parity import check_grads
    w = Workload("two_tiles", 1, 2, 200, 64, "bf16", True, 0.125, True, seed=2)
    x = {k: v.cuda() for k, v in make_inputs(w, with_grad=True).items()}
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], scale=w.scale, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    assert fa.fa_debug_set_wait_limit_ms(100) == fa.FA_OK
    assert fa.fa_debug_set_flags(2) == fa.FA_OK
    try:
        fa.fa_bwd(x["q"], x["k"], x["v"], o, x["do"], lse, scale=w.scale, causal=True)
        assert fa.fa_last_device_status() == fa.FA_ERR_TIMEOUT
        assert fa.fa_last_device_status() == fa.FA_OK
    finally:
        fa.fa_debug_set_flags(0)
        fa.fa_debug_set_wait_limit_ms(1000)
    dq, dk, dv = fa.fa_bwd(x["q"], x["k"], x["v"], o, x["do"], lse, scale=w.scale, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    ref = attn_bwd_ref(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["do"]), w.scale, True)
    check_grads([to64(dq), to64(dk), to64(dv)], ref, "after backward timeout")
