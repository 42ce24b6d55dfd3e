"""fa_debug_set_timing_events: the backward records the caller's events right
around the launch of its main kernel (the benchmark times the dominant kernel
with them), the gradients are those of an untimed call, and clearing the
setting stops the recording."""

import numpy as np
import pytest
import torch

import exact_io_aware_84_b200 as fa
from exact_io_aware_84_b200.inputs import Workload, make_inputs
from parity import rel_fro, to64

pytestmark = pytest.mark.gpu


def _events(n):
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    return evs


def test_events_bracket_the_main_kernel_and_clear():
    w = Workload("timing", 2, 4, 2048, 128, "bf16", False, 128 ** -0.5, True, seed=5)
    x = make_inputs(w)
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fa_fwd(g["q"], g["k"], g["v"], scale=w.scale, o_fp32=True)
    ref = fa.fa_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, scale=w.scale)
    outer_s, outer_e, kb, ka = _events(4)
    torch.cuda.synchronize()
    assert fa.fa_debug_set_timing_events(kb, ka) == fa.FA_OK
    outer_s.record()
    got = fa.fa_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, scale=w.scale)
    outer_e.record()
    assert fa.fa_debug_set_timing_events(None, None) == fa.FA_OK
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    main_ms, call_ms = kb.elapsed_time(ka), outer_s.elapsed_time(outer_e)
    # the main kernel lies inside the call (which also spans the other two
    # launches and the host's work between the events)
    assert 0.0 < main_ms <= call_ms, (main_ms, call_ms)
    for a, r in zip(got, ref):
        assert rel_fro(to64(a), to64(r)) < 1e-3
    # cleared: a later call leaves the events where they were
    before = kb.elapsed_time(ka)
    fa.fa_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, scale=w.scale)
    torch.cuda.synchronize()
    assert kb.elapsed_time(ka) == before
