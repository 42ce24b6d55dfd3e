"""The end-to-end leg of bench.py overlaps uploads, kernels and downloads on
three streams with alternating device buffers.  Its ordering is checked
here: the results it downloads for its last step equal those of direct
fa_fwd / fa_bwd calls on the same inputs, so no download read a buffer
before its kernels had finished and no upload overwrote inputs still in use.
"""

import argparse

import pytest
import torch

import bench
import exact_io_aware_84_b200 as fa
from exact_io_aware_84_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("backward", [True, False])
def test_e2e_pipeline_delivers_each_steps_results(backward):
    w = Workload("e2e", 2, 3, 700, 64, "bf16", True, 0.125, backward, seed=5)
    x = make_inputs(w)
    dev = torch.device("cuda:0")
    got = {}
    r = bench._e2e(fa, torch, w, x, dev, torch.cuda.current_stream(dev), 1.0, 1,
                   argparse.Namespace(warmup=3, steps=5), outputs=got)
    assert r["ms_per_step"] > 0
    assert r["h2d_bytes_per_step"] == sum(t.numel() * t.element_size() for t in x.values())
    g = {k: v.cuda() for k, v in x.items()}
    o, lse = fa.fa_fwd(g["q"], g["k"], g["v"], scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert torch.equal(got["o"], o.cpu()) and torch.equal(got["lse"], lse.cpu())
    if backward:
        dq, dk, dv = fa.fa_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, scale=w.scale, causal=w.causal)
        torch.cuda.synchronize()
        assert torch.equal(got["dk"], dk.cpu()) and torch.equal(got["dv"], dv.cpu())
        # dQ is summed by float reductions whose order is not fixed
        assert torch.allclose(got["dq"].float(), dq.cpu().float(), rtol=2e-2, atol=2e-3)
    else:
        assert set(got) == {"o", "lse"}
