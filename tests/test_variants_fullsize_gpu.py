"""The NEXT-row variants at the benchmark's size and launch configuration
(d128_n8192_nc: B=2, H=16, N=8192, d=128, seeded inputs, as
``bench.py --workload d128_n8192_nc --variant ...`` runs them), checked on
sampled rows or heads against the oracle:

* grouped-query attention (H_kv = 4): sampled rows of every query head,
  each against its key/value head;
* block-sparse (the bench's seeded 50% tile mask): two whole heads;
* FP8 forward with the bench's signs: two whole heads against the oracle's
  attention of the dequantised operands (the FP8 tolerance);
* ring attention over 4 ranks emulated on this GPU: sampled rows of four
  heads of the forward.
"""

import numpy as np
import pytest
import torch

import exact_io_aware_84_b200 as fa
from exact_io_aware_84_b200.inputs import make_inputs, workload
from exact_io_aware_84_b200.ring import ThreadRing, ring_attention_fwd
from oracle import attn_fwd_rows_ref, blocksparse_fwd_ref, fp8_attn_fwd_ref
from parity import check_o_lse, sample_rows, to64

pytestmark = pytest.mark.gpu

TOL_FP8_O_MAX = 5e-2
TOL_FP8_O_MEAN = 5e-3
TOL_FP8_LSE = 1e-3


@pytest.fixture(scope="module")
def d128():
    w = workload("d128_n8192_nc")
    x = make_inputs(w, with_grad=False)
    return w, x, {k: t.cuda() for k, t in x.items()}


def _pairs(B, H, n):
    allp = [(b, h) for b in range(B) for h in range(H)]
    return [allp[i] for i in sorted(set(int(i) for i in np.linspace(0, len(allp) - 1, n)))]


def test_gqa_full_size_sampled(d128):
    w, x, g = d128
    hkv = w.H // 4
    k, v = x["k"][:, :hkv].contiguous(), x["v"][:, :hkv].contiguous()
    o, lse = fa.fa_fwd_gqa(g["q"], k.cuda(), v.cuda(), scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    rng = np.random.default_rng(1)
    o_c, lse_c = o.cpu(), lse.cpu()
    for b in range(w.B):
        for h in range(w.H):
            rows = sample_rows(w.N, rng, 128)
            kvh = h // (w.H // hkv)
            o_ref, lse_ref = attn_fwd_rows_ref(to64(x["q"][b, h]), to64(k[b, kvh]), to64(v[b, kvh]), w.scale,
                                               w.causal, rows=rows)
            check_o_lse(to64(o_c[b, h, rows]), to64(lse_c[b, h, rows]), o_ref, lse_ref, f"gqa b={b} h={h}")


def test_blocksparse_full_size_two_heads(d128):
    w, x, g = d128
    nb = (w.N + 127) // 128
    rng = np.random.default_rng(1234)          # the bench's seeded mask (rank 0)
    mask = (rng.random((w.B, w.H, nb, nb)) < 0.5).astype(np.uint8)
    o, lse = fa.fa_fwd_blocksparse(g["q"], g["k"], g["v"], torch.from_numpy(mask).cuda(), scale=w.scale,
                                   causal=w.causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    for b, h in _pairs(w.B, w.H, 2):
        o_ref, lse_ref = blocksparse_fwd_ref(to64(x["q"][b, h]), to64(x["k"][b, h]), to64(x["v"][b, h]), w.scale,
                                             w.causal, mask[b, h].astype(bool))
        live = np.isfinite(lse_ref)
        assert np.array_equal(np.isneginf(to64(lse[b, h])), ~live)
        check_o_lse(to64(o[b, h])[live], to64(lse[b, h])[live], o_ref[live], lse_ref[live],
                    f"block-sparse b={b} h={h}")


def test_fp8_full_size_two_heads(d128):
    w, x, g = d128
    signs = (torch.randint(0, 2, (128,), generator=torch.Generator().manual_seed(77)) * 2 - 1).float()
    o, lse = fa.fa_fwd_fp8(g["q"], g["k"], g["v"], signs.cuda(), scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    for b, h in _pairs(w.B, w.H, 2):
        sl = (slice(b, b + 1), slice(h, h + 1))
        o_ref, lse_ref = fp8_attn_fwd_ref(x["q"][sl].float().numpy(), x["k"][sl].float().numpy(),
                                          x["v"][sl].float().numpy(), w.scale, w.causal, signs=signs.numpy())
        d = np.abs(to64(o[sl]) - o_ref)
        dl = np.abs(to64(lse[sl]) - lse_ref)
        assert d.max() <= TOL_FP8_O_MAX and d.mean() <= TOL_FP8_O_MEAN and dl.max() <= TOL_FP8_LSE, \
            f"fp8 b={b} h={h}: O max {d.max():.3e} mean {d.mean():.3e} LSE {dl.max():.3e}"


def test_ring_full_size_forward_sampled(d128):
    w, x, g = d128
    R = 4
    n = w.N // R
    ring = ThreadRing(R)
    res = [None] * R

    def run(r):
        c = {k: t[:, :, r * n:(r + 1) * n].contiguous() for k, t in g.items()}
        o, lse, _ = ring_attention_fwd(c["q"], c["k"], c["v"], scale=w.scale, causal=w.causal, comm=ring.comm(r))
        torch.cuda.synchronize()
        res[r] = (o.cpu(), lse.cpu())

    ring.run(run)
    o = torch.cat([res[r][0] for r in range(R)], dim=2)
    lse = torch.cat([res[r][1] for r in range(R)], dim=2)
    rng = np.random.default_rng(2)
    for b, h in _pairs(w.B, w.H, 4):
        rows = sample_rows(w.N, rng, 256)
        o_ref, lse_ref = attn_fwd_rows_ref(to64(x["q"][b, h]), to64(x["k"][b, h]), to64(x["v"][b, h]), w.scale,
                                           w.causal, rows=rows)
        check_o_lse(to64(o[b, h, rows]), to64(lse[b, h, rows]), o_ref, lse_ref, f"ring b={b} h={h}")
