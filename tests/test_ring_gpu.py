"""Ring attention's device steps on one GPU.

* fa_merge / fa_grad_accumulate / fa_convert against the oracle's merge and
  the plain definitions (fp32 sums, round-to-nearest-even conversion).
* The whole ring (``ring_attention_fwd`` / ``ring_attention_bwd`` with the
  CUDA kernels) for 2 and 4 ranks, emulated on one GPU by one host thread per
  rank and an in-process exchange (a copy on the shared stream); the kernels
  of different ranks never wait on one another, the host threads meet on a
  barrier.  The concatenated results must match the oracle's full attention.
"""

import numpy as np
import pytest
import torch

import exact_io_aware_84_b200 as fa
from exact_io_aware_84_b200.ring import ThreadRing, ring_attention_bwd, ring_attention_fwd
from oracle import attn_bwd_ref, attn_fwd_ref, merge_partials_ref
from parity import check_grads, check_o_lse, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_merge_matches_oracle(d):
    g = torch.Generator().manual_seed(d)
    rows = 1000
    o_a, o_b = (torch.randn(2, rows // 2, d, generator=g) for _ in range(2))
    l_a, l_b = (torch.randn(2, rows // 2, generator=g) * 4 for _ in range(2))
    l_a[0, :7] = -float("inf")            # partial a saw no key in these rows
    l_b[0, 3:11] = -float("inf")          # partial b in these (rows 3..6: neither)
    want_o, want_l = merge_partials_ref(to64(o_a), to64(l_a), to64(o_b), to64(l_b))
    go, gl = o_a.cuda(), l_a.cuda()
    out = torch.empty(go.shape, dtype=torch.bfloat16, device="cuda")
    fa.fa_merge(go, gl, o_b.cuda(), l_b.cuda(), out=out)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to64(go), want_o, atol=2e-6, rtol=2e-6)
    assert np.array_equal(np.isneginf(to64(gl)), np.isneginf(want_l))
    fin = np.isfinite(want_l)
    np.testing.assert_allclose(to64(gl)[fin], want_l[fin], atol=2e-6)
    assert not to64(go)[0, 3:7].any()
    assert torch.equal(out.cpu(), go.cpu().to(torch.bfloat16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n", [1, 7, 8, 4099, 1 << 20])
def test_accumulate_and_convert(dtype, n):
    g = torch.Generator().manual_seed(n)
    acc = torch.randn(n, generator=g)
    src = torch.randn(n, generator=g).to(dtype)
    want = acc + src.float()              # fp32 + exactly widened 16-bit value
    gacc = acc.cuda()
    fa.fa_grad_accumulate(gacc, src.cuda())
    out = fa.fa_convert(gacc, dtype)
    torch.cuda.synchronize()
    assert torch.equal(gacc.cpu(), want)
    assert torch.equal(out.cpu(), want.to(dtype))   # round to nearest even


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("world,n,d", [(2, 384, 64), (4, 300, 128), (3, 1000, 64)])
def test_ring_emulated_on_one_gpu_matches_full_attention(world, n, d, causal):
    B, H = 1, 3
    g = torch.Generator().manual_seed(world * 100 + n + d)
    q, k, v, do = (torch.randn(B, H, world * n, d, generator=g).to(torch.bfloat16) for _ in range(4))
    scale = d ** -0.5
    ring = ThreadRing(world)
    res = [None] * world

    def run(r):
        sl = slice(r * n, (r + 1) * n)
        lq, lk, lv, ldo = (x[:, :, sl].contiguous().cuda() for x in (q, k, v, do))
        comm = ring.comm(r)
        o, lse, o32 = ring_attention_fwd(lq, lk, lv, scale=scale, causal=causal, comm=comm)
        grads = ring_attention_bwd(lq, lk, lv, o32, ldo, lse, scale=scale, causal=causal, comm=comm)
        torch.cuda.synchronize()
        res[r] = (o, lse) + tuple(grads)

    ring.run(run)
    assert fa.fa_last_device_status() == fa.FA_OK
    cat = lambda i: torch.cat([res[r][i] for r in range(world)], dim=-2 if i != 1 else -1)
    o_ref, lse_ref = attn_fwd_ref(to64(q), to64(k), to64(v), scale, causal)
    check_o_lse(to64(cat(0)), to64(cat(1)), o_ref, lse_ref, f"ring fwd world={world}")
    ref = attn_bwd_ref(to64(q), to64(k), to64(v), to64(do), scale, causal)
    check_grads([to64(cat(2)), to64(cat(3)), to64(cat(4))], ref, f"ring bwd world={world}")
