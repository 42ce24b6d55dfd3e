"""FP8 forward with incoherent processing, through the C ABI.

* The preparation (rotation, scales, e4m3 codes) is compared with the oracle
  bit for bit: scales exactly, code values exactly (both sides divide in fp32
  and round to e4m3 the same way; the rotation is the same fp32 butterfly
  sequence).
* The attention is compared with the oracle's attention of the dequantised
  operands.  The kernel also rounds P to e4m3 before the P V product (the
  oracle keeps P exact), which is what the tolerance covers: with P in e4m3's
  normal range each term's relative error is at most 2^-4 and the errors of
  different keys are independent, so for N(0,1) inputs (row sums l of tens,
  N >= 300) the expected |dO| is ~2e-3 with a tail a few times that.
  Bound used: max |dO| <= 5e-2, mean |dO| <= 5e-3; LSE (from the unrounded
  P) within 1e-3.
* The error against exact attention on inputs with outlier channels, with
  and without the rotation: the rotation must lower it (the pages report
  2.6x lower error than plain FP8).
"""

import numpy as np
import pytest
import torch

import exact_io_aware_84_b200 as fa
from oracle import attn_fwd_ref, fp8_attn_fwd_ref, fp8_inputs_ref
from parity import to64

pytestmark = pytest.mark.gpu

TOL_FP8_O_MAX = 5e-2
TOL_FP8_O_MEAN = 5e-3
TOL_FP8_LSE = 1e-3


def _inputs(B, H, N, seed, dtype=torch.bfloat16, outliers=0.0):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, N, 128, generator=g) for _ in range(3))
    if outliers:
        q[..., :2] *= outliers
        k[..., :2] *= outliers
    return q.to(dtype), k.to(dtype), v.to(dtype)


def _signs(seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randint(0, 2, (128,), generator=g) * 2 - 1).float()


def _decode(codes):
    return codes.cpu().view(torch.float8_e4m3fn).double().numpy()


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("N", [128, 300, 1000])
def test_quantisation_matches_oracle_bit_for_bit(N, rotate):
    q, k, v = _inputs(2, 2, N, seed=N + rotate)
    s = _signs(N) if rotate else None
    z = fa.fa_fp8_quantize(q.cuda(), k.cuda(), v.cuda(), signs=s.cuda() if rotate else None)
    torch.cuda.synchronize()
    ref = fp8_inputs_ref(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                         signs=s.numpy() if rotate else None)
    np.testing.assert_array_equal(z["sq"].cpu().numpy(), ref["sq"])
    np.testing.assert_array_equal(z["sk"].cpu().numpy(), ref["sk"])
    np.testing.assert_array_equal(z["sv"].cpu().numpy(), ref["sv"])
    np.testing.assert_array_equal(_decode(z["q8"])[:, :, :N], ref["q"])
    np.testing.assert_array_equal(_decode(z["k8"])[:, :, :N], ref["k"])
    np.testing.assert_array_equal(np.swapaxes(_decode(z["v8t"]), -1, -2)[:, :, :N], ref["v"])
    n_pad = z["q8"].shape[2]
    if n_pad > N:   # padding rows / keys hold zero codes
        assert not z["q8"][:, :, N:].any() and not z["k8"][:, :, N:].any() and not z["v8t"][..., N:].any()


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 1000, 2048])
def test_fp8_forward_matches_oracle(N, causal, rotate):
    q, k, v = _inputs(1, 3, N, seed=7 * N + causal)
    s = _signs(N + 1) if rotate else None
    scale = 128 ** -0.5
    o, lse = fa.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), signs=s.cuda() if rotate else None, scale=scale,
                           causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    o_ref, lse_ref = fp8_attn_fwd_ref(q.float().numpy(), k.float().numpy(), v.float().numpy(), scale, causal,
                                      signs=s.numpy() if rotate else None)
    d = np.abs(to64(o) - o_ref)
    dl = np.abs(to64(lse) - lse_ref)
    msg = f"N={N} causal={causal} rotate={rotate}: O max {d.max():.3e} mean {d.mean():.3e}; LSE {dl.max():.3e}"
    assert d.max() <= TOL_FP8_O_MAX and d.mean() <= TOL_FP8_O_MEAN and dl.max() <= TOL_FP8_LSE, msg


def test_fp8_forward_fp16_inputs_and_fp32_output():
    q, k, v = _inputs(2, 2, 640, seed=3, dtype=torch.float16)
    s = _signs(5)
    o, lse = fa.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), signs=s.cuda(), o_fp32=True)
    torch.cuda.synchronize()
    assert o.dtype == torch.float32
    o_ref, lse_ref = fp8_attn_fwd_ref(q.float().numpy(), k.float().numpy(), v.float().numpy(), 128 ** -0.5,
                                      signs=s.numpy())
    assert np.abs(to64(o) - o_ref).mean() <= TOL_FP8_O_MEAN
    assert np.abs(to64(lse) - lse_ref).max() <= TOL_FP8_LSE


def test_rotation_lowers_the_fp8_error_with_outlier_channels():
    q, k, v = _inputs(1, 4, 2048, seed=11, outliers=10.0)
    s = _signs(11)
    scale = 128 ** -0.5
    exact, _ = attn_fwd_ref(to64(q), to64(k), to64(v), scale)
    gq, gk, gv = q.cuda(), k.cuda(), v.cuda()
    plain, _ = fa.fa_fwd_fp8(gq, gk, gv, scale=scale, o_fp32=True)
    rot, _ = fa.fa_fwd_fp8(gq, gk, gv, signs=s.cuda(), scale=scale, o_fp32=True)
    torch.cuda.synchronize()
    e_plain = float(np.sqrt(np.mean((to64(plain) - exact) ** 2)))
    e_rot = float(np.sqrt(np.mean((to64(rot) - exact) ** 2)))
    print(f"fp8 rmse vs exact: plain {e_plain:.4e}, rotated {e_rot:.4e}, ratio {e_plain / e_rot:.2f}")
    assert e_rot * 1.5 < e_plain


def test_fp8_rejects_head_dim_64():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fa_fwd_fp8(q, q, q)
