"""Host-side argument checks of the Python binding (no GPU needed).

A host tensor or a tensor on another GPU handed to the C ABI would reach the
kernels as a pointer they cannot (or must not) dereference; the binding must
refuse it before the library is called.
"""

import types

import pytest
import torch

import exact_io_aware_84_b200 as fa


class _FakeCuda:
    """Stands in for a CUDA tensor on a machine without a GPU: only the
    attributes the binding's checks read."""

    def __init__(self, shape, dtype=torch.bfloat16, device="cuda:0", is_cuda=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.is_cuda = is_cuda

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True


def test_lse_on_the_host_is_refused():
    q = _FakeCuda((1, 2, 8, 64))
    lse = torch.zeros((1, 2, 8), dtype=torch.float32)      # CPU tensor
    with pytest.raises(ValueError, match="CUDA"):
        fa._check_lse(lse, q)


def test_lse_on_another_device_is_refused():
    q = _FakeCuda((1, 2, 8, 64), device="cuda:0")
    lse = _FakeCuda((1, 2, 8), dtype=torch.float32, device="cuda:1")
    with pytest.raises(ValueError, match="device"):
        fa._check_lse(lse, q)


def test_lse_shape_and_type():
    q = _FakeCuda((1, 2, 8, 64))
    fa._check_lse(_FakeCuda((1, 2, 8), dtype=torch.float32), q)   # accepted
    with pytest.raises(ValueError):
        fa._check_lse(_FakeCuda((1, 2, 9), dtype=torch.float32), q)
    with pytest.raises(ValueError):
        fa._check_lse(_FakeCuda((1, 2, 8), dtype=torch.float16), q)


def test_workspace_must_be_on_the_device():
    q = _FakeCuda((1, 2, 8, 64))
    with pytest.raises(ValueError):
        fa._check_workspace(torch.zeros(16, dtype=torch.uint8), q)
    with pytest.raises(ValueError):
        fa._check_workspace(_FakeCuda((16,), dtype=torch.uint8, device="cuda:1"), q)


@pytest.mark.parametrize("entry", ["fa_bwd", "fa_bwd_noalloc", "fa_fwd"])
def test_wrappers_refuse_a_host_lse_before_calling_the_library(entry, monkeypatch):
    def no_library():
        raise AssertionError("the library must not be reached with a host lse")

    monkeypatch.setattr(fa, "load_library", no_library)
    monkeypatch.setattr(fa, "_check_bhnd", lambda *a, **k: None)   # the fakes pass the tensor checks
    q = _FakeCuda((1, 2, 8, 64))
    lse = torch.zeros((1, 2, 8), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        if entry == "fa_fwd":
            fa.fa_fwd(q, q, q, o=q, lse=lse)
        else:
            getattr(fa, entry)(q, q, q, q, q, lse, dq=q, dk=q, dv=q)


def test_stream_handle_of_an_explicit_stream():
    s = types.SimpleNamespace(cuda_stream=1234)
    assert fa._stream_handle(s) == 1234
    assert fa._stream_handle(5678) == 5678
