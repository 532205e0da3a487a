"""Argument checks the Python binding makes before it calls the library, on the CPU with
stand-in tensors: a tensor on another GPU than the current one, and a per-SM busy
buffer with fewer entries than the kernel writes, are refused before any launch."""
import types

import pytest
import torch

import free_adaptive_block_b200 as fv


class FakeCuda:
    """The attributes of a CUDA tensor the binding reads."""

    def __init__(self, shape, dtype, device=0, contiguous=True, ptr=0x10000):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.is_cuda = True
        self.device = types.SimpleNamespace(index=device)
        self._contiguous = contiguous
        self._ptr = ptr

    def is_contiguous(self):
        return self._contiguous

    def data_ptr(self):
        return self._ptr

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n


@pytest.fixture
def on_device0(monkeypatch):
    monkeypatch.setattr(fv, "_current_device", lambda: 0)
    monkeypatch.setattr(fv, "fvattn_num_sms", lambda: 148)

    def no_library():
        raise AssertionError("the library must not be called")

    monkeypatch.setattr(fv, "lib", no_library)


def test_tensor_on_another_device_is_refused(on_device0):
    ok = FakeCuda((2, 3), torch.float32, device=0)
    assert fv._ptr(ok, torch.float32, (2, 3), "x") == 0x10000
    other = FakeCuda((2, 3), torch.float32, device=1)
    with pytest.raises(ValueError, match="cuda:1.*cuda:0"):
        fv._ptr(other, torch.float32, (2, 3), "x")


def test_shape_dtype_layout_checks(on_device0):
    with pytest.raises(ValueError, match="shape"):
        fv._ptr(FakeCuda((2, 4), torch.float32), torch.float32, (2, 3), "x")
    with pytest.raises(ValueError, match="must be torch.float32"):
        fv._ptr(FakeCuda((2, 3), torch.bfloat16), torch.float32, (2, 3), "x")
    with pytest.raises(ValueError, match="contiguous"):
        fv._ptr(FakeCuda((2, 3), torch.float32, contiguous=False), torch.float32, (2, 3), "x")
    assert fv._ptr(None, torch.float32, (2, 3), "x") is None


def test_small_busy_buffer_is_refused_before_launch(on_device0):
    g = fv.Geometry(1, 2, 4, 8, 8, 64, 2, 4, 4)
    tok = (g.B, g.H, g.N, g.d)
    q = FakeCuda(tok, torch.bfloat16)
    mask = FakeCuda((g.B, g.H, g.nB, g.words), torch.int32)
    out = FakeCuda(tok, torch.bfloat16)
    lse = FakeCuda(tok[:3], torch.float32)
    ws = FakeCuda((4096,), torch.uint8)
    small = FakeCuda((100,), torch.int64)
    with pytest.raises(ValueError, match="148 entries, got 100"):
        fv.fvattn_block_sparse_attn(g, q, q, q, mask, 0.125, out, lse, ws, small, stream=0)
    with pytest.raises(ValueError, match="148 entries"):
        fv.fvattn_dense_attn(g, q, q, q, 0.125, out, lse, ws, small, stream=0)
    with pytest.raises(ValueError, match="148 entries"):
        fv.fvattn_block_sparse_attn_noalloc(g, q, q, q, mask, 0.125, out, lse, small, stream=0)
    fv._check_busy(None)
    fv._check_busy(FakeCuda((148,), torch.int64))
