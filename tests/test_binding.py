"""Argument checks of the Python binding, on the CPU: the library works on the current
device, so a tensor, workspace or stream from another device is refused before any
call into it, and a workspace's size is passed in bytes whatever its element type."""
import pytest
import torch

from rank_linear_lora_b200 import lora_linear as L


class FakeCuda:
    """Just enough of a CUDA tensor for the binding's checks."""

    def __init__(self, shape, dtype, index=0, contiguous=True):
        self.shape, self.dtype, self.is_cuda = tuple(shape), dtype, True
        self.device = torch.device("cuda", index)
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def numel(self):
        n = 1
        for d in self.shape:
            n *= d
        return n

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()

    def data_ptr(self):
        return 0x10000


class FakeStream:
    def __init__(self, index):
        self.device_index, self.cuda_stream = index, 0


@pytest.fixture
def on_device_0(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)


def test_tensors_on_another_device_are_refused(on_device_0):
    L._bf16(FakeCuda((4, 8), torch.bfloat16, 0), "x", (4, 8))
    with pytest.raises(ValueError, match="cuda:1"):
        L._bf16(FakeCuda((4, 8), torch.bfloat16, 1), "x", (4, 8))
    with pytest.raises(ValueError, match="dA"):
        L._f32(FakeCuda((8, 16), torch.float32, 1), "dA", (8, 16))
    with pytest.raises(ValueError, match="Wq"):
        L._q4(FakeCuda((8, 32), torch.uint8, 1), FakeCuda((8, 1), torch.bfloat16, 0), 8, 64)


def test_workspace_checks_and_size_in_bytes(on_device_0):
    _, n = L._ws(FakeCuda((1024,), torch.uint8))
    assert n == 1024
    _, n = L._ws(FakeCuda((256,), torch.float32))  # bytes, not elements
    assert n == 1024
    with pytest.raises(ValueError, match="workspace"):
        L._ws(FakeCuda((1024,), torch.uint8, 1))
    with pytest.raises(ValueError, match="contiguous"):
        L._ws(FakeCuda((1024,), torch.uint8, 0, contiguous=False))
    with pytest.raises(ValueError):
        L._ws(None)


def test_stream_of_another_device_is_refused(on_device_0):
    assert L._stream(FakeStream(0)).value in (None, 0)
    with pytest.raises(ValueError, match="stream"):
        L._stream(FakeStream(1))
