"""Argument checks of the Python binding that run before any library call.

The library launches on the calling thread's current device, so the binding
refuses calls whose tensors (or stream) sit on different devices and checks
the one-element device outputs (status word, norms).  These checks need no
GPU: stand-in objects with the attributes the binding reads take the place of
CUDA tensors, and every case here is refused before the library is reached.
"""
import pytest
import torch

import newton_schulz_grad_b200 as nsg


class FakeCuda:
    """Just enough of a CUDA tensor for the binding's checks."""

    def __init__(self, shape, dtype=torch.bfloat16, index=0, contiguous=True, cuda=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.is_cuda = cuda
        self.device = torch.device("cuda", index) if cuda else torch.device("cpu")
        self._contiguous = contiguous

    def dim(self):
        return len(self.shape)

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def is_contiguous(self):
        return self._contiguous

    def data_ptr(self):  # pragma: no cover - never reached: the checks refuse first
        raise AssertionError("the binding reached the library")


class FakeStream:
    def __init__(self, index):
        self.device = torch.device("cuda", index)
        self.cuda_stream = 0


def test_ns_refuses_tensors_on_two_devices():
    with pytest.raises(ValueError, match="one device"):
        nsg.dmuon_ns(FakeCuda((64, 128), index=0), FakeCuda((64, 128), index=1))


def test_ns_refuses_a_stream_of_another_device():
    with pytest.raises(ValueError, match="stream belongs"):
        nsg.dmuon_ns(FakeCuda((64, 128)), FakeCuda((64, 128)), stream=FakeStream(1))


def test_ns_refuses_host_tensors():
    with pytest.raises(ValueError, match="CUDA device"):
        nsg.dmuon_ns(FakeCuda((64, 128), cuda=False), FakeCuda((64, 128)))


def test_step_refuses_mixed_devices():
    ps = [FakeCuda((64, 128)), FakeCuda((32, 32))]
    gs = [FakeCuda((64, 128)), FakeCuda((32, 32), index=2)]
    bs = [FakeCuda((64, 128)), FakeCuda((32, 32))]
    with pytest.raises(ValueError, match="one device"):
        nsg.dmuon_step(ps, gs, bs)


@pytest.mark.parametrize("bad", ["empty", "strided", "dtype", "device"])
def test_noalloc_status_word_checks(bad):
    X, out = FakeCuda((64, 128)), FakeCuda((64, 128))
    status = {"empty": FakeCuda((0,), torch.int32), "strided": FakeCuda((2,), torch.int32, contiguous=False),
              "dtype": FakeCuda((1,), torch.int64), "device": FakeCuda((1,), torch.int32, index=3)}[bad]
    with pytest.raises(ValueError):
        nsg.dmuon_ns_noalloc(X, out, status=status)


def test_clipped_step_total_norm_checks():
    ps, gs, bs = [FakeCuda((8, 8))], [FakeCuda((8, 8))], [FakeCuda((8, 8))]
    with pytest.raises(ValueError, match="total_norm"):
        nsg.dmuon_step(ps, gs, bs, max_norm=1.0, total_norm=FakeCuda((0,), torch.float64))
    with pytest.raises(ValueError, match="one device"):
        nsg.dmuon_step(ps, gs, bs, max_norm=1.0, total_norm=FakeCuda((1,), torch.float64, index=1))
