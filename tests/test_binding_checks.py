"""The Python binding's buffer checks (CPU): a caller's buffer is refused
before its pointer reaches the library when it has the wrong dtype, too few
elements, a gap (not contiguous) or another device, so a wrong-size output
can never become an out-of-bounds write on the GPU.  The CUDA-residency part
of the check is replaced here by a CPU stand-in; everything else is the
binding's own code."""
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M


@pytest.fixture
def cpu_dev(monkeypatch):
    def dev(t, dtype=None, name="tensor"):
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
        if dtype is not None and t.dtype != dtype:
            raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
        return t
    monkeypatch.setattr(M, "_dev", dev)
    return torch.device("cpu")


def test_real_check_refuses_host_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        M._buf(torch.zeros(4, dtype=torch.int32), torch.int32, 4, "x")


def test_out_allocates_or_checks(cpu_dev):
    t = M._out(None, (3, 5), torch.float32, cpu_dev, "y")
    assert t.shape == (3, 5) and t.dtype == torch.float32
    big = torch.empty(20, dtype=torch.float32)
    assert M._out(big, (3, 5), torch.float32, cpu_dev, "y") is big          # at least 15 elements: accepted
    with pytest.raises(ValueError, match="needs 15"):
        M._out(torch.empty(14, dtype=torch.float32), (3, 5), torch.float32, cpu_dev, "y")
    with pytest.raises(ValueError, match="must be torch.float32"):
        M._out(torch.empty(15, dtype=torch.float64), (3, 5), torch.float32, cpu_dev, "y")
    with pytest.raises(ValueError, match="contiguous"):
        M._out(torch.empty(6, 5).t(), (3, 5), torch.float32, cpu_dev, "y")
    with pytest.raises(ValueError, match="is on"):
        M._buf(torch.empty(15), torch.float32, 15, "y", torch.device("meta"))


def test_workspace_size_counts_bytes():
    assert M._ws_bytes(torch.empty(10, dtype=torch.float32)) == 40
    assert M._ws_bytes(torch.empty(7, dtype=torch.uint8)) == 7


class _ReportsCuda(torch.Tensor):
    """A host tensor that answers is_cuda = True: it takes the checks' common
    path the way a device tensor does."""
    @property
    def is_cuda(self):
        return True


def test_common_path_and_failures_with_a_device_like_tensor():
    t = torch.empty(15, dtype=torch.float32).as_subclass(_ReportsCuda)
    assert M._buf(t, torch.float32, 15, "y", t.device) is t
    assert M._out(t, (3, 5), torch.float32, t.device, "y") is t
    assert M._buf(t, None, 0, "y") is t
    with pytest.raises(ValueError, match="needs 16"):
        M._buf(t, torch.float32, 16, "y", t.device)
    with pytest.raises(ValueError, match="must be torch.int32"):
        M._buf(t, torch.int32, 1, "y")
    with pytest.raises(ValueError, match="is on"):
        M._buf(t, torch.float32, 1, "y", torch.device("meta"))
    g = torch.empty(6, 5).t().as_subclass(_ReportsCuda)
    with pytest.raises(ValueError, match="contiguous"):
        M._buf(g, torch.float32, 1, "g")
