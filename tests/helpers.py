"""Shared test helpers: moving seeded numpy inputs to the GPU and back."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import synth

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def to_dev(a: np.ndarray, bf16: bool = False) -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays (bf16 bit patterns) become bfloat16."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16 or bf16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def to_np(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy; bfloat16 becomes uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def as_f64(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return synth.bf16_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def assert_layer_close(got: np.ndarray, ref: np.ndarray, rel: float = 2e-2):
    """max|y - y_ref| <= rel * max|y_ref| (the bf16 layer tolerance)."""
    g, r = as_f64(got), as_f64(ref)
    scale = np.abs(r).max()
    err = np.abs(g - r).max()
    assert np.isfinite(g).all()
    assert err <= rel * scale, "max err %.4g > %.3g * max|ref| %.4g" % (err, rel, scale)
    return err / scale if scale else 0.0
