"""Shared test helpers: moving seeded numpy inputs to the GPU and back, and
sampling full-size layers for the oracle."""
import concurrent.futures as cf
import os

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


# ------------------------------------------------ full-size layer sampling
BLOCK_ROWS = 128          # the grouped GEMMs' m-tile: a CTA pair's 256-row tile is two of these


def host_cores() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def oracle_map(fn, chunks):
    """fn over the chunks on the host cores.  Each fn call is a run of the
    single-threaded C oracle; ctypes releases the interpreter lock while C
    code runs, so the chunks proceed on separate cores.  The oracle is only
    the checker here: nothing of its arithmetic changes."""
    chunks = [c for c in chunks if len(c)]
    if not chunks:
        return []
    with cf.ThreadPoolExecutor(max_workers=min(host_cores(), len(chunks))) as ex:
        return list(ex.map(fn, chunks))


def token_chunks(tokens, per_core: int = 4):
    tokens = np.asarray(tokens, np.int64)
    n = max(1, min(tokens.size, host_cores() * per_core))
    return np.array_split(tokens, n)


def expert_blocks(offsets):
    """(start, end) of every 128-row block of every expert's rows."""
    off = np.asarray(offsets, np.int64)
    out = []
    for e in range(off.size - 1):
        a, b = int(off[e]), int(off[e + 1])
        out += [(s, min(s + BLOCK_ROWS, b)) for s in range(a, b, BLOCK_ROWS)]
    return out


def one_row_per_block(offsets, rng):
    """A seeded row inside every 128-row block of every expert."""
    return np.asarray([int(rng.integers(a, b)) for a, b in expert_blocks(offsets)], np.int64)


def assert_blocks_covered(offsets, row_token, tokens):
    """Every 128-row block of every expert holds at least one row of a
    checked token, so each half of every 256-row pair tile is compared."""
    checked = np.isin(np.asarray(row_token), np.asarray(tokens))
    blocks = expert_blocks(offsets)
    missing = [(a, b) for a, b in blocks if not checked[a:b].any()]
    assert not missing, "%d of %d 128-row blocks have no checked row" % (len(missing), len(blocks))
    return len(blocks)
