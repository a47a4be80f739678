"""moe_permute_noalloc: the permutation for callers that cannot allocate.

Some callers may not allocate device memory at all - a host framework that
owns every device byte and forbids allocation once it runs (an inference
plugin, a serving loop with a fixed memory plan), or a hot path that cannot
take cudaMalloc's implicit synchronisation.  For them the library keeps
the permutation's scratch in a fixed device array.  These tests call that
entry point through the C ABI and compare it with moe_permute (caller
workspace) on two calls in a row, the second on a different problem, so
the scratch left behind by the first call must not leak into the second.
The file is named to run last; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, synth, workloads as W
from oracle import oracle as O
from tests.helpers import needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]

SCRATCH_LIMIT = 4 << 20          # MOE_PERMUTE_NOALLOC_SCRATCH_BYTES


def outputs(x, idx, E, cf, goe, G):
    T, k = idx.shape
    R_max = max(M.permute_max_rows(T, k, E, cf, G if goe is not None else 0), 1)
    dev = "cuda"
    return dict(buffer=torch.empty((R_max, x.shape[1]), dtype=x.dtype, device=dev),
                row_map=torch.empty((T, k), dtype=torch.int32, device=dev),
                row_token=torch.empty(R_max, dtype=torch.int32, device=dev),
                counts=torch.empty(E, dtype=torch.int32, device=dev),
                offsets=torch.empty((G if goe is not None else E) + 1, dtype=torch.int32, device=dev),
                dropped=torch.empty(1, dtype=torch.int32, device=dev))


def call_noalloc(x, idx, E, cf, goe, G, out):
    T, k = idx.shape
    st = M.lib().moe_permute_noalloc(
        x.data_ptr(), M._act_dtype(x), T, x.shape[1], idx.data_ptr(), k, E, ctypes.c_double(cf),
        None if goe is None else goe.data_ptr(), G if goe is not None else 0,
        out["buffer"].data_ptr(), out["row_map"].data_ptr(), out["row_token"].data_ptr(),
        out["counts"].data_ptr(), out["offsets"].data_ptr(), out["dropped"].data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    return st


def compare(x_np, idx_np, E, cf, goe_np=None):
    G = int(goe_np.max()) + 1 if goe_np is not None else 0
    x, idx = to_dev(x_np), to_dev(idx_np)
    goe = None if goe_np is None else to_dev(goe_np)
    ref = M.permute(x, idx, E, cf, goe, G)                       # caller workspace
    out = outputs(x, idx, E, cf, goe, G)
    assert call_noalloc(x, idx, E, cf, goe, G, out) == 0
    torch.cuda.synchronize()
    assert M.device_error() == 0
    R = int(ref["offsets"][-1])
    assert int(out["offsets"][-1]) == R
    for key in ("row_map", "counts", "offsets", "dropped"):
        assert torch.equal(out[key], ref[key]), key
    assert torch.equal(out["row_token"][:R], ref["row_token"][:R])
    assert torch.equal(out["buffer"][:R].view(torch.int16), ref["buffer"][:R].view(torch.int16))
    return R


def test_noalloc_matches_workspace_path_on_two_calls_in_a_row():
    # call 1: the Mixtral-shaped routing (expert-major, experts overflow)
    w = W.MIXTRAL
    idx1, _ = O.route_topk(W.make_logits(w), w.k)
    R1 = compare(W.make_x(w)[:, :512], idx1, w.E, w.capacity_factor)
    # call 2: a different, smaller problem in group-major layout
    w2 = W.SWEEP.with_(T=2048)
    idx2, _ = O.route_topk(W.make_logits(w2), w2.k, True)
    R2 = compare(W.make_x(w2)[:, :256], idx2, w2.E, 0.0, W.equal_groups(w2.E, 8))
    assert R1 > 0 and R2 > 0
    # call 3: back to expert-major with drops, fp32 rows
    idx3, _ = O.route_topk(synth.normal_f32(9, 1, (3000, 16)), 4)
    compare(synth.normal_f32(9, 2, (3000, 20)), idx3, 16, 0.7)
    # call 4: the clustered top-6 routing, large enough for the two-launch
    # expert-major path (counting cluster, then rank and copy per chunk)
    w4 = W.FINE
    idx4, _ = O.route_topk(W.make_logits(w4), w4.k)
    assert idx4.size >= 32768
    compare(W.make_x(w4)[:, :256], idx4, w4.E, w4.capacity_factor)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """A valid problem whose scratch exceeds the fixed array is refused with
    MOE_ERR_WORKSPACE before anything is launched.  Real device buffers of
    the refused problem's shape are passed (rows of d = 8, about 60 MB), so
    the call could not touch an invalid address even if it did launch; the
    outputs must be left exactly as they were."""
    T, k, E, G, d = 262144, 8, 256, 64, 8
    assert M.permute_workspace_bytes(T, k, E, G) > SCRATCH_LIMIT
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    idx = (torch.arange(T * k, device="cuda", dtype=torch.int32) % E).view(T, k)
    goe = to_dev(W.equal_groups(E, G))
    out = outputs(x, idx, E, 0.0, goe, G)
    for t in out.values():
        t.fill_(-7) if t.dtype == torch.int32 else t.view(torch.int16).fill_(-7)
    torch.cuda.synchronize()
    launches = M.kernel_launches()
    assert call_noalloc(x, idx, E, 0.0, goe, G, out) == 4               # MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert M.kernel_launches() == launches
    for t in out.values():
        assert bool(((t if t.dtype == torch.int32 else t.view(torch.int16)) == -7).all())
