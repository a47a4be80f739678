"""GPU vs oracle: token permutation (bit-exact indices, byte-identical rows)."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, synth, workloads as W
from oracle import oracle as O
from tests.helpers import needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]


def run(x, idx, E, cf, goe=None, sample_rows=None):
    """Permute on both sides and compare.  x may be None (indices only)."""
    G = int(goe.max()) + 1 if goe is not None else 0
    out = M.permute(None if x is None else to_dev(x), to_dev(idx), E, cf,
                    None if goe is None else to_dev(goe), G)
    cap = O.capacity(cf, idx.shape[0], idx.shape[1], E)
    ref = O.permute(idx, E, cap, goe)
    R = ref["R"]
    assert np.array_equal(to_np(out["row_map"]), ref["row_map"])
    assert np.array_equal(to_np(out["counts"]), ref["counts"])
    assert np.array_equal(to_np(out["offsets"]), ref["offsets"])
    assert int(to_np(out["dropped"])[0]) == ref["dropped"]
    assert np.array_equal(to_np(out["row_token"])[:R], ref["row_token"])
    assert M.device_error() == 0
    if x is not None and R:
        if sample_rows is None:
            buf = to_np(out["buffer"][:R])
            want = O.gather_rows(x, ref["row_token"])
            assert buf.tobytes() == want.tobytes()
        else:
            rows = np.random.default_rng(0).choice(R, size=min(sample_rows, R), replace=False)
            rows = np.union1d(rows, [0, R - 1])
            buf = to_np(out["buffer"][torch.from_numpy(rows).cuda()])
            assert buf.tobytes() == x[ref["row_token"][rows]].tobytes()
    return out, ref


def routed(T, E, k, seed=3, skew=0.0):
    lg = synth.normal_f32(seed, 1, (T, E))
    if skew:
        lg[:, 0] += skew
    return O.route_topk(lg, k)[0]


@pytest.fixture(params=["rankcopy", "bulk", "vector"])
def copy_kind(request, monkeypatch):
    """Run a test on each way the rows can be moved: the two-launch
    expert-major path (counting cluster, then rank and copy per chunk of
    tokens: the library's choice for expert-major rows that fit its
    shared-memory slots), the count / rank / bulk-copy kernels, and the
    count / rank / vectorised-copy kernels.  Group-major calls and calls
    without rows take the count / rank kernels under every setting."""
    monkeypatch.setenv("LIBMOE_BULK_COPY", "0" if request.param == "vector" else "1")
    monkeypatch.setenv("LIBMOE_PERM_RANKCOPY", "1" if request.param == "rankcopy" else "0")
    return request.param


@pytest.mark.parametrize("T,E,k,cf,d,bf16", [
    (1, 1, 1, 1.0, 8, False), (1, 4, 2, 0.5, 8, True), (33, 3, 1, 0.7, 4, False), (1000, 8, 2, 0.5, 40, False),
    (1000, 8, 2, 1.25, 64, True), (4099, 16, 4, 0.9, 24, True), (777, 1024, 32, 2.0, 16, True),
    (2000, 64, 6, 0.0, 8, True), (513, 5, 5, 1.0, 64, False),
    (20011, 64, 6, 1.2, 16, True),                 # 2502 chunks of 8 tokens: 313 per counting CTA, the last 311
    (300, 8, 2, 0.9, 10240, True),                 # 20 KB rows: the largest the rank-and-copy slots take
    (300, 8, 2, 0.9, 10248, True),                 # one 16-byte vector more: rank, then the bulk copy
    (70001, 256, 8, 1.1, 8, True)])                # many index blocks: the scans run as separate kernels
def test_expert_major(T, E, k, cf, d, bf16, copy_kind):
    idx = routed(T, E, k, skew=1.0)
    x = synth.normal_bf16(1, 2, (T, d)) if bf16 else synth.normal_f32(1, 2, (T, d))
    _, ref = run(x, idx, E, cf)
    if 0 < cf < 1 and T >= 100:
        assert ref["dropped"] > 0


@pytest.mark.parametrize("T,E,k,G,cf", [(1000, 8, 2, 4, 0.0), (1000, 8, 3, 2, 0.6), (3001, 64, 6, 8, 1.5),
                                        (3001, 64, 6, 64, 0.0), (500, 16, 4, 1, 0.0), (4096, 256, 8, 32, 0.0)])
def test_group_major(T, E, k, G, cf, copy_kind):
    idx = routed(T, E, k)
    x = synth.normal_bf16(1, 2, (T, 72))
    run(x, idx, E, cf, W.equal_groups(E, G))


def test_group_major_arbitrary_placement():
    T, E, k, G = 2000, 16, 4, 4
    idx = routed(T, E, k)
    goe = np.random.default_rng(2).permutation(np.repeat(np.arange(G), E // G)).astype(np.int32)
    run(synth.normal_f32(1, 2, (T, 12)), idx, E, 1.0, goe)


def test_group_major_identity_groups_equal_expert_major():
    T, E, k = 3000, 16, 3
    idx = routed(T, E, k, skew=0.5)
    x = synth.normal_bf16(1, 2, (T, 64))
    a, _ = run(x, idx, E, 0.8)
    b, _ = run(x, idx, E, 0.8, np.arange(E, dtype=np.int32))
    for key in ("row_map", "counts", "offsets", "dropped"):
        assert torch.equal(a[key], b[key])


def test_indices_only():
    idx = routed(5000, 32, 4)
    run(None, idx, 32, 1.1)
    run(None, routed(7, 256, 8), 256, 0.5)


def test_empty():
    out = M.permute(torch.empty((0, 8), device="cuda"), torch.empty((0, 2), dtype=torch.int32, device="cuda"), 4, 1.0)
    assert int(out["dropped"][0]) == 0 and int(out["offsets"][-1]) == 0


def test_out_of_range_expert_is_skipped_and_reported():
    idx = routed(100, 8, 2)
    idx[5, 1] = 8
    assert M.device_error(clear=True) == 0
    out = M.permute(None, to_dev(idx), 8, 0.0)
    assert M.device_error(clear=True) == 8          # MOE_ERR_DEVICE_INDEX
    assert M.device_error(clear=True) == 0          # cleared
    assert int(to_np(out["row_map"])[5, 1]) == -1


def test_out_of_range_expert_with_rows_is_skipped_and_reported(copy_kind):
    idx = routed(3000, 8, 2)
    idx[700, 0] = 8
    idx[2999, 1] = 9
    x = synth.normal_bf16(1, 2, (3000, 32))
    assert M.device_error(clear=True) == 0
    out = M.permute(to_dev(x), to_dev(idx), 8, 0.0)
    assert M.device_error(clear=True) == 8          # MOE_ERR_DEVICE_INDEX
    rm = to_np(out["row_map"])
    assert rm[700, 0] == -1 and rm[2999, 1] == -1
    keep = np.ones_like(idx, bool)
    keep[700, 0] = keep[2999, 1] = False
    # the other slots keep distinct rows holding their own token
    rows = rm[keep]
    assert np.unique(rows).size == rows.size and (rows >= 0).all()
    buf = to_np(out["buffer"])
    toks = np.nonzero(keep)[0]
    assert buf[rows].tobytes() == x[toks].tobytes()


@pytest.mark.parametrize("w", [W.MIXTRAL, W.FINE], ids=lambda w: w.name)
def test_workload_full(w, copy_kind):
    idx, _ = O.route_topk(W.make_logits(w), w.k)
    _, ref = run(W.make_x(w), idx, w.E, w.capacity_factor)
    if w is W.MIXTRAL:
        assert ref["dropped"] > 0           # the skewed layer overflows experts


@pytest.mark.parametrize("G", W.SWEEP_G)
def test_sweep_group_major_small(G):
    w = W.SWEEP.with_(T=4096)
    idx, _ = O.route_topk(W.make_logits(w), w.k, True)
    run(W.make_x(w), idx, w.E, 0.0, W.equal_groups(w.E, G))


def test_sweep_full_size_sampled_rows():
    w = W.SWEEP
    idx, _ = O.route_topk(W.make_logits(w), w.k, True)
    x = W.make_x(w)
    run(x, idx, w.E, 0.0, W.equal_groups(w.E, 8), sample_rows=4000)
