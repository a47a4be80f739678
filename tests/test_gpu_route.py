"""GPU vs oracle: top-k and expert-choice routing (bit-exact indices)."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, synth, workloads as W
from oracle import oracle as O
from tests.helpers import needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]

GATE_RTOL = 1e-6   # expf (<= 2 ulp) + fp32 rounding; the sum and the ratio are fp64


def check_topk(logits, k, norm=False):
    idx, gate = M.route_topk(to_dev(logits), k, norm)
    ridx, rgate = O.route_topk(logits, k, norm)
    gi, gg = to_np(idx), to_np(gate)
    bad = np.nonzero((gi != ridx).any(1))[0]
    assert bad.size == 0, "token %d: gpu %s oracle %s" % (bad[0], gi[bad[0]], ridx[bad[0]])
    np.testing.assert_allclose(gg, rgate, rtol=GATE_RTOL, atol=1e-30)


@pytest.fixture(params=["rows", "warp"])
def topk_kind(request, monkeypatch):
    """Run a test with the thread-per-token top-k kernel and with the
    warp-per-token ones (the library picks by T; the tests force each)."""
    monkeypatch.setenv("LIBMOE_TOPK_ROWS", "1" if request.param == "rows" else "0")
    return request.param


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (7, 3, 2), (1000, 8, 2), (333, 33, 5), (512, 64, 6), (300, 100, 7),
                                   (1025, 256, 8), (200, 1024, 32), (64, 160, 32), (50, 5, 5), (129, 36, 4),
                                   (300, 1020, 8), (77, 12, 1), (1001, 64, 2), (999, 128, 8), (1003, 192, 5),
                                   (70, 256, 3), (1001, 128, 1), (65, 64, 1), (2049, 96, 8), (33, 224, 4)])
@pytest.mark.parametrize("norm", [False, True])
def test_topk_random(T, E, k, norm, topk_kind):
    check_topk(synth.normal_f32(11, 1, (T, E), 0.0, 2.0), k, norm)


def test_topk_ties_lower_index_wins(topk_kind):
    rng = np.random.default_rng(0)
    for E, k in ((8, 3), (40, 6), (256, 8)):
        logits = rng.integers(-2, 3, size=(2000, E)).astype(np.float32)
        check_topk(logits, k)
    check_topk(np.zeros((10, 70), np.float32), 7, True)
    z = np.zeros((300, 64), np.float32)
    z[:, ::3] = -0.0                                  # -0 and +0 are equal logits: the lower expert wins
    check_topk(z, 8)


def test_topk_concentrated_and_sorted_rows(topk_kind):
    """Rows whose largest logits sit in a strided subset of the experts
    (every fourth group of four), and sorted rows: the threshold of the
    thread-per-token kernel rises late or at once."""
    for E in (64, 256):
        T = 999
        base = synth.normal_f32(13, 1, (T, E), 0.0, 0.1)
        e = np.arange(E)
        lane0 = ((e // 4) % 8) == 0
        base[:, lane0] += 10.0
        for k in (2, 8):
            check_topk(base, k)
            check_topk(base, k, True)
        check_topk(np.tile(-np.arange(E, dtype=np.float32), (T, 1)), 8)      # sorted rows
        check_topk(np.tile(np.arange(E, dtype=np.float32), (T, 1)), 8)


def test_topk_near_ties_in_the_last_bits(topk_kind):
    """Logits that differ in their last few bits: at the k-th / (k+1)-th
    boundary (the thread-per-token kernel ranks those rows again with full
    comparisons), among the winners (put back in exact order), and rows of
    values a few hundred units in the last place apart."""
    rng = np.random.default_rng(5)
    for E, k in ((256, 8), (64, 6), (128, 4)):
        T = 600
        x = synth.normal_f32(14, 1, (T, E), 0.0, 1.0).copy()
        order = np.argsort(-x, axis=1, kind="stable")
        rows = np.arange(T)
        kth = x[rows, order[:, k - 1]]
        bits = kth.view(np.uint32).astype(np.int64)
        one_ulp_down = np.where(kth > 0, bits - 1, bits + 1).astype(np.uint32).view(np.float32)
        a = rows % 3 == 0                      # the (k+1)-th one unit below the k-th
        x[rows[a], order[a, k]] = one_ulp_down[a]
        b = rows % 3 == 1                      # the (k+1)-th equal to the k-th
        x[rows[b], order[b, k]] = kth[b]
        top = x[rows, order[:, 0]]             # the 2nd best one unit below the best
        tb = top.view(np.uint32).astype(np.int64)
        x[rows, order[:, 1]] = np.where(top > 0, tb - 1, tb + 1).astype(np.uint32).view(np.float32)
        check_topk(x, k)
        check_topk(x, k, True)
    for v0 in (1.0, -3.0):
        base = np.float32(v0).view(np.uint32)
        x = (base + rng.integers(0, 600, size=(300, 256)).astype(np.uint32)).view(np.float32)
        check_topk(x, 8)
    # masked experts (-inf) with more than k finite logits left per row
    x = synth.normal_f32(15, 1, (500, 64), 0.0, 1.0).copy()
    x[:, 16:] = -np.inf
    check_topk(x, 8)
    check_topk(x, 8, True)


@pytest.mark.parametrize("E,k,norm", [(256, 8, True), (64, 6, False), (8, 2, False), (128, 1, False)])
def test_topk_large_T_default_choice(E, k, norm):
    """T large enough for the thread-per-token kernel to be the default."""
    check_topk(synth.normal_f32(12, 1, (70001, E)), k, norm)


def test_topk_empty():
    idx, gate = M.route_topk(torch.empty((0, 8), dtype=torch.float32, device="cuda"), 2)
    assert idx.shape == (0, 2)


@pytest.mark.parametrize("w", [W.TINY, W.MIXTRAL, W.FINE, W.SWEEP], ids=lambda w: w.name)
def test_topk_workloads(w):
    check_topk(W.make_logits(w), w.k, w.norm_topk)


def test_top1_both_layers_of_expert_choice_workload():
    w = W.EXPERT_CHOICE
    l1 = W.make_logits(w)
    check_topk(l1, 1)
    check_topk(W.make_layer2_logits(w, l1), 1)


def check_ec(logits, C):
    out = M.route_ec(to_dev(logits), C)
    ec_token, ec_gate, tok_ptr, tok_row = [to_np(t) for t in out]
    r_token, r_gate, r_ptr, r_row = O.route_ec(logits, C)
    bad = np.nonzero((ec_token != r_token).any(1))[0]
    assert bad.size == 0, "expert %d differs" % bad[0]
    np.testing.assert_allclose(ec_gate, r_gate, rtol=GATE_RTOL, atol=1e-30)
    assert np.array_equal(tok_ptr, r_ptr)
    assert np.array_equal(tok_row, r_row)


@pytest.mark.parametrize("T,E,C", [(1, 1, 1), (40, 4, 10), (1000, 7, 333), (3000, 64, 100), (2048, 33, 2048),
                                   (5000, 128, 79), (50001, 8, 7001),
                                   (70001, 4, 9000)])   # the last: T above the binned selection, keys in global memory
def test_expert_choice_random(T, E, C):
    check_ec(synth.normal_f32(5, 1, (T, E)), C)


def test_expert_choice_ties():
    # boundary bins of equal keys: the radix over the full keys, ties in token order
    rng = np.random.default_rng(1)
    check_ec(rng.integers(-1, 2, size=(3000, 16)).astype(np.float32), 700)
    check_ec(np.zeros((257, 3), np.float32), 100)


def test_expert_choice_one_crowded_bin():
    # logits within 1e-4 of each other: every key of an expert in one 1/256-wide
    # bin, all distinct, so the boundary bin's 3000 keys go through the radix
    check_ec((1e-4 * synth.normal_f32(5, 3, (3000, 16))).astype(np.float32), 700)
    # two experts, logits scaled so that the boundary bins hold a few hundred
    # keys: 243 and 248 (ranked pairwise; the second taken whole), then 331
    # and 321 (above the pairwise limit of 256: the radix)
    for a in (0.15, 0.12):
        check_ec((a * synth.normal_f32(5, 4, (20000, 2))).astype(np.float32), 5000)


def test_expert_choice_workload():
    w = W.EXPERT_CHOICE
    check_ec(W.make_logits(w), w.C)
