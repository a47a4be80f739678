"""GPU vs oracle: correlated placement, group affinity, predicted homes and
local-slot counts (all integer: bit-exact)."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, synth, workloads as W
from oracle import oracle as O
from tests.helpers import needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]


def check_place(C, G):
    got = to_np(M.place_experts(to_dev(np.ascontiguousarray(C, np.int32)), G))
    assert np.array_equal(got, O.place_experts(C, G))
    return got


def test_place_hand_example_and_ties():
    check_place(np.array([[5, 3, 0, 1], [3, 4, 0, 0], [0, 0, 6, 2], [1, 0, 2, 3]], np.int32), 2)
    check_place(np.zeros((6, 6), np.int32), 3)
    check_place(np.ones((10, 10), np.int32), 5)


@pytest.mark.parametrize("E,G,k,T", [(8, 2, 2, 1000), (64, 16, 6, 5000), (64, 8, 6, 5000), (256, 32, 8, 4000),
                                     (1024, 8, 4, 3000), (12, 1, 3, 300), (16, 16, 2, 100)])
def test_place_random_routing(E, G, k, T):
    idx, _ = O.route_topk(synth.normal_f32(21, 1, (T, E)), k)
    check_place(O.coselect(idx, E), G)


def test_place_recovers_scrambled_clusters():
    w = W.FINE.with_(T=8192)
    idx, _ = O.route_topk(W.make_logits(w), w.k)
    perm = np.random.default_rng(7).permutation(w.E).astype(np.int32)
    goe = check_place(O.coselect(perm[idx], w.E), w.n_clusters)
    inv = np.argsort(perm)
    for g in range(w.n_clusters):
        assert len(set((inv[np.nonzero(goe == g)[0]] // 4).tolist())) == 1


@pytest.mark.parametrize("T,E,G,k1,k2", [(1000, 16, 4, 1, 1), (3000, 64, 8, 2, 3), (2000, 1000, 10, 1, 2)])
def test_affinity_home_and_local_counts(T, E, G, k1, k2):
    i1, _ = O.route_topk(synth.normal_f32(22, 1, (T, E)), k1)
    i2, _ = O.route_topk(synth.normal_f32(22, 2, (T, E)), k2)
    Mt = O.transition(i1, i2, E)
    goe = np.random.default_rng(3).permutation(np.repeat(np.arange(G), E // G)).astype(np.int32)
    aff = to_np(M.group_affinity(to_dev(Mt), to_dev(goe), G))
    assert np.array_equal(aff, O.group_affinity(Mt, goe, G))
    home = to_np(M.predict_home(to_dev(i1), to_dev(aff)))
    assert np.array_equal(home, O.predict_home(i1, aff))
    got = int(to_np(M.count_local(to_dev(i2), to_dev(goe), G, to_dev(home)))[0])
    assert got == O.count_local(i2, goe, G, home)
    got0 = int(to_np(M.count_local(to_dev(i2), to_dev(goe), G))[0])
    assert got0 == O.count_local(i2, goe, G)
    assert M.device_error() == 0


def test_shuffling_statistic_on_the_correlated_layers():
    w = W.EXPERT_CHOICE
    l1 = W.make_logits(w)
    l2 = W.make_layer2_logits(w, l1)
    G = 8
    goe = to_dev(W.equal_groups(w.E, G))
    a, _ = M.route_topk(to_dev(l1), 1)
    b, _ = M.route_topk(to_dev(l2), 1)
    trans = M.transition(a, b, w.E)
    home = M.predict_home(a, M.group_affinity(trans, goe, G))
    before = int(M.count_local(b, goe, G)[0]) / w.T
    after = int(M.count_local(b, goe, G, home)[0]) / w.T
    ra, _ = O.route_topk(l1, 1)
    rb, _ = O.route_topk(l2, 1)
    rhome = O.predict_home(ra, O.group_affinity(O.transition(ra, rb, w.E), W.equal_groups(w.E, G), G))
    assert np.array_equal(to_np(home), rhome)
    assert after * w.T == O.count_local(rb, W.equal_groups(w.E, G), G, rhome)
    assert abs(before - 1 / G) < 0.01 and after > 2 * before
