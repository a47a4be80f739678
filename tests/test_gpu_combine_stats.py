"""GPU vs oracle: combine (unpermute) within 1e-5 in fp32, and the
co-selection / transition histograms bit-exact."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, synth, workloads as W
from oracle import oracle as O
from tests.helpers import as_f64, needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]
REL = 1e-5


def bound_scale(Y, row_map, gate, shared=None):
    """sum_j |gate_j| |Y[row_j]| (+ |shared|): the magnitude a combine's
    rounding error scales with."""
    Yf = np.abs(as_f64(Y))
    T, k = row_map.shape
    s = np.zeros((T, Y.shape[1]))
    for j in range(k):
        r = row_map[:, j]
        m = r >= 0
        s[m] += np.abs(gate[m, j].astype(np.float64))[:, None] * Yf[r[m]]
    if shared is not None:
        s += np.abs(as_f64(shared))
    return s


def check_combine(Y, row_map, gate, shared=None, out_bf16=False):
    got = M.unpermute(to_dev(Y), to_dev(row_map), to_dev(gate), None if shared is None else to_dev(shared),
                      torch.bfloat16 if out_bf16 else torch.float32)
    ref = O.unpermute(Y, row_map, gate, shared)
    g = as_f64(to_np(got))
    scale = bound_scale(Y, row_map, gate, shared)
    tol = REL * scale + 1e-30
    if out_bf16:
        tol = tol + np.abs(ref) * 2.0 ** -8          # output rounding to bf16
    err = np.abs(g - ref)
    assert (err <= tol).all(), "max excess %.3g" % (err - tol).max()


@pytest.fixture(params=["bulk", "register"])
def combine_kind(request, monkeypatch):
    """Run a test with the bulk-staged combine and with the register one (the
    library picks by k; the tests force each)."""
    monkeypatch.setenv("LIBMOE_BULK_COMBINE", "1" if request.param == "bulk" else "0")
    return request.param


@pytest.mark.parametrize("T,E,k,cf,d,bf16", [(256, 8, 2, 1.25, 64, False), (1000, 8, 2, 0.5, 40, False),
                                             (777, 64, 6, 1.5, 136, True), (300, 256, 8, 0.0, 7168, True),
                                             (50, 4, 3, 0.9, 9, False), (64, 1024, 32, 0.0, 16, False)])
def test_combine_expert_major(T, E, k, cf, d, bf16, combine_kind):
    lg = synth.normal_f32(2, 1, (T, E))
    idx, gate = O.route_topk(lg, k)
    p = O.permute(idx, E, O.capacity(cf, T, k, E))
    R = max(p["R"], 1)
    Y = synth.normal_bf16(2, 9, (R, d)) if bf16 else synth.normal_f32(2, 9, (R, d))
    check_combine(Y, p["row_map"], gate)
    sh = synth.normal_bf16(2, 10, (T, d)) if bf16 else synth.normal_f32(2, 10, (T, d))
    check_combine(Y, p["row_map"], gate, shared=sh)
    if bf16:
        check_combine(Y, p["row_map"], gate, shared=sh, out_bf16=True)


@pytest.mark.parametrize("G", [8, 32, 64])
def test_combine_group_major_identity_experts(G, combine_kind):
    w = W.SWEEP.with_(T=2048)
    idx, gate = O.route_topk(W.make_logits(w), w.k, True)
    p = O.permute(idx, w.E, O.capacity(0.0, w.T, w.k, w.E), W.equal_groups(w.E, G))
    x = W.make_x(w)
    Y = O.gather_rows(x, p["row_token"])
    check_combine(Y, p["row_map"], gate)
    # identity experts with renormalised gates: y == x (up to fp32 rounding)
    got = as_f64(to_np(M.unpermute(to_dev(Y), to_dev(p["row_map"]), to_dev(gate), None, torch.float32)))
    np.testing.assert_allclose(got, as_f64(x), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("T,E,C,d", [(40, 4, 10, 8), (3000, 64, 100, 64), (5000, 128, 79, 1024), (300, 16, 250, 136),
                                     (2000, 32, 1500, 2048)])
def test_combine_expert_choice(T, E, C, d, combine_kind):
    lg = synth.normal_f32(4, 1, (T, E))
    ec_token, ec_gate, tok_ptr, tok_row = O.route_ec(lg, C)
    Y = synth.normal_bf16(4, 9, (E * C, d))
    got = as_f64(to_np(M.unpermute_ec(to_dev(Y), to_dev(tok_ptr), to_dev(tok_row), to_dev(ec_gate.reshape(-1)),
                                      torch.float32)))
    ref = O.unpermute_ec(Y, tok_ptr, tok_row, ec_gate)
    scale = O.unpermute_ec(synth.f32_to_bf16(np.abs(as_f64(Y)).astype(np.float32)), tok_ptr, tok_row, ec_gate)
    assert (np.abs(got - ref) <= REL * scale + 1e-30).all()


@pytest.mark.parametrize("bulk", ["1", "0"])
@pytest.mark.parametrize("d", [64, 1024, 7168])
def test_gather_rows_matches_token_csr(bulk, d, monkeypatch):
    monkeypatch.setenv("LIBMOE_BULK_COPY", bulk)          # bulk-copy engine, then the vectorised copy
    T, E, C = 3000, 64, 100
    lg = synth.normal_f32(4, 1, (T, E))
    ec_token, _, tok_ptr, tok_row = O.route_ec(lg, C)
    x = synth.normal_bf16(4, 2, (T, d))
    buf = to_np(M.gather_rows(to_dev(x), to_dev(tok_ptr), to_dev(tok_row), E * C))
    assert buf.tobytes() == O.gather_rows(x, ec_token.reshape(-1)).tobytes()


# -------------------------------------------------------------- histograms
@pytest.fixture(params=["cluster", "sym", "ordered"])
def cosel_kind(request, monkeypatch):
    """Co-selection through the thread-per-token cluster kernel (the default
    for k <= 8), the kernel that counts each unordered slot pair once and
    mirrors it, and the ordered-pair kernel."""
    monkeypatch.setenv("LIBMOE_COSEL_CLUSTER", "1" if request.param == "cluster" else "0")
    monkeypatch.setenv("LIBMOE_COSEL_SYM", "1" if request.param == "sym" else "0")
    return request.param


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (100, 8, 2), (16384, 64, 6), (5000, 1000, 3), (20000, 256, 8),
                                   (3000, 7, 7), (70000, 256, 8), (999, 130, 5), (4096, 1024, 8),
                                   (131072, 256, 8), (3, 256, 8)])
def test_coselect(T, E, k, cosel_kind):
    idx, _ = O.route_topk(synth.normal_f32(6, 1, (T, E)), k)
    got = M.coselect(to_dev(idx), E)
    ref = O.coselect(idx, E)
    assert np.array_equal(to_np(got), ref)
    M.coselect(to_dev(idx), E, into=got)               # accumulates
    assert np.array_equal(to_np(got), 2 * ref)


def test_coselect_duplicates_and_bad_indices(cosel_kind):
    """Rows that repeat an expert (every ordered slot pair still counts, so a
    repeated expert adds 2 to its diagonal per extra pair) and entries out of
    range (pairs that touch one are skipped and the fault word is set)."""
    rng = np.random.default_rng(11)
    for T, E, k in ((3000, 6, 4), (2000, 40, 7), (500, 256, 8), (1000, 3, 1)):
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        assert np.array_equal(to_np(M.coselect(to_dev(idx), E)), O.coselect(idx, E))
        assert M.device_error() == 0
        bad = idx.copy()
        bad[::17, 0] = E
        bad[5::23, -1] = -1
        got = to_np(M.coselect(to_dev(bad), E))
        assert M.device_error() == 8
        ok = (bad >= 0) & (bad < E)
        ref = np.zeros((E, E), np.int64)
        for t in range(T):
            v = bad[t][ok[t]]
            np.add.at(ref, (v[:, None], v[None, :]), 1)      # every ordered pair of valid slots
        assert np.array_equal(got, ref)


def test_coselect_workloads(cosel_kind):
    for w in (W.FINE, W.SWEEP):
        idx, _ = O.route_topk(W.make_logits(w), w.k, w.norm_topk)
        assert np.array_equal(to_np(M.coselect(to_dev(idx), w.E)), O.coselect(idx, w.E))


@pytest.mark.parametrize("T,E,k1,k2", [(1000, 16, 1, 1), (4000, 64, 2, 3), (3000, 300, 4, 2)])
def test_transition(T, E, k1, k2):
    a, _ = O.route_topk(synth.normal_f32(7, 1, (T, E)), k1)
    b, _ = O.route_topk(synth.normal_f32(7, 2, (T, E)), k2)
    assert np.array_equal(to_np(M.transition(to_dev(a), to_dev(b), E)), O.transition(a, b, E))


def test_transition_workload():
    w = W.EXPERT_CHOICE
    l1 = W.make_logits(w)
    l2 = W.make_layer2_logits(w, l1)
    # each side routes its own top-1 for both layers
    ga, _ = M.route_topk(to_dev(l1), 1)
    gb, _ = M.route_topk(to_dev(l2), 1)
    got = to_np(M.transition(ga, gb, w.E))
    ra, _ = O.route_topk(l1, 1)
    rb, _ = O.route_topk(l2, 1)
    ref = O.transition(ra, rb, w.E)
    assert np.array_equal(got, ref)
    assert got.sum() == w.T
