"""Pins for the CPU oracle: each check ties it to something other than itself
(brute-force enumeration, closed forms, independent library routines, values
the pages state).  CPU only."""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special as sps
import torch

from oracle import oracle as O
from mixture_experts_routing_top_b200 import synth, workloads as W

RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------- top-k
def _beats(la, ea, lb, eb):
    """(logit desc, index asc): does expert ea beat expert eb?"""
    return la > lb or (la == lb and ea < eb)


@pytest.mark.parametrize("E", [1, 2, 3, 5, 8])
def test_topk_matches_subset_enumeration(E):
    # small integer logits make exact ties common
    T = 150
    logits = RNG.integers(-2, 3, size=(T, E)).astype(np.float32)
    for k in range(1, E + 1):
        idx, _ = O.route_topk(logits, k)
        for t in range(T):
            l = logits[t]
            winners = [S for S in itertools.combinations(range(E), k)
                       if all(_beats(l[a], a, l[b], b) for a in S for b in range(E) if b not in S)]
            assert len(winners) == 1
            S = winners[0]
            assert set(idx[t].tolist()) == set(S)
            # slot order: best first
            for j in range(k - 1):
                assert _beats(l[idx[t, j]], idx[t, j], l[idx[t, j + 1]], idx[t, j + 1])


def test_topk_all_equal_logits():
    T, E, k = 7, 6, 3
    logits = np.full((T, E), 0.25, np.float32)
    idx, gate = O.route_topk(logits, k)
    assert (idx == np.arange(k)[None, :]).all()
    np.testing.assert_allclose(gate, 1.0 / E, rtol=1e-7)
    _, gate_n = O.route_topk(logits, k, norm_topk=True)
    np.testing.assert_allclose(gate_n, 1.0 / k, rtol=1e-7)


def test_gate_two_experts_is_logistic():
    T = 64
    logits = RNG.normal(size=(T, 2)).astype(np.float32) * 3
    idx, gate = O.route_topk(logits, 2)
    for t in range(T):
        a, b = float(logits[t, idx[t, 0]]), float(logits[t, idx[t, 1]])
        p = 1.0 / (1.0 + math.exp(b - a))
        assert gate[t, 0] == pytest.approx(p, rel=1e-7)
        assert gate[t, 1] == pytest.approx(1.0 - p, rel=1e-6)


def test_gates_are_softmax_probabilities():
    T, E, k = 300, 16, 4
    logits = RNG.normal(size=(T, E)).astype(np.float32) * 2
    idx, gate = O.route_topk(logits, k)
    p = sps.softmax(logits.astype(np.float64), axis=1)
    np.testing.assert_allclose(gate, np.take_along_axis(p, idx, 1), rtol=2e-7, atol=0)
    _, gate_n = O.route_topk(logits, k, norm_topk=True)
    sel = np.take_along_axis(p, idx, 1)
    np.testing.assert_allclose(gate_n, sel / sel.sum(1, keepdims=True), rtol=2e-7, atol=0)
    np.testing.assert_allclose(gate_n.astype(np.float64).sum(1), 1.0, atol=1e-6)
    _, gate_all = O.route_topk(logits, E)
    np.testing.assert_allclose(gate_all.astype(np.float64).sum(1), 1.0, atol=1e-6)


def test_topk_rejects_bad_k():
    with pytest.raises(ValueError):
        O.route_topk(np.zeros((2, 4), np.float32), 5)


# ------------------------------------------------------------- capacity
def test_capacity_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "capacity_factor.json")))
    for c in g["cases"]:
        assert c["T"] * c["k"] / c["E"] == c["average_load"]
        assert O.capacity(c["capacity_factor"], c["T"], c["k"], c["E"]) == c["capacity"]


@pytest.mark.parametrize("w", [W.TINY, W.MIXTRAL, W.FINE])
def test_capacity_is_exact_ceiling(w):
    q = Fraction(w.capacity_factor) * w.T * w.k / w.E
    cap = O.capacity(w.capacity_factor, w.T, w.k, w.E)
    assert cap - 1 < q <= cap
    assert cap == {"tiny_fp32": 80, "mixtral_top2_bf16": 2560, "fine_top6_shared_bf16": 2304}[w.name]


@pytest.mark.parametrize("cf,T,k,E", [(1.25, 100, 3, 7), (1.0, 10, 1, 3), (0.5, 7, 1, 2), (1.3, 1000, 6, 64),
                                      (2.0, 1, 1, 3)])
def test_capacity_rounds_fractional_loads_up(cf, T, k, E):
    """Whole rows: a fractional cf * T * k / E is rounded up (the exact
    rational ceiling of the double cf), never down."""
    q = Fraction(cf) * T * k / E
    assert q.denominator != 1
    cap = O.capacity(cf, T, k, E)
    assert cap - 1 < q <= cap


def test_capacity_unbounded():
    assert O.capacity(0.0, 100, 3, 7) >= 300
    assert O.capacity(-1.0, 100, 3, 7) >= 300


# -------------------------------------------------------------- permute
def _brute_ranks(idx):
    flat = idx.reshape(-1)
    seen = {}
    ranks = np.empty(flat.size, np.int64)
    for s, e in enumerate(flat):
        ranks[s] = seen.get(e, 0)
        seen[e] = ranks[s] + 1
    return ranks.reshape(idx.shape)


@pytest.mark.parametrize("T,E,k,cf", [(64, 4, 2, 0.5), (97, 8, 3, 1.0), (33, 3, 1, 0.7), (50, 6, 6, 0.0)])
def test_drops_match_brute_force_rank(T, E, k, cf):
    logits = RNG.normal(size=(T, E)).astype(np.float32)
    logits[:, 0] += 1.5                       # skew the load so experts overflow
    idx, _ = O.route_topk(logits, k)
    cap = O.capacity(cf, T, k, E)
    p = O.permute(idx, E, cap)
    ranks = _brute_ranks(idx)
    assert ((p["row_map"] < 0) == (ranks >= cap)).all()
    load = np.bincount(idx.reshape(-1), minlength=E)
    assert (p["load"] == load).all()
    assert (p["counts"] == np.minimum(load, cap)).all()
    assert (p["counts"] <= cap).all()
    assert p["counts"].sum() + p["dropped"] == T * k
    assert p["R"] == p["counts"].sum()
    if cf > 0 and cf < 1:
        assert p["dropped"] > 0


def test_expert_major_layout_and_round_trip():
    T, E, k, d = 120, 5, 1, 9
    logits = RNG.normal(size=(T, E)).astype(np.float32)
    logits[:, 2] += 1.0
    idx, _ = O.route_topk(logits, k)
    cap = O.capacity(1.0, T, k, E)
    p = O.permute(idx, E, cap)
    off, rt = p["offsets"], p["row_token"]
    assert off[0] == 0 and (np.diff(off) == p["counts"]).all()
    for e in range(E):
        toks = rt[off[e]:off[e + 1]]
        assert (np.diff(toks) > 0).all()                      # ascending token order
        assert (idx[toks, 0] == e).all()
    x = RNG.normal(size=(T, d)).astype(np.float32)
    buf = O.gather_rows(x, rt)
    for r in range(p["R"]):
        assert buf[r].tobytes() == x[rt[r]].tobytes()
    # identity experts, unit gates: unpermute(permute(x)) == x for kept tokens, 0 for dropped
    y = O.unpermute(buf, p["row_map"], np.ones((T, k), np.float32))
    kept = p["row_map"][:, 0] >= 0
    assert (y[kept] == x[kept].astype(np.float64)).all()
    assert (y[~kept] == 0).all()
    assert (~kept).sum() == p["dropped"] > 0


@pytest.mark.parametrize("cf", [0.0, 0.6])
def test_group_major_with_identity_groups_is_expert_major(cf):
    T, E, k = 80, 6, 2
    idx, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k)
    cap = O.capacity(cf, T, k, E)
    a = O.permute(idx, E, cap)
    b = O.permute(idx, E, cap, group_of_expert=np.arange(E, dtype=np.int32))
    for key in ("row_map", "row_token", "counts", "offsets", "dropped", "R"):
        assert np.array_equal(np.asarray(a[key]), np.asarray(b[key])), key


@pytest.mark.parametrize("G,cf", [(2, 0.0), (4, 0.0), (4, 0.8), (8, 1.0)])
def test_group_major_matches_distinct_pairs(G, cf):
    T, E, k = 90, 8, 3
    idx, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k)
    goe = W.equal_groups(E, G)
    cap = O.capacity(cf, T, k, E)
    p = O.permute(idx, E, cap, group_of_expert=goe)
    kept = _brute_ranks(idx) < cap
    pairs = sorted({(int(goe[idx[t, j]]), t) for t in range(T) for j in range(k) if kept[t, j]})
    assert p["R"] == len(pairs)
    row_of = {pair: r for r, pair in enumerate(pairs)}
    assert [t for _, t in pairs] == p["row_token"].tolist()
    for t in range(T):
        for j in range(k):
            want = row_of[(int(goe[idx[t, j]]), t)] if kept[t, j] else -1
            assert p["row_map"][t, j] == want
    starts = [next((r for r, (g, _) in enumerate(pairs) if g == gg), None) for gg in range(G)]
    for gg in range(G):
        n_g = sum(1 for g, _ in pairs if g == gg)
        assert p["offsets"][gg + 1] - p["offsets"][gg] == n_g
        if n_g:
            assert p["offsets"][gg] == starts[gg]


def _expected_group_rows_per_slot(E, k, G):
    L = E // G
    return G * (1.0 - math.comb(E - L, k) / math.comb(E, k)) / k


@pytest.mark.parametrize("G,expected", [(8, 0.662), (32, 0.908), (64, 0.959)])
def test_group_major_row_count_under_uniform_routing(G, expected):
    E, k, T = 256, 8, 4096
    assert _expected_group_rows_per_slot(E, k, G) == pytest.approx(expected, abs=1e-3)
    logits = synth.normal_f32(7, 1, (T, E))
    idx, _ = O.route_topk(logits, k)
    p = O.permute(idx, E, O.capacity(0.0, T, k, E), group_of_expert=W.equal_groups(E, G))
    ratio = p["R"] / (T * k)
    # per-token row count has std < sqrt(k)/2 rows; 4 sigma over T tokens
    tol = 4 * (math.sqrt(k) / 2) / math.sqrt(T) / k
    assert abs(ratio - _expected_group_rows_per_slot(E, k, G)) < tol


def test_local_fraction_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "local_fraction.json")))
    for c in g["cases"]:
        E, G = c["E"], c["G"]
        assert E // G == c["L"]
        T, k = 20000, 2
        idx, _ = O.route_topk(synth.normal_f32(3, 1, (T, E)), k)
        f = O.local_fraction(idx, W.equal_groups(E, G), G)
        # binomial standard error over T*k slots (slots of one token are dependent: use T)
        tol = 4 * math.sqrt(c["expected_local_fraction"] * (1 - c["expected_local_fraction"]) / T)
        assert abs(f - c["expected_local_fraction"]) < tol


def test_local_fraction_extremes():
    T, E, G = 40, 4, 2
    goe = W.equal_groups(E, G)
    home = (np.arange(T) * G) // T
    idx = (home * 2).astype(np.int32)[:, None]           # every token in its home group
    assert O.local_fraction(idx, goe, G) == 1.0
    idx = ((1 - home) * 2).astype(np.int32)[:, None]     # every token away
    assert O.local_fraction(idx, goe, G) == 0.0


# ------------------------------------------------------------------ FFN
def test_activation_values():
    assert O.silu(0.0) == 0.0
    assert O.gelu(0.0) == 0.0
    assert O.gelu(1.0) == pytest.approx(0.8413447460685429, rel=1e-15)   # Phi(1)
    for z in (-3.1, -0.4, 0.7, 2.5, 9.0):
        assert O.silu(z) - O.silu(-z) == pytest.approx(z, abs=1e-14)
        assert O.gelu(-z) == pytest.approx(O.gelu(z) - z, abs=1e-14)
        assert O.silu(z) == pytest.approx(z * sps.expit(z), rel=1e-14)
        assert O.gelu(z) == pytest.approx(z * sps.ndtr(z), rel=1e-13, abs=1e-300)


def test_round_bf16():
    assert O.round_bf16(1.0 + 2 ** -8) == 1.0                       # tie -> even
    assert O.round_bf16(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6          # tie -> even (up)
    assert O.round_bf16(1.0 + 2 ** -8 + 2 ** -30) == 1.0 + 2 ** -7   # just above the tie
    assert O.round_bf16(1.0 / 3.0) == 0.333984375
    assert O.round_bf16(-2.0 ** -130) == -(2.0 ** -130)              # subnormal, exact
    vals = RNG.normal(size=5000).astype(np.float32) * np.float32(10.0) ** RNG.integers(-30, 30, 5000).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([O.round_bf16(float(v)) for v in vals])
    assert np.array_equal(got, ref)
    # below 2^-126 bf16 values are evenly spaced (2^-133 apart): fp32 subnormals, rounded as torch rounds them
    sub = (RNG.random(3000) * 2.0 ** -126).astype(np.float32)
    sub = np.concatenate([sub, -sub, np.float32([1e-45, 3 * 2.0 ** -134, 2.0 ** -126])])
    ref = torch.from_numpy(sub).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.array([O.round_bf16(float(v)) for v in sub]), ref)


def test_ffn_scalar_closed_form():
    x = np.array([[1.5], [-0.75]], np.float32)
    W1 = np.array([[[0.5]], [[-2.0]]], np.float32)
    W3 = np.array([[[3.0]], [[0.25]]], np.float32)
    W2 = np.array([[[-1.25]], [[4.0]]], np.float32)
    for e in (0, 1):
        y = O.expert_ffn_rows(x, np.array([e, e], np.int32), W1, W3, W2)
        for i in range(2):
            a = float(W1[e, 0, 0] * x[i, 0])
            want = float(W2[e, 0, 0]) * (a / (1 + math.exp(-a))) * float(W3[e, 0, 0] * x[i, 0])
            assert y[i, 0] == pytest.approx(want, rel=1e-15)
        yg = O.expert_ffn_rows(x, np.array([e, e], np.int32), W1, None, W2, act="gelu")
        for i in range(2):
            a = float(W1[e, 0, 0] * x[i, 0])
            assert yg[i, 0] == pytest.approx(float(W2[e, 0, 0]) * a * sps.ndtr(a), rel=1e-13)


def test_ffn_one_hot_rows_pick_columns():
    E, F, d = 3, 5, 4
    W1 = RNG.normal(size=(E, F, d)).astype(np.float32)
    W3 = RNG.normal(size=(E, F, d)).astype(np.float32)
    W2 = RNG.normal(size=(E, d, F)).astype(np.float32)
    for e in range(E):
        for c in range(d):
            x = np.zeros((1, d), np.float32)
            x[0, c] = 1.0
            y = O.expert_ffn_rows(x, np.array([e], np.int32), W1, W3, W2)[0]
            a, b = W1[e, :, c].astype(np.float64), W3[e, :, c].astype(np.float64)
            h = a * sps.expit(a) * b
            np.testing.assert_allclose(y, W2[e].astype(np.float64) @ h, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_ffn_matches_float64_matmul(act):
    E, F, d, n = 4, 24, 16, 30
    x = RNG.normal(size=(n, d)).astype(np.float32)
    W1 = RNG.normal(size=(E, F, d)).astype(np.float32) * 0.3
    W3 = RNG.normal(size=(E, F, d)).astype(np.float32) * 0.3
    W2 = RNG.normal(size=(E, d, F)).astype(np.float32) * 0.3
    re = RNG.integers(0, E, n).astype(np.int32)
    y = O.expert_ffn_rows(x, re, W1, W3 if act == "swiglu" else None, W2, act=act)
    for i in range(n):
        xe = x[i].astype(np.float64)
        a = W1[re[i]].astype(np.float64) @ xe
        h = a * sps.expit(a) * (W3[re[i]].astype(np.float64) @ xe) if act == "swiglu" else a * sps.ndtr(a)
        np.testing.assert_allclose(y[i], W2[re[i]].astype(np.float64) @ h, rtol=1e-11, atol=1e-13)


def test_ffn_bf16_rounds_hidden_and_output():
    # small integers: every product and sum before the nonlinearity is exact
    E, F, d, n = 2, 6, 8, 5
    x = synth.f32_to_bf16(RNG.integers(-3, 4, (n, d)).astype(np.float32))
    W1 = synth.f32_to_bf16(RNG.integers(-2, 3, (E, F, d)).astype(np.float32) * 0.25)
    W3 = synth.f32_to_bf16(RNG.integers(-2, 3, (E, F, d)).astype(np.float32) * 0.25)
    W2 = synth.f32_to_bf16(RNG.integers(-2, 3, (E, d, F)).astype(np.float32) * 0.25)
    re = np.array([0, 1, 1, 0, 1], np.int32)
    y = O.expert_ffn_rows(x, re, W1, W3, W2)
    f = lambda a: synth.bf16_to_f32(a).astype(np.float64)
    for i in range(n):
        a = f(W1)[re[i]] @ f(x)[i]
        b = f(W3)[re[i]] @ f(x)[i]
        h = np.array([O.round_bf16(v) for v in a * sps.expit(a) * b])
        want = np.array([O.round_bf16(v) for v in f(W2)[re[i]] @ h])
        np.testing.assert_allclose(y[i], want, rtol=1e-15, atol=0)
        # every value is a bf16 number
        assert np.array_equal(y[i], synth.bf16_to_f32(synth.f32_to_bf16(y[i].astype(np.float32))))


# ------------------------------------------------------- router linear gate
def test_router_logits_match_float64_matmul():
    x = synth.normal_bf16(3, 1, (37, 128))
    Wr = synth.normal_bf16(3, 2, (24, 128), 0.0, 0.1)
    got = O.router_logits(x, Wr)
    want = synth.bf16_to_f32(x).astype(np.float64) @ synth.bf16_to_f32(Wr).astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    xf, Wf = RNG.normal(size=(9, 17)).astype(np.float32), RNG.normal(size=(5, 17)).astype(np.float32)
    np.testing.assert_allclose(O.router_logits(xf, Wf), xf.astype(np.float64) @ Wf.astype(np.float64).T, rtol=1e-12)


def test_router_logits_exact_on_small_integers_and_one_hot_rows():
    xi = RNG.integers(-8, 9, size=(50, 64))
    Wi = RNG.integers(-8, 9, size=(16, 64))
    got = O.router_logits(xi.astype(np.float32), Wi.astype(np.float32))
    assert np.array_equal(got, (xi @ Wi.T).astype(np.float64))
    # one-hot hidden states pick out one column of W_r
    W = RNG.normal(size=(6, 10)).astype(np.float32)
    eye = np.eye(10, dtype=np.float32)
    assert np.array_equal(O.router_logits(eye, W), W.T.astype(np.float64))


# -------------------------------------------------------------- combine
def test_combine_identity_experts_closed_form():
    T, E, k, d = 70, 6, 3, 5
    logits = RNG.normal(size=(T, E)).astype(np.float32)
    logits[:, 1] += 1.0
    idx, gate = O.route_topk(logits, k)
    cap = O.capacity(0.8, T, k, E)
    p = O.permute(idx, E, cap)
    x = RNG.normal(size=(T, d)).astype(np.float32)
    y = O.unpermute(O.gather_rows(x, p["row_token"]), p["row_map"], gate)
    kept_gate = np.where(p["row_map"] >= 0, gate.astype(np.float64), 0.0).sum(1)
    np.testing.assert_allclose(y, kept_gate[:, None] * x.astype(np.float64), rtol=1e-15, atol=0)
    sh = RNG.normal(size=(T, d)).astype(np.float32)
    y2 = O.unpermute(O.gather_rows(x, p["row_token"]), p["row_map"], gate, shared=sh)
    np.testing.assert_allclose(y2, y + sh.astype(np.float64), rtol=1e-15, atol=1e-15)


def test_combine_group_major_identity_experts():
    T, E, k, d, G = 60, 8, 4, 3, 4
    idx, gate = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k, norm_topk=True)
    p = O.permute(idx, E, O.capacity(0.0, T, k, E), group_of_expert=W.equal_groups(E, G))
    x = RNG.normal(size=(T, d)).astype(np.float32)
    y = O.unpermute(O.gather_rows(x, p["row_token"]), p["row_map"], gate)
    # renormalised gates sum to 1 and nothing is dropped: y == x
    np.testing.assert_allclose(y, x.astype(np.float64), rtol=1e-6, atol=1e-7)


# ------------------------------------------------ group-major expert path
def _two_group_example():
    idx = np.array([[0, 2, 1], [3, 2, 0]], np.int32)
    gate = np.array([[0.5, 0.25, 0.125], [0.5, 0.25, 0.25]], np.float32)
    goe = np.array([0, 0, 1, 1], np.int32)
    return idx, gate, goe


def test_group_path_hand_example():
    """Two tokens, experts {0,1} in group 0 and {2,3} in group 1; the output
    of expert e for token t is (10e + t, e - t).  Group rows and token sums
    worked out by hand."""
    idx, gate, goe = _two_group_example()
    E = 4
    pe = O.permute(idx, E, O.capacity(0.0, 2, 3, E))
    pg = O.permute(idx, E, O.capacity(0.0, 2, 3, E), group_of_expert=goe)
    # group-major rows: group 0 (tokens 0, 1), then group 1 (tokens 0, 1)
    assert pg["row_map"].tolist() == [[0, 2, 0], [3, 3, 1]]
    row_e = np.repeat(np.arange(E), pe["counts"])
    Y = np.stack([10.0 * row_e + pe["row_token"], row_e - pe["row_token"]], 1).astype(np.float32)
    P = O.group_precombine(Y, pe["row_map"], pg["row_map"], gate, 4)
    assert P.tolist() == [[1.25, 0.125], [0.25, -0.25], [5.0, 0.5], [20.75, 1.25]]
    out = O.unpermute_groups(O.to_dtype_bits(P, Y), pg["row_map"])
    assert out.tolist() == [[6.25, 0.625], [21.0, 1.0]]
    sh = np.array([[1, 2], [3, 4]], np.float32)
    assert O.unpermute_groups(O.to_dtype_bits(P, Y), pg["row_map"], shared=sh).tolist() == [[7.25, 2.625], [24.0, 5.0]]


@pytest.mark.parametrize("cf,G", [(0.0, 4), (0.7, 4), (0.7, 16), (1.0, 1)])
def test_group_path_equals_plain_unpermute(cf, G):
    """Summing per group and then over groups is the plain gate-weighted sum."""
    T, E, k, d = 300, 16, 4, 6
    logits = RNG.normal(size=(T, E)).astype(np.float32)
    logits[:, 3] += 1.5                             # a hot expert, so cf < 1 drops
    idx, gate = O.route_topk(logits, k)
    cap = O.capacity(cf, T, k, E)
    goe = RNG.permutation(W.equal_groups(E, G)).astype(np.int32)
    pe = O.permute(idx, E, cap)
    pg = O.permute(idx, E, cap, group_of_expert=goe)
    assert np.array_equal(pe["row_map"] >= 0, pg["row_map"] >= 0)      # same kept assignments
    if cf > 0:
        assert pe["dropped"] > 0
    Y = RNG.normal(size=(int(pe["offsets"][-1]), d)).astype(np.float32)
    R_g = int(pg["offsets"][-1])
    P = O.group_precombine(Y, pe["row_map"], pg["row_map"], gate, R_g)
    assert not np.isnan(P).any()                    # every group row is produced
    got = O.unpermute_groups(O.to_dtype_bits(P, Y), pg["row_map"])
    want = O.unpermute(Y, pe["row_map"], gate)
    np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-6)


def test_group_path_one_expert_per_group_is_one_rounding():
    """G = E: each group row is one gated expert output, rounded once to bf16
    (checked against torch's float64 -> bfloat16 conversion)."""
    T, E, k, d = 64, 8, 3, 16
    idx, gate = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k)
    cap = O.capacity(0.0, T, k, E)
    pe = O.permute(idx, E, cap)
    pg = O.permute(idx, E, cap, group_of_expert=np.arange(E, dtype=np.int32))
    Yb = synth.f32_to_bf16(RNG.normal(size=(int(pe["offsets"][-1]), d)).astype(np.float32))
    P = O.group_precombine(Yb, pe["row_map"], pg["row_map"], gate, int(pg["offsets"][-1]))
    Yd = torch.from_numpy(synth.bf16_to_f32(Yb).astype(np.float64))
    for t in range(T):
        for j in range(k):
            want = (float(gate[t, j]) * Yd[pe["row_map"][t, j]]).to(torch.bfloat16).to(torch.float64).numpy()
            assert np.array_equal(P[pg["row_map"][t, j]], want)


def test_copy_slot_rows_turns_group_rows_into_expert_rows():
    T, E, k, d, G = 120, 8, 3, 5, 2
    idx, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k)
    cap = O.capacity(0.9, T, k, E)
    goe = W.equal_groups(E, G)
    pe = O.permute(idx, E, cap)
    pg = O.permute(idx, E, cap, group_of_expert=goe)
    x = RNG.normal(size=(T, d)).astype(np.float32)
    xg = O.gather_rows(x, pg["row_token"][:pg["offsets"][-1]])
    R_e = int(pe["offsets"][-1])
    xe = np.full((R_e, d), np.nan, np.float32)
    O.copy_slot_rows(xg, pg["row_map"], pe["row_map"], xe)
    assert np.array_equal(xe, O.gather_rows(x, pe["row_token"][:R_e]))


# --------------------------------------------------------- expert choice
@pytest.mark.parametrize("T,E,C", [(40, 4, 10), (33, 5, 33), (25, 3, 1)])
def test_expert_choice_matches_sort(T, E, C):
    logits = RNG.normal(size=(T, E)).astype(np.float32)
    ec_token, ec_gate, tok_ptr, tok_row = O.route_ec(logits, C)
    p = sps.softmax(logits.astype(np.float64), axis=1)
    for e in range(E):
        order = np.lexsort((np.arange(T), -p[:, e]))        # prob desc, token asc
        want = np.sort(order[:C])
        assert (ec_token[e] == want).all()
        np.testing.assert_allclose(ec_gate[e], p[want, e], rtol=1e-6)
    assert tok_ptr[0] == 0 and tok_ptr[-1] == E * C
    assert sorted(tok_row.tolist()) == list(range(E * C))
    for t in range(T):
        rows = tok_row[tok_ptr[t]:tok_ptr[t + 1]]
        assert (np.diff(rows // C) > 0).all()               # ascending expert
        assert all(ec_token.reshape(-1)[r] == t for r in rows)
        assert len(rows) == sum(t in set(ec_token[e].tolist()) for e in range(E))


def test_expert_choice_ties_prefer_lower_token():
    T, E, C = 12, 2, 5
    logits = np.zeros((T, E), np.float32)                    # all scores equal
    ec_token, ec_gate, _, _ = O.route_ec(logits, C)
    assert (ec_token == np.arange(C)[None, :]).all()
    np.testing.assert_allclose(ec_gate, 0.5, rtol=1e-7)


def test_expert_choice_combine():
    T, E, C, d = 30, 4, 9, 6
    logits = RNG.normal(size=(T, E)).astype(np.float32)
    ec_token, ec_gate, tok_ptr, tok_row = O.route_ec(logits, C)
    x = RNG.normal(size=(T, d)).astype(np.float32)
    Y = O.gather_rows(x, ec_token.reshape(-1))               # identity experts
    y = O.unpermute_ec(Y, tok_ptr, tok_row, ec_gate)
    gsum = np.zeros(T)
    for e in range(E):
        for i in range(C):
            gsum[ec_token[e, i]] += ec_gate[e, i]
    np.testing.assert_allclose(y, gsum[:, None] * x.astype(np.float64), rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------ histograms
@pytest.mark.parametrize("E,k", [(8, 2), (16, 6), (5, 5)])
def test_coselect_properties_and_brute_force(E, k):
    T = 200
    idx, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k)
    C = O.coselect(idx, E)
    assert (C == C.T).all()
    load = np.bincount(idx.reshape(-1), minlength=E)
    assert (np.diag(C) == load).all()
    off = C - np.diag(np.diag(C))
    assert off.sum() == T * k * (k - 1)
    assert (off.sum(1) == (k - 1) * load).all()
    want = np.zeros((E, E), np.int64)
    for t in range(T):
        s = set(idx[t].tolist())
        for a in range(E):
            for b in range(E):
                want[a, b] += (a in s) and (b in s)
    assert (C == want).all()
    C2 = O.coselect(idx, E, into=C.copy())                   # accumulates
    assert (C2 == 2 * C).all()


def test_transition_properties_and_brute_force():
    T, E = 300, 12
    for k1, k2 in ((1, 1), (2, 3)):
        i1, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k1)
        i2, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), k2)
        M = O.transition(i1, i2, E)
        assert M.sum() == T * k1 * k2
        assert (M.sum(1) == k2 * np.bincount(i1.reshape(-1), minlength=E)).all()
        assert (M.sum(0) == k1 * np.bincount(i2.reshape(-1), minlength=E)).all()
        want = np.zeros((E, E), np.int64)
        for t in range(T):
            for a in i1[t]:
                for b in i2[t]:
                    want[a, b] += 1
        assert (M == want).all()


def test_transition_detects_correlation():
    # layer-2 logits built from layer-1's top-1: the transition matrix is
    # concentrated (its top entry per row holds far more than 1/E of the row)
    w = W.EXPERT_CHOICE.with_(T=4096)
    l1 = W.make_logits(w)
    l2 = W.make_layer2_logits(w, l1)
    a, _ = O.route_topk(l1, 1)
    b, _ = O.route_topk(l2, 1)
    M = O.transition(a, b, w.E)
    rows = M.sum(1)
    nz = rows > 0
    assert (M.max(1)[nz] / rows[nz]).mean() > 5.0 / w.E


# ---------------------------------------------------------------- inputs
def test_generator_deterministic_and_distribution():
    a = synth.normal_f32(0, 1, (1000, 37))
    b = synth.normal_f32(0, 1, (1000, 37))
    assert a.tobytes() == b.tobytes()
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1) < 0.01
    c = synth.normal_f32(0, 1, (500, 37))                    # prefix property
    assert c.tobytes() == a[:500].tobytes()
    h = synth.normal_bf16(0, 1, (1000, 37))
    assert np.array_equal(h, synth.f32_to_bf16(a))
    # the generator's bf16 is round-to-nearest-even of the fp32 draw, as torch converts it
    tb = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(h, tb)
    assert not np.array_equal(synth.u64(0, 1, 10), synth.u64(0, 2, 10))


# ------------------------------------------------ placement and shuffling
def test_place_experts_hand_traced():
    # off-diagonal masses 4, 3, 2, 3 -> seed 0; affinities to {0}: 3, 0, 1 -> add 1;
    # remaining {2, 3}: masses 2, 3 -> seed 3, then 2
    C = np.array([[5, 3, 0, 1], [3, 4, 0, 0], [0, 0, 6, 2], [1, 0, 2, 3]], np.int32)
    assert O.place_experts(C, 2).tolist() == [0, 0, 1, 1]
    # a group grows by the co-selection summed over all its members: seed 0 (mass 18); affinities to {0}:
    # 1 -> 10, 2 -> 8 -> add 1; summed over {0, 1}: 2 -> 8 + 0, 3 -> 0 + 5 -> add 2 (expert 3 would win on
    # its co-selection with the newest member alone); the rest form group 1
    C = np.zeros((6, 6), np.int32)
    for a, b, n in ((0, 1, 10), (0, 2, 8), (1, 3, 5), (4, 5, 1)):
        C[a, b] = C[b, a] = n
    assert O.place_experts(C, 2).tolist() == [0, 0, 0, 1, 1, 1]
    # all ties: lowest indices first
    assert O.place_experts(np.zeros((6, 6), np.int32), 2).tolist() == [0, 0, 0, 1, 1, 1]
    with pytest.raises(ValueError):
        O.place_experts(np.zeros((6, 6), np.int32), 4)


def test_place_experts_is_a_balanced_partition():
    for E, G in ((12, 3), (64, 16), (32, 1), (10, 10)):
        idx, _ = O.route_topk(RNG.normal(size=(500, E)).astype(np.float32), min(4, E))
        goe = O.place_experts(O.coselect(idx, E), G)
        assert (np.bincount(goe, minlength=G) == E // G).all()


def test_place_experts_recovers_planted_clusters():
    # the clustered top-6 recipe with expert ids scrambled: each group found
    # must be exactly one of the 16 planted clusters
    w = W.FINE.with_(T=4096)
    idx, _ = O.route_topk(W.make_logits(w), w.k)
    perm = np.random.default_rng(7).permutation(w.E).astype(np.int32)
    scrambled = perm[idx]
    goe = O.place_experts(O.coselect(scrambled, w.E), w.n_clusters)
    inv = np.argsort(perm)
    for g in range(w.n_clusters):
        members = inv[np.nonzero(goe == g)[0]]
        assert len(set((members // 4).tolist())) == 1
    # so the group-major layout needs exactly the rows of the true clusters,
    # fewer than contiguous groups of the scrambled ids
    cap = O.capacity(0.0, w.T, w.k, w.E)
    rows_placed = O.permute(scrambled, w.E, cap, goe)["R"]
    rows_true = O.permute(idx, w.E, cap, W.equal_groups(w.E, w.n_clusters))["R"]
    rows_contig = O.permute(scrambled, w.E, cap, W.equal_groups(w.E, w.n_clusters))["R"]
    assert rows_placed == rows_true
    assert rows_placed < 0.8 * rows_contig


def test_group_affinity_and_home_brute_force():
    T, E, G = 400, 12, 3
    i1, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), 2)
    i2, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), 3)
    M = O.transition(i1, i2, E)
    goe = RNG.permutation(np.repeat(np.arange(G), E // G)).astype(np.int32)
    aff = O.group_affinity(M, goe, G)
    want = np.zeros((E, G), np.int64)
    for a in range(E):
        for b in range(E):
            want[a, goe[b]] += M[a, b]
    assert (aff == want).all()
    assert (aff.sum(1) == M.sum(1)).all()
    home = O.predict_home(i1, aff)
    score = aff[i1].sum(1)                                   # [T, G]
    assert (home == np.argmax(score, axis=1)).all()           # argmax: first maximum
    local = O.count_local(i2, goe, G, home)
    assert local == sum(int(goe[i2[t, j]] == home[t]) for t in range(T) for j in range(3))


def test_count_local_closed_forms():
    T, E, G = 240, 8, 4
    goe = W.equal_groups(E, G)
    idx, _ = O.route_topk(RNG.normal(size=(T, E)).astype(np.float32), 1)
    # sequence-sharded home: same as the local-fraction definition
    assert O.count_local(idx, goe, G) == round(O.local_fraction(idx, goe, G) * T)
    # next layer identical to this one: the transition matrix is diagonal and
    # every token's predicted home holds its expert
    aff = O.group_affinity(O.transition(idx, idx, E), goe, G)
    assert O.count_local(idx, goe, G, O.predict_home(idx, aff)) == T


def test_shuffling_raises_local_share_on_correlated_layers():
    w = W.EXPERT_CHOICE.with_(T=8192)
    l1 = W.make_logits(w)
    a, _ = O.route_topk(l1, 1)
    b, _ = O.route_topk(W.make_layer2_logits(w, l1), 1)
    G = 8
    goe = W.equal_groups(w.E, G)
    before = O.count_local(b, goe, G) / w.T
    home = O.predict_home(a, O.group_affinity(O.transition(a, b, w.E), goe, G))
    after = O.count_local(b, goe, G, home) / w.T
    assert abs(before - 1 / G) < 0.02
    assert after > 2 * before


# ------------------------------------------ per-token layer compositions
def _layer_case(dtype, cf, F_shared):
    w = W.TINY.with_(dtype=dtype, capacity_factor=cf, T=300, F_shared=F_shared)
    return w, W.make_logits(w), W.make_x(w), W.make_weights(w), W.make_shared_weights(w)


@pytest.mark.parametrize("dtype,cf,F_shared", [("f32", 1.25, 0), ("bf16", 0.75, 96)])
def test_layer_tokens_equal_the_whole_batch_path(dtype, cf, F_shared):
    """The per-token layer (routing and drops over all tokens, the listed
    tokens' expert MLPs and their gated sum) equals the whole batch through
    the oracle's permutation, row copy, expert MLPs and unpermutation, bit
    for bit, for tokens listed in any order."""
    w, logits, x, Wt, Ws = _layer_case(dtype, cf, F_shared)
    idx, gate = O.route_topk(logits, w.k)
    p = O.permute(idx, w.E, O.capacity(w.capacity_factor, w.T, w.k, w.E))
    assert p["dropped"] > 0 or cf > 1
    buf = O.gather_rows(x, p["row_token"])
    Y = O.to_dtype_bits(O.expert_ffn_rows(buf, np.repeat(np.arange(w.E, dtype=np.int32), p["counts"]), *Wt, w.act), x)
    sh = None
    if Ws is not None:
        sh = O.to_dtype_bits(O.expert_ffn_rows(x, np.zeros(w.T, np.int32), *Ws, "swiglu"), x)
    full = O.unpermute(Y, p["row_map"], gate, sh)
    toks = RNG.permutation(w.T)[:120]
    got, info = O.topk_layer_tokens(w, logits, x, Wt, Ws, toks)
    if dtype == "bf16":
        assert np.array_equal(got, full[toks])           # Y is a bf16 tensor on both paths
    else:
        # fp32 layers round nothing; the whole-batch path hands Y to the unpermutation as fp32,
        # one rounding per expert output: within 2^-24 of sum_j |g_j Y_j|
        Yabs = O.to_dtype_bits(np.abs(O.expert_ffn_rows(buf, np.repeat(np.arange(w.E, dtype=np.int32), p["counts"]),
                                                        *Wt, w.act)), x)
        scale = O.unpermute(Yabs, p["row_map"], np.abs(gate))
        assert (np.abs(got - full[toks]) <= 2.0 ** -24 * scale[toks] + 1e-300).all()
        assert not np.array_equal(got, np.zeros_like(got))
    assert np.array_equal(info["perm"]["row_map"], p["row_map"])


def test_group_layer_tokens_equal_the_whole_batch_group_path():
    """The same for the group-major expert path: group rows -> each group's
    local copy to expert rows -> expert MLPs -> per-group gated pre-combine
    -> unit sum of the token's group rows, on scattered groups with drops."""
    w, logits, x, Wt, _ = _layer_case("bf16", 0.75, 0)
    G = 4
    goe = RNG.permutation(W.equal_groups(w.E, G)).astype(np.int32)
    idx, gate = O.route_topk(logits, w.k)
    cap = O.capacity(w.capacity_factor, w.T, w.k, w.E)
    pe, pg = O.permute(idx, w.E, cap), O.permute(idx, w.E, cap, group_of_expert=goe)
    xg = O.gather_rows(x, pg["row_token"])
    xe = np.zeros((pe["R"], w.d), x.dtype)
    O.copy_slot_rows(xg, pg["row_map"], pe["row_map"], xe)
    Ye = O.to_dtype_bits(O.expert_ffn_rows(xe, np.repeat(np.arange(w.E, dtype=np.int32), pe["counts"]), *Wt, w.act), x)
    P = O.group_precombine(Ye, pe["row_map"], pg["row_map"], gate, pg["R"])
    full = O.unpermute_groups(O.to_dtype_bits(P, x), pg["row_map"])
    toks = RNG.permutation(w.T)[:120]
    got, _ = O.topk_group_layer_tokens(w, logits, x, Wt, None, goe, toks)
    assert np.array_equal(got, full[toks])
