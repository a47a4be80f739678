"""GPU vs oracle: the router's linear gate fused with top-k.

The fused kernel returns its fp32 logits on request.  Parity is checked in
three parts:
  - logits within the fp32 accumulation bound of the fp64 oracle:
    |l - l_ref| <= d * 2^-23 * sum_c |x_c w_c| (every product of two bf16
    values is exact in fp32; each of the d additions rounds once);
  - the experts and gates the kernel chose from those logits are exactly the
    oracle's top-k of the same logits (indices bit-exact, gates 1e-6);
  - against the oracle's top-k of its own logits: identical wherever the
    gaps around the k-th logit exceed twice that bound, and otherwise a
    valid choice (every chosen logit within the bound of the oracle's k-th).
Small-integer inputs make every logit exact, so there the ranking, ties
included, must equal the oracle's outright."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, synth, workloads as W
from oracle import oracle as O
from tests.helpers import needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]
GATE_RTOL = 1e-6


def _f64(a):
    return synth.bf16_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def check_router(x, Wr, k, norm=False, tokens=None):
    """Runs the fused router on x (all rows) and checks the listed tokens."""
    T, d = x.shape
    idx, gate, lg = M.router_topk(to_dev(x), to_dev(Wr), k, norm, want_logits=True)
    assert M.device_error() == 0
    gi, gg, gl = to_np(idx), to_np(gate), to_np(lg)
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    # 1. logits vs the fp64 oracle
    ref = O.router_logits(x[toks], Wr)
    bound = d * 2.0 ** -23 * O.router_logits(np.abs(_f64(x[toks])).astype(np.float32),
                                             np.abs(_f64(Wr)).astype(np.float32))
    err = np.abs(gl[toks] - ref)
    assert (err <= bound + 1e-30).all(), "logit error %.3g over bound" % (err - bound).max()
    # 2. the kernel's choice from its own logits is the oracle's top-k of them
    ridx, rgate = O.route_topk(gl[toks], k, norm)
    bad = np.nonzero((gi[toks] != ridx).any(1))[0]
    assert bad.size == 0, "token %d: gpu %s oracle %s" % (toks[bad[0]], gi[toks[bad[0]]], ridx[bad[0]])
    np.testing.assert_allclose(gg[toks], rgate, rtol=GATE_RTOL, atol=1e-30)
    # 3. vs the oracle's ranking of its own logits
    oidx, _ = O.route_topk(ref.astype(np.float32), k, norm)
    tol = 2 * bound.max(1)
    srt = -np.sort(-ref, 1)[:, :min(k + 1, ref.shape[1])]
    gaps = -np.diff(srt, axis=1).min(1) if srt.shape[1] > 1 else np.full(len(toks), np.inf)
    clear = gaps > tol
    assert np.array_equal(gi[toks][clear], oidx[clear])
    kth = srt[:, k - 1]
    chosen = np.take_along_axis(ref, gi[toks].astype(np.int64), 1)
    assert (chosen >= kth[:, None] - tol[:, None]).all()
    # 4. the same choice without the logits output
    idx2, gate2, _ = M.router_topk(to_dev(x), to_dev(Wr), k, norm)
    assert torch.equal(idx2, idx) and torch.equal(gate2, gate)
    return clear.mean()


@pytest.fixture(params=["persistent", "pair"])
def router_kind(request, monkeypatch):
    """Run a test with the persistent router kernel and with the one that
    splits K over a CTA pair (the library picks by T; the tests force each)."""
    monkeypatch.setenv("LIBMOE_ROUTER_PAIR", "1" if request.param == "pair" else "0")
    return request.param


@pytest.mark.parametrize("T,d,E,k", [(1, 64, 8, 2), (77, 128, 16, 1), (1000, 256, 8, 2), (1000, 64, 64, 6),
                                     (4097, 512, 128, 4), (300, 1024, 256, 8), (129, 192, 24, 3),
                                     (2500, 2048, 72, 8), (700, 192, 8, 2)])
@pytest.mark.parametrize("norm", [False, True])
def test_router_bf16_random(T, d, E, k, norm, router_kind):
    x = synth.normal_bf16(21, 1, (T, d))
    Wr = synth.normal_bf16(21, 2, (E, d), 0.0, d ** -0.5)
    assert check_router(x, Wr, k, norm) > 0.95


def test_router_exact_integers_and_ties(router_kind):
    """Small integers: exact logits, many ties (and all-zero rows, where the
    k lowest experts win)."""
    rng = np.random.default_rng(5)
    for T, d, E, k in ((1000, 64, 8, 2), (700, 128, 64, 6), (300, 256, 256, 8)):
        xi = rng.integers(-2, 3, size=(T, d)).astype(np.float32)
        xi[::7] = 0.0
        Wi = rng.integers(-1, 2, size=(E, d)).astype(np.float32)
        x, Wr = synth.f32_to_bf16(xi), synth.f32_to_bf16(Wi)
        idx, gate, lg = M.router_topk(to_dev(x), to_dev(Wr), k, want_logits=True)
        ref = O.router_logits(x, Wr)
        assert np.array_equal(to_np(lg), ref.astype(np.float32))
        ridx, rgate = O.route_topk(ref.astype(np.float32), k)
        assert np.array_equal(to_np(idx), ridx)
        assert (to_np(idx)[::7] == np.arange(k)).all()
        np.testing.assert_allclose(to_np(gate), rgate, rtol=GATE_RTOL, atol=1e-30)


@pytest.mark.parametrize("w", [W.MIXTRAL, W.FINE], ids=lambda w: w.name)
def test_router_full_size(w, router_kind):
    x = W.make_x(w)
    Wr = W.make_router_weights(w)
    rng = np.random.default_rng(1)
    toks = np.unique(np.concatenate([rng.choice(w.T, 2000, replace=False), [0, w.T - 1]]))
    check_router(x, Wr, w.k, w.norm_topk, tokens=toks)


def test_router_sweep_shape_sampled():
    w = W.SWEEP.with_(T=16384)
    x = W.make_x(w)
    Wr = W.make_router_weights(w)
    toks = np.unique(np.concatenate([np.random.default_rng(2).choice(w.T, 200, replace=False), [w.T - 1]]))
    check_router(x, Wr, w.k, True, tokens=toks)


def test_router_fp32():
    w = W.TINY
    x = W.make_x(w)
    Wr = W.make_router_weights(w)
    idx, gate, lg = M.router_topk(to_dev(x), to_dev(Wr), w.k)
    ref = O.router_logits(x, Wr)
    bound = w.d * 2.0 ** -23 * O.router_logits(np.abs(x), np.abs(Wr))
    assert (np.abs(to_np(lg) - ref) <= bound).all()
    ridx, rgate = O.route_topk(to_np(lg), w.k)
    assert np.array_equal(to_np(idx), ridx)
    np.testing.assert_allclose(to_np(gate), rgate, rtol=GATE_RTOL, atol=1e-30)


def test_router_edges():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    idx, gate, _ = M.router_topk(x, Wr, 2)
    assert idx.shape == (0, 2)
    x1 = torch.zeros((5, 64), dtype=torch.bfloat16, device="cuda")
    for E, k, d, status in ((12, 2, 64, 2), (16, 9, 64, 2), (8, 2, 96, 2), (264, 2, 64, 2), (8, 9, 64, 1)):
        with pytest.raises(M.MoeError) as ei:
            M.router_topk(torch.zeros((5, d), dtype=torch.bfloat16, device="cuda"),
                          torch.zeros((E, d), dtype=torch.bfloat16, device="cuda"), k)
        assert ei.value.status == status
    assert M.device_error() == 0
    idx, gate, _ = M.router_topk(x1, Wr, 2)
    assert to_np(idx).tolist() == [[0, 1]] * 5
