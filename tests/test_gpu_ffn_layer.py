"""GPU vs oracle: grouped expert MLPs and whole MoE layers.

Tolerance (bf16 layers): max|y - y_ref| <= 2e-2 * max|y_ref|; the fp32
layer must also meet a 1e-4 bound (fp32 FMA against the fp64 oracle)."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, layer as Lyr, synth, workloads as W
from oracle import oracle as O
from tests.helpers import as_f64, assert_layer_close, needs_gpu, to_dev, to_np

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(params=["pair", "single"])
def gemm_kind(request, monkeypatch):
    """Run a test with the CTA-pair grouped GEMMs and with the one-CTA ones."""
    monkeypatch.setenv("LIBMOE_GEMM_PAIR", "1" if request.param == "pair" else "0")
    return request.param


def ffn_case(counts, d, F, act, bf16=True, seed=0):
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    R_max = R + 37                                   # rows past R must stay untouched
    gen = (lambda s, shp, std: synth.normal_bf16(seed, s, shp, 0.0, std)) if bf16 else \
          (lambda s, shp, std: synth.normal_f32(seed, s, shp, 0.0, std))
    x = gen(1, (R_max, d), 1.0)
    W1 = gen(2, (E, F, d), 0.05)
    W3 = gen(3, (E, F, d), 0.05) if act == "swiglu" else None
    W2 = gen(4, (E, d, F), 0.05)
    y = torch.full((R_max, d), 7.0, dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")
    M.expert_ffn(to_dev(x), to_dev(offsets), to_dev(W1), None if W3 is None else to_dev(W3), to_dev(W2), act, y=y)
    assert M.device_error() == 0
    got = to_np(y)
    row_e = np.repeat(np.arange(E, dtype=np.int32), counts)
    ref = O.expert_ffn_rows(x[:R], row_e, W1, W3, W2, act)
    assert (as_f64(got[R:]) == 7.0).all()
    return got[:R], ref


@pytest.mark.parametrize("counts,d,F,act", [
    ([0, 130, 300], 128, 192, "swiglu"),           # empty expert, ragged tiles, partial n-tiles
    ([257, 1, 128, 0, 64], 256, 128, "swiglu"),
    ([200, 333], 512, 1024, "swiglu"),             # several k-blocks and n-tiles
    ([0, 130, 300], 128, 256, "gelu"),
    ([129, 511], 320, 448, "gelu"),
    ([1000], 64, 64, "swiglu"),
    ([600, 0, 900, 257], 256, 320, "swiglu"),     # 256-row tiles with ragged tails, partial n-tiles
    ([513, 1100], 320, 256, "gelu")])
def test_expert_ffn_bf16(counts, d, F, act, gemm_kind):
    got, ref = ffn_case(counts, d, F, act)
    assert_layer_close(got, ref)


def test_gelu_epilogue_matches_exact_erf(gemm_kind):
    """One expert whose W1 and W2 are identities: the MLP returns gelu(x)
    itself.  fp32: within the erf approximation's bound (A&S 7.1.28, 2e-6
    absolute in fp32) plus fp32 rounding; bf16: the exact GELU rounded to
    bf16, up to one bf16 step where the exact value sits on a rounding
    boundary."""
    import math
    d = 64
    xs = np.concatenate([np.linspace(-8.0, 8.0, 4091), [0.0, 1e-6, -1e-6, 1e-3, -1e-3]])
    n = xs.size
    eye = np.eye(d)
    for bf16 in (False, True):
        rows = np.zeros((n, d))
        rows[:, 0] = xs
        if bf16:
            x = synth.f32_to_bf16(rows.astype(np.float32))
            W = synth.f32_to_bf16(eye.astype(np.float32))
        else:
            x, W = rows.astype(np.float32), eye.astype(np.float32)
        xv = as_f64(x)[:, 0]
        y = torch.zeros((n, d), dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")
        M.expert_ffn(to_dev(x), to_dev(np.array([0, n], np.int32)), to_dev(W[None]), None, to_dev(W[None]), "gelu",
                     y=y)
        got = as_f64(to_np(y))[:, 0]
        exact = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in xv])
        # absolute error of 0.5 x (1 + erf): the approximation's 2e-6 on erf (in fp32, where 1 + erf also
        # cancels to 0 in the far negative tail) times 0.5 |x|
        approx = 1.1e-6 * np.abs(xv)
        if bf16:
            want = as_f64(synth.f32_to_bf16(exact.astype(np.float32)))
            step = np.abs(want) * 2.0 ** -7 + 1e-38
            assert (np.abs(got - want) <= step + approx).all()
            # where |gelu| >= 0.05 the fp32 value of 1 + erf keeps its relative precision: bf16 values agree
            big = np.abs(exact) >= 0.05
            assert (got[big] == want[big]).mean() > 0.99
        else:
            assert (np.abs(got - exact) <= approx + 1e-6 * np.abs(exact) + 1e-30).all()


def test_expert_ffn_fp32():
    got, ref = ffn_case([70, 0, 90, 100], 64, 128, "swiglu", bf16=False)
    assert_layer_close(got, ref, rel=1e-4)
    got, ref = ffn_case([10, 20], 24, 40, "gelu", bf16=False)
    assert_layer_close(got, ref, rel=1e-4)


# ------------------------------------------------------------------ layers
def weights_dev(ws):
    return tuple(None if a is None else to_dev(a) for a in ws)


def test_layer_tiny_fp32_all_tokens():
    w = W.TINY
    logits, x = W.make_logits(w), W.make_x(w)
    Wt = W.make_weights(w)
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, torch.float32, *weights_dev(Wt))
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    ref, info = O.topk_layer_tokens(w, logits, x, Wt, None, np.arange(w.T))
    assert_layer_close(got, ref, rel=1e-4)


def test_layer_tiny_forced_drops():
    w = W.TINY.with_(T=999, capacity_factor=0.5)
    logits, x = W.make_logits(w), W.make_x(w)
    Wt = W.make_weights(w)
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, torch.float32, *weights_dev(Wt))
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    ref, info = O.topk_layer_tokens(w, logits, x, Wt, None, np.arange(w.T))
    assert info["perm"]["dropped"] > 0
    assert int(L.perm["dropped"][0]) == info["perm"]["dropped"]
    assert_layer_close(got, ref, rel=1e-4)
    all_dropped = (info["perm"]["row_map"] < 0).all(1)
    assert all_dropped.any() and (got[all_dropped] == 0).all()


def sampled_tokens(info, T, n, seed=0):
    """n tokens: some with dropped slots first, the rest uniform."""
    rng = np.random.default_rng(seed)
    dropped = np.nonzero((info["perm"]["row_map"] < 0).any(1))[0]
    pick = list(rng.choice(dropped, size=min(n // 2, dropped.size), replace=False)) if dropped.size else []
    rest = rng.choice(T, size=n - len(pick), replace=False)
    return np.unique(np.concatenate([np.asarray(pick, np.int64), rest, [0, T - 1]]))


def boundary_tokens(perm, E, inner_tiles):
    """Tokens owning the buffer rows at each expert's first and last row, at
    the first row of its last (ragged) 128-row tile and on both sides of its
    first `inner_tiles` 128-row tile boundaries: the rows where the grouped
    GEMMs' tiles start, end and straddle experts."""
    off, rt = perm["offsets"], perm["row_token"]
    rows = []
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b <= a:
            continue
        rows += [a, b - 1, a + ((b - 1 - a) // 128) * 128]
        for j in range(1, inner_tiles + 1):
            if a + 128 * j < b:
                rows += [a + 128 * j - 1, a + 128 * j]
    return np.unique(rt[np.asarray(rows)])


_FULL_REF = {}


def full_size_reference(w, logits, x, Wt, Ws):
    """The oracle's outputs on the sampled tokens of a full-size layer,
    computed once per workload (the test runs once per GEMM kernel)."""
    if w.name not in _FULL_REF:
        _, info = O.topk_layer_tokens(w, logits, x, Wt, Ws, [])
        toks = np.union1d(sampled_tokens(info, w.T, 12), boundary_tokens(info["perm"], w.E, 1 if w.E <= 8 else 0))
        ref, _ = O.topk_layer_tokens(w, logits, x, Wt, Ws, toks)
        _FULL_REF[w.name] = (toks, ref, info["idx"])
    return _FULL_REF[w.name]


@pytest.mark.parametrize("w", [W.MIXTRAL, W.FINE], ids=lambda w: w.name)
def test_layer_full_size_sampled(w, gemm_kind):
    """Full-size layer in the bench's launch configuration against the
    oracle on sampled tokens: some with dropped slots, some uniform, and
    those owning each expert's first and last rows and rows at 128-row tile
    boundaries."""
    logits, x = W.make_logits(w), W.make_x(w)
    Wt = W.make_weights(w)
    Ws = W.make_shared_weights(w)
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, torch.bfloat16, *weights_dev(Wt),
                      shared_weights=None if Ws is None else weights_dev(Ws))
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    assert M.device_error() == 0
    toks, ref, idx = full_size_reference(w, logits, x, Wt, Ws)
    assert toks.size > 30
    assert_layer_close(got[toks], ref)
    # co-selection of this layer's routing, bit-exact
    assert np.array_equal(to_np(M.coselect(L.idx, w.E)), O.coselect(idx, w.E))


@pytest.mark.parametrize("G", W.SWEEP_G)
def test_layer_dispatch_combine_identity(G):
    w = W.SWEEP.with_(T=4096)
    logits, x = W.make_logits(w), W.make_x(w)
    goe = W.equal_groups(w.E, G)
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, 0, 0.0, torch.bfloat16, None, None, None, norm_topk=True,
                      group_of_expert=to_dev(goe), G=G, out_dtype=torch.float32)
    got = as_f64(to_np(L.forward(to_dev(logits), to_dev(x))))
    idx, gate = O.route_topk(logits, w.k, True)
    p = O.permute(idx, w.E, O.capacity(0.0, w.T, w.k, w.E), goe)
    ref = O.unpermute(O.gather_rows(x, p["row_token"]), p["row_map"], gate)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(got, as_f64(x), rtol=1e-5, atol=1e-6)   # renormalised gates: y == x


def test_layer_expert_choice_sampled(gemm_kind):
    w = W.EXPERT_CHOICE
    logits, x = W.make_logits(w), W.make_x(w)
    W1, _, W2 = W.make_weights(w)
    L = Lyr.ExpertChoiceLayer(w.T, w.d, w.E, w.C, w.F, torch.bfloat16, to_dev(W1), None, to_dev(W2), "gelu")
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    assert M.device_error() == 0
    ec_token, ec_gate, tok_ptr, tok_row = O.route_ec(logits, w.C)
    rng = np.random.default_rng(0)
    chosen = np.nonzero(np.diff(tok_ptr) > 0)[0]
    unchosen = np.nonzero(np.diff(tok_ptr) == 0)[0]
    toks = np.unique(np.concatenate([rng.choice(chosen, 10, replace=False), unchosen[:3]]))
    ref = np.zeros((toks.size, w.d))
    for i, t in enumerate(toks):
        rows = tok_row[tok_ptr[t]:tok_ptr[t + 1]]
        if rows.size:
            y = O.expert_ffn_rows(x[[t] * rows.size], (rows // w.C).astype(np.int32), W1, None, W2, "gelu")
            ref[i] = (ec_gate.reshape(-1)[rows].astype(np.float64)[:, None] * y).sum(0)
    assert_layer_close(got[toks], ref)
    assert (as_f64(got[unchosen]) == 0).all()


def test_host_pipeline_matches_plain_forward():
    """Batches streamed through HostPipeline (copies overlapped with compute)
    give exactly the outputs of one forward per batch."""
    w = W.TINY
    Wt = weights_dev(W.make_weights(w))
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, torch.float32, *Wt)
    batches = [w.with_(seed=s) for s in (3, 4, 5, 6, 7)]
    h_in = [[torch.from_numpy(W.make_logits(b)).pin_memory(), torch.from_numpy(W.make_x(b)).pin_memory()]
            for b in batches]
    h_out = [torch.empty((w.T, w.d), dtype=torch.float32).pin_memory() for _ in batches]
    d_lg, d_x = torch.empty((w.T, w.E), device="cuda"), torch.empty((w.T, w.d), device="cuda")
    pipe = Lyr.HostPipeline(lambda lg, x, out: L.forward(lg, x, out=out), [d_lg, d_x], torch.empty_like(L.out))
    pipe.run(h_in, h_out)
    torch.cuda.synchronize()
    for (lg, x), got in zip(h_in, h_out):
        want = L.forward(lg.cuda(), x.cuda()).cpu()
        assert torch.equal(got, want)


@pytest.mark.parametrize("bf16", [False, True])
def test_captured_forward_matches_eager(bf16):
    """The whole top-k layer recorded as one CUDA graph: replays give exactly
    the eager outputs, and follow new contents of the input tensors."""
    w = W.TINY if not bf16 else W.FINE.with_(T=2048, F_shared=0)
    dt = torch.bfloat16 if bf16 else torch.float32
    Wt = weights_dev(W.make_weights(w))
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, dt, *Wt)
    lg0, x0 = to_dev(W.make_logits(w)), to_dev(W.make_x(w))
    want0 = L.forward(lg0, x0).clone()
    w1 = w.with_(seed=5)
    lg1, x1 = to_dev(W.make_logits(w1)), to_dev(W.make_x(w1))
    want1 = L.forward(lg1, x1).clone()
    lg, x = lg0.clone(), x0.clone()
    cap = Lyr.CapturedForward(lambda a, b, out: L.forward(a, b, out=out), [lg, x], torch.empty_like(L.out))
    assert torch.equal(cap.replay(), want0)
    lg.copy_(lg1)
    x.copy_(x1)
    assert torch.equal(cap.replay(), want1)
    assert M.device_error() == 0
