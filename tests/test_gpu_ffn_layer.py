"""GPU vs oracle: grouped expert MLPs and whole MoE layers.

Tolerance (bf16 layers): max|y - y_ref| <= 2e-2 * max|y_ref|; the fp32
layer must also meet a 1e-4 bound (fp32 FMA against the fp64 oracle)."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import libmoe as M, layer as Lyr, synth, workloads as W
from oracle import oracle as O
from tests.helpers import (as_f64, assert_blocks_covered, assert_layer_close, needs_gpu, one_row_per_block, oracle_map,
                           to_dev, to_np, token_chunks)

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
    ([513, 1100], 320, 256, "gelu"),
    ([31, 32, 33, 96, 127, 129, 1, 255, 257], 128, 128, "swiglu"),   # 32-row warp boxes: full, straddling, short
    ([31, 32, 33, 96, 127, 129, 1, 255, 257], 128, 192, "gelu")])
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


FULL_UNIFORM = 1024      # seeded uniform tokens per full-size layer


def boundary_tokens(perm, E):
    """Tokens owning each expert's first and last buffer rows and the first
    row of its last (ragged) 128-row tile: where the grouped GEMMs' tiles
    start, end and straddle experts."""
    off, rt = perm["offsets"], perm["row_token"]
    rows = []
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            rows += [a, b - 1, a + ((b - 1 - a) // 128) * 128]
    return np.unique(rt[np.asarray(rows, np.int64)]) if rows else np.zeros(0, np.int64)


def full_size_tokens(info, w, seed=0):
    """The tokens a full-size layer is checked on: every token with a
    dropped slot, 1024 seeded uniform tokens, the owner of one seeded row in
    every 128-row block of every expert, the tile-boundary owners, and the
    first and last tokens."""
    rng = np.random.default_rng(seed)
    perm = info["perm"]
    dropped = np.nonzero((perm["row_map"] < 0).any(1))[0]
    uniform = rng.choice(w.T, size=min(FULL_UNIFORM, w.T), replace=False)
    blocks = perm["row_token"][one_row_per_block(perm["offsets"], rng)]
    return np.unique(np.concatenate([dropped, uniform, blocks, boundary_tokens(perm, w.E), [0, w.T - 1]])), dropped


_FULL_REF = {}


def full_size_reference(w, logits, x, Wt, Ws):
    """The oracle's outputs on the checked tokens of a full-size layer,
    computed once per workload (the test runs once per GEMM kernel family),
    token chunks spread over the host cores."""
    if w.name not in _FULL_REF:
        _, info = O.topk_layer_tokens(w, logits, x, Wt, Ws, [])
        toks, dropped = full_size_tokens(info, w)
        parts = oracle_map(lambda c: O.topk_layer_tokens(w, logits, x, Wt, Ws, c)[0], token_chunks(toks))
        _FULL_REF[w.name] = (toks, np.concatenate(parts), info, dropped)
    return _FULL_REF[w.name]


@pytest.mark.parametrize("w", [W.MIXTRAL, W.FINE], ids=lambda w: w.name)
def test_layer_full_size(w, gemm_kind):
    """Full-size layer in the bench's launch configuration against the
    oracle on every token with a dropped slot, 1024 seeded tokens and one
    row of every 128-row block of every expert (so each half of every
    256-row CTA-pair tile of the persistent schedule is compared)."""
    logits, x = W.make_logits(w), W.make_x(w)
    Wt = W.make_weights(w)
    Ws = W.make_shared_weights(w)
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, torch.bfloat16, *weights_dev(Wt),
                      shared_weights=None if Ws is None else weights_dev(Ws))
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    assert M.device_error() == 0
    toks, ref, info, dropped = full_size_reference(w, logits, x, Wt, Ws)
    perm = info["perm"]
    # the sample's contract: all dropped-slot tokens, >= 1024 tokens, every block covered
    assert np.isin(dropped, toks).all() and toks.size >= FULL_UNIFORM
    assert assert_blocks_covered(perm["offsets"], perm["row_token"], toks) >= (perm["R"] + 127) // 128
    # the layer's own routing and permutation are those of the oracle, on all tokens
    assert np.array_equal(to_np(L.perm["offsets"]), perm["offsets"])
    assert np.array_equal(to_np(L.perm["row_map"]).reshape(w.T, w.k), perm["row_map"])
    assert_layer_close(got[toks], ref)
    # tokens whose every slot dropped (and no shared expert) output exactly zero
    if Ws is None:
        gone = np.nonzero((perm["row_map"] < 0).all(1))[0]
        assert (as_f64(got[gone]) == 0).all()
    # co-selection of this layer's routing, bit-exact
    assert np.array_equal(to_np(M.coselect(L.idx, w.E)), O.coselect(info["idx"], w.E))


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


_EC_REF = {}


def ec_reference(w, x, W1, W2):
    """The oracle's expert-choice layer on the checked tokens: 1024 seeded
    chosen tokens and the owner of one seeded row in every 128-row block of
    every expert's C rows; each token's expert outputs gate-summed in the
    token CSR's order (ascending expert).  Computed once, token chunks
    spread over the host cores."""
    if w.name in _EC_REF:
        return _EC_REF[w.name]
    logits = W.make_logits(w)
    ec_token, ec_gate, tok_ptr, tok_row = O.route_ec(logits, w.C)
    rng = np.random.default_rng(0)
    chosen = np.nonzero(np.diff(tok_ptr) > 0)[0]
    offsets = np.arange(w.E + 1, dtype=np.int64) * w.C
    blocks = ec_token.reshape(-1)[one_row_per_block(offsets, rng)]
    toks = np.unique(np.concatenate([rng.choice(chosen, min(FULL_UNIFORM, chosen.size), replace=False), blocks]))
    g = ec_gate.reshape(-1).astype(np.float64)

    def chunk(ts):
        rows = [tok_row[tok_ptr[t]:tok_ptr[t + 1]] for t in ts]
        y = O.expert_ffn_rows(x[np.repeat(ts, [r.size for r in rows])],
                              (np.concatenate(rows) // w.C).astype(np.int32), W1, None, W2, "gelu")
        out = np.zeros((len(ts), w.d))
        n = 0
        for i, r in enumerate(rows):
            for q in r:
                out[i] += g[q] * y[n]
                n += 1
        return out

    ref = np.concatenate(oracle_map(chunk, token_chunks(toks)))
    _EC_REF[w.name] = (toks, ref, (ec_token, tok_ptr), offsets)
    return _EC_REF[w.name]


def test_layer_expert_choice_full_size(gemm_kind):
    """The expert-choice GELU layer at full size (T=32768, E=128, C=512):
    1024 seeded tokens plus one row of every 128-row block of every
    expert against the oracle; every unchosen token outputs exactly 0."""
    w = W.EXPERT_CHOICE
    logits, x = W.make_logits(w), W.make_x(w)
    W1, _, W2 = W.make_weights(w)
    L = Lyr.ExpertChoiceLayer(w.T, w.d, w.E, w.C, w.F, torch.bfloat16, to_dev(W1), None, to_dev(W2), "gelu")
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    assert M.device_error() == 0
    toks, ref, (ec_token, tok_ptr), offsets = ec_reference(w, x, W1, W2)
    assert toks.size >= FULL_UNIFORM
    assert assert_blocks_covered(offsets, ec_token.reshape(-1), toks) == w.E * ((w.C + 127) // 128)
    assert_layer_close(got[toks], ref)
    unchosen = np.nonzero(np.diff(tok_ptr) == 0)[0]
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
