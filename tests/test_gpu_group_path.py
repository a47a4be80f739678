"""GPU vs oracle: the group-major expert path (send-once dispatcher with real
experts): local row copy bit-exact, group pre-combine and group unpermute
within the fp32 bound (plus one bf16 rounding where the result is bf16), and
whole layers within the bf16 layer tolerance."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_top_b200 import layer as Lyr, libmoe as M, synth, workloads as W
from oracle import oracle as O
from tests.helpers import (as_f64, assert_blocks_covered, assert_layer_close, needs_gpu, one_row_per_block, oracle_map,
                           to_dev, to_np, token_chunks)

pytestmark = [pytest.mark.gpu, needs_gpu]
REL = 1e-5
MOE_ERR_DEVICE_INDEX = 8          # moe_device_error: an index past its buffer was skipped


def routing(T, E, k, cf, G, seed=0, scatter=True):
    """Top-k routing with a hot expert (so small cf drops), both layouts."""
    lg = synth.normal_f32(seed, 1, (T, E))
    lg[:, E // 3] += 1.5
    idx, gate = O.route_topk(lg, k)
    cap = O.capacity(cf, T, k, E)
    goe = W.equal_groups(E, G)
    if scatter:                                  # groups that are not contiguous expert ranges
        goe = goe[np.random.default_rng(seed).permutation(E)].astype(np.int32)
    pe = O.permute(idx, E, cap)
    pg = O.permute(idx, E, cap, group_of_expert=goe)
    return idx, gate, goe, pe, pg


def gpu_routes(idx, E, cf, goe, G):
    d_idx = to_dev(idx)
    pg = M.permute(None, d_idx, E, cf, to_dev(goe), G)
    pe = M.permute(None, d_idx, E, cf)
    return pe, pg


CASES = [(300, 8, 2, 1.25, 2, 64, True), (2049, 16, 4, 0.7, 4, 256, True), (1000, 64, 6, 0.0, 8, 136, True),
         (777, 32, 1, 0.5, 4, 40, False), (64, 256, 8, 0.0, 64, 7168, True), (5000, 64, 8, 1.0, 16, 512, False)]


@pytest.mark.parametrize("T,E,k,cf,G,d,bf16", CASES)
def test_copy_slot_rows_exact(T, E, k, cf, G, d, bf16):
    idx, gate, goe, pe, pg = routing(T, E, k, cf, G)
    pe_d, pg_d = gpu_routes(idx, E, cf, goe, G)
    assert np.array_equal(to_np(pe_d["row_map"]), pe["row_map"])
    assert np.array_equal(to_np(pg_d["row_map"]), pg["row_map"])
    x = synth.normal_bf16(1, 2, (T, d)) if bf16 else synth.normal_f32(1, 2, (T, d))
    xg = O.gather_rows(x, pg["row_token"][:pg["R"]])
    R_e = pe["R"]
    dst = torch.full((R_e + 5, d), 3.0, dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")
    M.copy_slot_rows(to_dev(xg), pg_d["row_map"], pe_d["row_map"], dst)
    assert M.device_error() == 0
    got = to_np(dst)
    assert got[:R_e].tobytes() == O.gather_rows(x, pe["row_token"][:R_e]).tobytes()
    assert (as_f64(got[R_e:]) == 3.0).all()


@pytest.mark.parametrize("T,E,k,cf,G,d,bf16", CASES)
def test_group_precombine(T, E, k, cf, G, d, bf16):
    idx, gate, goe, pe, pg = routing(T, E, k, cf, G, seed=1)
    R_e, R_g = max(pe["R"], 1), max(pg["R"], 1)
    Y = synth.normal_bf16(1, 3, (R_e, d)) if bf16 else synth.normal_f32(1, 3, (R_e, d))
    y_g = torch.full((R_g + 3, d), 5.0, dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")
    M.group_precombine(to_dev(Y), to_dev(pe["row_map"]), to_dev(pg["row_map"]), to_dev(gate), y_g)
    assert M.device_error() == 0
    got = as_f64(to_np(y_g))
    ref = O.group_precombine(Y, pe["row_map"], pg["row_map"], gate, R_g)
    absY = (Y & 0x7FFF) if bf16 else np.abs(Y)
    scale = O.group_precombine(absY, pe["row_map"], pg["row_map"], np.abs(gate), R_g)
    n = pg["R"]
    tol = REL * scale[:n] + 1e-30
    if bf16:
        tol = tol + 2.0 ** -7 * np.abs(ref[:n])        # both sides round once to bf16
    assert (np.abs(got[:n] - ref[:n]) <= tol).all()
    if bf16:
        assert (got[:n] == ref[:n]).mean() > 0.99
    assert (got[R_g:] == 5.0).all()


@pytest.mark.parametrize("bulk", ["1", "0"])
@pytest.mark.parametrize("T,E,k,cf,G,d,bf16", CASES)
def test_unpermute_groups(T, E, k, cf, G, d, bf16, bulk, monkeypatch):
    monkeypatch.setenv("LIBMOE_BULK_COMBINE", bulk)       # bulk-staged kernel (k <= 8), then the register one
    idx, gate, goe, pe, pg = routing(T, E, k, cf, G, seed=2)
    R_g = max(pg["R"], 1)
    Yg = synth.normal_bf16(2, 3, (R_g, d)) if bf16 else synth.normal_f32(2, 3, (R_g, d))
    sh = synth.normal_bf16(2, 4, (T, d)) if bf16 else synth.normal_f32(2, 4, (T, d))
    absYg = np.abs(as_f64(Yg)).astype(np.float32)
    abssh = np.abs(as_f64(sh)).astype(np.float32)
    for shared in (None, sh):
        for out_dt in ((torch.float32, torch.bfloat16) if bf16 else (torch.float32,)):
            got = as_f64(to_np(M.unpermute_groups(to_dev(Yg), to_dev(pg["row_map"]),
                                                  None if shared is None else to_dev(shared), out_dt)))
            assert M.device_error() == 0
            ref = O.unpermute_groups(Yg, pg["row_map"], shared)
            scale = O.unpermute_groups(absYg, pg["row_map"], None if shared is None else abssh)
            tol = REL * scale + 1e-30
            if out_dt == torch.bfloat16:
                tol = tol + 2.0 ** -8 * np.abs(ref)
            assert (np.abs(got - ref) <= tol).all()
            if shared is None:
                dead = (pg["row_map"] < 0).all(1)
                assert (got[dead] == 0).all()


def test_group_path_empty_and_bad_rows():
    """T = 0 launches nothing; a row index past the buffer is skipped and
    reported through the device error word, not dereferenced."""
    z = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    g = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    y = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    before = M.kernel_launches()
    M.group_precombine(y, z, z, g, y.clone())
    out = M.unpermute_groups(y, z)
    assert out.shape == (0, 64) and M.kernel_launches() == before
    rm = torch.tensor([[0, 9], [1, -1]], dtype=torch.int32, device="cuda")       # 9 >= R_g = 4
    M.unpermute_groups(y, rm)
    assert M.device_error() == MOE_ERR_DEVICE_INDEX
    M.copy_slot_rows(y, rm.view(-1), torch.tensor([0, 1, 2, 3], dtype=torch.int32, device="cuda"), y.clone())
    assert M.device_error() == MOE_ERR_DEVICE_INDEX
    M.group_precombine(y, rm, rm, torch.ones((2, 2), device="cuda"), y.clone())
    assert M.device_error() == MOE_ERR_DEVICE_INDEX
    assert M.device_error() == 0                                               # cleared


# ------------------------------------------------------------------ layers
def weights_dev(ws):
    return tuple(None if a is None else to_dev(a) for a in ws)


@pytest.mark.parametrize("G,cf", [(2, 1.25), (4, 0.5), (8, 0.0)])
def test_group_layer_tiny_fp32_all_tokens(G, cf):
    w = W.TINY.with_(capacity_factor=cf, T=999)
    logits, x = W.make_logits(w), W.make_x(w)
    Wt = W.make_weights(w)
    goe = W.equal_groups(w.E, G)
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, torch.float32, *weights_dev(Wt),
                      group_of_expert=to_dev(goe), G=G)
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    assert M.device_error() == 0
    ref, info = O.topk_group_layer_tokens(w, logits, x, Wt, None, goe, np.arange(w.T))
    assert_layer_close(got, ref, rel=1e-4)
    # the same layer through the expert-major path
    ref_e, _ = O.topk_layer_tokens(w, logits, x, Wt, None, np.arange(w.T))
    assert_layer_close(ref, ref_e, rel=1e-6)
    assert int(L.perm["offsets"][-1].item()) == O.permute(info["idx"], w.E, info["cap"], goe)["R"]


@pytest.mark.parametrize("G", [4, 16])
def test_group_layer_fine_full_size(G):
    """Fine-grained layer (64 experts, top-6, shared expert) with placed
    (non-contiguous) groups, at full size, against the oracle on 1024
    seeded tokens, every token with a dropped slot, and one row of every
    128-row block of every expert's rows (the rows the grouped GEMMs tile)."""
    w = W.FINE
    logits, x = W.make_logits(w), W.make_x(w)
    Wt, Ws = W.make_weights(w), W.make_shared_weights(w)
    idx, _ = O.route_topk(logits, w.k)
    goe = O.place_experts(O.coselect(idx, w.E), G)
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, torch.bfloat16, *weights_dev(Wt),
                      shared_weights=weights_dev(Ws), group_of_expert=to_dev(goe), G=G)
    got = to_np(L.forward(to_dev(logits), to_dev(x)))
    assert M.device_error() == 0
    _, info = O.topk_group_layer_tokens(w, logits, x, Wt, Ws, goe, [])
    pe = info["perm"]                                   # expert-major rows: what the GEMMs run on
    rng = np.random.default_rng(G)
    dropped = np.nonzero((pe["row_map"] < 0).any(1))[0]
    toks = np.unique(np.concatenate([rng.choice(w.T, 1024, replace=False), dropped,
                                     pe["row_token"][one_row_per_block(pe["offsets"], rng)], [0, w.T - 1]]))
    assert assert_blocks_covered(pe["offsets"], pe["row_token"], toks) >= (pe["R"] + 127) // 128
    assert np.array_equal(to_np(L.perm_e["offsets"]), pe["offsets"])
    parts = oracle_map(lambda c: O.topk_group_layer_tokens(w, logits, x, Wt, Ws, goe, c)[0], token_chunks(toks))
    assert_layer_close(got[toks], np.concatenate(parts))
    # fewer rows cross to the groups than there are kept assignments
    R_g = int(L.perm["offsets"][-1].item())
    R_e = int(L.perm_e["offsets"][-1].item())
    assert R_g == O.permute(info["idx"], w.E, info["cap"], goe)["R"] and R_g < R_e
