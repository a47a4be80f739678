"""bench.py's CPU-baseline leg (CPU): each runner times the oracle on a
sample sized by a time budget and reports it in the contract's form.  The
runners are built here without their device state (the leg only reads the
host copies of the inputs)."""
import time
import types

import numpy as np
import pytest

import bench
from mixture_experts_routing_top_b200 import workloads as W
from oracle import oracle as O


def topk_runner(w):
    r = object.__new__(bench.TopKRunner)
    r.w = w
    r.logits_np, r.x_np = W.make_logits(w), W.make_x(w)
    r.weights_np = W.make_weights(w) if w.F else (None, None, None)
    r.shared_np = W.make_shared_weights(w)
    r.Wr_np = W.make_router_weights(w) if w.router else None
    r.goe = W.equal_groups(w.E, w.G) if w.G else None
    r.L = types.SimpleNamespace(grouped=bool(w.G and w.F))
    return r


def check(res, budget):
    assert res["kind"] == "oracle" and res["cores"] == 1 and res["unit"] == "tokens/s"
    assert res["value"] > 0 and res["sample"]


@pytest.mark.parametrize("w", [W.TINY.with_(T=2000), W.FINE.with_(T=1024, d=256, F=128, F_shared=256),
                               W.FINE.with_(T=1024, d=256, F=128, G=8)], ids=["tiny", "shared", "grouped"])
def test_topk_baseline_fills_its_budget(w):
    r = topk_runner(w)
    t0 = time.perf_counter()
    res = r.cpu_baseline(0.5)
    took = time.perf_counter() - t0
    check(res, 0.5)
    assert "expert MLP on" in res["sample"]
    n = int(res["sample"].split("expert MLP on ")[1].split(" of ")[0])
    assert n > 4 and took < 30


def test_mlp_sample_spreads_over_all_experts_and_respects_the_budget():
    w = W.TINY.with_(T=2000)
    x = W.make_x(w)
    idx, _ = O.route_topk(W.make_logits(w), w.k)
    p = O.permute(idx, w.E, O.capacity(w.capacity_factor, w.T, w.k, w.E))
    buf = O.gather_rows(x, p["row_token"])
    seen = []
    row_expert = lambda rows: (seen.append(rows) or
                               (np.searchsorted(p["offsets"], rows, side="right") - 1).astype(np.int32))
    n, t_row = bench.time_mlp_rows(O, buf, row_expert, W.make_weights(w), w.act, 0.2)
    assert 4 < n <= p["R"] and t_row > 0
    experts = np.searchsorted(p["offsets"], seen[-1], side="right") - 1
    assert set(experts.tolist()) == set(np.nonzero(p["counts"])[0].tolist())
    n0, _ = bench.time_mlp_rows(O, buf, row_expert, W.make_weights(w), w.act, 0.0)
    assert n0 == 4                              # no budget: the probe alone


def test_routing_baseline_scales_its_token_sample():
    w = W.SWEEP.with_(T=20000)
    r = object.__new__(bench.RoutingRunner)
    r.w = w
    r.in_np = [W.make_logits(w)]
    r.Wr_np = None
    res = r.cpu_baseline(0.3)
    check(res, 0.3)
    Ts = int(res["sample"].split(" on ")[1].split(" of ")[0])
    assert 256 < Ts <= w.T


def test_expert_choice_baseline_fills_its_budget():
    w = W.EXPERT_CHOICE.with_(T=2048, d=128, F=256, C=32)
    r = object.__new__(bench.ExpertChoiceRunner)
    r.w = w
    r.logits_np, r.x_np = W.make_logits(w), W.make_x(w)
    r.logits2_np = W.make_layer2_logits(w, r.logits_np)
    r.weights_np = W.make_weights(w)
    res = r.cpu_baseline(0.5)
    check(res, 0.5)
    n = int(res["sample"].split("expert MLP on ")[1].split(" of ")[0])
    assert 4 < n <= w.E * w.C
