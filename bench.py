#!/usr/bin/env python
"""Benchmark of one MoE layer step on B200 through libmoe.

A step is one pass of the whole hot path over one batch.  Default workload:
the Mixtral-shaped top-2 layer (T=8192 tokens, d=4096, E=8 experts, SwiGLU
4096->14336->4096, capacity factor 1.25, bf16 with fp32 accumulation); its
step is top-k routing -> capacity-bounded permutation -> grouped expert MLPs
(tcgen05 GEMMs) -> gate-weighted combine -> co-selection histogram.  Other
workloads (``--workload``): the fine-grained top-6 layer with a shared expert,
the dispatch/combine sweep (identity experts, group-major rows), and the
expert-choice layer with its layer-to-layer transition histogram.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libmoe|reference]

One JSON line on rank 0.  Under torchrun each rank runs its own batch (its
own seed) against the same expert weights: independent replicas, no
collective on the data path, weak scaling; the timed region is bracketed by
a barrier and a device synchronise on both sides and the slowest rank's
time is taken.  ``--impl reference`` times the CPU oracle (single-threaded C)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s; permute/combine HBM GB/s and grouped-GEMM TFLOP/s vs peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs of the run: N > 1 needs one process per GPU (torch.distributed.run)")
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="libmoe", choices=["libmoe", "reference"])
    ap.add_argument("--workload", default="mixtral_top2_bf16")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU-baseline budget: the oracle's expert-MLP (or routing) sample takes about this long")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--graph", action="store_true",
                    help="time the step as one CUDA-graph replay (stage times from an eager pass before it)")
    ap.add_argument("--routing-only", action="store_true",
                    help="time routing and co-selection alone at the workload's shape (top-k workloads)")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field (e.g. T=4096) - for smaller profiling cases, not bench lines")
    return ap.parse_args(argv)


def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def workload_from_args(args):
    from mixture_experts_routing_top_b200 import workloads as W

    w = W.BY_NAME[args.workload]
    for kv in args.set:
        key, val = kv.split("=", 1)
        w = w.with_(**{key: type(getattr(w, key))(val)})
    if args.set:
        w = w.with_(name=w.name + "[" + ",".join(args.set) + "]")
    if getattr(args, "routing_only", False):
        w = w.with_(name=w.name + "[routing only]")
    return w


def kind_of(w):
    if w.routing == "ec":
        return "ec"
    return "sweep" if w.F == 0 else "topk"


# ------------------------------------------------------------- clocks
class Clocks:
    """nvidia-smi samples (every 100 ms) across the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL,
                                         stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"samples": 0}
        num = lambda v: v.replace(".", "", 1).isdigit()
        sm = [float(r[1]) for r in rows if num(r[1])]
        mx = [float(r[2]) for r in rows if num(r[2])]
        pw = [float(r[3]) for r in rows if num(r[3])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------- ranks
def rank_batch(w, rank):
    """Workload of one rank: its own batch (seed = rank), same shapes."""
    return w.with_(seed=rank)


def reduce_over_ranks(elapsed_ms, launches, device):
    """Slowest rank's time and total launches over all ranks (identity on one
    process).  Runs on any torch.distributed backend (NCCL on GPUs, gloo on
    CPU in the tests)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(elapsed_ms), int(launches)
    t = torch.tensor([float(elapsed_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    c = torch.tensor([int(launches)], dtype=torch.int64, device=device)
    dist.all_reduce(c, op=dist.ReduceOp.SUM)
    return float(t.item()), int(c.item())


def job_histogram(name, hist, world, device):
    """The job's histogram from the ranks' accumulated ones: one int32 SUM
    all-reduce of the E x E counts (outside the timed steps).  Every rank ran
    the same number of passes over T tokens, so the job total must be the
    world size times this rank's; returns the record for the JSON line."""
    import torch

    from mixture_experts_routing_top_b200 import layer as Lyr

    local_total = int(hist.sum().item())
    job = hist.clone()
    if device.type == "cuda":
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        Lyr.reduce_histogram(job)
        b.record()
        torch.cuda.synchronize()
        us = 1e3 * a.elapsed_time(b)
    else:
        t0 = time.perf_counter()
        Lyr.reduce_histogram(job)
        us = 1e6 * (time.perf_counter() - t0)
    E = int(hist.shape[0])
    total = int(job.sum().item())
    return job, {"name": name, "E": E, "bytes": E * E * 4, "ranks": world,
                 "collective": "all_reduce sum int32" if world > 1 else "none (one rank)",
                 "allreduce_us": round(us, 1) if world > 1 else 0.0,
                 "total": total, "consistent": total == world * local_total}


def time_mlp_rows(O, buf, row_expert_of, weights, act, budget_s):
    """(rows timed, seconds per row) of the oracle's expert MLP on buffer
    rows spread evenly over all experts: a 4-row probe, then as many rows as
    fit the budget (at most all of them)."""
    R = buf.shape[0]

    def run(n):
        rows = np.linspace(0, R - 1, num=min(n, R)).astype(np.int64)
        t0 = time.perf_counter()
        O.expert_ffn_rows(buf[rows], row_expert_of(rows), *weights, act)
        return len(rows), time.perf_counter() - t0

    n, t = run(4)
    want = int(min(R, budget_s / max(t / n, 1e-9)))
    if want > n:
        n, t = run(want)
    return n, t / n


def workload_config(w, world):
    """The `config` object of both arms' JSON lines: the workload's name and
    shape, the batch over all ranks and how it is spread."""
    cfg = {"workload": w.name, "T": w.T, "d": w.d, "E": w.E}
    cfg.update({"k": w.k, "capacity_factor": w.capacity_factor} if w.routing == "topk" else {"C": w.C})
    if w.F:
        cfg.update({"F": w.F, "act": w.act})
    if w.F_shared:
        cfg["F_shared"] = w.F_shared
    if w.G and not w.F:
        cfg["G"] = w.G
    cfg.update({"global_batch": world * w.T, "parallelism": "independent replicas, one batch per GPU"})
    return cfg


def held_under_power_cap(elapsed_ms, clk):
    """True when a tensor-bound stage ran in the sustained regime: a timed
    region of a second or more, or a clock record whose median SM clock sat
    below 90 % of its maximum with the power cap among the reasons."""
    if elapsed_ms >= 1000.0:
        return True
    if not clk or not clk.get("sm_mhz") or not clk.get("sm_max_mhz"):
        return False
    return "sw_power_cap" in (clk.get("reasons") or []) and clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"]


def throughput(world, tokens_per_rank, steps, max_elapsed_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_elapsed_ms / 1e3)


def traffic_for(kernel_key):
    """Per-step DRAM bytes of a stage from the committed ncu summary, or None
    if missing or taken on another version of the kernel's source."""
    try:
        with open(TRAFFIC_FILE) as f:
            entry = json.load(f)[kernel_key]
        src = open(os.path.join(ROOT, entry["source"]), "rb").read()
        if entry.get("source_sha256") != hashlib.sha256(src).hexdigest():
            return None
        return entry.get("bytes_per_step")
    except (OSError, ValueError, KeyError):
        return None


def _cpu_name():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip() + " (%d cores visible)" % os.cpu_count()
    except OSError:
        pass
    return "unknown"


def _dev(a, device):
    import torch

    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def _pinned(a):
    import torch

    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
    return t.pin_memory()


# ----------------------------------------------------------- runners
class TopKRunner:
    """Top-k layers (with or without experts/shared expert) and the
    dispatch/combine sweep (identity experts, group-major rows)."""

    def __init__(self, w, rank, device):
        import torch

        from mixture_experts_routing_top_b200 import layer as Lyr, libmoe as M, workloads as W

        self.w, self.M = w, M
        wr = rank_batch(w, rank)
        self.logits_np, self.x_np = W.make_logits(wr), W.make_x(wr)
        self.weights_np = W.make_weights(w) if w.F else (None, None, None)
        self.shared_np = W.make_shared_weights(w)
        self.logits, self.x = _dev(self.logits_np, device), _dev(self.x_np, device)
        self.Wr_np = W.make_router_weights(w) if w.router else None       # logits from x on the device
        self.Wr = None if self.Wr_np is None else _dev(self.Wr_np, device)
        weights = tuple(_dev(a, device) for a in self.weights_np)
        shared = None if self.shared_np is None else tuple(_dev(a, device) for a in self.shared_np)
        self.goe = W.equal_groups(w.E, w.G) if w.G else None
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, dt, *weights, act=w.act,
                               norm_topk=w.norm_topk, shared_weights=shared,
                               group_of_expert=None if self.goe is None else _dev(self.goe, device),
                               G=w.G if self.goe is not None else 0, device=device, W_r=self.Wr)
        self.cosel = torch.zeros((w.E, w.E), dtype=torch.int32, device=device)
        route_in = self.Wr if w.router else self.logits
        self.resident_bytes = (sum(t.numel() * t.element_size() for t in weights if t is not None) +
                               route_in.numel() * route_in.element_size() + self.x.numel() * self.x.element_size())
        if w.router:
            self.stages = [("route", lambda: self.L.route_x(self.x))]
        else:
            self.stages = [("route", lambda: self.L.route(self.logits))]
        self.stages.append(("permute", lambda: self.L.dispatch(self.x)))
        if self.L.grouped:
            # send-once dispatcher with experts: group rows -> expert rows -> MLPs -> group rows
            self.stages.append(("local_permute", lambda: self.L.local_permute()))
        if w.F:
            self.stages.append(("ffn", self._ffn))
        if self.L.grouped:
            self.stages.append(("precombine", self._precombine))
        self.stages.append(("combine", self._combine))
        self.stages.append(("coselect", lambda: M.coselect(self.L.idx, w.E, into=self.cosel)))
        self._y = self._sh = None

    def _ffn(self):
        self._y = self.L.expert_mlps() if self.L.grouped else self.L.experts()
        self._sh = self.L.shared_expert(self.x)

    def _precombine(self):
        self._y = self.L.precombine(self._y)

    def _combine(self):
        y = self._y if self.w.F else self.L.perm["buffer"]
        self.L.combine(y, self._sh)

    def histogram(self):
        return "coselect", self.cosel

    def after_warmup(self):
        self.R = int(self.L.perm["offsets"][-1].item())
        self.dropped = int(self.L.perm["dropped"][0].item())
        self.R_e = int(self.L.perm_e["offsets"][-1].item()) if self.L.grouped else self.R

    def work(self):
        """Algorithmic bytes (memory stages) and FLOPs (expert MLPs) per step.
        With groups, R counts the (token, group) rows and R_e the expert rows."""
        w, R, R_e = self.w, self.R, self.R_e
        b = 2 if w.dtype == "bf16" else 4
        T, d, E, k = w.T, w.d, w.E, w.k
        shared = T * d * b if w.F_shared else 0
        route_bytes = (T * d * b + E * d * b if w.router else T * E * 4) + T * k * 8
        out = {"route": ("bytes", route_bytes),
               "permute": ("bytes", T * d * b + R * d * b + T * k * 8 + R * 4),
               "coselect": ("bytes", T * k * 4 + E * E * 4)}
        if self.L.grouped:
            out["permute"] = ("bytes", out["permute"][1] + T * k * 8 + R_e * 4)     # + the index-only permute
            out["local_permute"] = ("bytes", 2 * R_e * d * b + T * k * 8)
            out["precombine"] = ("bytes", R_e * d * b + R * d * b + T * k * 12)
            out["combine"] = ("bytes", R * d * b + T * d * b + T * k * 4 + shared)
        else:
            out["combine"] = ("bytes", R * d * b + T * d * b + T * k * 8 + shared)
        if w.F:
            f = 2.0 * R_e * d * w.F * (3 if w.act == "swiglu" else 2)
            if w.F_shared:
                f += 2.0 * T * d * w.F_shared * 3
            out["ffn"] = ("flops", f)
        return out

    def e2e_setup(self):
        import torch

        from mixture_experts_routing_top_b200 import layer as Lyr

        self.h_out = torch.empty(self.L.out.shape, dtype=self.L.out.dtype).pin_memory()
        if self.w.router:                      # the router runs on the device: x is the only input
            self.h_in = [_pinned(self.x_np)]
            self.pipe = Lyr.HostPipeline(lambda x, out: self.L.forward(None, x, out=out), [self.x], self.L.out)
        else:
            self.h_in = [_pinned(self.logits_np), _pinned(self.x_np)]
            self.pipe = Lyr.HostPipeline(lambda lg, x, out: self.L.forward(lg, x, out=out), [self.logits, self.x],
                                         self.L.out)

    def e2e_run(self, n):
        self.pipe.run([self.h_in] * n, [self.h_out] * n)

    def e2e_bytes(self):
        return (sum(h.numel() * h.element_size() for h in self.h_in), self.h_out.numel() * self.h_out.element_size())

    def extra(self):
        out = {"rows": self.R, "dropped": self.dropped}
        if self.L.grouped:
            out.update(expert_rows=self.R_e, G=self.w.G, rows_removed=round(1.0 - self.R / max(self.R_e, 1), 4))
        if self.w.cluster_bias:
            out["correlated_placement"] = self.placement_stat()
        return out

    def placement_stat(self):
        """Correlated placement on this batch: the expert ids are scrambled
        by a fixed seeded permutation (so that contiguous groups no longer
        coincide with the routing clusters), the co-selection counts feed
        moe_place_experts, and the group-major row counts with the placed
        and with contiguous groups are compared (one group per cluster)."""
        import torch

        M, w = self.M, self.w
        dev = self.L.idx.device
        G = w.n_clusters
        perm = torch.from_numpy(np.random.default_rng(7).permutation(w.E).astype(np.int32)).to(dev)
        scr = perm[self.L.idx.long()].contiguous()
        cosel = M.coselect(scr, w.E)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        goe = M.place_experts(cosel, G)
        b.record()
        torch.cuda.synchronize()
        contig = torch.arange(w.E, dtype=torch.int32, device=dev) // (w.E // G)
        rows = {}
        for name, g in (("placed", goe), ("contiguous", contig)):
            p = M.permute(None, scr, w.E, 0.0, g, G)
            rows[name] = int(p["offsets"][-1].item())
        return {"G": G, "rows_placed": rows["placed"], "rows_contiguous": rows["contiguous"],
                "rows_removed": round(1.0 - rows["placed"] / rows["contiguous"], 4),
                "assignments": w.T * w.k, "place_us": round(1e3 * a.elapsed_time(b), 1),
                "inputs": "this batch's routing, expert ids scrambled (seed 7)"}

    def cpu_baseline(self, budget_s):
        """The oracle as it stands, single-threaded, on a bounded sample."""
        from oracle import oracle as O
        from mixture_experts_routing_top_b200 import synth

        w = self.w
        Ts = min(w.T, 8192)                    # token sample for the routing/permute/combine part
        logits, x = self.logits_np[:Ts], self.x_np[:Ts]
        grouped = self.L.grouped
        t0 = time.perf_counter()
        if w.router:
            logits = O.router_logits(x, self.Wr_np).astype(np.float32)
        idx, gate = O.route_topk(logits, w.k, w.norm_topk)
        cap = O.capacity(w.capacity_factor, Ts, w.k, w.E)
        p = O.permute(idx, w.E, cap, self.goe)
        buf = O.gather_rows(x, p["row_token"])
        pe = p
        if grouped:                            # the group's local permutation to expert rows
            pe = O.permute(idx, w.E, cap)
            buf = O.copy_slot_rows(buf, p["row_map"], pe["row_map"], np.empty((pe["R"], w.d), buf.dtype))
        t_rp = time.perf_counter() - t0
        R = pe["R"]
        Y = buf if not w.F else (synth.normal_bf16(99, 1, (R, w.d)) if w.dtype == "bf16"
                                 else synth.normal_f32(99, 1, (R, w.d)))
        t0 = time.perf_counter()
        if grouped:
            P = O.group_precombine(Y, pe["row_map"], p["row_map"], gate, p["R"])
            O.unpermute_groups(O.to_dtype_bits(P, Y), p["row_map"])
        else:
            O.unpermute(Y, p["row_map"], gate)
        t_comb = time.perf_counter() - t0
        per_token = (t_rp + t_comb) / Ts
        sample = "%sroute, capacity, permute, row copy and combine on %d of %d tokens (%.2f s)" % (
            "router gate, " if w.router else "", Ts, w.T, t_rp + t_comb)
        if w.F:
            row_expert = lambda rows: (np.searchsorted(pe["offsets"], rows, side="right") - 1).astype(np.int32)
            n, t_row = time_mlp_rows(O, buf, row_expert, self.weights_np, w.act, budget_s)
            per_token += t_row * R / Ts
            sample += "; expert MLP on %d of %d rows, %.4f s per row (%.1f s), extrapolated to all rows" % (
                n, R, t_row, n * t_row)
            if self.shared_np is not None:
                t0 = time.perf_counter()
                O.expert_ffn_rows(x[:2], np.zeros(2, np.int32), *self.shared_np, "swiglu")
                per_token += (time.perf_counter() - t0) / 2
                sample += "; shared expert on 2 tokens"
        return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample,
                "cpu": _cpu_name()}


class ExpertChoiceRunner:
    """Expert-choice layer plus the two top-1 routings and the layer-to-layer
    transition histogram."""

    def __init__(self, w, rank, device):
        import torch

        from mixture_experts_routing_top_b200 import layer as Lyr, libmoe as M, workloads as W

        self.w, self.M = w, M
        wr = rank_batch(w, rank)
        self.logits_np, self.x_np = W.make_logits(wr), W.make_x(wr)
        self.logits2_np = W.make_layer2_logits(wr, self.logits_np)
        self.weights_np = W.make_weights(w)
        self.logits, self.logits2 = _dev(self.logits_np, device), _dev(self.logits2_np, device)
        self.x = _dev(self.x_np, device)
        W1, W3, W2 = (_dev(a, device) for a in self.weights_np)
        self.L = Lyr.ExpertChoiceLayer(w.T, w.d, w.E, w.C, w.F, torch.bfloat16, W1, W3, W2, w.act, device=device)
        self.top1 = [torch.empty((w.T, 1), dtype=torch.int32, device=device) for _ in range(2)]
        self.g1 = [torch.empty((w.T, 1), dtype=torch.float32, device=device) for _ in range(2)]
        self.trans = torch.zeros((w.E, w.E), dtype=torch.int32, device=device)
        self.resident_bytes = (sum(t.numel() * t.element_size() for t in (W1, W2)) + 2 * self.logits.numel() * 4 +
                               self.x.numel() * 2)
        L = self.L
        self.stages = [("route_ec", lambda: M.route_ec(self.logits, w.C, workspace=L.route_ws, out=L.routing)),
                       ("dispatch", lambda: M.gather_rows(self.x, L.routing[2], L.routing[3], L.R, buffer=L.buffer)),
                       ("ffn", lambda: M.expert_ffn(L.buffer, L.offsets, L.W1, L.W3, L.W2, w.act, y=L.y,
                                                    workspace=L.ffn_ws)),
                       ("combine", lambda: M.unpermute_ec(L.y, L.routing[2], L.routing[3], L.routing[1].view(-1),
                                                          out=L.out)),
                       ("transition", self._transition)]

    def _transition(self):
        M = self.M
        M.route_topk(self.logits, 1, False, self.top1[0], self.g1[0])
        M.route_topk(self.logits2, 1, False, self.top1[1], self.g1[1])
        M.transition(self.top1[0], self.top1[1], self.w.E, into=self.trans)

    def histogram(self):
        return "transition", self.trans

    def after_warmup(self):
        tp = self.L.routing[2]
        self.chosen = int((tp[1:] > tp[:-1]).sum().item())

    def work(self):
        w = self.w
        T, d, E, C = w.T, w.d, w.E, w.C
        R = E * C
        return {"route_ec": ("bytes", T * E * 4 + R * 12 + (T + 1) * 4),
                "dispatch": ("bytes", self.chosen * d * 2 + R * d * 2 + (T + 1 + R) * 4),
                "ffn": ("flops", 2.0 * R * d * w.F * (3 if w.act == "swiglu" else 2)),
                "combine": ("bytes", R * d * 2 + T * d * 2 + (T + 1 + 2 * R) * 4),
                "transition": ("bytes", 2 * T * E * 4 + 2 * T * 8)}

    def e2e_setup(self):
        import torch

        from mixture_experts_routing_top_b200 import layer as Lyr

        self.h_in = [_pinned(self.logits_np), _pinned(self.x_np)]
        self.h_out = torch.empty(self.L.out.shape, dtype=self.L.out.dtype).pin_memory()
        self.pipe = Lyr.HostPipeline(lambda lg, x, out: self.L.forward(lg, x, out=out), [self.logits, self.x],
                                     self.L.out)

    def e2e_run(self, n):
        self.pipe.run([self.h_in] * n, [self.h_out] * n)

    def e2e_bytes(self):
        return (sum(h.numel() * h.element_size() for h in self.h_in), self.h_out.numel() * self.h_out.element_size())

    def extra(self):
        return {"rows": self.w.E * self.w.C, "tokens_chosen": self.chosen, "token_shuffling": self.shuffle_stat()}

    def shuffle_stat(self, G=8):
        """Share of layer-2 assignments served in the token's home group of
        G contiguous expert groups: sequence-sharded homes vs homes predicted
        from this batch's layer-1 -> layer-2 transition counts."""
        import torch

        M, w = self.M, self.w
        goe = torch.arange(w.E, dtype=torch.int32, device=self.x.device) // (w.E // G)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        home = M.predict_home(self.top1[0], M.group_affinity(self.trans, goe, G))
        b.record()
        before = int(M.count_local(self.top1[1], goe, G)[0].item())
        after = int(M.count_local(self.top1[1], goe, G, home)[0].item())
        torch.cuda.synchronize()
        return {"G": G, "local_before": round(before / w.T, 4), "local_after": round(after / w.T, 4),
                "predict_us": round(1e3 * a.elapsed_time(b), 1),
                "note": "transition counts accumulated over all timed steps (identical batches)"}

    def cpu_baseline(self, budget_s):
        from oracle import oracle as O
        from mixture_experts_routing_top_b200 import synth

        w = self.w
        t0 = time.perf_counter()
        ec_token, ec_gate, tok_ptr, tok_row = O.route_ec(self.logits_np, w.C)
        buf = O.gather_rows(self.x_np, ec_token.reshape(-1))
        R = w.E * w.C
        Y = synth.normal_bf16(99, 1, (R, w.d))
        O.unpermute_ec(Y, tok_ptr, tok_row, ec_gate)
        a, _ = O.route_topk(self.logits_np, 1)
        b, _ = O.route_topk(self.logits2_np, 1)
        O.transition(a, b, w.E)
        t_rest = time.perf_counter() - t0
        n, t_row = time_mlp_rows(O, buf, lambda rows: (rows // w.C).astype(np.int32), self.weights_np, w.act,
                                 budget_s)
        per_token = t_rest / w.T + t_row * R / w.T
        return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": "expert-choice routing, dispatch, combine and both top-1 routings + transitions on all "
                          "%d tokens (%.2f s); expert MLP on %d of %d rows, %.4f s per row (%.1f s), extrapolated"
                          % (w.T, t_rest, n, R, t_row, n * t_row), "cpu": _cpu_name()}


class RoutingRunner:
    """Routing and its statistic alone (top-k, or the fused router with
    router=1, then co-selection) at a workload's shape: the routing step
    measured where its inputs are large enough for HBM to matter."""

    def __init__(self, w, rank, device):
        import torch

        from mixture_experts_routing_top_b200 import libmoe as M, workloads as W

        self.w, self.M = w, M
        wr = rank_batch(w, rank)
        self.idx = torch.empty((w.T, w.k), dtype=torch.int32, device=device)
        self.gate = torch.empty((w.T, w.k), dtype=torch.float32, device=device)
        self.cosel = torch.zeros((w.E, w.E), dtype=torch.int32, device=device)
        if w.router:
            self.in_np = [W.make_x(wr)]
            self.Wr_np = W.make_router_weights(w)
            self.Wr = _dev(self.Wr_np, device)
            route = lambda inp: M.router_topk(inp, self.Wr, w.k, w.norm_topk, self.idx, self.gate)
        else:
            self.in_np = [W.make_logits(wr)]
            route = lambda inp: M.route_topk(inp, w.k, w.norm_topk, self.idx, self.gate)
        self.inp = _dev(self.in_np[0], device)
        self.route = route
        self.resident_bytes = self.inp.numel() * self.inp.element_size()
        self.stages = [("route", lambda: route(self.inp)),
                       ("coselect", lambda: M.coselect(self.idx, w.E, into=self.cosel))]

    def histogram(self):
        return "coselect", self.cosel

    def after_warmup(self):
        pass

    def work(self):
        w = self.w
        T, E, k = w.T, w.E, w.k
        b = 2 if w.dtype == "bf16" else 4
        route_in = T * w.d * b + E * w.d * b if w.router else T * E * 4
        return {"route": ("bytes", route_in + T * k * 8), "coselect": ("bytes", T * k * 4 + E * E * 4)}

    def e2e_setup(self):
        import torch

        self.h_in = _pinned(self.in_np[0])
        self.h_out = [torch.empty(self.idx.shape, dtype=torch.int32).pin_memory(),
                      torch.empty(self.gate.shape, dtype=torch.float32).pin_memory()]
        self.d_in = [self.inp, torch.empty_like(self.inp)]

    def e2e_run(self, n):
        for i in range(n):
            d = self.d_in[i & 1]
            d.copy_(self.h_in, non_blocking=True)
            self.route(d)
            self.h_out[0].copy_(self.idx, non_blocking=True)
            self.h_out[1].copy_(self.gate, non_blocking=True)

    def e2e_bytes(self):
        return self.h_in.numel() * self.h_in.element_size(), sum(h.numel() * h.element_size() for h in self.h_out)

    def extra(self):
        return {"routing_only": True}

    def cpu_baseline(self, budget_s):
        from oracle import oracle as O

        w = self.w

        def run(n):
            t0 = time.perf_counter()
            if w.router:
                lg = O.router_logits(self.in_np[0][:n], self.Wr_np).astype(np.float32)
            else:
                lg = self.in_np[0][:n]
            idx, _ = O.route_topk(lg, w.k, w.norm_topk)
            O.coselect(idx, w.E)
            return time.perf_counter() - t0

        Ts = min(w.T, 256)
        t = run(Ts)
        want = int(min(w.T, budget_s * Ts / max(t, 1e-9)))       # as many tokens as fit the budget
        if want > Ts:
            Ts = want
            t = run(Ts)
        return {"value": Ts / t, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": "routing and co-selection on %d of %d tokens (%.2f s)" % (Ts, w.T, t), "cpu": _cpu_name()}


def make_runner(w, rank, device, routing_only=False):
    if routing_only:
        if kind_of(w) == "ec":
            raise SystemExit("--routing-only times top-k routing; the expert-choice workload routes inside its step")
        return RoutingRunner(w, rank, device)
    return ExpertChoiceRunner(w, rank, device) if kind_of(w) == "ec" else TopKRunner(w, rank, device)


# ------------------------------------------------------------ libmoe arm
def run_libmoe(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from mixture_experts_routing_top_b200 import build as B, libmoe as M

    B.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    run = make_runner(w, rank, device, args.routing_only)
    stream = torch.cuda.current_stream(device)
    names = [n for n, _ in run.stages]
    ns = len(names)
    # inputs smaller than L2: flush it between timed steps (outside the events)
    flush = None
    if run.resident_bytes < 2 * L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    def step(ev=None):
        for j, (_, fn) in enumerate(run.stages):
            if ev:
                ev[j].record(stream)
            fn()
        if ev:
            ev[ns].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if M.device_error() != 0:
        raise RuntimeError("device fault word set during warm-up")
    run.after_warmup()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ns + 1)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph = None
    if args.graph:
        # stage times from an eager pass, then the whole step captured once and replayed
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
        stage_ms_eager = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(names)}
        n_cap = M.kernel_launches()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        per_step = M.kernel_launches() - n_cap
        graph.replay()
        torch.cuda.synchronize()
    clocks = Clocks()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = M.kernel_launches()
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
        if graph is None:
            step(evs[i])
        else:
            evs[i][0].record(stream)
            graph.replay()
            evs[i][ns].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    # graph replays launch their kernels without the host: count them from the capture
    launches = M.kernel_launches() - n0 if graph is None else per_step * args.steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop() if rank == 0 else None
    if flush is None:
        elapsed_ms = t_start.elapsed_time(t_end)
    else:
        elapsed_ms = sum(e[0].elapsed_time(e[ns]) for e in evs)
    if graph is None:
        stage_ms = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(names)}
    else:
        stage_ms = stage_ms_eager
    if M.device_error() != 0:
        raise RuntimeError("device fault word set during the timed steps")
    elapsed_ms, launches = reduce_over_ranks(elapsed_ms, launches, device)
    _, hist_rec = job_histogram(*run.histogram(), world, device)

    # end to end through the public API: pinned host inputs -> layer -> host output
    e2e = None
    if args.e2e_steps > 0:
        run.e2e_setup()
        run.e2e_run(3)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run.e2e_run(args.e2e_steps)               # each step: its inputs in, the layer, its output out
        b.record(stream)
        torch.cuda.synchronize()
        e_ms, _ = reduce_over_ranks(a.elapsed_time(b), 0, device)
        hb, db = run.e2e_bytes()
        e2e = {"value": round(throughput(world, w.T, args.e2e_steps, e_ms), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db}

    if rank != 0:
        return None
    pk, pk_kind = peaks()
    work = run.work()
    report = {}
    for n in names:
        kind, amount = work[n]
        ms = stage_ms[n]
        r = {"ms": round(ms, 4)}
        if kind == "bytes":
            gbs = amount / (ms / 1e3) / 1e9
            r.update({"GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 3), "bytes": amount})
        else:
            tf = amount / (ms / 1e3) / 1e12
            r.update({"TFLOP/s": round(tf, 1), "flops": amount,
                      "frac_burst": round(tf / pk["bf16_tflops"], 3)})
        report[n] = r
    dom = max(names, key=lambda n: stage_ms[n])
    kind, amount = work[dom]
    if kind == "flops":
        # The stage runs inside a step of a few ms.  In a timed region of well under a second the burst
        # figure (cuBLAS timed alone) is its peak; in a region of a second or more, or once the power cap
        # has pulled the SM clock well below its maximum, the seconds-long sustained figure is.  The
        # other fraction is kept beside it.
        sustained = held_under_power_cap(elapsed_ms, clk) and "bf16_tflops_sustained" in pk
        peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
        ach = report[dom]["TFLOP/s"]
        roof = {"bound": "tensor", "stage": dom, "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": round(ach / peak, 4),
                "peak_kind": pk_kind + (" sustained bf16 (cuBLAS held under the power cap)" if sustained
                                        else " burst bf16 (cuBLAS timed alone)")}
        if sustained:
            roof["frac_burst"] = round(ach / pk["bf16_tflops"], 4)
        elif "bf16_tflops_sustained" in pk:
            roof["frac_sustained"] = round(ach / pk["bf16_tflops_sustained"], 4)
    else:
        peak = pk["hbm_gbs"]
        ach = report[dom]["GB/s"]
        roof = {"bound": "hbm", "stage": dom, "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "peak_kind": pk_kind + " HBM copy"}
    roof["traffic"] = traffic_for("%s/%s" % (w.name, dom))
    value = throughput(world, w.T, args.steps, elapsed_ms)
    cfg = workload_config(w, world)
    if graph is not None:
        cfg["launch"] = "step replayed as one CUDA graph; stage times from an eager pass"
    cfg["l2"] = ("flushed between timed steps (256 MB write outside the events)" if flush is not None else
                 "inputs larger than L2: %.2f GB resident inputs read every step" % (run.resident_bytes / 1e9))
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic: seeded normals (logits, activations) and random-init expert weights",
        "config": cfg, "roofline": roof, "stages": report, "gpu_launches": launches, "clocks": clk,
    }
    res.update(run.extra())
    res["job_histogram"] = hist_rec
    if e2e:
        res["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = run.cpu_baseline(args.cpu_seconds)
    return res


# --------------------------------------------------------- reference arm
def run_reference(args, w, world=1):
    """The oracle as it stands (single-threaded C) on the host cores.  Each
    step: routing, capacity, permutation (with the row copy) and the combine
    over a token sample, plus the expert MLP of one buffer row (rotating);
    throughput is extrapolated per token from those parts."""
    from oracle import oracle as O
    from mixture_experts_routing_top_b200 import synth, workloads as W

    Ts = min(w.T, 8192)
    logits, x = W.make_logits(w)[:Ts], W.make_x(w)[:Ts]
    is_ec = kind_of(w) == "ec"
    Wt = W.make_weights(w) if w.F else None
    Ws = W.make_shared_weights(w)
    goe = W.equal_groups(w.E, w.G) if w.G else None
    grouped = bool(w.G and w.F)                 # send-once dispatcher with experts
    Wr = W.make_router_weights(w) if w.router else None
    if is_ec:
        C = max(1, w.C * Ts // w.T)
        R_probe = w.E * C
    else:
        lg0 = O.router_logits(x, Wr).astype(np.float32) if Wr is not None else logits
        R_probe = O.permute(O.route_topk(lg0, w.k, w.norm_topk)[0], w.E,
                            O.capacity(w.capacity_factor, Ts, w.k, w.E), None if grouped else goe)["R"]
    Y = synth.normal_bf16(99, 1, (R_probe, w.d)) if w.dtype == "bf16" else synth.normal_f32(99, 1, (R_probe, w.d))

    routing_only = getattr(args, "routing_only", False) and not is_ec

    def step(i):
        t0 = time.perf_counter()
        if routing_only:                       # routing and co-selection alone
            lg = O.router_logits(x, Wr).astype(np.float32) if Wr is not None else logits
            idx, _ = O.route_topk(lg, w.k, w.norm_topk)
            O.coselect(idx, w.E)
            t1 = time.perf_counter()
            return (t1 - t0) / Ts, t1 - t0
        if is_ec:
            ec_token, ec_gate, tok_ptr, tok_row = O.route_ec(logits, C)
            buf = O.gather_rows(x, ec_token.reshape(-1))
            O.unpermute_ec(Y, tok_ptr, tok_row, ec_gate)
            R = w.E * C
            row_e = lambda r: r // C
        else:
            lg = O.router_logits(x, Wr).astype(np.float32) if Wr is not None else logits
            idx, gate = O.route_topk(lg, w.k, w.norm_topk)
            cap = O.capacity(w.capacity_factor, Ts, w.k, w.E)
            p = O.permute(idx, w.E, cap, goe)
            buf = O.gather_rows(x, p["row_token"])
            pe = p
            if grouped:
                pe = O.permute(idx, w.E, cap)
                buf = O.copy_slot_rows(buf, p["row_map"], pe["row_map"], np.empty((pe["R"], w.d), buf.dtype))
                P = O.group_precombine(Y, pe["row_map"], p["row_map"], gate, p["R"])
                O.unpermute_groups(O.to_dtype_bits(P, Y), p["row_map"])
            else:
                O.unpermute(Y if w.F else buf, p["row_map"], gate)
            R = pe["R"]
            row_e = lambda r: int(np.searchsorted(pe["offsets"], r, side="right") - 1)
        t1 = time.perf_counter()
        if w.F:
            r = (i * 7919) % R
            O.expert_ffn_rows(buf[r:r + 1], np.array([row_e(r)], np.int32), *Wt, w.act)
            if Ws is not None:
                O.expert_ffn_rows(x[:1], np.zeros(1, np.int32), *Ws, "swiglu")
        t2 = time.perf_counter()
        return (t1 - t0) / Ts + (t2 - t1) * (R / Ts if w.F else 0.0), t2 - t0

    for i in range(args.warmup):
        step(i)
    per_token, wall = [], []
    for i in range(args.steps):
        pt, wt = step(args.warmup + i)
        per_token.append(pt)
        wall.append(wt)
    value = len(per_token) / sum(per_token)
    sample = ("per step: routing, capacity, permutation, row copy and combine over %d of %d tokens%s, "
              "extrapolated per token" % (Ts, w.T, ", plus the expert MLP of one buffer row" if w.F else ""))
    if routing_only:
        sample = "per step: routing and co-selection over %d of %d tokens, extrapolated per token" % (Ts, w.T)
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(wall), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: seeded normals and random-init expert weights",
            "config": dict(workload_config(w, world), l2="host run of the oracle: no GPU cache involved"),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": sample, "cpu": _cpu_name()},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    w = workload_from_args(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.gpus > 1 and world == 1:
        raise SystemExit("--gpus %d needs one process per GPU: launch with python -m torch.distributed.run "
                         "--nproc-per-node %d" % (args.gpus, args.gpus))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w, world)), flush=True)
        return
    if world > 1:
        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_libmoe(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
