#!/usr/bin/env python
"""Benchmark of one MoE layer step on B200 through libmoe.

A step is one pass of the whole hot path over one batch: top-k routing,
capacity-bounded permutation, the grouped expert MLPs (tcgen05 GEMMs), the
gate-weighted combine and the co-selection histogram.  Default workload:
the Mixtral-shaped top-2 layer (T=8192 tokens, d=4096, E=8 experts, SwiGLU
4096->14336->4096, capacity factor 1.25, bf16 with fp32 accumulation).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libmoe|reference]

One JSON line on rank 0.  Under torchrun each rank runs its own batch (its
own seed) against the same expert weights: independent replicas, no
collective on the data path, weak scaling; the timed region is bracketed by
a barrier and a device synchronise on both sides and the slowest rank's
time is taken.  `--impl reference` times the CPU oracle (single-threaded C)
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
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ffn_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="libmoe", choices=["libmoe", "reference"])
    ap.add_argument("--workload", default="mixtral_top2_bf16")
    ap.add_argument("--cpu-rows", type=int, default=24, help="expert-MLP rows in the CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field (e.g. T=4096) - for smaller profiling cases, not bench lines")
    return ap.parse_args()


def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


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

    def stop(self, gpu_index=None):
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
                if len(parts) < 9:
                    continue
                if gpu_index is not None and parts[0] != str(gpu_index):
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


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


def throughput(world, tokens_per_rank, steps, max_elapsed_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_elapsed_ms / 1e3)


# ------------------------------------------------------------ libmoe arm
def make_problem(w, rank, device):
    import torch

    from mixture_experts_routing_top_b200 import workloads as W

    wr = rank_batch(w, rank)                   # this rank's batch
    logits = W.make_logits(wr)
    x = W.make_x(wr)
    Wt = W.make_weights(w)                     # one model on every rank
    Ws = W.make_shared_weights(w)

    def dev(a):
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    return dict(logits_np=logits, x_np=x, weights_np=Wt, shared_np=Ws, logits=dev(logits), x=dev(x),
                weights=tuple(dev(a) for a in Wt), shared=None if Ws is None else tuple(dev(a) for a in Ws))


def stage_bytes(w, R, b):
    """Algorithmic bytes per launch of the memory-bound stages (kept rows only)."""
    T, d, E, k = w.T, w.d, w.E, w.k
    return {
        "route": T * E * 4 + T * k * 8,
        "permute": T * d * b + R * d * b + T * k * (4 + 4) + R * 4,
        "combine": R * d * b + T * d * b + T * k * (4 + 4) + (T * d * b if w.F_shared else 0),
        "coselect": T * k * 4 + E * E * 4,
    }


def ffn_flops(w, R):
    mats = 3 if w.act == "swiglu" else 2
    f = 2.0 * R * w.d * w.F * mats
    if w.F_shared:
        f += 2.0 * w.T * w.d * w.F_shared * 3
    return f


def traffic_of_ffn():
    """Per-launch DRAM bytes of the FFN stage from the committed ncu summary,
    or None if missing or taken on another version of the kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        src = open(os.path.join(ROOT, "mixture_experts_routing_top_b200", "csrc", "ffn.cu"), "rb").read()
        if t.get("source_sha256") != hashlib.sha256(src).hexdigest():
            return None
        return t.get("bytes_per_step")
    except (OSError, ValueError):
        return None


def cpu_baseline(w, prob, n_rows):
    """The oracle as it stands, single-threaded, on a bounded sample."""
    from oracle import oracle as O
    from mixture_experts_routing_top_b200 import synth

    logits, x = prob["logits_np"], prob["x_np"]
    t0 = time.perf_counter()
    idx, gate = O.route_topk(logits, w.k, w.norm_topk)
    p = O.permute(idx, w.E, O.capacity(w.capacity_factor, w.T, w.k, w.E))
    buf = O.gather_rows(x, p["row_token"])
    t_rp = time.perf_counter() - t0
    R = p["R"]
    rows = np.linspace(0, R - 1, num=min(n_rows, R)).astype(np.int64)
    row_e = np.searchsorted(p["offsets"], rows, side="right").astype(np.int32) - 1
    W1, W3, W2 = prob["weights_np"]
    t0 = time.perf_counter()
    O.expert_ffn_rows(buf[rows], row_e, W1, W3, W2, w.act)
    t_row = (time.perf_counter() - t0) / len(rows)
    Y = synth.normal_bf16(99, 1, (R, w.d)) if w.dtype == "bf16" else synth.normal_f32(99, 1, (R, w.d))
    t0 = time.perf_counter()
    O.unpermute(Y, p["row_map"], gate)
    t_comb = time.perf_counter() - t0
    t_shared_row = 0.0
    if prob["shared_np"] is not None:
        sW1, sW3, sW2 = prob["shared_np"]
        t0 = time.perf_counter()
        O.expert_ffn_rows(x[:2], np.zeros(2, np.int32), sW1, sW3, sW2, "swiglu")
        t_shared_row = (time.perf_counter() - t0) / 2
    per_token = (t_rp + t_comb) / w.T + t_row * R / w.T + t_shared_row
    return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "route, capacity, permute and combine on all %d tokens (%.2f s); expert MLP on %d of %d "
                      "rows, %.3f s per row, extrapolated to all rows" % (w.T, t_rp + t_comb, len(rows), R, t_row),
            "cpu": _cpu_name()}


def _cpu_name():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip() + " (%d cores visible)" % os.cpu_count()
    except OSError:
        pass
    return "unknown"


def run_libmoe(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from mixture_experts_routing_top_b200 import build as B, layer as Lyr, libmoe as M

    B.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    prob = make_problem(w, rank, device)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    L = Lyr.TopKLayer(w.T, w.d, w.E, w.k, w.F, w.capacity_factor, dt, *prob["weights"], act=w.act,
                      norm_topk=w.norm_topk, shared_weights=prob["shared"], device=device)
    cosel = torch.zeros((w.E, w.E), dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    stages = ["route", "permute", "ffn", "shared", "combine", "coselect"]

    def step(ev=None):
        if ev: ev[0].record(stream)
        L.route(prob["logits"])
        if ev: ev[1].record(stream)
        L.dispatch(prob["x"])
        if ev: ev[2].record(stream)
        y = L.experts()
        if ev: ev[3].record(stream)
        sh = L.shared_expert(prob["x"])
        if ev: ev[4].record(stream)
        L.combine(y, sh)
        if ev: ev[5].record(stream)
        M.coselect(L.idx, w.E, into=cosel)
        if ev: ev[6].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if M.device_error() != 0:
        raise RuntimeError("device fault word set during warm-up")
    R = int(L.perm["offsets"][-1].item())
    dropped = int(L.perm["dropped"][0].item())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    launches = M.kernel_launches() - n0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop() if rank == 0 else None
    elapsed_ms = t_start.elapsed_time(t_end)
    stage_ms = {s: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, s in enumerate(stages)}
    if M.device_error() != 0:
        raise RuntimeError("device fault word set during the timed steps")

    # max over ranks (slowest rank), total launches
    elapsed_ms, launches = reduce_over_ranks(elapsed_ms, launches, device)

    # end to end through the public API: pinned host inputs -> layer -> host output
    e2e = None
    if args.e2e_steps > 0:
        lg_h = torch.from_numpy(prob["logits_np"]).pin_memory()
        xn = prob["x_np"]
        x_h = (torch.from_numpy(xn.view(np.int16)).view(torch.bfloat16) if xn.dtype == np.uint16
               else torch.from_numpy(xn)).pin_memory()
        out_h = torch.empty(L.out.shape, dtype=L.out.dtype).pin_memory()
        lg_d, x_d = torch.empty_like(prob["logits"]), torch.empty_like(prob["x"])

        def e2e_step():
            lg_d.copy_(lg_h, non_blocking=True)
            x_d.copy_(x_h, non_blocking=True)
            out = L.forward(lg_d, x_d)
            out_h.copy_(out, non_blocking=True)

        for _ in range(3):
            e2e_step()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms, _ = reduce_over_ranks(a.elapsed_time(b), 0, device)
        e2e = {"value": throughput(world, w.T, args.e2e_steps, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": lg_h.numel() * 4 + x_h.numel() * x_h.element_size(),
               "d2h_bytes_per_step": out_h.numel() * out_h.element_size()}

    if rank != 0:
        return None
    pk, pk_kind = peaks()
    b = 2 if w.dtype == "bf16" else 4
    sb = stage_bytes(w, R, b)
    flops = ffn_flops(w, R)
    ffn_ms = stage_ms["ffn"] + stage_ms["shared"]
    achieved = flops / (ffn_ms / 1e3) / 1e12
    peak_s = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    stage_report = {
        s: {"ms": round(stage_ms[s], 4),
            **({"GB/s": round(sb[s] / (stage_ms[s] / 1e3) / 1e9, 1),
                "frac_hbm": round(sb[s] / (stage_ms[s] / 1e3) / 1e9 / pk["hbm_gbs"], 3)} if s in sb else {})}
        for s in stages}
    stage_report["ffn"].update({"TFLOP/s": round(achieved, 1), "flops": flops,
                                "frac_burst": round(achieved / pk["bf16_tflops"], 3)})
    value = throughput(world, w.T, args.steps, elapsed_ms)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic: seeded normals (logits, activations) and random-init expert weights",
        "config": {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "F": w.F, "F_shared": w.F_shared,
                   "capacity_factor": w.capacity_factor, "act": w.act, "global_batch": world * w.T,
                   "parallelism": "independent replicas, one batch per GPU",
                   "l2": "inputs larger than L2: %.2f GB of expert weights read every step" %
                         (sum(t.numel() * t.element_size() for t in prob["weights"] if t is not None) / 1e9)},
        "roofline": {"bound": "tensor", "kernel": "expert MLP (2 tcgen05 grouped-GEMM launches)",
                     "achieved": round(achieved, 1), "peak": peak_s, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_s, 4), "peak_kind": pk_kind + " sustained bf16 (cuBLAS)",
                     "traffic": traffic_of_ffn()},
        "stages": stage_report,
        "rows": R, "dropped": dropped,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if e2e:
        res["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, prob, args.cpu_rows)
    return res


# --------------------------------------------------------- reference arm
def run_reference(args, w):
    """The oracle as it stands (single-threaded C) on the host cores.  Each
    step: routing, capacity, permutation (with the row copy) and the combine
    over all T tokens, plus the expert MLP of one buffer row (rotating);
    throughput is extrapolated per token from those parts."""
    from oracle import oracle as O
    from mixture_experts_routing_top_b200 import synth, workloads as W

    logits, x = W.make_logits(w), W.make_x(w)
    W1, W3, W2 = W.make_weights(w)
    Ws = W.make_shared_weights(w)
    R_probe = O.permute(O.route_topk(logits, w.k, w.norm_topk)[0], w.E,
                        O.capacity(w.capacity_factor, w.T, w.k, w.E))["R"]
    Y = synth.normal_bf16(99, 1, (R_probe, w.d)) if w.dtype == "bf16" else synth.normal_f32(99, 1, (R_probe, w.d))

    def step(i):
        t0 = time.perf_counter()
        idx, gate = O.route_topk(logits, w.k, w.norm_topk)
        p = O.permute(idx, w.E, O.capacity(w.capacity_factor, w.T, w.k, w.E))
        buf = O.gather_rows(x, p["row_token"])
        O.unpermute(Y, p["row_map"], gate)
        t1 = time.perf_counter()
        r = (i * 7919) % p["R"]
        e = int(np.searchsorted(p["offsets"], r, side="right") - 1)
        O.expert_ffn_rows(buf[r:r + 1], np.array([e], np.int32), W1, W3, W2, w.act)
        if Ws is not None:
            O.expert_ffn_rows(x[:1], np.zeros(1, np.int32), *Ws, "swiglu")
        t2 = time.perf_counter()
        shared_t = 0.0
        return (t1 - t0) / w.T + (t2 - t1) * p["R"] / w.T, t2 - t0, shared_t

    for i in range(args.warmup):
        step(i)
    per_token, wall = [], []
    for i in range(args.steps):
        pt, wt, _ = step(args.warmup + i)
        per_token.append(pt)
        wall.append(wt)
    value = len(per_token) / sum(per_token)
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(wall), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: seeded normals and random-init expert weights",
            "config": {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "F": w.F,
                       "capacity_factor": w.capacity_factor},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": "per step: route, capacity, permute, row copy and combine over all %d "
                                       "tokens, expert MLP of one buffer row, extrapolated per token" % w.T,
                             "cpu": _cpu_name()},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    from mixture_experts_routing_top_b200 import workloads as W

    w = W.BY_NAME[args.workload]
    for kv in args.set:
        key, val = kv.split("=", 1)
        cur = getattr(w, key)
        w = w.with_(**{key: type(cur)(val)})
    if args.set:
        w = w.with_(name=w.name + "[" + ",".join(args.set) + "]")
    if w.routing != "topk":
        raise SystemExit("bench.py times top-k layers; %s is measured by its tests" % w.name)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
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
