#!/usr/bin/env python
"""Benchmark of the dynamic-hash embedding step (RecIS Embedding Engine hot path).

One step = recis_feature_hash + recis_lookup_pooled + recis_backward_update
over one batch of the 26-feature one-hot workload (26 categorical features,
batch 8192, int64 IDs Zipf(1.05) over 10^7 per feature, hashed then mod 2^40,
tagged and merged into one dim-64 fp32 table with Adam state, sum pooling).

Prints one JSON line: IDs/s (device time, inputs resident, L2 flushed between
steps), the same through the API with host buffers (e2e), the roofline of the
dominant kernel, and the CPU oracle's rate on this host as a baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU runs (torchrun, one rank per GPU) are independent replicas: each rank
owns its own table and batches; only the timing is reduced (max over ranks).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "lookups/sec (IDs/s) fwd+bwd+update per step; achieved HBM GB/s vs B200 peak"
WORKLOAD = "criteo26"
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _config(w: W.Workload, extra=None):
    t = w.tables[0]
    c = {"workload": f"{w.name}: F={w.F} one-hot features, B={w.B}, IDs Zipf({w.zipf_a}) over "
                     f"{w.n_ids:.0e} per feature, hash->mod 2^40->tag, one merged dim-{t.dim} fp32 "
                     f"table, {t.optimizer}, {t.combiner} pooling",
         "F": w.F, "B": w.B, "dim": t.dim, "optimizer": t.optimizer, "combiner": t.combiner,
         "l2": "flushed (256 MiB write) between timed steps", "parallelism": "replicas"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------ CPU oracle
def _oracle_rate(w: W.Workload, budget_s: float, batches):
    """The CPU oracle (single thread) on full steps of the workload, ~budget_s."""
    import oracle as O
    t = w.tables[0]
    ops = [O.FeatureOp(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                       tag_shift=f.tag_shift) for f in w.features]
    tab = O.Table(t.dim, O.ADAM if t.optimizer == "adam" else O.ADAGRAD, t.lr, init_seed=t.init_seed)
    n_ids, steps, t0 = 0, 0, time.perf_counter()
    times = []
    while True:
        b, g = batches[steps % len(batches)]
        s0 = time.perf_counter()
        keys = O.feature_hash(ops, b.values, b.feat_offsets)
        tab.lookup(keys, b.bag_offsets, w.F, w.B)
        tab.backward_update(g)
        times.append(time.perf_counter() - s0)
        n_ids += len(b.values)
        steps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = sum(times)
    return {"value": n_ids / el, "unit": "IDs/s", "cores": 1, "kind": "oracle",
            "sample": f"{steps} full {w.name} steps (feature hash + lookup + backward/Adam) "
                      f"on the single-threaded CPU oracle, {el:.1f} s",
            "ms_per_step": 1e3 * el / steps, "steps": steps}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = W.WORKLOADS[WORKLOAD]
    t = w.tables[0]
    batches = [(W.make_batch(w, i), W.make_grad((w.B, w.F, t.dim), 100 + i)) for i in range(2)]
    warm = _oracle_rate(w, 0.0, batches) if args.warmup > 0 else None  # one untimed step
    del warm
    res = _oracle_rate(w, max(5.0, 2.0 * args.steps), batches)
    line = {"impl": "reference", "metric": METRIC, "value": res["value"], "unit": "IDs/s",
            "n_gpus": args.gpus, "steps": res["steps"], "warmup": args.warmup,
            "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64-accumulate/f32-store", "data": "synthetic",
            "config": _config(w),
            "cpu_baseline": {k: res[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": res["value"], "unit": "IDs/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        self.proc = None
        self.index = index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), "--query-gpu=clocks.sm,clocks.max.sm,"
                 "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap,utilization.gpu",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                clk, cmax, util = float(parts[0]), float(parts[1]), float(parts[7])
            except ValueError:
                continue
            mx = max(mx, cmax)
            if util > 0:
                sm.append(clk)
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples_under_load": len(sm)}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    from recommender_sparse_embedding_b200 import build as rbuild
    if rank == 0:
        rbuild.build()
    if world > 1:
        dist.barrier()
    import recommender_sparse_embedding_b200 as R
    R.load()

    w = W.WORKLOADS[WORKLOAD]
    spec = w.tables[0]
    D = spec.dim
    nb = args.warmup + args.steps
    n_distinct = min(nb, args.batches)
    seed = 2025 + w.index + 1000 * rank
    host = []
    for i in range(n_distinct):
        b = W.make_batch(w, i, seed=seed)
        g = W.make_grad((w.B, w.F, D), seed + i)
        host.append((b, g))
    feats = [R.Feature(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                       tag_shift=f.tag_shift) for f in w.features]
    devb = []
    for b, g in host:
        devb.append((torch.from_numpy(b.values).to(dev), b.feat_offsets.tolist(),
                     torch.from_numpy(b.bag_offsets).to(dev), torch.from_numpy(g).to(dev),
                     len(b.values)))
    opt = R.ADAM if spec.optimizer == "adam" else R.ADAGRAD
    table = R.Table(D, opt, spec.lr, init_seed=spec.init_seed,
                    initial_capacity=1_000_000 if args.small else 8_000_000)
    batch = R.Batch()
    keys = torch.empty(max(x[4] for x in devb), dtype=torch.int64, device=dev)
    pooled = torch.empty((w.B, w.F, D), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        vals, foffs, boffs, grad, n = devb[i % n_distinct]
        k = keys[:n]
        R.feature_hash(feats, vals, foffs, keys_out=k)
        table.lookup_pooled(batch, k, boffs, w.F, w.B, R.SUM, pooled_out=pooled)
        table.backward_update(batch, grad)
        return n

    # unique keys per batch (for the algorithmic bytes), outside any timing
    uniq_counts = []
    for i in range(n_distinct):
        vals, foffs, _, _, n = devb[i]
        k = R.feature_hash(feats, vals, foffs)
        uniq_counts.append(int(torch.unique(k).numel()))

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    table.status_sync()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    R.profile_enable(True)
    R.profile_collect()
    launches0 = R.launch_count()
    clocks = Clocks(torch.cuda.current_device()) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ids = 0
    for j in range(args.steps):
        flush.zero_()
        ev[j][0].record(stream)
        ids += step(args.warmup + j)
        ev[j][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = R.launch_count() - launches0
    clk = clocks.stop() if clocks else None
    prof = R.profile_collect()
    R.profile_enable(False)
    table.status_sync()
    dev_ms = sum(a.elapsed_time(b) for a, b in ev)

    # ---- e2e through the API with host buffers (pinned), copies inside the timing
    e2e_ids, e2e_ms, h2d, d2h = 0, 0.0, 0, 0
    pin = []
    for b, g in host[: min(4, n_distinct)]:
        pin.append((torch.from_numpy(b.values).pin_memory(), b.feat_offsets.tolist(),
                    torch.from_numpy(b.bag_offsets).pin_memory(), torch.from_numpy(g).pin_memory(),
                    len(b.values)))
    pooled_h = torch.empty((w.B, w.F, D), dtype=torch.float32).pin_memory()
    dv = torch.empty(max(x[4] for x in pin), dtype=torch.int64, device=dev)
    dbo = torch.empty(w.F * w.B + 1, dtype=torch.int64, device=dev)
    dg = torch.empty((w.B, w.F, D), dtype=torch.float32, device=dev)
    e2e_steps = max(3, args.steps // 2)
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(e2e_steps)]
    torch.cuda.synchronize()
    for j in range(e2e_steps):
        vals_h, foffs, bo_h, g_h, n = pin[j % len(pin)]
        flush.zero_()
        eev[j][0].record(stream)
        v = dv[:n]
        v.copy_(vals_h, non_blocking=True)
        dbo.copy_(bo_h, non_blocking=True)
        dg.copy_(g_h, non_blocking=True)
        k = keys[:n]
        R.feature_hash(feats, v, foffs, keys_out=k)
        table.lookup_pooled(batch, k, dbo, w.F, w.B, R.SUM, pooled_out=pooled)
        table.backward_update(batch, dg)
        pooled_h.copy_(pooled, non_blocking=True)
        eev[j][1].record(stream)
        e2e_ids += n
        h2d = vals_h.numel() * 8 + bo_h.numel() * 8 + g_h.numel() * 4
        d2h = pooled_h.numel() * 4
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in eev)
    table.status_sync()

    # ---- reduce over ranks: max time, summed work
    t_dev = torch.tensor([dev_ms, e2e_ms, float(ids), float(e2e_ids)], dtype=torch.float64, device=dev)
    if world > 1:
        mx = t_dev.clone()
        dist.all_reduce(mx[:2], op=dist.ReduceOp.MAX)
        sm = t_dev.clone()
        dist.all_reduce(sm[2:], op=dist.ReduceOp.SUM)
        dev_ms, e2e_ms, ids, e2e_ids = float(mx[0]), float(mx[1]), float(sm[2]), float(sm[3])
    value = ids / (dev_ms / 1e3)
    e2e_value = e2e_ids / (e2e_ms / 1e3)

    if rank == 0:
        peak, peak_kind = _peaks()
        # algorithmic bytes per launch of each kernel of the step
        Nm = statistics.mean(x[4] for x in devb)
        Um = statistics.mean(uniq_counts)
        nb_ = w.F * w.B
        s = 2 if spec.optimizer == "adam" else 1
        alg = {
            "reduce_update": 4 * D * nb_ + 2 * 4 * D * (1 + s) * Um,
            "gather_pool": 4 * D * Um + 4 * D * nb_,
            "feature_hash": 16 * Nm,
            "unique_insert": 16 * Um,
        }
        kern = {k: {"launches": v[0], "total_ms": v[1], "avg_us": 1e3 * v[1] / max(v[0], 1)}
                for k, v in prof.items()}
        top = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else None
        roof = None
        if top in alg:
            avg_s = prof[top][1] / prof[top][0] / 1e3
            achieved = alg[top] / avg_s / 1e9
            roof = {"bound": "hbm", "kernel": top, "achieved": achieved, "peak": peak,
                    "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                    "traffic": None, "alg_bytes_per_launch": alg[top]}
        step_alg = (8 * Nm + 16 * Um + 4 * D * Um + 4 * D * nb_) + alg["reduce_update"]
        line = {
            "metric": METRIC, "value": value, "unit": "IDs/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dev_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": _config(w, {"ids_per_step": Nm, "unique_per_step": Um,
                                  "distinct_batches": n_distinct}),
            "roofline": roof,
            "step_alg_gbs": step_alg / (dev_ms / args.steps / 1e3) / 1e9,
            "e2e": {"value": e2e_value, "unit": "IDs/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "kernels": kern,
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            res = _oracle_rate(w, args.cpu_seconds, host[:2])
            line["cpu_baseline"] = {k: res[k] for k in ("value", "unit", "cores", "kind", "sample")}
        print(json.dumps(line), flush=True)

    table.close()
    batch.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--batches", type=int, default=32, help="distinct batches generated")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--small", action="store_true",
                    help="smaller table reservation (for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "own":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
