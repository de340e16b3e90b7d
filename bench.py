#!/usr/bin/env python
"""Benchmark of the dynamic-hash embedding step (RecIS Embedding Engine hot path).

One step = recis_feature_hash + recis_lookup_pooled + recis_backward_update
over one batch of a synthetic workload.

The headline workload is the large table: about 50M live IDs pre-inserted
(100 features, dim-64 fp32 rows with Adam m and v beside them, ~38 GB), batch
65536 x 100 features with bag lengths geometric (mean 5), each occurrence a
never-seen ID with probability 0.05 (fresh IDs for every step) and otherwise a
Zipf(1.05) draw over its feature's share of the live set, sum pooling.  The
same line carries sub-records for the 26-feature one-hot workload (criteo26),
the long behaviour sequence (longseq) and the 8 multi-hot sequence features
(seq8); `--workload` selects another headline and `--subs` the sub-records.

Per workload: IDs/s (device time, inputs resident in HBM, L2 flushed between
steps), the same through the API with host buffers (e2e: torch copies of
pinned host buffers around the library's device-pointer calls, pipelined),
the roofline of the dominant kernel group, SM clocks sampled during the timed
region, and the CPU oracle's rate on this host as a baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--workload NAME] [--subs a,b,c|none]
Multi-GPU runs (torchrun, one rank per GPU) are independent replicas: each rank
owns its own tables and batches; only the timing is reduced (max over ranks).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "lookups/sec (IDs/s) fwd+bwd+update per step; achieved HBM GB/s vs B200 peak"
DEFAULT_WORKLOAD = "large"
DEFAULT_SUBS = "criteo26,longseq,seq8"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, the nominal figure (the measured copy peak is the roofline)
TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
# the large-table workload's CPU baseline runs at this fraction of its batch
# and of its live set (the full live set would need ~40 GB of host memory)
LARGE_ORACLE_SCALE = 16


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _describe(w: W.Workload) -> str:
    tabs = ", ".join(f"dim-{t.dim} {t.optimizer} {t.combiner}"
                     + (" pooled" if t.pooled else "") + (" +unpooled" if t.unpooled else "")
                     for t in w.tables)
    f0 = w.features[0]
    tf = "hash->mod 2^40->tag" if f0.flags & W.HASH else "tag"
    if w.live_ids:
        ids = (f"{w.live_ids:.0e} live IDs pre-inserted, each occurrence fresh with p={w.fresh_frac} "
               f"(never-seen IDs every step) else Zipf({w.zipf_a}) over its feature's "
               f"{w.live_ids // w.F} live IDs")
    else:
        ids = f"IDs Zipf({w.zipf_a}) over {w.n_ids:.0e} per feature"
    return (f"{w.name}: F={w.F} features, B={w.B}, bag length {w.length}, {ids}, {tf}, "
            f"fp32 tables [{tabs}]")


def _workload(name: str, scale: int) -> W.Workload:
    """The named workload, or for profiler captures the same recipe with a
    batch 1/scale as large (and, for the large table, 1/(2 scale) of its live
    rows)."""
    w = W.WORKLOADS[name]
    if scale <= 1:
        return w
    s = w.scaled(max(1, w.B // scale))
    s.live_ids = w.live_ids // (2 * scale)
    s.scale = scale
    return s


def _config(w: W.Workload, extra=None):
    c = {"workload": _describe(w), "F": w.F, "B": w.B,
         "tables": [{"dim": t.dim, "features": len(t.features), "optimizer": t.optimizer,
                     "combiner": t.combiner, "pooled": t.pooled, "unpooled": t.unpooled}
                    for t in w.tables],
         "l2": "flushed (256 MiB write) between timed steps", "parallelism": "replicas"}
    if getattr(w, "scale", 1) > 1:
        c["scale"] = f"batch 1/{w.scale} of the workload's (profiler capture case)"
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------ CPU oracle
def _host_cpu() -> str:
    """CPU model and hardware threads of this host, for the CPU baseline."""
    model = "unknown CPU"
    try:
        with open("/proc/cpuinfo") as fh:
            for ln in fh:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return f"{model}, {os.cpu_count()} hardware threads"


def _grads(w: W.Workload, b: W.Batch, seed: int):
    """Upstream gradients of one batch: (grad_pooled, grad_unpooled) per table."""
    out = []
    for i, t in enumerate(w.tables):
        lo, hi, _ = b.table_slice(t, w.B)
        gp = W.make_grad((w.B, len(t.features), t.dim), seed + 17 * i) if t.pooled else None
        gu = W.make_grad((hi - lo, t.dim), seed + 17 * i + 1) if t.unpooled else None
        out.append((gp, gu))
    return out


def _oracle_sample(w: W.Workload):
    """(workload the oracle runs, its pre-inserted live keys per table or None,
    a description of the sample).  The large-table workload runs at
    1/LARGE_ORACLE_SCALE of its batch and live set; the others in full."""
    if not w.live_ids:
        return w, None, "full steps"
    s = LARGE_ORACLE_SCALE
    ws = w.scaled(w.B // s)
    ws.live_ids = w.live_ids // s
    per = ws.live_ids // ws.F
    live = np.concatenate([(np.int64(ws.features[f].tag) << np.int64(ws.features[f].tag_shift))
                           | W.live_ids(ws, f, per) for f in range(ws.F)])
    live.sort()
    return ws, [live], (f"1/{s}-scale steps: batch {ws.B} x {ws.F} features against a table "
                        f"pre-filled with {len(live)} live keys (1/{s} of the live set)")


def _oracle_rate(w: W.Workload, budget_s: float, nbatch: int = 2, n_steps: int = 0, n_warm: int = 0):
    """The CPU oracle (single thread) on steps of the workload for ~budget_s,
    or, when n_steps > 0, on exactly n_warm untimed and n_steps timed steps."""
    import oracle as O
    ws, live, what = _oracle_sample(w)
    batches = []
    for i in range(nbatch):
        b = W.make_batch(ws, i)
        batches.append((b, _grads(ws, b, 100 + i)))
    ops = [O.FeatureOp(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                       tag_shift=f.tag_shift, boundaries=list(f.boundaries)) for f in ws.features]
    tabs = [O.Table(t.dim, O.ADAM if t.optimizer == "adam" else O.ADAGRAD, t.lr,
                    init_seed=t.init_seed) for t in ws.tables]
    if live is not None:  # pre-insert the live set (untimed)
        for tab, keys in zip(tabs, live):
            for c0 in range(0, len(keys), 1 << 20):
                k = keys[c0:c0 + (1 << 20)]
                tab.lookup(k, np.arange(len(k) + 1, dtype=np.int64), 1, len(k), pooled=False)
    n_ids, steps, t0 = 0, 0, time.perf_counter()
    times = []
    for j in range(n_warm + n_steps if n_steps > 0 else 1 << 62):
        b, grads = batches[j % len(batches)]
        vals = b.values if live is None else W.with_fresh_ids(ws, b, 200 + j)
        s0 = time.perf_counter()
        keys = O.feature_hash(ops, vals, b.feat_offsets)
        for t, tab, (gp, gu) in zip(ws.tables, tabs, grads):
            lo, hi, bo = b.table_slice(t, ws.B)
            tab.lookup(keys[lo:hi], bo, len(t.features), ws.B,
                       O.SUM if t.combiner == "sum" else O.MEAN, pooled=t.pooled,
                       unpooled=t.unpooled)
            tab.backward_update(gp, gu)
        if j < n_warm:
            continue  # untimed warm-up step
        times.append(time.perf_counter() - s0)
        n_ids += len(vals)
        steps += 1
        if n_steps == 0 and time.perf_counter() - t0 >= budget_s:
            break
    el = sum(times)
    return {"value": n_ids / el, "unit": "IDs/s", "cores": 1, "kind": "oracle", "host": _host_cpu(),
            "sample": f"{steps} {what} of {w.name} (feature hash + lookup + backward/optimiser) "
                      f"on the single-threaded CPU oracle, {el:.1f} s",
            "ms_per_step": 1e3 * el / steps, "steps": steps}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    # exactly W untimed and K timed steps, each a bounded sample of the
    # workload (the large table's at 1/16 scale: about a second of CPU work)
    res = _oracle_rate(w, 0.0, n_steps=max(1, args.steps), n_warm=max(0, args.warmup))
    line = {"impl": "reference", "metric": METRIC, "value": res["value"], "unit": "IDs/s",
            "n_gpus": args.gpus, "steps": res["steps"], "warmup": args.warmup,
            "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64-accumulate/f32-store", "data": "synthetic",
            "config": _config(w),
            "cpu_baseline": {k: res[k] for k in ("value", "unit", "cores", "kind", "sample", "host")},
            "e2e": {"value": res["value"], "unit": "IDs/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
class Clocks:
    """SM clock and clock-event reasons, sampled through NVML every few ms on a
    background thread; only samples inside [t0, t1] (the timed region) count."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, torch_index: int, period_s: float = 0.002):
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml as N
            import torch
            N.nvmlInit()
            self.N = N
            uuid = str(torch.cuda.get_device_properties(torch_index).uuid)
            handle = None
            for i in range(N.nvmlDeviceGetCount()):
                h = N.nvmlDeviceGetHandleByIndex(i)
                u = N.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    handle = h
                    break
            if handle is None:
                handle = N.nvmlDeviceGetHandleByIndex(torch_index)
            self.h = handle
            self.max_mhz = float(N.nvmlDeviceGetMaxClockInfo(handle, N.NVML_CLOCK_SM))
            self.masks = [(name, getattr(N, attr, 0)) for name, attr in self.REASONS]
            self._thread = threading.Thread(target=self._run, args=(period_s,), daemon=True)
            self._thread.start()
        except Exception as e:  # NVML missing: report no clocks rather than fail the bench
            self.error = f"{type(e).__name__}: {e}"

    def _run(self, period_s):
        N = self.N
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                clk = N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM)
                rs = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((t, float(clk), int(rs)))
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            time.sleep(period_s)

    def stop(self, t0: float, t1: float):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        reasons = set()
        for _, _, rs in inside:
            for name, m in getattr(self, "masks", []):
                if m and rs & m:
                    reasons.add(name)
        out = {"sm_mhz": statistics.median(s[1] for s in inside) if inside else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
               "samples": len(inside), "source": "nvml, 2 ms period, timed region only"}
        if self.error:
            out["error"] = self.error
        return out


def _code_only(text: str) -> str:
    """Source text without // and /* */ comments and blank lines: what a
    capture depends on (a comment edit leaves the kernels as they were)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def _files_sha(files):
    """sha256 of the code (comments dropped) of a kernel's source files."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()


def _traffic(workload: str, kernel: str, units: float):
    """(DRAM bytes per launch, L2 hit rate %, note) of `kernel` on `workload` from
    the committed ncu summary, scaled to `units` occurrences when it was
    captured on another size; bytes None when the kernel's sources changed
    since the capture."""
    if not os.path.exists(TRAFFIC):
        return None, None, "no capture"
    with open(TRAFFIC) as fh:
        d = json.load(fh)
    e = d.get(workload, {}).get(kernel)
    if not e:
        return None, None, "no capture of this kernel on this workload"
    try:
        if _files_sha(e["files"]) != e["sha256"]:
            return None, None, "kernel changed since the capture"
    except OSError:
        return None, None, "kernel sources missing"
    scale = units / e["units"] if e.get("units") else 1.0
    note = e.get("note", "")
    if abs(scale - 1.0) > 0.01:
        note += f"; captured at {e['units']} occurrences, scaled by {scale:.3f}"
    return e["dram_bytes_per_launch"] * scale, e.get("l2_hit_pct"), note


# kernels of the step, grouped by the row of the method they implement
GROUPS = {
    "feature_hash": ("feature_hash",),
    "dedup": ("ss_rank", "ss_probe", "ss_count", "ss_tilescan", "ss_scatter", "ss_local", "ss_finish",
              "sort_hist", "sort_pass", "unique_insert"),
    "gather_pool": ("bag_prep", "gather_pool"),
    "backward": ("seg_partial", "seg_combine", "row_update"),
}


def _alg_bytes(w: W.Workload, stats):
    """Algorithmic bytes per step of each group (what the method must move; the
    dedup's sort scratch is not credited).  stats[i] = (N, U, n_new) of table i."""
    total_N = sum(s[0] for s in stats)
    out = {"feature_hash": 16.0 * total_N, "dedup": 0.0, "gather_pool": 0.0, "backward": 0.0}
    for t, (N, U, n_new) in zip(w.tables, stats):
        D, s = t.dim, (2 if t.optimizer == "adam" else 1)
        bags = len(t.features) * w.B
        out["dedup"] += 8 * N + 4 * N + 16 * U + 16 * U + 4 * D * (1 + s) * n_new
        out["gather_pool"] += 4 * D * U + (4 * D * bags if t.pooled else 0) + \
            (4 * D * N if t.unpooled else 0) + 8 * bags
        out["backward"] += (4 * D * bags if t.pooled else 0) + (4 * D * N if t.unpooled else 0) \
            + 2 * 4 * D * (1 + s) * U
    return out


def _live_keys(w: W.Workload, seed: int):
    """Pre-inserted keys of the large-table workload, tagged, ascending."""
    per = w.live_ids // w.F
    live = np.concatenate([(np.int64(w.features[f].tag) << np.int64(w.features[f].tag_shift))
                           | W.live_ids(w, f, per, seed=seed) for f in range(w.F)])
    live.sort()
    return live


def measure(w: W.Workload, args, R, dist, world: int, rank: int, dev, headline: bool):
    """One workload: setup, warm-up, timed steps, traced steps (per-kernel
    event times), e2e steps with host buffers, the CPU baseline.  Returns the
    record on rank 0 (None elsewhere)."""
    import torch

    large = bool(w.live_ids)
    prof_steps = min(args.steps, 10 if large else 50)
    e2e_steps = 4 if large else max(3, min(args.steps, 50) // 2)
    seed = 2025 + w.index + 1000 * rank
    feats = [R.Feature(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                       tag_shift=f.tag_shift,
                       boundaries=(torch.tensor(list(f.boundaries), dtype=torch.int64, device=dev)
                                   if f.boundaries else None)) for f in w.features]

    # ---- inputs: every step's batch resident on the device before timing
    n_steps = args.warmup + args.steps + prof_steps
    if large:
        # two drawn batches; every step gives their fresh-ID positions IDs never
        # seen before (stream index = step), so 5% of occurrences are new each step
        base = [W.make_batch(w, i, seed=seed) for i in range(2)]
        host = [(b, _grads(w, b, seed + i)) for i, b in enumerate(base)]
        step_vals = [W.with_fresh_ids(w, base[j % 2], 10 + j, seed=seed) for j in range(n_steps)]
    else:
        n_distinct = min(n_steps, args.batches)
        host = []
        for i in range(n_distinct):
            b = W.make_batch(w, i, seed=seed)
            host.append((b, _grads(w, b, seed + i)))
        step_vals = None

    def dev_batch(b, grads, vals=None, pin=False):
        mv = (lambda a: torch.from_numpy(a).pin_memory()) if pin else \
            (lambda a: torch.from_numpy(a).to(dev))
        per_table = []
        for t, (gp, gu) in zip(w.tables, grads):
            lo, hi, bo = b.table_slice(t, w.B)
            per_table.append((lo, hi, mv(bo), None if gp is None else mv(gp),
                              None if gu is None else mv(gu)))
        v = b.values if vals is None else vals
        return mv(v), b.feat_offsets.tolist(), per_table, len(v)

    if large:
        base_dev = [dev_batch(b, g) for b, g in host]
        devb = []
        for j, v in enumerate(step_vals):
            _, foffs, per_table, n = base_dev[j % 2]
            devb.append((torch.from_numpy(v).to(dev), foffs, per_table, n))
        del step_vals
    else:
        devb = [dev_batch(b, g) for b, g in host]
    nb = len(devb)

    maxN = max(x[3] for x in devb)
    if large:
        live = _live_keys(w, seed)
        new_est = int(1.1 * w.fresh_frac * maxN) * (n_steps + e2e_steps + 2)
        cap = len(live) + new_est + maxN
    else:
        live = None
        cap = 1_000_000 if args.small else 8_000_000
    tables = [R.Table(t.dim, R.ADAM if t.optimizer == "adam" else R.ADAGRAD, t.lr,
                      init_seed=t.init_seed, initial_capacity=cap) for t in w.tables]
    batches = [R.Batch() for _ in w.tables]
    if large:  # pre-insert the live set, in chunks the dedup takes in one call
        b_ins = R.Batch()
        chunk = 1_500_000
        for c0 in range(0, len(live), chunk):
            tables[0].insert(b_ins, torch.from_numpy(live[c0:c0 + chunk]).to(dev))
        torch.cuda.synchronize()
        tables[0].status_sync()
        b_ins.close()
        assert tables[0].size()[0] == len(live)
    keys = torch.empty(maxN, dtype=torch.int64, device=dev)
    pooled = [torch.empty((w.B, len(t.features), t.dim), dtype=torch.float32, device=dev)
              if t.pooled else None for t in w.tables]
    max_n = [max(x[2][i][1] - x[2][i][0] for x in devb) for i in range(len(w.tables))]
    unpooled = [torch.empty((max_n[i], t.dim), dtype=torch.float32, device=dev)
                if t.unpooled else None for i, t in enumerate(w.tables)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    combiner = [R.SUM if t.combiner == "sum" else R.MEAN for t in w.tables]

    def run_step(vals, foffs, per_table, n, kbuf, pooled_bufs=None, unpooled_bufs=None):
        pb = pooled if pooled_bufs is None else pooled_bufs
        ub = unpooled if unpooled_bufs is None else unpooled_bufs
        k = kbuf[:n]
        R.feature_hash(feats, vals, foffs, keys_out=k)
        for i, t in enumerate(w.tables):
            lo, hi, bo, gp, gu = per_table[i]
            up = ub[i][: hi - lo] if ub[i] is not None else None
            tables[i].lookup_pooled(batches[i], k[lo:hi], bo, len(t.features), w.B, combiner[i],
                                    pooled_out=pb[i], unpooled_out=up)
            tables[i].backward_update(batches[i], gp, gu)
        return n

    # unique keys per table (for the algorithmic bytes) on a few batches, untimed
    uniq = []
    for vals, foffs, per_table, n in devb[: min(nb, 4)]:
        k = R.feature_hash(feats, vals, foffs)
        uniq.append([int(torch.unique(k[lo:hi]).numel()) for (lo, hi, *_r) in per_table])
        del k

    rows_pre = [t.size()[0] for t in tables]
    for i in range(args.warmup):
        run_step(*devb[i % nb], keys)
    torch.cuda.synchronize()
    for t in tables:
        t.status_sync()
    rows0 = [t.size()[0] for t in tables]
    # make room now for every row the remaining steps may add (from the
    # warm-up's growth), so that no block is mapped and no IDMap rehashed
    # inside the timed region
    for t, r_pre, r0, (lo, hi, *_r) in zip(tables, rows_pre, rows0, devb[0][2]):
        per_step = (r0 - r_pre) / max(args.warmup, 1)
        t.reserve(int(r0 + 1.1 * per_step * (args.steps + prof_steps + e2e_steps + 2)) + (hi - lo))

    # ---- timed region: K steps, no tracing events between the kernels
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    launches0 = R.launch_count()
    clocks = Clocks(torch.cuda.current_device()) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    ids = 0
    for j in range(args.steps):
        flush.zero_()
        ev[j][0].record(stream)
        ids += run_step(*devb[(args.warmup + j) % nb], keys)
        ev[j][1].record(stream)
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    launches = R.launch_count() - launches0
    clk = clocks.stop(h0, h1) if clocks else None
    for t in tables:
        t.status_sync()
    new_rows = [(t.size()[0] - r0) / args.steps for t, r0 in zip(tables, rows0)]
    dev_ms = sum(a.elapsed_time(b) for a, b in ev)
    step_ms = sorted(a.elapsed_time(b) for a, b in ev)  # this rank's steps, each between its events

    # ---- traced region: further steps with CUDA events around every launch of
    # the library (per-kernel durations for the roofline)
    R.profile_enable(True)
    R.profile_collect()
    torch.cuda.synchronize()
    for j in range(prof_steps):
        flush.zero_()
        run_step(*devb[(args.warmup + args.steps + j) % nb], keys)
    torch.cuda.synchronize()
    prof = R.profile_collect()
    R.profile_enable(False)
    for t in tables:
        t.status_sync()
    Nm = statistics.mean(x[3] for x in devb)
    stats_N = [statistics.mean(x[2][i][1] - x[2][i][0] for x in devb) for i in range(len(w.tables))]
    del devb
    if large:
        del base_dev
    torch.cuda.empty_cache()

    # ---- e2e through the API with host buffers (pinned), copies inside the timing.
    # Steps are pipelined the way a training loop feeds the engine: step j+1's
    # inputs go up on a copy stream while step j computes, and step j's pooled
    # rows come down on another, so the two PCIe directions and the kernels
    # overlap.  Two sets of device buffers alternate.  The timed region runs
    # from the first copy up to the last copy down and holds every step's
    # copies, its L2 flush and its kernels.  The copies are torch copies of
    # pinned host tensors; the library calls take the device buffers.
    e2e_ids, h2d, d2h = 0, 0, 0
    if large:
        # every e2e step has never-seen fresh IDs too; the gradients and bag
        # offsets of the two drawn batches are pinned once and shared
        pin_base = [dev_batch(b, g, pin=True) for b, g in host]
        pin = []
        for j in range(e2e_steps):
            _, foffs, per_h, n = pin_base[j % 2]
            vals = W.with_fresh_ids(w, host[j % 2][0], 10 + n_steps + j, seed=seed)
            pin.append((torch.from_numpy(vals).pin_memory(), foffs, per_h, n))
    else:
        pin = [dev_batch(b, g, pin=True) for b, g in host[: min(4, len(host))]]
    NBUF = 2
    dv = [torch.empty(maxN, dtype=torch.int64, device=dev) for _ in range(NBUF)]
    dbo = [[torch.empty(w.F * w.B + 1, dtype=torch.int64, device=dev) for _ in w.tables]
           for _ in range(NBUF)]
    dgp = [[torch.empty_like(p) if p is not None else None for p in pooled] for _ in range(NBUF)]
    dgu = [[torch.empty_like(u) if u is not None else None for u in unpooled] for _ in range(NBUF)]
    dpool = [[torch.empty_like(p) if p is not None else None for p in pooled] for _ in range(NBUF)]
    pooled_h = [torch.empty(p.shape, dtype=p.dtype).pin_memory() if p is not None else None
                for p in pooled]
    up_s, down_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_down = [torch.cuda.Event() for _ in range(e2e_steps)]
    t_first, t_last = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def upload(j):
        """Step j's inputs into buffer set j % NBUF (once step j - NBUF is done with it)."""
        nonlocal h2d
        vals_h, foffs, per_h, n = pin[j % len(pin)]
        sb = j % NBUF
        with torch.cuda.stream(up_s):
            if j >= NBUF:
                up_s.wait_event(ev_done[j - NBUF])
            v = dv[sb][:n]
            v.copy_(vals_h, non_blocking=True)
            nbytes = vals_h.numel() * 8
            per_d = []
            for i, (lo, hi, bo_h, gp_h, gu_h) in enumerate(per_h):
                bo = dbo[sb][i][: bo_h.numel()]
                bo.copy_(bo_h, non_blocking=True)
                nbytes += bo_h.numel() * 8
                gp = gu = None
                if gp_h is not None:
                    gp = dgp[sb][i]
                    gp.copy_(gp_h, non_blocking=True)
                    nbytes += gp_h.numel() * 4
                if gu_h is not None:
                    gu = dgu[sb][i][: gu_h.shape[0]]
                    gu.copy_(gu_h, non_blocking=True)
                    nbytes += gu_h.numel() * 4
                per_d.append((lo, hi, bo, gp, gu))
            ev_up[j].record(up_s)
        h2d = nbytes
        return v, foffs, per_d, n

    torch.cuda.synchronize()
    t_first.record(up_s)
    staged = upload(0)
    for j in range(e2e_steps):
        nxt = upload(j + 1) if j + 1 < e2e_steps else None
        sb = j % NBUF
        stream.wait_event(ev_up[j])
        if j >= NBUF:
            stream.wait_event(ev_down[j - NBUF])  # pooled buffers of set sb copied down
        flush.zero_()
        v, foffs, per_d, n = staged
        run_step(v, foffs, per_d, n, keys, pooled_bufs=dpool[sb])
        ev_done[j].record(stream)
        with torch.cuda.stream(down_s):
            down_s.wait_event(ev_done[j])
            d2h = 0
            for i, ph in enumerate(pooled_h):
                if ph is not None:
                    ph.copy_(dpool[sb][i], non_blocking=True)
                    d2h += ph.numel() * 4
            ev_down[j].record(down_s)
        e2e_ids += n
        staged = nxt
    t_last.record(down_s)
    torch.cuda.synchronize()
    e2e_ms = t_first.elapsed_time(t_last)
    for t in tables:
        t.status_sync()

    # ---- reduce over ranks: max time, summed work
    t_dev = torch.tensor([dev_ms, e2e_ms, float(ids), float(e2e_ids)], dtype=torch.float64,
                         device=dev)
    if world > 1:
        mx = t_dev.clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        sm = t_dev.clone()
        dist.all_reduce(sm, op=dist.ReduceOp.SUM)
        dev_ms, e2e_ms, ids, e2e_ids = float(mx[0]), float(mx[1]), float(sm[2]), float(sm[3])
    value = ids / (dev_ms / 1e3)
    e2e_value = e2e_ids / (e2e_ms / 1e3)

    rec = None
    if rank == 0:
        peak, peak_kind = _peaks()
        stats = []
        for i, t in enumerate(w.tables):
            Ui = statistics.mean(u[i] for u in uniq)
            stats.append((stats_N[i], Ui, new_rows[i]))
        alg = _alg_bytes(w, stats)
        kern = {k: {"launches": v[0], "total_ms": v[1], "avg_us": 1e3 * v[1] / max(v[0], 1)}
                for k, v in prof.items()}
        # the dominant kernel, and its row of the method
        roof = None
        if prof:
            top = max(prof.items(), key=lambda kv: kv[1][1])[0]
            grp = next((g for g, ks in GROUPS.items() if top in ks), None)
            if grp is not None:
                members = [k for k in GROUPS[grp] if k in prof]
                # bytes of the row per step; time of the row's kernels per step
                row_s = sum(prof[k][1] for k in members) / prof_steps / 1e3
                top_launches_per_step = prof[top][0] / prof_steps
                top_s = prof[top][1] / prof[top][0] / 1e3
                if len(members) == 1:
                    per_launch = alg[grp] / top_launches_per_step
                    achieved = per_launch / top_s / 1e9
                else:
                    per_launch = alg[grp]
                    achieved = alg[grp] / row_s / 1e9
                traffic, l2hit, tnote = _traffic(w.name, top, Nm / top_launches_per_step)
                roof = {"bound": "hbm", "kernel": top, "row": grp,
                        "row_kernels": members, "achieved": achieved, "peak": peak,
                        "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                        "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                        "traffic": traffic, "traffic_note": tnote,
                        "l2_hit_rate_pct": l2hit,
                        "alg_bytes_per_launch": per_launch,
                        "note": ("algorithmic bytes of the row / its kernels' event time"
                                 if len(members) > 1 else
                                 "algorithmic bytes per launch / CUDA-event time per launch")}
        # actual DRAM traffic (ncu capture) of the kernels that have one:
        # per kernel, and over those kernels' share of the step
        l2 = {}
        dram_b = dram_t = 0.0
        for k, v in prof.items():
            lps = v[0] / prof_steps  # launches per step
            tb, hit, _n = _traffic(w.name, k, Nm / max(lps, 1e-9))
            if hit is not None:
                l2[k] = hit
            if tb is not None:
                kern[k]["dram_bytes_per_launch"] = tb
                kern[k]["dram_gbs"] = tb / (kern[k]["avg_us"] * 1e-6) / 1e9
                kern[k]["dram_frac"] = kern[k]["dram_gbs"] / peak
                dram_b += tb * lps
                dram_t += kern[k]["avg_us"] * 1e-6 * lps
        dram = ({"gbs": dram_b / dram_t / 1e9, "frac": dram_b / dram_t / 1e9 / peak,
                 "kernels": sorted(k for k in kern if "dram_gbs" in kern[k]),
                 "share_of_step_kernel_time": dram_t / (sum(v[1] for v in prof.values()) / prof_steps / 1e3),
                 "note": "ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of these kernels "
                         "(profiles/traffic.json) / their CUDA-event time"} if dram_t > 0 else None)
        step_alg = sum(alg.values()) - alg["feature_hash"] + 16 * Nm
        step_s = dev_ms / args.steps / 1e3
        rec = {
            "metric": METRIC, "value": value, "unit": "IDs/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dev_ms / args.steps,
            "ms_per_step_p50": statistics.median(step_ms),
            "ms_per_step_p90": step_ms[min(len(step_ms) - 1, round(0.9 * (len(step_ms) - 1)))],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": _config(w, {"ids_per_step": Nm,
                                  "unique_per_step": [s[1] for s in stats],
                                  "new_rows_per_step": [s[2] for s in stats],
                                  "distinct_batches": nb,
                                  **({"live_rows_at_start": len(live)} if large else {})}),
            "roofline": roof,
            "step_alg_bytes": step_alg,
            "step_alg_gbs": step_alg / step_s / 1e9,
            "step_frac_of_peak": step_alg / step_s / 1e9 / peak,
            "l2_hit_rate_pct": l2 or None,
            "dram_achieved": dram,
            "e2e": {"value": e2e_value, "unit": "IDs/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "note": "torch copies of pinned host buffers around the library's "
                            "device-pointer calls, inside the timed region; steps pipelined: step "
                            "j+1's inputs up and step j-1's pooled rows down overlap step j's "
                            "kernels; timed from the first copy up to the last copy down"},
            "gpu_launches": launches,
            "kernels": kern,
            "kernels_note": f"CUDA events around every launch, {prof_steps} further steps after "
                            "the timed region (the timed region itself runs without them)",
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            res = _oracle_rate(w, args.cpu_seconds if headline else args.cpu_seconds / 2)
            rec["cpu_baseline"] = {k: res[k] for k in ("value", "unit", "cores", "kind", "sample",
                                                       "host")}

    for t in tables:
        t.close()
    for b in batches:
        b.close()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
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

    subs = [] if args.subs in ("", "none") else [s for s in args.subs.split(",")
                                                 if s != args.workload]
    line = measure(_workload(args.workload, args.scale), args, R, dist, world, rank, dev, headline=True)
    sub_recs = {}
    for name in subs:
        r = measure(_workload(name, args.scale), args, R, dist, world, rank, dev, headline=False)
        if r is not None:
            keep = ("value", "unit", "ms_per_step", "ms_per_step_p50", "ms_per_step_p90", "config",
                    "roofline", "step_alg_bytes", "step_alg_gbs", "step_frac_of_peak",
                    "l2_hit_rate_pct", "dram_achieved", "e2e", "gpu_launches", "kernels", "clocks",
                    "cpu_baseline")
            sub_recs[name] = {k: r[k] for k in keep if k in r}
    if rank == 0:
        if sub_recs:
            line["configs"] = sub_recs
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--subs", default=DEFAULT_SUBS,
                    help="comma-separated workloads measured after the headline one, or none")
    ap.add_argument("--batches", type=int, default=32, help="distinct batches generated")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--small", action="store_true",
                    help="smaller table reservation (for profiler captures)")
    ap.add_argument("--scale", type=int, default=1,
                    help="run each workload with a batch 1/scale as large (profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "own":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
