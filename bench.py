#!/usr/bin/env python
"""Benchmark of the TriAttention KV-cache compression pass on B200.

Workload: the Qwen3-32B-shape long-reasoning decode cache (64 layers, 64 query
/ 8 KV heads, head_dim 128, 32768 cached tokens, budget 2048, window 256,
NEOX pairing, theta 1e4), seeded synthetic bf16 K/V.  One step = one full
compression pass (coefficients, scoring + normalize-then-max + selection,
in-place compaction of K, V and positions) through the C ABI.

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
on the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "keys scored+selected/s (Qwen3-32B-shape 32K pass)"
UNIT = "keys/s"


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("tria_score_tc.cu", "tria_tc.cuh", "tria_device.cuh", "tria_internal.h"):
        with open(os.path.join(ROOT, "key_retention_scoring_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if it
    was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch_full_size")


class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML while the
    timed region runs (reads only)."""

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples = []
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml as N

            N.nvmlInit()
            self._N = N
            self._h = N.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self._h, N.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception as e:  # NVML missing: report it, do not fail the bench
            self.error = repr(e)
        return self

    def _run(self):
        N = self._N
        while not self._stop.is_set():
            try:
                mhz = N.nvmlDeviceGetClockInfo(self._h, N.NVML_CLOCK_SM)
                reasons = N.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                pw = N.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                self.samples.append((mhz, reasons, pw))
            except Exception as e:
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        names = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                 0x100: "display_clock_setting"}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "error": self.error}
        mhz = [s[0] for s in self.samples]
        seen = set()
        for _, r, _ in self.samples:
            for bit, n in names.items():
                if r & bit:
                    seen.add(n)
        seen.discard("gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(seen), "samples": len(mhz),
                "power_w_median": round(statistics.median(s[2] for s in self.samples), 1)}


# ---------------------------------------------------------------------------
# oracle (CPU baseline and reference arm): worker processes (spawned, one
# numpy thread each) that time the fp64 oracle on whole units of a workload,
# generated on the host with the same recipe
# ---------------------------------------------------------------------------
def _single_thread_env():
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                             "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    return saved


def _restore_env(saved):
    for k, v in saved.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_units(task):
    """Worker: the fp64 oracle (scores in `form`, normalize-then-max,
    selection) on units of workload `cfg_idx` until `seconds` of compute (at
    least one unit, at most `max_units`).  Returns (keys, seconds, units)."""
    cfg_idx, form, seconds, max_units, seed = task
    import synth
    from oracle import tria_oracle as O

    cfg = synth.CONFIGS[cfg_idx]
    re, im, am = synth.make_stats(cfg)
    centers = synth.make_centers(cfg)
    omega = O.band_frequencies(cfg.head_dim, cfg.theta)
    G = cfg.group
    lens = synth.seq_lengths(cfg)
    rng = np.random.default_rng(seed)
    spent, keys, units = 0.0, 0, 0
    while units == 0 or (spent < seconds and units < max_units):
        s = int(rng.integers(cfg.n_seq))
        l, h = int(rng.integers(cfg.n_layers)), int(rng.integers(cfg.n_kv_heads))
        N = int(lens[s])
        bits = synth.host_key_rows(cfg, centers, s, l, h, np.arange(N))
        k = O.bf16_bits_to_f64(bits)
        qc = re[l, h * G:(h + 1) * G].astype(np.float64) + 1j * im[l, h * G:(h + 1) * G]
        qa = am[l, h * G:(h + 1) * G].astype(np.float64)
        t0 = time.perf_counter()
        O.compress_unit(k, np.arange(N), N - 1, qc, qa, omega, cfg.pairing, cfg.budget,
                        cfg.window, cfg.sinks, cfg.offset_log2_max, form=form)
        spent += time.perf_counter() - t0
        keys += N
        units += 1
    return keys, spent, units


def oracle_rate(cfg_idx: int, form: str, seconds: float, workers: int, max_units: int = 64,
                seed: int = 0):
    """keys/s of the oracle on `workers` processes in parallel (the sum of
    their rates), with the sample it took."""
    tasks = [(cfg_idx, form, seconds, max_units, seed * 1000 + i) for i in range(workers)]
    if workers == 1:
        saved = _single_thread_env()
        try:
            res = [_oracle_units(tasks[0])]
        finally:
            _restore_env(saved)
    else:
        import multiprocessing as mp

        saved = _single_thread_env()
        try:
            with mp.get_context("spawn").Pool(workers) as pool:
                res = pool.map(_oracle_units, tasks)
        finally:
            _restore_env(saved)
    rate = sum(k / t for k, t, _ in res)
    units = sum(u for _, _, u in res)
    keys = sum(k for k, _, _ in res)
    return rate, {"units": units, "keys": keys, "cpu_seconds": round(sum(t for _, t, _ in res), 2)}


def cpu_baseline(args, cfg_main):
    """The fp64 oracle on the host cores: the folded form (Eq. 7) on every
    workload, and the direct 17-offset form (Eq. 4, the reference-style
    scorer) on the two smallest both on all cores and on one."""
    import synth

    cores = host_cores()
    per = max(2.0, args.cpu_seconds / 6)
    out = {"kind": "oracle", "cores": cores, "cpu_model": cpu_model(), "unit": UNIT,
           "workloads": {}}
    for ci in sorted(synth.CONFIGS):
        rate, smp = oracle_rate(ci, "folded", per, cores, seed=ci)
        out["workloads"][synth.CONFIGS[ci].name] = {
            "value": rate, "sample": f"{smp['units']} units ({smp['keys']} keys) on {cores} "
                                     f"processes, {smp['cpu_seconds']} CPU s, folded form + z-norm "
                                     f"+ selection"}
    direct = {}
    for ci in (0, 1):
        r_all, s_all = oracle_rate(ci, "direct", per / 2, cores, max_units=1, seed=10 + ci)
        r_one, s_one = oracle_rate(ci, "direct", per / 2, 1, max_units=1, seed=20 + ci)
        direct[synth.CONFIGS[ci].name] = {"all_cores": r_all, "one_core": r_one,
                                           "sample": f"{s_all['units']} units on {cores} processes; "
                                                     f"{s_one['units']} unit on one",
                                           "unit": UNIT}
    out["direct_form"] = direct
    main = out["workloads"][cfg_main.name]
    out["value"] = main["value"]
    out["sample"] = main["sample"]
    return out


def _ref_worker(conn, cfg_idx, unit, form):
    """Reference-arm worker: prepares one unit's inputs (the oracle's fp64 key
    rows and statistics), then runs the oracle on it once per "go"."""
    import synth
    from oracle import tria_oracle as O

    cfg = synth.CONFIGS[cfg_idx]
    re, im, am = synth.make_stats(cfg)
    centers = synth.make_centers(cfg)
    omega = O.band_frequencies(cfg.head_dim, cfg.theta)
    G = cfg.group
    s, l, h = unit
    N = int(synth.seq_lengths(cfg)[s])
    k = O.bf16_bits_to_f64(synth.host_key_rows(cfg, centers, s, l, h, np.arange(N)))
    qc = re[l, h * G:(h + 1) * G].astype(np.float64) + 1j * im[l, h * G:(h + 1) * G]
    qa = am[l, h * G:(h + 1) * G].astype(np.float64)
    conn.send(N)
    while conn.recv() is not None:
        O.compress_unit(k, np.arange(N), N - 1, qc, qa, omega, cfg.pairing, cfg.budget,
                        cfg.window, cfg.sinks, cfg.offset_log2_max, form=form)
        conn.send(N)
    conn.close()


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle (folded form, z-norm, selection) on
    the host cores, one process per core.  Each process holds one unit of the
    workload (its inputs prepared before timing); a step runs every process's
    unit once, and the timed region covers only those runs."""
    import multiprocessing as mp

    import synth

    if rank != 0:
        return 0
    cfg = synth.CONFIGS[args.config]
    cores = host_cores()
    rng = np.random.default_rng(7)
    units = [(int(rng.integers(cfg.n_seq)), int(rng.integers(cfg.n_layers)),
              int(rng.integers(cfg.n_kv_heads))) for _ in range(cores)]
    ctx = mp.get_context("spawn")
    saved = _single_thread_env()  # inherited by the workers: one thread each
    try:
        pipes, procs = [], []
        for u in units:
            a, b = ctx.Pipe()
            pr = ctx.Process(target=_ref_worker, args=(b, args.config, u, "folded"), daemon=True)
            pr.start()
            pipes.append(a)
            procs.append(pr)
    finally:
        _restore_env(saved)
    n_keys = [c.recv() for c in pipes]

    def step():
        for c in pipes:
            c.send(1)
        for c in pipes:
            c.recv()

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    wall = time.perf_counter() - t0
    for c in pipes:
        c.send(None)
    for pr in procs:
        pr.join(timeout=10)
    keys_per_step = sum(n_keys)
    value = keys_per_step * args.steps / wall
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wall / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_desc(cfg),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"{cores} units x {args.steps} steps ({keys_per_step} keys per "
                                   f"step, G={cfg.group}) on {cores} processes, fp64 numpy, folded "
                                   "form + z-norm + selection; inputs prepared before timing"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def rank_config(base, rank: int):
    """Weak scaling: every rank compresses its own sequence of the workload
    (same shape, its own seed); no data crosses ranks."""
    return base.scaled(seed=base.seed + 1000 * rank)


def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time (all ranks call it in the same order)."""
    import torch

    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def config_desc(cfg, extra=None):
    import synth

    k_gb = float(np.sum(synth.seq_lengths(cfg))) * cfg.n_layers * cfg.n_kv_heads * cfg.head_dim * 2 / 1e9
    d = {"workload": cfg.name, "layers": cfg.n_layers, "q_heads": cfg.n_q_heads,
         "kv_heads": cfg.n_kv_heads, "head_dim": cfg.head_dim, "seq_len": cfg.seq_len,
         "n_seq": cfg.n_seq, "budget": cfg.budget, "window": cfg.window, "sinks": cfg.sinks,
         "pairing": "neox" if cfg.pairing == 0 else "interleaved", "theta": cfg.theta,
         "offsets": f"2^0..2^{cfg.offset_log2_max}",
         "l2": (f"inputs ({k_gb:.1f} GB of K) larger than L2, plus a 256 MB L2 flush before each pass"
                if k_gb > 0.126 else
                f"inputs ({k_gb * 1e3:.0f} MB of K) fit in L2; a 256 MB L2 flush before each pass"),
         "restore": "rows overwritten by compaction restored between passes, outside the "
                    "per-pass CUDA events"}
    if extra:
        d["sample"] = extra
    return d


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tria", choices=["tria", "reference"])
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-extras", action="store_true", help="skip e2e, run16 and CPU baseline")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (small profiling cases)")
    ap.add_argument("--only-extra", default="",
                    choices=["", "decode_attention", "offset_max", "layer_budgets", "calibration",
                             "workload"],
                    help="after the warm-up passes run just this extra and print its result "
                         "(profiling of one kernel on a small case)")
    ap.add_argument("--seqs", type=int, default=0,
                    help="with --only-extra workload: override the workload's sequence count")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    local = _env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist

    import key_retention_scoring_b200 as T
    import synth
    from key_retention_scoring_b200 import build as tria_build

    torch.cuda.set_device(local)
    if args.only_extra == "workload":
        # one pass of a workload shape (any layout), optionally cut to fewer
        # layers / sequences: the `workloads` measurement on a small case
        tria_build.build()
        synth.build()
        wcfg = synth.CONFIGS[args.config]
        if args.layers:
            wcfg = wcfg.scaled(n_layers=args.layers)
        if args.seqs:
            wcfg = wcfg.scaled(n_seq=args.seqs)
        hbm, _ = peaks()
        res = workload_pass(T, torch, args.config, hbm, cfg=wcfg)
        if rank == 0:
            print(json.dumps({"extra": "workload", "config": config_desc(wcfg), **res}), flush=True)
        return 0
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    tria_build.build()
    synth.build()

    base = synth.CONFIGS[args.config]
    if args.layers:
        base = base.scaled(n_layers=args.layers)
    cfg = rank_config(base, rank)
    w = synth.Workload(cfg)
    re, im, am = w.stats
    st = T.tria_load_stats(T.model_desc(cfg.n_layers, cfg.n_q_heads, cfg.n_kv_heads, cfg.pairing,
                                        cfg.theta, cfg.offset_log2_max), re, im, am)
    cache = T.Cache.from_workload(w)
    prm = T.params(cfg.budget, cfg.window, cfg.sinks)
    ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
    T.tria_read_device_status(ws)
    B = cfg.budget
    kept = torch.empty((cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, B), dtype=torch.int32,
                       device="cuda")
    # backups of what compaction overwrites
    kb = [t[:, :, :B].clone() for t in w.k]
    vb = [t[:, :, :B].clone() for t in w.v]
    pb = w.positions[..., :B].clone()
    lens0 = w.seq_lens.clone()
    qpos0 = w.query_pos.clone()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def restore():
        for l in range(cfg.n_layers):
            w.k[l][:, :, :B].copy_(kb[l])
            w.v[l][:, :, :B].copy_(vb[l])
        w.positions[..., :B].copy_(pb)
        w.seq_lens.copy_(lens0)
        w.query_pos.copy_(qpos0)
        flush.zero_()

    stream = torch.cuda.current_stream()

    def timed_pass():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        T.tria_set_pass_events(evs)
        T.tria_compress_pass(st, cache, prm, kept, ws, stream=stream)
        T.tria_set_pass_events(None)
        return evs

    for _ in range(args.warmup):
        restore()
        timed_pass()
    torch.cuda.synchronize()
    if T.tria_read_device_status(ws) != 0:
        raise RuntimeError("device status flags set")
    if args.only_extra:
        hbm, _ = peaks()
        run = {"decode_attention": lambda: decode_attention(T, torch, w, st, cache, prm, ws, kept,
                                                            restore, cfg, hbm),
               "offset_max": lambda: offset_max(T, torch, st, cache, cfg, kept, restore, hbm),
               "layer_budgets": lambda: layer_budgets(T, torch, w, st, cfg, restore, hbm),
               "calibration": lambda: calibration(T, torch, hbm)}[args.only_extra]
        res = run()
        st.free()
        if rank == 0:
            print(json.dumps({"extra": args.only_extra, "config": config_desc(cfg), **res}), flush=True)
        return 0
    # moved rows of one pass (for the compaction bytes)
    kh = kept.cpu().numpy()
    moved = int(np.sum(kh != np.arange(B)[None, None, None, :]))

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    all_evs = []
    with ClockSampler(local) as clk:
        br0 = torch.cuda.Event(enable_timing=True)
        br1 = torch.cuda.Event(enable_timing=True)
        br0.record()
        for _ in range(args.steps):
            restore()
            all_evs.append(timed_pass())
        br1.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    seg = split_events(all_evs)
    ms = seg["pass"]
    if world > 1:
        ms = max_over_ranks(ms, dist, "cuda")

    N = cfg.seq_len
    units = cfg.n_seq * cfg.n_layers * cfg.n_kv_heads
    keys = units * N
    C = N - cfg.window - cfg.sinks
    k_bytes = units * C * 256
    compact_bytes = moved * 1024
    hbm, peak_kind = peaks()
    score_ms = seg["score"]
    line = {
        "metric": METRIC, "value": keys * world / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_desc(cfg),
        "numerics": "bf16 K/V cache; scores accumulate in fp32 (tensor cores, bf16 hi/lo "
                    "operands), moments in fp64, selection on fp32 agg",
        "us_per_pass": ms * 1e3,
        "keys_per_s_per_query_head": keys * world * cfg.group / (ms * 1e-3),
        "kernels_us": {"coef": 1e3 * seg["coef"], "score": 1e3 * score_ms,
                       "normalize_select": 1e3 * seg["select"], "compact": 1e3 * seg["compact"]},
        # the dominant kernel: scoring; its algorithmic bytes are the K rows
        # it reads once
        "roofline": {"bound": "hbm",
                     "kernel": "score_tc_kernel (scores of every candidate key)",
                     "achieved": k_bytes / (score_ms * 1e-3) / 1e9, "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": k_bytes / (score_ms * 1e-3) / 1e9 / hbm,
                     "traffic": recorded_traffic("score_kernel"), "algorithmic_bytes": k_bytes,
                     "pass": pass_roofline(k_bytes, compact_bytes, ms, hbm)},
        "pass_roofline": pass_roofline(k_bytes, compact_bytes, ms, hbm),
        "compact_roofline": {
            "kernel": "compact_kernel", "achieved": compact_bytes / (seg["compact"] * 1e-3) / 1e9,
            "peak": hbm, "unit": "GB/s",
            "frac": compact_bytes / (seg["compact"] * 1e-3) / 1e9 / hbm,
            "algorithmic_bytes": compact_bytes, "moved_rows": moved},
        "bracket_ms_per_step": br0.elapsed_time(br1) / args.steps,
        "clocks": clk.summary(),
        # coefficients, scoring, normalize-then-max + selection, compaction
        "gpu_launches": 4 * args.steps,
    }

    if not args.no_extras:
        line["decode_attention"] = decode_attention(T, torch, w, st, cache, prm, ws, kept, restore,
                                                    cfg, hbm)
        line["run16"] = run16(T, w, st, cache, prm, ws, kept, restore, hbm)
        line["calibration"] = calibration(T, torch, hbm)
        line["offset_max"] = offset_max(T, torch, st, cache, cfg, kept, restore, hbm)
        line["layer_budgets"] = layer_budgets(T, torch, w, st, cfg, restore, hbm)
        line["e2e"] = e2e(T, torch, w, st, cache, prm, ws, kept, restore, args.e2e_steps, keys, world)
        if world > 1:
            # the job's end-to-end time is the slowest rank's (every rank
            # takes this collective)
            ms_e2e = max_over_ranks(line["e2e"]["ms_per_step"], dist, "cuda")
            line["e2e"]["ms_per_step"] = ms_e2e
            line["e2e"]["value"] = keys * world / (ms_e2e * 1e-3)
    T.tria_set_pass_events(None)
    st.free()
    del w, kb, vb, pb, ws, kept, cache, flush
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if not args.no_extras and world == 1:
        # the other workload shapes, each timed on its own (one GPU)
        line["workloads"] = {}
        for ci in (1, 4, 3):
            if ci == args.config:
                continue
            try:
                line["workloads"][synth.CONFIGS[ci].name] = workload_pass(T, torch, ci, hbm)
            except torch.cuda.OutOfMemoryError as e:
                line["workloads"][synth.CONFIGS[ci].name] = {"error": f"out of memory: {e}"}
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        if rank == 0:
            line["cpu_baseline"] = cpu_baseline(args, cfg)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def split_events(all_evs):
    """Mean per-kernel times (ms) of a list of tria_set_pass_events records:
    coefficients, scoring, normalize-then-max + selection, compaction, and
    the whole pass."""
    seg = [statistics.mean(e[k].elapsed_time(e[k + 1]) for e in all_evs) for k in range(4)]
    return {"coef": seg[0], "score": seg[1], "select": seg[2], "compact": seg[3],
            "pass": statistics.mean(e[0].elapsed_time(e[4]) for e in all_evs)}


def pass_roofline(k_bytes, compact_bytes, ms, hbm):
    """The whole pass against the HBM bandwidth: K rows read once plus the
    moved K/V rows read and written, over the pass time."""
    tot = k_bytes + compact_bytes
    return {"bound": "hbm", "achieved": tot / (ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": tot / (ms * 1e-3) / 1e9 / hbm, "algorithmic_bytes": tot, "k_bytes": k_bytes,
            "compact_bytes": compact_bytes, "us": ms * 1e3}


def workload_pass(T, torch, ci, hbm, passes=None, cfg=None):
    """One full compression pass of workload `ci` (the other shapes of the
    pages' workloads; `cfg`, when given, a cut-down instance of it), timed
    with the pass's own CUDA events.  Contiguous
    caches restore the rows compaction overwrites between passes; the paged
    batch (157.5 GB of K + V, no room for backups) is generated afresh
    before each pass, after a warm-up pass of the same kernels on a small
    instance of it."""
    import synth

    cfg = synth.CONFIGS[ci] if cfg is None else cfg
    paged = cfg.layout == synth.LAYOUT_PAGED
    passes = passes or (2 if paged else 5)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def load(wl):
        re, im, am = wl.stats
        return T.tria_load_stats(T.model_desc(wl.cfg.n_layers, wl.cfg.n_q_heads, wl.cfg.n_kv_heads,
                                              wl.cfg.pairing, wl.cfg.theta,
                                              wl.cfg.offset_log2_max), re, im, am)

    if paged:
        small = synth.Workload(cfg.scaled(n_layers=1, n_seq=2, len_range=(4096, 6000)),
                               with_positions=False)
        sst = load(small)
        scache = T.Cache.from_workload(small)
        sprm = T.params(small.cfg.budget, small.cfg.window, small.cfg.sinks)
        sws = T.alloc_workspace(T.tria_workspace_size(sst, scache, sprm))
        T.tria_compress_pass(sst, scache, sprm, None, sws)
        torch.cuda.synchronize()
        sst.free()
        del small, scache, sws
        torch.cuda.empty_cache()
    w = synth.Workload(cfg, with_positions=not paged)
    st = load(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks)
        ws_bytes = T.tria_workspace_size(st, cache, prm)
        ws = T.alloc_workspace(ws_bytes)
        T.tria_read_device_status(ws)
        B = cfg.budget
        kept = torch.empty((cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, B), dtype=torch.int32,
                           device="cuda")
        lens = w.seq_lens.clone()
        if not paged:
            kb = [t[:, :, :B].clone() for t in w.k]
            vb = [t[:, :, :B].clone() for t in w.v]
        zero = np.zeros(cfg.n_seq, dtype=np.int64)

        def reset():
            if paged:
                w._fill(zero.astype(np.int32), w.lens.astype(np.int32), zero)
            else:
                for l in range(cfg.n_layers):
                    w.k[l][:, :, :B].copy_(kb[l])
                    w.v[l][:, :, :B].copy_(vb[l])
            w.seq_lens.copy_(lens)
            flush.zero_()

        evs_all, moved = [], 0
        for i in range(passes + (0 if paged else 2)):
            reset()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            T.tria_set_pass_events(evs)
            T.tria_compress_pass(st, cache, prm, kept, ws)
            T.tria_set_pass_events(None)
            if paged or i >= 2:
                evs_all.append(evs)
        torch.cuda.synchronize()
        if T.tria_read_device_status(ws) != 0:
            raise RuntimeError(f"device status flags set ({cfg.name})")
        kh = kept.cpu().numpy()
        moved = int(np.sum((kh >= 0) & (kh != np.arange(B)[None, None, None, :])))
        seg = split_events(evs_all)
        ms = seg["pass"]
        lens_h = w.lens.astype(np.int64)
        units = cfg.n_layers * cfg.n_kv_heads
        keys = int(lens_h.sum()) * units
        comp = lens_h > B
        k_bytes = int(np.sum(lens_h[comp] - cfg.window - cfg.sinks)) * units * 256
        compact_bytes = moved * 1024
        out = {"workload": cfg.name, "us_per_pass": ms * 1e3, "keys_per_s": keys / (ms * 1e-3),
               "keys": keys, "passes": passes,
               "kernels_us": {"coef": 1e3 * seg["coef"], "score": 1e3 * seg["score"],
                              "normalize_select": 1e3 * seg["select"],
                              "compact": 1e3 * seg["compact"]},
               "roofline": {"bound": "hbm",
                            "kernel": "scoring (score_tc_kernel; score_grp_kernel for paged blocks "
                                      "of 128 rows over all KV heads)",
                            "achieved": k_bytes / (seg["score"] * 1e-3) / 1e9, "peak": hbm,
                            "unit": "GB/s",
                            "frac": k_bytes / (seg["score"] * 1e-3) / 1e9 / hbm,
                            "algorithmic_bytes": k_bytes},
               "pass_roofline": pass_roofline(k_bytes, compact_bytes, ms, hbm),
               "moved_rows": moved,
               "footprint_bytes": {"kv_cache": w.footprint_bytes(), "workspace": ws_bytes},
               "restore": "cache generated afresh before each pass" if paged else
                          "overwritten rows restored between passes, outside the events"}
        if paged:
            out["lengths"] = {"sum": int(lens_h.sum()), "min": int(lens_h.min()),
                              "max": int(lens_h.max())}
        return out
    finally:
        st.free()
        del w
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def calibration(T, torch, hbm, reps=5):
    """Calibration reduction (tria_calib_accumulate) of one Qwen3-32B-shape
    layer: 32768 pre-RoPE query tokens x 64 heads x 128 bf16 = 512 MB, larger
    than L2, generated on the device (seeded)."""
    hq, n = 64, 32768
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    q = (torch.randn((n, hq, 128), generator=g, device="cuda") + 0.5).to(torch.bfloat16)
    acc = torch.zeros((hq, 64, 3), dtype=torch.float64, device="cuda")
    desc = T.model_desc(1, hq, 8, T.PAIR_NEOX, 1e4)
    for _ in range(2):
        T.tria_calib_accumulate(desc, q, acc)
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        T.tria_calib_accumulate(desc, q, acc)
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ms = statistics.mean(ts)
    nbytes = n * hq * 128 * 2
    del q
    return {"workload": "one layer, 32768 tokens x 64 query heads x 128 (bf16, 512 MB)",
            "ms": ms, "tokens_per_s": n / (ms * 1e-3), "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "reps": reps}


def offset_max(T, torch, st, cache, cfg, kept, restore, hbm, passes=5):
    """The same pass with the maximum over the offsets instead of the folded
    mean (tria_params.offset_reduce = OFFSET_MAX): per-kernel CUDA-event
    times over `passes` passes, rows restored between them."""
    prm = T.params(cfg.budget, cfg.window, cfg.sinks, T.OFFSET_MAX)
    ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
    T.tria_read_device_status(ws)
    evs_all = []
    for i in range(passes + 2):
        restore()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        T.tria_set_pass_events(evs)
        T.tria_compress_pass(st, cache, prm, kept, ws)
        T.tria_set_pass_events(None)
        if i >= 2:
            evs_all.append(evs)
    torch.cuda.synchronize()
    if T.tria_read_device_status(ws) != 0:
        raise RuntimeError("device status flags set (max-over-offsets pass)")
    seg = [[e[k].elapsed_time(e[k + 1]) for e in evs_all] for k in range(4)]
    ms = statistics.mean(e[0].elapsed_time(e[4]) for e in evs_all)
    units = cfg.n_seq * cfg.n_layers * cfg.n_kv_heads
    C = cfg.seq_len - cfg.window - cfg.sinks
    score_ms = statistics.mean(seg[1])
    del ws
    return {"us_per_pass": 1e3 * ms, "keys_per_s": units * cfg.seq_len / (ms * 1e-3),
            "kernels_us": {"coef": 1e3 * statistics.mean(seg[0]), "score": 1e3 * score_ms,
                           "normalize_select": 1e3 * statistics.mean(seg[2]),
                           "compact": 1e3 * statistics.mean(seg[3])},
            "score_roofline": {"bound": "hbm", "achieved": units * C * 256 / (score_ms * 1e-3) / 1e9,
                               "peak": hbm, "unit": "GB/s",
                               "frac": units * C * 256 / (score_ms * 1e-3) / 1e9 / hbm},
            "score_tflops": units * C * 2.0 * 128 * (2 * 17 * cfg.group) / (score_ms * 1e-3) / 1e12,
            "passes": passes}


def layer_budgets(T, torch, w, st, cfg, restore, hbm, passes=5):
    """The same pass with per-layer budgets (tria_params.layer_budget_scales,
    linear from 0.5 to 1.5 over the layers, mean 1) and lengths per (sequence,
    layer) (tria_cache_view.layer_seq_lens): per-kernel CUDA-event times over
    `passes` passes, rows and lengths restored between them."""
    L = cfg.n_layers
    scales = [0.5 + l / max(1, L - 1) for l in range(L)]
    ll = torch.full((cfg.n_seq, L), cfg.seq_len, dtype=torch.int32, device="cuda")
    cache = T.Cache.from_workload(w, layer_seq_lens=ll)
    prm = T.params(cfg.budget, cfg.window, cfg.sinks, layer_budget_scales=scales)
    budgets, bmax = T.tria_layer_budgets(st, cache, prm)
    B = cfg.budget
    # rows past the default budget that this variant's compaction overwrites
    kx = [t[:, :, B:bmax].clone() for t in w.k]
    vx = [t[:, :, B:bmax].clone() for t in w.v]
    kept = torch.empty((cfg.n_seq, L, cfg.n_kv_heads, bmax), dtype=torch.int32, device="cuda")
    ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
    T.tria_read_device_status(ws)
    evs_all = []
    for i in range(passes + 2):
        restore()
        for l in range(L):
            w.k[l][:, :, B:bmax].copy_(kx[l])
            w.v[l][:, :, B:bmax].copy_(vx[l])
        ll.fill_(cfg.seq_len)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        T.tria_set_pass_events(evs)
        T.tria_compress_pass(st, cache, prm, kept, ws)
        T.tria_set_pass_events(None)
        if i >= 2:
            evs_all.append(evs)
    torch.cuda.synchronize()
    if T.tria_read_device_status(ws) != 0:
        raise RuntimeError("device status flags set (per-layer budgets pass)")
    if sorted(set(ll[0].cpu().tolist())) != sorted(set(budgets)):
        raise RuntimeError("per-layer lengths after the pass differ from the budgets")
    seg = [[e[k].elapsed_time(e[k + 1]) for e in evs_all] for k in range(4)]
    ms = statistics.mean(e[0].elapsed_time(e[4]) for e in evs_all)
    units = cfg.n_seq * L * cfg.n_kv_heads
    C = cfg.seq_len - cfg.window - cfg.sinks
    score_ms = statistics.mean(seg[1])
    kept_rows = cfg.n_seq * cfg.n_kv_heads * sum(budgets)  # every unit is compressed
    del ws, kx, vx
    return {"workload": f"scales 0.5 .. 1.5 linear over {L} layers (budgets {min(budgets)} .. "
                        f"{max(budgets)}), lengths per (sequence, layer)",
            "us_per_pass": 1e3 * ms, "keys_per_s": units * cfg.seq_len / (ms * 1e-3),
            "kernels_us": {"coef": 1e3 * statistics.mean(seg[0]), "score": 1e3 * score_ms,
                           "normalize_select": 1e3 * statistics.mean(seg[2]),
                           "compact_and_lengths": 1e3 * statistics.mean(seg[3])},
            "score_roofline": {"bound": "hbm", "achieved": units * C * 256 / (score_ms * 1e-3) / 1e9,
                               "peak": hbm, "unit": "GB/s",
                               "frac": units * C * 256 / (score_ms * 1e-3) / 1e9 / hbm},
            "kept_rows": kept_rows, "passes": passes}


def decode_attention(T, torch, w, st, cache, prm, ws, kept, restore, cfg, hbm, reps=3):
    """Decode-step attention (tria_decode_attention) of every layer with
    seeded decode queries at the next position: over the full cache, and over
    the cache one compression pass pruned to the budget.  Per-layer time is
    the mean over all layers run back to back from one CUDA graph (the
    layers' K and V together exceed L2).  Also the share of each head's full-cache attention mass that
    the kept rows hold, on sampled layers, next to a random kept set of the
    same size (window included)."""
    import synth

    L, S, Hq, Hkv, G = cfg.n_layers, cfg.n_seq, cfg.n_q_heads, cfg.n_kv_heads, cfg.group
    N, B, W = cfg.seq_len, cfg.budget, cfg.window
    pos = w.query_pos.cpu().numpy() + 1
    qs = [torch.from_numpy(synth.decode_queries(cfg, l, pos).view(np.int16)).cuda()
          .view(torch.bfloat16) for l in range(L)]
    scale = 1.0 / math.sqrt(128.0)
    out = torch.empty((S, Hq, 128), device="cuda")
    dws = T.alloc_workspace(T.tria_decode_workspace_size(st, cache))
    T.tria_read_device_status(dws)

    def per_layer_us():
        # the layers' launches captured once in a CUDA graph (a decode step
        # replays it), then replayed `reps` times
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for l in range(L):
                T.tria_decode_attention(st, cache, l, qs[l], scale, out, dws)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for l in range(L):
                T.tria_decode_attention(st, cache, l, qs[l], scale, out, dws)
        graph.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(1e3 * a.elapsed_time(b) / L)
        del graph
        return statistics.mean(ts)

    restore()
    torch.cuda.synchronize()
    sample = sorted({0, L // 3, 2 * L // 3, L - 1})
    zbuf = torch.empty((S, Hq, w.max_seq_len), device="cuda")
    full_z = {}
    for l in sample:
        T.tria_decode_attention(st, cache, l, qs[l], scale, out, dws, logits=zbuf)
        full_z[l] = zbuf[:, :, :N].cpu().numpy().astype(np.float64)
    full_us = per_layer_us()
    T.tria_compress_pass(st, cache, prm, kept, ws)
    torch.cuda.synchronize()
    pruned_us = per_layer_us()
    if T.tria_read_device_status(dws) != 0:
        raise RuntimeError("device status flags set (decode attention)")
    kh = kept.cpu().numpy()
    rng = np.random.default_rng(0)
    rec, rnd = [], []
    for l in sample:
        for s in range(S):
            for h in range(Hkv):
                z = full_z[l][s, h * G:(h + 1) * G]
                p = np.exp(z - z.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                rec.append(float(p[:, kh[s, l, h]].sum(axis=1).mean()))
                r = np.concatenate([rng.choice(N - W, B - W, replace=False), np.arange(N - W, N)])
                rnd.append(float(p[:, r].sum(axis=1).mean()))
    restore()
    torch.cuda.synchronize()
    full_bytes = S * Hkv * N * 512
    pruned_bytes = S * Hkv * B * 512
    del dws, zbuf
    return {"workload": f"one decode query per sequence and query head, every layer, over {N} rows "
                        f"(full) and {B} rows (pruned) per KV head",
            "full_us_per_layer": full_us, "pruned_us_per_layer": pruned_us,
            "full_roofline": {"bound": "hbm", "kernel": "decode_kernel",
                              "achieved": full_bytes / (full_us * 1e-6) / 1e9, "peak": hbm,
                              "unit": "GB/s", "frac": full_bytes / (full_us * 1e-6) / 1e9 / hbm,
                              "algorithmic_bytes": full_bytes},
            "pruned_gbs": pruned_bytes / (pruned_us * 1e-6) / 1e9,
            "attention_mass_kept": statistics.mean(rec),
            "attention_mass_random_same_size": statistics.mean(rnd),
            "sampled_layers": sample, "reps": reps}


def run16(T, w, st, cache, prm, ws, kept, restore, hbm):
    """The decode run: a first pass at 32K, then 15 passes each after 128
    appended tokens (append excluded from the pass times).  The steady
    passes see N = budget + 128 rows per unit: their algorithmic bytes are
    the candidates' K rows plus the moved K/V rows (read and written)."""
    import torch

    restore()
    torch.cuda.synchronize()
    cfg = w.cfg
    B = cfg.budget
    units = cfg.n_seq * cfg.n_layers * cfg.n_kv_heads
    pass_us, append_ms, moved, kbytes = [], [], [], []
    for i in range(16):
        if i:
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            w.append(128)
            a1.record()
            torch.cuda.synchronize()
            append_ms.append(a0.elapsed_time(a1))
        n = int(w.seq_lens[0].item())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        T.tria_compress_pass(st, cache, prm, kept, ws)
        e1.record()
        torch.cuda.synchronize()
        pass_us.append(1e3 * e0.elapsed_time(e1))
        kh = kept.cpu().numpy()
        moved.append(int(np.sum((kh >= 0) & (kh != np.arange(B)[None, None, None, :]))))
        kbytes.append(units * (n - cfg.window - cfg.sinks) * 256)
    w.next_pos = w.lens.astype(np.int64).copy()
    restore()
    steady_us = statistics.mean(pass_us[1:])
    steady_bytes = statistics.mean(kb + 1024 * m for kb, m in zip(kbytes[1:], moved[1:]))
    return {"first_pass_us": pass_us[0], "steady_pass_us_mean": steady_us,
            "steady_keys_per_pass": int(units * (B + 128)),
            "steady_moved_rows_mean": statistics.mean(moved[1:]),
            "steady_roofline": {"bound": "hbm", "algorithmic_bytes": steady_bytes,
                                "achieved": steady_bytes / (steady_us * 1e-6) / 1e9, "peak": hbm,
                                "unit": "GB/s",
                                "frac": steady_bytes / (steady_us * 1e-6) / 1e9 / hbm},
            "total_pass_ms": sum(pass_us) / 1e3, "append_ms_mean": statistics.mean(append_ms)}


def e2e(T, torch, w, st, cache, prm, ws, kept, restore, steps, keys, world):
    """Same metric through the C ABI with host buffers: every step copies the
    K, V and positions of the cache from pinned host memory, runs the pass and
    reads the kept lists back."""
    restore()
    torch.cuda.synchronize()
    hk = [t.cpu().pin_memory() for t in w.k]
    hv = [t.cpu().pin_memory() for t in w.v]
    hp = w.positions.cpu().pin_memory()
    hl = w.seq_lens.cpu().pin_memory()
    hq = w.query_pos.cpu().pin_memory()
    hkept = torch.empty(kept.shape, dtype=kept.dtype).pin_memory()
    h2d = sum(t.numel() * 2 for t in hk) + sum(t.numel() * 2 for t in hv) + hp.numel() * 4 \
        + hl.numel() * 4 + hq.numel() * 8
    d2h = hkept.numel() * 4
    times = []
    for i in range(steps + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for l in range(len(hk)):
            w.k[l].copy_(hk[l], non_blocking=True)
            w.v[l].copy_(hv[l], non_blocking=True)
        w.positions.copy_(hp, non_blocking=True)
        w.seq_lens.copy_(hl, non_blocking=True)
        w.query_pos.copy_(hq, non_blocking=True)
        T.tria_compress_pass(st, cache, prm, kept, ws)
        hkept.copy_(kept, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        if i:
            times.append(e0.elapsed_time(e1))
    ms = statistics.mean(times)
    del hk, hv, hp
    return {"value": keys * world / (ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "steps": steps}


if __name__ == "__main__":
    sys.exit(main())
