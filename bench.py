"""Benchmark of the e-means hot path on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload emb768] [--impl ours|reference]

A step is one mini-batch step of training: gather in the per-pass order, fused
nearest-centroid search, grouping by label with segmented sums and the EMA
update, and every 5th step the revival check (runs restart with a fresh begin
when they end, finalize included). `value` is points assigned per second over the
K timed steps with the training matrix resident in HBM (fp32, cast to the bf16
search copy inside each begin). Under torchrun every rank trains its own replica
on its own GPU (no data-path collective); the time is the max over ranks.

Extra keys: roofline (the assignment kernel against the measured bf16 peak, from
CUDA events around every assignment launch inside the timed region), e2e (the same
metric through em_train with a pinned host matrix: host->device copy, training,
centroid read-back), cpu_baseline (the fp64 oracle on a bounded sample, rank 0 at
N = 1), lloyd25 (wall-clock and epochs to the test MSE of 25 Lloyd iterations).
--impl reference times the fp64 oracle on the host cores instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "pts assigned/s & wall-clock to Lloyd-25 test MSE, 1M×768 k=4096, 1×B200"
UNIT = "pts/s"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def workload_desc(w):
    return (f"{w.name}: n={w.n_train:,} train + {w.n_test:,} test, d={w.d}, k={w.k:,}, {w.epochs:g} epochs, "
            f"{w.storage} storage / bf16 search; {w.recipe}")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.2)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- the fp64 oracle on the host

def oracle_step(O, xb, c, N, S, k, t, rec, spherical):
    """One oracle mini-batch step: search, per-cluster statistics, EMA update (and
    the rescaling to norm 1 of spherical e-means)."""
    cq = O.search_copy_of_centroids(c)
    labels = (O.assign_dot(xb, cq) if spherical else O.assign(xb, cq))[0]
    n_j, s_j = O.batch_stats(xb, labels, k)
    N, S, c = O.ema_update(N, S, c, n_j, s_j, O.alpha_at(t, rec["total_steps"], rec["alpha0"]))
    return N, S, (O.unit_rows(c) if spherical else c)


def oracle_sample_rate(w, xt_dev, seconds, rows_per_step=None, log_prefix="cpu", spherical=False):
    """Times oracle mini-batch steps (search + statistics + EMA update) on the
    first batches of pass 0, copied to the host. Returns (pts/s, sample text, threads)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import emeans_oracle as O

    rec = O.recipe(w.n_train, w.k, w.epochs)
    B = rec["batch_size"] if rows_per_step is None else int(rows_per_step)
    order = O.pass_order(w.n_train, 1234, 0)
    start_rows = O.starting_rows(w.n_train, w.k, 1234)
    import torch

    idx = torch.from_numpy(start_rows).to(xt_dev.device)
    c = O.search_copy_of_data(xt_dev.index_select(0, idx).float().cpu().numpy())
    if spherical:
        c = O.unit_rows(c)
    N = np.zeros(w.k)
    S = np.zeros((w.k, w.d))
    t_total, rows_total, steps = 0.0, 0, 0
    # the batches of pass 0 (a full batch each, the last one possibly shorter)
    while t_total < seconds and steps < rec["total_steps"] and steps * B < w.n_train:
        ids = torch.from_numpy(order[steps * B:(steps + 1) * B]).to(xt_dev.device)
        xb = O.search_copy_of_data(xt_dev.index_select(0, ids).float().cpu().numpy())
        t0 = time.perf_counter()
        N, S, c = oracle_step(O, xb, c, N, S, w.k, steps, rec, spherical)
        t_total += time.perf_counter() - t0
        rows_total += len(xb)
        steps += 1
        log(f"[{log_prefix}] oracle step {steps}: {len(xb)} rows, {t_total:.1f} s so far")
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    sample = (f"{steps} oracle steps, {rows_total} rows in all (batches of up to {B}; search against all {w.k} "
              f"centroids, per-cluster sums, EMA update{', spherical' if spherical else ''}) from pass 0 of "
              f"{w.name}; {t_total:.3g} s of host time")
    return rows_total / t_total, sample, threads


# ---------------------------------------------------------------- our arm

class stdout_to_stderr:
    """Sends what native code writes to stdout (NCCL prints its version when a
    communicator is created) to stderr, so that stdout carries only the JSON line."""

    def __enter__(self):
        sys.stdout.flush()
        self.saved = os.dup(1)
        os.dup2(2, 1)
        return self

    def __exit__(self, *exc):
        sys.stdout.flush()
        os.dup2(self.saved, 1)
        os.close(self.saved)
        return False


def dp_join(em, m, world):
    """Data-parallel mode for model m: the torch.distributed group's ranks, or one rank."""
    with stdout_to_stderr():
        if world > 1:
            m.dp_init()
        else:
            m.dp_init_id(1, 0, em.dp_unique_id())


def reduce_over_ranks(ms, rows, device, world):
    """The job's time is the slowest rank's; its rows are every rank's."""
    if world <= 1:
        return ms, rows
    import torch

    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    r = torch.tensor([rows], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(r)
    return float(t.item()), int(r.item())


def step_rows(rec, n_train, s):
    """Rows that step s of a run (0-based, over all passes) processes: a full batch,
    or what is left of its pass for a pass's last step."""
    B, full = rec["batch_size"], rec["steps_full_pass"]
    p = s // full
    rows_pass = rec["rows_last_pass"] if p == rec["passes"] - 1 else n_train
    return min(B, rows_pass - (s - p * full) * B)


def run_ours(args, rank, world):
    import torch

    import datagen
    import mini_ema_means_b200 as em

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    t0 = time.time()
    # replicas train on the same rows; data-parallel ranks each hold their own
    w, xt, xs = datagen.make(args.workload, device=dev, seed=rank if args.dp else 0)
    torch.cuda.synchronize()
    log(f"[rank {rank}] data {w.name} ready in {time.time() - t0:.1f} s")
    stream = torch.cuda.current_stream(dev)
    m = em.Model(w.d, w.k, seed=1234, spherical=int(args.spherical), prefetch=args.prefetch,
                 search_format=args.search, pdl=args.pdl)
    m.set_stream(stream.cuda_stream)
    if args.dp:
        dp_join(em, m, world)
    m.set_option("input_dtype", 1 if w.storage == "bf16" else 0)
    rec = m.begin(xt, epochs=w.epochs)
    total = rec["total_steps"]

    # bookkeeping without synchronising: steps left in the current run on the host side
    state = {"in_run": 0}

    def steps_loop(K):
        done = 0
        rows = 0
        while done < K:
            left = total - state["in_run"]
            take = min(left, K - done)
            m.step(take)
            for s in range(state["in_run"], state["in_run"] + take):
                rows += step_rows(rec, w.n_train, s)
            state["in_run"] += take
            done += take
            if state["in_run"] >= total:
                m.finalize()
                m.begin(xt, epochs=w.epochs)
                state["in_run"] = 0
        return rows

    # warm-up (untimed)
    steps_loop(args.warmup)
    torch.cuda.synchronize()

    def timed_pass(profile):
        """K steps from a fresh begin between barriers and device syncs; returns (ms, rows)."""
        m.finalize()
        m.begin(xt, epochs=w.epochs)
        state["in_run"] = 0
        m.set_option("profile", 1 if profile else 0)
        m.profile(reset=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        rows = steps_loop(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        return e0.elapsed_time(e1), rows

    # the timed schedule once, untimed: every step range it asks for is captured as a
    # CUDA graph here, so that the timed pass only replays graphs
    timed_pass(profile=False)
    # pass 1: the headline number (step graphs replayed, no per-launch events)
    sampler = ClockSampler(dev.index)
    sampler.start()
    ms, rows = timed_pass(profile=False)
    clocks = sampler.stop()
    launches = m.profile(reset=True)["launches"]
    # pass 2: the same K steps with CUDA events around every phase of every step
    # (graphs are bypassed while profiling): per-kernel durations for the roofline
    ms_prof, _ = timed_pass(profile=True)
    prof = m.profile(reset=True)
    m.set_option("profile", 0)
    ms_max, rows_all = reduce_over_ranks(ms, rows, dev, world)
    if args.dp:  # every rank counted the rows of the whole batch
        rows_all = rows
    value = rows_all / (ms_max / 1e3)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if args.search == "fp8" else "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w), "method": "spherical e-means" if args.spherical else "e-means",
                   "search": args.search,
                   "batch_size": rec["batch_size"], "alpha0": round(rec["alpha0"], 6), "prefetch": args.prefetch,
                   "pdl": args.pdl,
                   "steps_per_run": total,
                   "l2": ("inputs larger than L2: the fp32 training matrix (%.2f GB) and its bf16 copy are re-read "
                          "in a fresh random order every pass" % (w.n_train * w.d * 4 / 1e9)
                          if w.n_train * w.d * 4 > L2_BYTES else
                          "inputs fit in L2 (the fp32 training matrix is %.1f MB) and L2 is not flushed between "
                          "steps" % (w.n_train * w.d * 4 / 1e6)),
                   "parallelism": (f"data-parallel dp{world} (NCCL all-reduce of the batch statistics)" if args.dp
                                   else "replicas" if world > 1 else "single GPU")},
    }
    # roofline of the dominant kernel: the fused assignment (tensor-core bound)
    a_ms = prof["ms"]["assign"]
    a_n = max(prof["spans"]["assign"], 1)
    achieved = prof["assign_flops"] / (a_ms / 1e3) / 1e12 if a_ms > 0 else 0.0
    # an E4M3 contraction takes the measured bf16 peak x the nominal fp8 / bf16 ratio (4.5 / 2.25)
    ratio = 2.0 if args.search == "fp8" else 1.0
    peak = peaks["bf16_tflops"] * ratio
    out["roofline"] = {
        "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
        "frac": achieved / peak,
        "traffic": (args.traffic if args.traffic is not None
                    else ASSIGN_TRAFFIC.get(args.workload) if args.search == "bf16" else None),
        "kernel": ("k_assign_tc (tcgen05 e4m3 x e4m3 -> fp32, fused |c'|^2/2 add + row argmin)" if args.search == "fp8"
                   else "k_assign_tc (tcgen05 bf16 x bf16 -> fp32, fused |c|^2 (added, or folded into the MMAs "
                        "at d < 128) + row argmin)"),
        "peak_source": (f"{peaks['source']} bf16 burst x 2 (nominal e4m3 / bf16 ratio)" if args.search == "fp8"
                        else f"{peaks['source']} bf16 burst"),
        "frac_of_sustained": (achieved / (peaks["bf16_tflops_sustained"] * ratio)
                              if peaks.get("bf16_tflops_sustained") else None),
        "avg_launch_ms": a_ms / a_n,
        "launches": prof["spans"]["assign"],
        "measured_in": "second timed pass of the same K steps with CUDA events around every launch",
    }
    u_ms = prof["ms"]["update"]
    out["phases_ms"] = {k: round(v, 4) for k, v in prof["ms"].items()}
    out["profiled_pass_ms_per_step"] = ms_prof / args.steps
    out["update_roofline"] = {
        "bound": "hbm", "achieved": prof["update_bytes"] / (u_ms / 1e3) / 1e9 if u_ms > 0 else 0.0,
        "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": (prof["update_bytes"] / (u_ms / 1e3) / 1e9) / peaks["hbm_gbs"] if u_ms > 0 else 0.0,
    }
    # the profiled pass assigns the same rows as the timed one
    out["assign_only_pts_per_s"] = (rows / (a_ms / 1e3)) if a_ms > 0 else None
    out["epochs_per_s"] = value / w.n_train
    out["gpu_launches"] = launches
    out["clocks"] = clocks

    if rank == 0 and not args.no_extras:
        out["lloyd25"] = lloyd25(m, w, xt, xs, rec)
    if not args.no_e2e:
        out["e2e"] = e2e(em, w, xt, stream, world, dev, spherical=args.spherical, dp=args.dp, search=args.search)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # steps of a whole batch where one takes a few seconds of host time, else of
        # fewer rows (the oracle's cost per row is the same: a search over all k)
        rows = min(rec["batch_size"], max(1024, int(4e11 / (2.0 * w.k * w.d))))
        v, sample, threads = oracle_sample_rate(w, xt, args.cpu_seconds, rows_per_step=rows,
                                                spherical=args.spherical)
        run_rows = w.n_train * w.epochs
        out["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
                               "full_run_s_extrapolated": run_rows / v,
                               "full_run_note": f"{run_rows:.4g} rows of a whole {w.epochs:g}-epoch run at the "
                                                f"sampled rate (extrapolated, not timed)"}
    m.close()
    return out


def lloyd25(m, w, xt, xs, rec):
    """Test MSE of 25 Lloyd iterations from the same starting rows, then the first
    e-means checkpoint (every ceil(S/20) steps and at pass ends; evaluation time
    excluded) whose test MSE is at or below it."""
    import torch

    t0 = time.time()
    m.lloyd(xt, 25)
    target = m.mse(xs)
    lloyd_s = time.time() - t0
    total = rec["total_steps"]
    every = math.ceil(total / 20)
    full = rec["steps_full_pass"]
    stream = torch.cuda.current_stream()
    # one untimed pass over the same checkpoint schedule first, so that the timed
    # pass replays step graphs instead of capturing them
    for timed in (False, True):
        m.begin(xt, epochs=w.epochs)
        train_ms, steps, hit, eval_s = 0.0, 0, None, 0.0
        history = []
        if timed:
            break
        while steps < total:
            nxt = min(total, (steps // every + 1) * every, (steps // full + 1) * full)
            m.step(nxt - steps)
            steps = nxt
        m.finalize()
    while steps < total:
        nxt = min(total, (steps // every + 1) * every, (steps // full + 1) * full)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        m.step(nxt - steps)
        e1.record(stream)
        torch.cuda.synchronize()
        train_ms += e0.elapsed_time(e1)
        steps = nxt
        t_eval = time.perf_counter()
        mse = m.mse(xs)
        eval_s += time.perf_counter() - t_eval
        epochs = steps / full
        history.append((round(epochs, 4), mse))
        if hit is None and mse <= target:
            hit = {"seconds": train_ms / 1e3, "epochs": epochs, "test_mse": mse}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    m.finalize()
    e1.record(stream)
    torch.cuda.synchronize()
    train_ms += e0.elapsed_time(e1)
    final = m.mse(xs)
    if hit is None and final <= target:
        hit = {"seconds": train_ms / 1e3, "epochs": w.epochs, "test_mse": final}
    return {"lloyd25_test_mse": target, "lloyd25_wall_s": lloyd_s, "emeans_final_test_mse": final,
            "emeans_train_s": train_ms / 1e3, "evaluation_s_excluded": eval_s, "reached": hit is not None,
            "time_to_target_s": hit["seconds"] if hit else None, "epochs_to_target": hit["epochs"] if hit else None,
            "final_ratio": final / target, "checkpoints": history}


def e2e(em, w, xt, stream, world, dev, spherical=False, dp=False, search="bf16"):
    """em_train through the C ABI with a pinned host matrix: H2D copy, training and
    the centroid read-back inside the timed region, with the timed arm's method and
    search format."""
    import torch

    xh = xt.cpu().pin_memory()
    m = em.Model(w.d, w.k, seed=1234, spherical=int(spherical), search_format=search)
    m.set_stream(stream.cuda_stream)
    if dp:
        dp_join(em, m, world)
    cent = torch.empty(w.k, w.d).pin_memory()
    m.train(xh, epochs=w.epochs)  # warm-up run
    m.centroids(cent)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    m.train(xh, epochs=w.epochs)
    m.centroids(cent)
    torch.cuda.synchronize()
    sec = time.perf_counter() - t0
    r = m.recipe()
    rows = w.n_train * w.epochs
    if world > 1:
        t = torch.tensor([sec], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        sec = float(t.item())
        rows *= world
    m.close()
    steps = r["total_steps"]
    return {"value": rows / sec, "unit": UNIT,
            "h2d_bytes_per_step": xh.numel() * xh.element_size() / steps,
            "d2h_bytes_per_step": (w.k * w.d * 4) / steps,
            "what": f"em_train on a pinned host {'fp32' if xh.dtype == torch.float32 else 'bf16'} matrix (copied to "
                    f"the device inside the call) + centroid read-back, one whole {w.epochs:g}-epoch run, "
                    f"{search} search, host wall clock"}


# ---------------------------------------------------------------- reference arm (the oracle)

def run_reference(args):
    import torch

    import datagen

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w, xt, _ = datagen.make(args.workload, device=dev, seed=0)
    budget = args.ref_seconds
    # calibrate the rows of one step so that warm-up + timed steps fit the budget
    v0, _, _ = oracle_sample_rate(w, xt, 0.1, rows_per_step=512, log_prefix="ref-calibrate",
                                  spherical=args.spherical)
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import emeans_oracle as O

    rec = O.recipe(w.n_train, w.k, w.epochs)
    # at most one batch of the workload (and never more rows than it has)
    rows = int(max(1, min(rec["batch_size"], w.n_train, max(64, v0 * budget / max(args.steps + args.warmup, 1)))))
    order = O.pass_order(w.n_train, 1234, 0)
    start = O.starting_rows(w.n_train, w.k, 1234)
    c = O.search_copy_of_data(xt.index_select(0, torch.from_numpy(start).to(xt.device)).float().cpu().numpy())
    if args.spherical:
        c = O.unit_rows(c)
    N, S = np.zeros(w.k), np.zeros((w.k, w.d))

    def one(t):
        nonlocal N, S, c
        start = (t * rows) % (w.n_train - rows + 1)
        ids = order[start:start + rows]
        xb = O.search_copy_of_data(xt.index_select(0, torch.from_numpy(ids).to(xt.device)).float().cpu().numpy())
        t0 = time.perf_counter()
        N, S, c = oracle_step(O, xb, c, N, S, w.k, t, rec, args.spherical)
        return time.perf_counter() - t0, len(xb)

    for t in range(args.warmup):
        one(t)
    timed = [one(args.warmup + t) for t in range(args.steps)]
    sec = sum(x[0] for x in timed)
    assert all(x[1] == rows for x in timed)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    value = args.steps * rows / sec
    sample = (f"{args.steps} oracle steps of {rows} rows each from pass 0 of {w.name} (search against all "
              f"{w.k} centroids, per-cluster sums, EMA update)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "method": "spherical e-means" if args.spherical else "e-means",
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_kernel_case(args):
    """A small standalone case for profiler captures: `--kernel-case assign` runs the
    fused assignment twice on `--case-rows` rows of the workload (bf16, larger than
    L2) against k starting centroids; `--kernel-case step` runs `--steps` training
    steps of the full workload."""
    import torch

    import datagen
    import mini_ema_means_b200 as em

    torch.cuda.set_device(0)
    if args.kernel_case == "assign":
        w, xt, _ = datagen.make(args.workload, device="cuda", seed=0, n_train=args.case_rows, n_test=1)
        xb = xt.to(torch.bfloat16).contiguous()
        m = em.Model(w.d, w.k, seed=1234, input_dtype=1, search_format=args.search)
        m.set_state(c=xt[: w.k].float().contiguous())
        lab = torch.empty(w.n_train, dtype=torch.int64, device="cuda")
        for _ in range(2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            m.assign(xb, labels=lab)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            log(f"assign pass {w.n_train} x {w.k} x {w.d}: {ms:.3f} ms, "
                f"{2.0 * w.n_train * w.k * w.d / ms / 1e9:.1f} TFLOP/s (whole call)")
    else:
        rows = args.case_rows if args.case_rows_step else None
        w, xt, _ = datagen.make(args.workload, device="cuda", seed=0, n_train=rows, n_test=1 if rows else None)
        m = em.Model(w.d, w.k, seed=1234, search_format=args.search)
        if args.case_batch:
            m.set_option("batch_size", args.case_batch)
        m.begin(xt, epochs=w.epochs)
        m.step(args.steps)
        m.sync()
    m.close()
    print(json.dumps({"kernel_case": args.kernel_case, "workload": args.workload, "ok": True}))


def run_ablation(args):
    """Revival ablation on one workload: split, resample and none over several
    seeds. After training, a full assignment pass of the training rows counts each
    cluster's rows: unused clusters hold fewer than a tenth of the mean count;
    test MSE with the same centroids."""
    import torch

    import datagen
    import mini_ema_means_b200 as em

    torch.cuda.set_device(0)
    w, xt, xs = datagen.make(args.workload, device="cuda", seed=0)
    labels = torch.empty(w.n_train, dtype=torch.int64, device="cuda")
    out = {"ablation": args.workload, "seeds": args.ablation_seeds, "modes": {}}
    for mode in ("split", "resample", "none"):
        rows = []
        for seed in range(args.ablation_seeds):
            m = em.Model(w.d, w.k, seed=seed, revival=mode)
            m.set_option("input_dtype", 1 if w.storage == "bf16" else 0)
            m.train(xt, epochs=w.epochs)
            m.assign(xt, labels=labels)
            cnt = torch.bincount(labels, minlength=w.k)
            # unused: fewer rows than a tenth of the mean (the revival criterion);
            # empty: no row at all (a cluster never revived keeps its starting row,
            # which it always wins, so this one rarely moves)
            unused = int((cnt.double() < 0.1 * cnt.double().mean()).sum().item())
            empty = int((cnt == 0).sum().item())
            rows.append({"seed": seed, "unused": unused, "empty": empty, "test_mse": m.mse(xs),
                         "splits": m.stats()["n_splits"]})
            m.close()
            log(f"[ablation] {mode} seed {seed}: {rows[-1]}")
        out["modes"][mode] = {"runs": rows, "unused_mean": statistics.mean(r["unused"] for r in rows),
                              "empty_mean": statistics.mean(r["empty"] for r in rows),
                              "test_mse_mean": statistics.mean(r["test_mse"] for r in rows)}
    return out


L2_BYTES = 126e6  # the B200's L2 (126 MB)

# DRAM bytes per assignment launch of the bench's batch, from ncu captures of the
# current kernel (emb768: 262,144 rows; deep96: 1,048,576 rows, 205.8 MB read and
# 24.4 MB written), scaled to one 65,536-row batch by rows for the batch and the
# keys, with the centroid operand counted once.
ASSIGN_TRAFFIC = {"emb768": 109.6e6, "deep96": 18.6e6}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2400)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--workload", default="emb768")
    ap.add_argument("--spherical", action="store_true", help="spherical e-means (unit centroids, highest dot product)")
    ap.add_argument("--prefetch", type=int, default=1, choices=[0, 1],
                    help="gather the next step's rows on a second stream during the update (default 1)")
    ap.add_argument("--pdl", type=int, default=1, choices=[0, 1],
                    help="programmatic dependent launch of the step's kernels (default 1)")
    ap.add_argument("--search", default="bf16", choices=["bf16", "fp8"],
                    help="search format: bf16 copies (default) or FP8 E4M3 codes with a fitted converter")
    ap.add_argument("--dp", action="store_true",
                    help="data-parallel e-means: each rank holds its own rows, the per-batch statistics are added "
                         "with NCCL (default for several GPUs: independent replicas)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per assignment launch from an ncu capture of the current kernel")
    ap.add_argument("--kernel-case", choices=["assign", "step"], default=None)
    ap.add_argument("--case-rows", type=int, default=262144)
    ap.add_argument("--case-rows-step", action="store_true", help="train the step case on --case-rows rows")
    ap.add_argument("--case-batch", type=int, default=0, help="batch size of the step case (0: the recipe's)")
    ap.add_argument("--ablation", action="store_true", help="revival ablation (split / resample / none)")
    ap.add_argument("--ablation-seeds", type=int, default=5)
    args = ap.parse_args()
    if args.ablation:
        print(json.dumps(run_ablation(args)), flush=True)
        return
    if args.kernel_case:
        run_kernel_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime

        import torch

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        out = run_ours(args, rank, world)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch

            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
