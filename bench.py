"""Throughput of teacher-forced KL scoring on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step scores one window of full-vocabulary logits (2047 positions x
248,320 vocabulary ids, bf16, seeded synthetic Zipf/Gumbel rows) with
kld_full_vocab and reduces it with kld_reduce_stats (mean, median, p99,
p99.9, top-1, perplexity).  Inputs are resident in HBM and larger than L2
(2.03 GB per step).  With N GPUs (torchrun) every rank scores its own window
(weak scaling) and the step's statistics cover every rank's positions: the
reduction runs as shard steps with an all-gather of one small block per rank
between them, the only collective on the data path; the timing is the max
over ranks.  Rank 0 prints one JSON line.

--impl reference times the f64 CPU oracle on the same workload instead.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "scored positions/sec at V=248,320 (KL+top-1)"
UNIT = "positions/s"
N_ROWS = 2047
VOCAB = 248_320
QUANTILES = (0.5, 0.99, 0.999)
WORKLOAD = "one-window full-vocabulary scoring: 2047 positions x 248,320 vocab, bf16 logits"
PROFILE = os.path.join(ROOT, "profiles", "full_vocab_kernel_window_bf16.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "quantization_fidelity_scoring_b200", "csrc", f)
                  for f in ("full_vocab.cu", "kld_common.cuh", "stream_common.cuh")]


def kernel_digest() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    if not os.path.exists(PROFILE):
        return None
    vals = {}
    with open(PROFILE) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_digest") != kernel_digest():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """NVML clock / throttle-reason sampling on a background thread (read only)."""

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples = []  # (t, sm_mhz, reasons_bitmask)
        self._stop = threading.Event()
        self._th = None
        self.max_mhz = None
        self.ok = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._th = threading.Thread(target=self._run, daemon=True)
        self._th.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._th:
            self._th.join()

    def summary(self, t0: float, t1: float, t_load: float | None = None) -> dict:
        """Clocks over the timed region [t0, t1]; when it holds fewer than
        five samples, over the load window [t_load, t1] (warm-up steps and
        the timed region back to back) instead."""
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        use = inside
        if len(inside) < 5:
            use = [s for s in self.samples if (t_load if t_load is not None else t0) <= s[0] <= t1] or self.samples
        names = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}
        seen = set()
        for _, _, rs in use:
            for bit, name in names.items():
                if rs & bit:
                    seen.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in use]) if use else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(seen),
                "samples_in_timed_region": len(inside), "samples": len(use),
                "window": "timed region" if use is inside else "warm-up + timed region"}


def rank_env(default_world: int = 1):
    """(world size, rank, local rank) from the torchrun environment."""
    world = int(os.environ.get("WORLD_SIZE", str(default_world)))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def window_seed(rank: int) -> int:
    """Every rank scores its own window: distinct seeded inputs per rank."""
    from synth import workloads as W
    return W.seed_for(2) + 1000 * rank


def max_over_ranks(x: float, device, world: int) -> float:
    """The slowest rank's time (all ranks take part; a no-op for one rank)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(n_per_rank: int, world: int, steps: int, seconds: float) -> float:
    """Positions scored by all ranks per second of the slowest rank."""
    return n_per_rank * world * steps / seconds


def oracle_rows(ref, cand, targets, rows):
    """Run the f64 oracle on the given row indices (host copies) on this
    thread; returns seconds (exact bf16 -> f64 conversion included)."""
    import numpy as np
    import torch
    from oracle import kld_oracle as O
    idx = torch.as_tensor(rows, device=ref.device)
    xb = ref[idx].cpu().view(torch.int16).numpy().view(np.uint16)
    yb = cand[idx].cpu().view(torch.int16).numpy().view(np.uint16)
    T = targets[idx].cpu().numpy()
    t0 = time.perf_counter()
    res = O.full_vocab(O.bf16_bits_to_f64(xb), O.bf16_bits_to_f64(yb), T)
    O.reduce_stats(res["kl"], res["ref_argmax"], res["cand_argmax"], None, res["ref_target_lp"],
                   res["cand_target_lp"], quantiles=QUANTILES)
    return time.perf_counter() - t0


def cpu_baseline(ref, cand, targets, single_rows: int) -> dict:
    """The f64 oracle timed on the host: every row of the window over all
    cores (the reported value), and a sample of rows on one thread."""
    from oracle import kld_oracle as O
    from oracle.pool import OraclePool
    n = ref.shape[0]
    rows = list(range(0, n, max(1, n // single_rows)))[:single_rows]
    dt1 = oracle_rows(ref, cand, targets, rows)
    with OraclePool() as pool:
        staged = {"X": pool.stage("x", ref, "bf16"), "Y": pool.stage("y", cand, "bf16"),
                  "targets": pool.stage("t", targets, "int")}
        t0 = time.perf_counter()
        res = pool.run("full_vocab", staged, n)
        O.reduce_stats(res["kl"], res["ref_argmax"], res["cand_argmax"], None, res["ref_target_lp"],
                       res["cand_target_lp"], quantiles=QUANTILES)
        dt = time.perf_counter() - t0
        cores = pool.cores
    return {"value": n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"all {n} rows of the window (f64 numpy oracle + reductions), one process per core",
            "single_thread": {"value": round(len(rows) / dt1, 2), "cores": 1, "sample": f"{len(rows)} rows"}}


def run_reference(args) -> int:
    """Reference arm: the f64 oracle on the host's cores, a bounded sample of
    the window's rows per step, spread over one process per core."""
    import torch
    from oracle import kld_oracle as O
    from oracle.pool import OraclePool
    from synth import workloads as W
    world, rank, _ = rank_env(default_world=args.gpus)
    if rank != 0:
        return 0
    with OraclePool() as pool:          # spawned before the first CUDA call
        # inputs drawn on the GPU when there is one (same bytes as our arm), else on the host
        dev = torch.device("cuda:0") if torch.cuda.is_available() else torch.device("cpu")
        per_row_s = 0.012 / pool.cores
        rows_per_step = int(args.ref_seconds / ((args.steps + args.warmup) * per_row_s))
        rows_per_step = max(pool.cores, min(N_ROWS, rows_per_step))
        n_avail = min(N_ROWS, max(2 * rows_per_step, 64))
        d = W.window_full_vocab(seed=W.seed_for(2), device=dev, n_rows=n_avail)
        staged = {"X": pool.stage("x", d["ref"], "bf16"), "Y": pool.stage("y", d["cand"], "bf16"),
                  "targets": pool.stage("t", d["targets"], "int")}
        del d

        def step(i):
            a = (i * rows_per_step) % (n_avail - rows_per_step + 1)
            res = pool.run("full_vocab", staged, rows_per_step, start=a)
            O.reduce_stats(res["kl"], res["ref_argmax"], res["cand_argmax"], None, res["ref_target_lp"],
                           res["cand_target_lp"], quantiles=QUANTILES)

        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        for i in range(args.steps):
            step(i)
        dt = time.perf_counter() - t0
        cores = pool.cores
    value = rows_per_step * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Zipf/Gumbel logits; no corpus or model)",
        "config": config_dict(),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} rows of the window per step, f64 numpy oracle, "
                                   f"{cores} processes (one per host core)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(rows: int = N_ROWS, world: int = 1, pipelined: bool = False) -> dict:
    workload = WORKLOAD if rows == N_ROWS else WORKLOAD.replace("2047 positions", f"{rows} positions") + \
        " (reduced profiling case)"
    return {"workload": workload, "n_rows": rows, "vocab": VOCAB, "input_dtype": "bf16",
            "step": "kld_full_vocab + kld_reduce_stats (mean, p50/p99/p99.9, top-1, ppl)" +
                    ("; stats on a second stream, overlapping the next window" if pipelined else ""),
            "l2": f"inputs larger than L2: {2 * rows * VOCAB * 2 / 1e9:.2f} GB of logits per step",
            "parallelism": "dp (each rank scores its own window)" if world == 1 else
            f"dp{world}: each rank scores its own window; the statistics cover all ranks' positions "
            "(shard steps with an all-gather of one 16.5 KB block per rank and step)"}


def run_ours(args) -> int:
    import torch
    import torch.distributed as dist

    import quantization_fidelity_scoring_b200 as kq
    from synth import workloads as W

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    kq.load_library()

    d = W.window_full_vocab(seed=window_seed(rank), device=dev, n_rows=args.rows)
    ref, cand, targets = d["ref"], d["cand"], d["targets"]
    n = ref.shape[0]
    stream = torch.cuda.current_stream()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    fws = torch.empty(kq.kld_full_vocab_workspace_size(n), dtype=torch.uint8, device=dev)

    def outputs():
        return dict(kl=torch.empty(n, dtype=torch.float32, device=dev),
                    ra=torch.empty(n, dtype=torch.int32, device=dev),
                    ca=torch.empty(n, dtype=torch.int32, device=dev),
                    lpr=torch.empty(n, dtype=torch.float32, device=dev),
                    lpc=torch.empty(n, dtype=torch.float32, device=dev),
                    ws=torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev),
                    stats=torch.empty(280, dtype=torch.uint8, device=dev))

    # With one GPU the statistics of window i run on a second stream while
    # window i + 1 is scored: the per-position outputs are double-buffered,
    # and events keep a buffer from being rewritten before its statistics
    # have read it.  (--serial runs them one after the other.)
    pipelined = world == 1 and not args.serial
    bufs = [outputs(), outputs()] if pipelined else [outputs()]
    side = torch.cuda.Stream(device=dev) if pipelined else stream
    scored = [torch.cuda.Event(), torch.cuda.Event()]
    reduced = [torch.cuda.Event(), torch.cuda.Event()]
    for e in reduced:
        e.record(side)
    count = [0]

    if world > 1:
        from quantization_fidelity_scoring_b200 import shards
        sws = torch.empty(kq.kld_reduce_shard_workspace_size(n), dtype=torch.uint8, device=dev)

    def step(ev=None):
        i = count[0] % len(bufs)
        count[0] += 1
        o = bufs[i]
        if pipelined:
            stream.wait_event(reduced[i])  # this buffer's previous statistics are done
        if ev is not None:
            ev[0].record(stream)
        kq.kld_full_vocab(ref, cand, targets, kl=o["kl"], ref_argmax=o["ra"], cand_argmax=o["ca"],
                          ref_target_lp=o["lpr"], cand_target_lp=o["lpc"], workspace=fws, dev_status=status,
                          stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if world > 1:
            # the statistics of every rank's positions: shard steps with an
            # all-gather of each step's 16.5 KB block
            shards.reduce_stats_across_ranks(o["kl"], o["ra"], o["ca"], None, o["lpr"], o["lpc"], None, QUANTILES,
                                             (), out=o["stats"], workspace=sws, dev_status=status, to_host=False)
        else:
            if pipelined:
                scored[i].record(stream)
                side.wait_event(scored[i])
            kq.kld_reduce_stats(o["kl"], o["ra"], o["ca"], None, o["lpr"], o["lpc"], None, QUANTILES, (),
                                out=o["stats"], workspace=o["ws"], dev_status=status, stream=side, to_host=False)
            if pipelined:
                reduced[i].record(side)

    sampler = ClockSampler(local).start()
    # warm-up: at least W steps and about a second of load so the clocks settle
    t_w = time.perf_counter()
    i = 0
    while i < args.warmup or time.perf_counter() - t_w < 1.0:
        step()
        i += 1
        if i % 50 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()

    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start.record(stream)
    for s in range(args.steps):
        step(kev[s])
    stream.wait_stream(side)  # the last window's statistics are inside the timed region
    stop.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    sampler.stop()
    ms = start.elapsed_time(stop)
    k_ms = [a.elapsed_time(b) for a, b in kev]
    ms = max_over_ranks(ms, dev, world)
    assert status.item() == 0, f"device status {status.item()}"

    value = whole_job_rate(n, world, args.steps, ms / 1e3)

    # roofline of the dominant kernel (full-vocabulary pass)
    alg_bytes = 2 * n * VOCAB * 2 + n * (4 + 4 * 5)   # both logit rows, targets, five outputs
    # the dominant kernel is the streaming pass; the events bracket it and the
    # small piece-merge kernel that follows it
    k_avg_s = statistics.mean(k_ms) / 1e3
    achieved = alg_bytes / k_avg_s / 1e9
    peak, peak_kind = measured_peaks()
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": profiled_traffic(),
                "kernel": "kld::stream_kernel<bf16> + kld::merge_kernel<bf16>",
                "kernel_ms": round(statistics.mean(k_ms), 5),
                "peak_source": "measured hbm_gbs" if peak_kind == "measured" else "fallback 6.65 TB/s"}

    e2e = measure_e2e(args, kq, d, dev, world)

    clocks = sampler.summary(t0, t1, t_w)
    if clocks.get("sm_mhz"):
        # clock-normalised step time (ms x median SM MHz), comparable across runs
        clocks["ms_per_step_x_sm_mhz"] = round(ms / args.steps * clocks["sm_mhz"], 2)

    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded Zipf/Gumbel logits; no corpus or model)",
            "config": config_dict(args.rows, world, pipelined), "roofline": roofline,
            "clocks": clocks, "gpu_launches": launches_per_step(n, world) * args.steps,
            "e2e": e2e,
        }
        if world == 1 and not args.no_extra:
            # one GPU only: under torchrun the other ranks would wait at the
            # closing barrier, within the process group's timeout, meanwhile.
            # The latency-bound paths run before the seconds-long GEMM loop, whose
            # power-capped clocks would otherwise linger into their timing
            extra = {"topk_tail": measure_topk(args, kq, dev),
                     "sparse_ref": measure_sparse_ref(args, kq, dev),
                     "sparse_capture": measure_sparse_capture(args, kq, dev),
                     "paired": measure_paired(args, kq, dev),
                     "shared_head": measure_shared_head(args, kq, dev),
                     "batched_f32": measure_batched(args, kq, dev)}
            torch.cuda.empty_cache()
            # each path's full record on its own line; the headline (printed
            # last) carries a compact summary of every path
            for name, rec in extra.items():
                print(json.dumps({"extra_path": name, **rec}), flush=True)
            line["extra_paths"] = {name: compact_path(rec) for name, rec in extra.items()}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(ref, cand, targets, args.cpu_rows)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def compact_path(rec: dict) -> dict:
    """The figures of one extra path that the headline line keeps."""
    r = rec["roofline"]
    return {"value": round(rec["value"], 1), "unit": rec["unit"], "ms": round(rec["ms_per_step"], 4),
            "kernel_ms": round(r["kernel_ms"], 4), "bound": r["bound"], "frac": round(r["frac"], 3)}


def launches_per_step(n: int, world: int = 1) -> int:
    """Library kernels per step: streaming pass + piece merge + reduction
    (one CTA up to 8192 positions, else a clearing launch + one cooperative
    grid; across ranks the five shard steps: 3 + 3 x 3 + 2 kernels)."""
    if world > 1:
        return 2 + 14
    return 2 + (1 if n <= 8192 else 2)


def measure_topk(args, kq, dev, windows=512, steps=None) -> dict:
    """Top-64 + tail bucket on its full workload (512 windows x 2047
    positions): kld_topk_tail + kld_reduce_stats (mean/p50/p99/p99.9, top-1,
    both perplexities), inputs resident, larger than L2."""
    import torch
    from synth import workloads as W
    d = W.topk_tail_windows(seed=W.seed_for(4), device=dev, windows=windows)
    ri, rl = d["ref_ids"].reshape(-1, 64), d["ref_lp"].reshape(-1, 64)
    ci, cl = d["cand_ids"].reshape(-1, 64), d["cand_lp"].reshape(-1, 64)
    rt, ct = d["ref_target_lp"].reshape(-1), d["cand_target_lp"].reshape(-1)
    n = ri.shape[0]
    kl = torch.empty(n, dtype=torch.float32, device=dev)
    top1 = torch.empty(n, dtype=torch.uint8, device=dev)
    ws = torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev)
    out = torch.empty(280, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        kq.kld_topk_tail(ri, rl, ci, cl, d["vocab"], kl=kl, top1=top1, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        kq.kld_reduce_stats(kl, None, None, top1, rt, ct, None, QUANTILES, (), out=out, workspace=ws,
                            stream=stream, to_host=False)

    steps = steps or max(1, min(args.steps, 100))
    for _ in range(max(3, args.warmup)):
        step()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        step(kev[i])
    stop.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(stop) / steps
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    alg = n * (2 * 64 * 4 + 2 * 64 * 2 + 4 + 1)   # both lists in, kl and top-1 out
    peak, _ = measured_peaks()
    return {"workload": f"top-64 + tail bucket: {windows} windows x 2047 positions, V=248,320",
            "value": n / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "step": "kld_topk_tail + kld_reduce_stats", "gpu_launches_per_step": 1 + launches_per_step(n) - 2,
            "roofline": {"bound": "hbm", "achieved": alg / (k_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": alg / (k_ms / 1e3) / 1e9 / peak, "kernel": "kld::topk_tail_kernel",
                         "kernel_ms": k_ms}}


def measure_sparse_ref(args, kq, dev, n_rows=N_ROWS, k=512, steps=None) -> dict:
    """The challenge score on one window: candidate full logits (2047 x
    248,320 bf16) against a 512-id sparse reference with stored tail masses,
    kld_sparse_ref_score + kld_reduce_stats, inputs resident, larger than L2."""
    import torch
    from synth import workloads as W
    d = W.sparse_ref_window(seed=W.seed_for(6), device=dev, n_rows=n_rows, k=k)
    cand, top, rows, tg = d["cand"], d["ref_top"], d["ref_rows"], d["targets"]
    n = cand.shape[0]
    kl = torch.empty(n, dtype=torch.float32, device=dev)
    am = torch.empty(n, dtype=torch.int32, device=dev)
    top1 = torch.empty(n, dtype=torch.uint8, device=dev)
    lpc = torch.empty(n, dtype=torch.float32, device=dev)
    lpr = torch.empty(n, dtype=torch.float32, device=dev)
    sws = torch.empty(kq.kld_sparse_ref_workspace_size(n, k), dtype=torch.uint8, device=dev)
    ws = torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev)
    out = torch.empty(280, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        kq.kld_sparse_ref_score(cand, top, rows, tg, kl=kl, cand_argmax=am, top1=top1, cand_target_lp=lpc,
                                ref_target_lp=lpr, workspace=sws, dev_status=status, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        kq.kld_reduce_stats(kl, None, None, top1, lpr, lpc, None, QUANTILES, (), out=out, workspace=ws,
                            stream=stream, to_host=False)

    steps = steps or max(1, min(args.steps, 200))
    for _ in range(max(3, args.warmup)):
        step()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        step(kev[i])
    stop.record(stream)
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item()}"
    ms = start.elapsed_time(stop) / steps
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    # candidate row, reference entries and stored row, target in; five outputs
    alg = n * (VOCAB * 2 + k * 8 + 12 + 4 + 17)
    peak, _ = measured_peaks()
    return {"workload": f"challenge score: {n} positions x 248,320 bf16 candidate logits vs "
                        f"{k}-id sparse reference + tail cell",
            "value": n / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "step": "kld_sparse_ref_score + kld_reduce_stats", "gpu_launches_per_step": launches_per_step(n),
            "roofline": {"bound": "hbm", "achieved": alg / (k_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": alg / (k_ms / 1e3) / 1e9 / peak,
                         "kernel": "kld::sparse_stream_kernel<bf16> + kld::sparse_merge_kernel<bf16>",
                         "kernel_ms": k_ms}}


def measure_sparse_capture(args, kq, dev, n_rows=N_ROWS, k=512, steps=None) -> dict:
    """The sparse reference record of one window: full logits (2047 x
    248,320 bf16) -> top-512 ids and log-probs, NLL, entropy, tail mass;
    kld_sparse_capture, inputs resident, larger than L2."""
    import torch
    from synth import workloads as W
    d = W.window_full_vocab(seed=W.seed_for(2), device=dev, n_rows=n_rows)
    x, tg = d["ref"], d["targets"]
    n = x.shape[0]
    top = torch.empty((n, k, 2), dtype=torch.int32, device=dev)
    rows = torch.empty((n, 3), dtype=torch.float32, device=dev)
    ws = torch.empty(kq.kld_sparse_capture_workspace_size(n, k), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        kq.kld_sparse_capture(x, k, tg, top=top, rows=rows, workspace=ws, dev_status=status, stream=stream)

    steps = steps or max(1, min(args.steps, 200))
    for _ in range(max(3, args.warmup)):
        step()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        step()
    stop.record(stream)
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item()}"
    ms = start.elapsed_time(stop) / steps
    # logits and targets in; k (id, lp) entries and the 3-float row out
    alg = n * (VOCAB * 2 + 4 + k * 8 + 12)
    peak, _ = measured_peaks()
    return {"workload": f"sparse capture: {n} positions x 248,320 bf16 logits -> top-{k} + (NLL, entropy, tail)",
            "value": n / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "step": "kld_sparse_capture (sample + stream + finish)", "gpu_launches_per_step": 3,
            "roofline": {"bound": "hbm", "achieved": alg / (ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": alg / (ms / 1e3) / 1e9 / peak,
                         "kernel": "kld::cap_sample_kernel + cap_stream_kernel + cap_finalize_kernel (bf16)",
                         "kernel_ms": ms}}


def measure_reduce(args, kq, dev, n=N_ROWS, steps=None) -> dict:
    """Only the statistics (kld_reduce_stats: mean, p50/p99/p99.9, top-1,
    perplexities) of n positions' results, resident on the device."""
    from synth import workloads as W
    import torch
    d = W.position_results(seed=window_seed(0) + 7, device=dev, n=n)
    out = torch.empty(280, dtype=torch.uint8, device=dev)
    ws = torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(s=stream):
        kq.kld_reduce_stats(d["kl"], d["ra"], d["ca"], None, d["lpr"], d["lpc"], None, QUANTILES, (), out=out,
                            workspace=ws, dev_status=status, stream=s, to_host=False)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    k = steps or args.steps
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(k):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    host_ms = a.elapsed_time(b) / k
    # the same calls replayed from a CUDA graph: device time without the
    # host's per-call cost
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for _ in range(k):
            step(side)
    graph.replay()
    torch.cuda.synchronize()
    a.record(stream)
    graph.replay()
    b.record(stream)
    torch.cuda.synchronize()
    assert status.item() == 0
    ms = a.elapsed_time(b) / k
    return {"path": "kld_reduce_stats", "positions": n, "ms": ms, "us": ms * 1e3, "us_host_loop": host_ms * 1e3,
            "launches_per_step": launches_per_step(n) - 2}


def measure_batched(args, kq, dev, steps=None) -> dict:
    """Batched full-vocabulary scoring (16 windows x 2047 rows of f32
    logits, 32.5 GB per side, resident): kld_full_vocab + kld_reduce_stats
    per step, inputs far larger than L2."""
    import torch
    from synth import workloads as W
    t0 = time.perf_counter()
    d = W.batched_full_vocab(device=dev)
    torch.cuda.synchronize()
    gen_s = time.perf_counter() - t0
    ref, cand, targets = d["ref"], d["cand"], d["targets"]
    n = ref.shape[0]
    kl = torch.empty(n, dtype=torch.float32, device=dev)
    ra = torch.empty(n, dtype=torch.int32, device=dev)
    ca = torch.empty(n, dtype=torch.int32, device=dev)
    lpr = torch.empty(n, dtype=torch.float32, device=dev)
    lpc = torch.empty(n, dtype=torch.float32, device=dev)
    fws = torch.empty(kq.kld_full_vocab_workspace_size(n), dtype=torch.uint8, device=dev)
    ws = torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev)
    out = torch.empty(280, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        kq.kld_full_vocab(ref, cand, targets, kl=kl, ref_argmax=ra, cand_argmax=ca, ref_target_lp=lpr,
                          cand_target_lp=lpc, workspace=fws, dev_status=status, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        kq.kld_reduce_stats(kl, ra, ca, None, lpr, lpc, None, QUANTILES, (), out=out, workspace=ws,
                            dev_status=status, stream=stream, to_host=False)

    steps = steps or max(1, min(args.steps, 20))
    for _ in range(3):
        step()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        step(kev[i])
    stop.record(stream)
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item()}"
    ms = start.elapsed_time(stop) / steps
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    alg = 2 * n * VOCAB * 4 + n * (4 + 4 * 5)
    peak, _ = measured_peaks()
    del d, ref, cand
    return {"workload": f"batched full-vocabulary scoring: {n} positions x 248,320 f32 logits (16 windows)",
            "value": n / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "step": "kld_full_vocab + kld_reduce_stats", "gpu_launches_per_step": 2 + 2,
            "generate_s": gen_s,
            "roofline": {"bound": "hbm", "achieved": alg / (k_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": alg / (k_ms / 1e3) / 1e9 / peak,
                         "kernel": "kld::stream_kernel<f32> + kld::merge_kernel<f32>", "kernel_ms": k_ms}}


def measure_paired(args, kq, dev, steps=None) -> dict:
    """Two candidates compared paired per context over one whole suite
    (5,120 contexts x 2,047 positions, 842 source clusters) with a
    10,000-replicate cluster bootstrap: kld_paired_compare.  Inputs are
    resident; L2 is flushed before every timed call (the inputs are about
    L2's size)."""
    import torch
    from synth import workloads as W
    d = W.paired_candidates(seed=W.seed_for(8), device=dev)
    a, b, cl, rs = d["kl_a"], d["kl_b"], d["cluster"], d["resample"]
    n_ctx, L = a.shape
    B, C = rs.shape
    out = torch.empty(144, dtype=torch.uint8, device=dev)
    boot = torch.empty(B, dtype=torch.float64, device=dev)
    ws = torch.empty(kq.kld_paired_workspace_size(n_ctx, C, B), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        kq.kld_paired_compare(a, b, cl, rs, (0.025, 0.975), None, boot_stats=boot, out=out, workspace=ws,
                              dev_status=status, stream=stream, to_host=False)

    steps = steps or max(1, min(args.steps, 100))
    for _ in range(max(3, args.warmup)):
        step()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        kev[i][0].record(stream)
        step()
        kev[i][1].record(stream)
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item()}"
    ms = statistics.mean(x.elapsed_time(y) for x, y in kev)
    # both candidates' KL, the cluster ids and the draws in; replicate statistics out
    alg = 2 * n_ctx * L * 4 + n_ctx * 4 + B * C * 4 + B * 8
    peak, _ = measured_peaks()
    return {"workload": f"paired comparison: {n_ctx} contexts x {L} positions, two candidates, {C} source "
                        f"clusters, {B}-replicate cluster bootstrap",
            "value": n_ctx * L / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "step": "kld_paired_compare", "gpu_launches_per_step": 4, "l2": "flushed before every call",
            "roofline": {"bound": "hbm", "achieved": alg / (ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": alg / (ms / 1e3) / 1e9 / peak,
                         "kernel": "kld::paired_{ctx,cluster,boot,select}_kernel", "kernel_ms": ms}}


def measured_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), float(d["bf16_tflops"]), "measured"
    return 1400.0, 1590.0, "fallback"


def measure_shared_head(args, kq, dev, n_rows=8192, hidden=5120, vocab=VOCAB, steps=None) -> dict:
    """Fused shared head (hidden states through one bf16 head, logits in
    tensor memory only): kld_from_hidden_shared_head + kld_reduce_stats."""
    import torch
    from synth import workloads as W
    d = W.shared_head_states(seed=W.seed_for(5), device=dev, n_rows=n_rows, hidden=hidden, vocab=vocab)
    n = n_rows
    kl = torch.empty(n, dtype=torch.float32, device=dev)
    ra = torch.empty(n, dtype=torch.int32, device=dev)
    ca = torch.empty(n, dtype=torch.int32, device=dev)
    lpr = torch.empty(n, dtype=torch.float32, device=dev)
    lpc = torch.empty(n, dtype=torch.float32, device=dev)
    hws = torch.empty(kq.kld_shared_head_workspace_size(n, hidden, vocab), dtype=torch.uint8, device=dev)
    ws = torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev)
    out = torch.empty(280, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        kq.kld_from_hidden_shared_head(d["h_ref"], d["h_cand"], d["W"], d["targets"], kl=kl, ref_argmax=ra,
                                       cand_argmax=ca, ref_target_lp=lpr, cand_target_lp=lpc, workspace=hws,
                                       dev_status=status, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        kq.kld_reduce_stats(kl, ra, ca, None, lpr, lpc, None, QUANTILES, (), out=out, workspace=ws,
                            stream=stream, to_host=False)

    steps = steps or max(1, min(args.steps, 10))
    for _ in range(3):
        step()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        step(kev[i])
    stop.record(stream)
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item()}"
    ms = start.elapsed_time(stop) / steps
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    flop = 2.0 * 2.0 * n * vocab * hidden          # both sides' logits
    sustained, burst, kind = measured_tensor_peak()
    achieved = flop / (k_ms / 1e3) / 1e12
    # the kernel is timed in isolation (a few calls of ~30 ms), so the burst
    # GEMM rate is its peak; the sustained one is reported beside it
    return {"workload": f"fused shared head: {n} positions, hidden {hidden}, head {vocab} x {hidden} bf16",
            "value": n / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "step": "kld_from_hidden_shared_head + kld_reduce_stats",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                         "frac": achieved / burst, "frac_of_sustained_peak": achieved / sustained,
                         "kernel": "kld::head_kernel + kld::head_merge_kernel", "kernel_ms": k_ms,
                         "peak_source": f"{kind} bf16_tflops (burst; sustained {sustained})"}}


def measure_e2e(args, kq, d, dev, world) -> dict:
    """The same step from pinned host buffers: per step the logits and targets
    are copied host -> device in row chunks on a copy stream, overlapped with
    scoring of the previous chunk, and the stats struct is read back."""
    import torch
    import torch.distributed as dist
    n = d["ref"].shape[0]
    chunk = 256
    h_ref = d["ref"].cpu().pin_memory()
    h_cand = d["cand"].cpu().pin_memory()
    h_t = d["targets"].cpu().pin_memory()
    d_ref = torch.empty_like(d["ref"])
    d_cand = torch.empty_like(d["cand"])
    d_t = torch.empty_like(d["targets"])
    kl = torch.empty(n, dtype=torch.float32, device=dev)
    ra = torch.empty(n, dtype=torch.int32, device=dev)
    ca = torch.empty(n, dtype=torch.int32, device=dev)
    lpr = torch.empty(n, dtype=torch.float32, device=dev)
    lpc = torch.empty(n, dtype=torch.float32, device=dev)
    ws = torch.empty(kq.kld_reduce_workspace_size(n), dtype=torch.uint8, device=dev)
    fws = torch.empty(kq.kld_full_vocab_workspace_size(chunk), dtype=torch.uint8, device=dev)
    stats_buf = torch.empty(280, dtype=torch.uint8, device=dev)
    h_stats = torch.empty(280, dtype=torch.uint8).pin_memory()
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream(device=dev)
    if world > 1:
        from quantization_fidelity_scoring_b200 import shards
        sws = torch.empty(kq.kld_reduce_shard_workspace_size(n), dtype=torch.uint8, device=dev)
    chunks = [(a, min(n, a + chunk)) for a in range(0, n, chunk)]

    def step():
        evs = []
        with torch.cuda.stream(copy):
            for a, b in chunks:
                d_ref[a:b].copy_(h_ref[a:b], non_blocking=True)
                d_cand[a:b].copy_(h_cand[a:b], non_blocking=True)
                d_t[a:b].copy_(h_t[a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(copy)
                evs.append(e)
        for (a, b), e in zip(chunks, evs):
            comp.wait_event(e)
            kq.kld_full_vocab(d_ref[a:b], d_cand[a:b], d_t[a:b], kl=kl[a:b], ref_argmax=ra[a:b],
                              cand_argmax=ca[a:b], ref_target_lp=lpr[a:b], cand_target_lp=lpc[a:b],
                              workspace=fws, stream=comp)
        if world > 1:
            shards.reduce_stats_across_ranks(kl, ra, ca, None, lpr, lpc, None, QUANTILES, (), out=stats_buf,
                                             workspace=sws, to_host=False)
        else:
            kq.kld_reduce_stats(kl, ra, ca, None, lpr, lpc, None, QUANTILES, (), out=stats_buf, workspace=ws,
                                stream=comp, to_host=False)
        h_stats.copy_(stats_buf, non_blocking=True)
        comp.synchronize()

    steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(3):
        step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = max_over_ranks(time.perf_counter() - t0, dev, world)
    h2d = h_ref.numel() * 2 + h_cand.numel() * 2 + h_t.numel() * 4
    return {"value": whole_job_rate(n, world, steps, dt), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": 280, "steps": steps,
            "how": "pinned host logits, 256-row H2D chunks overlapped with scoring, stats read back; wall clock"}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-rows", type=int, default=512)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--ref-seconds", type=float, default=90.0,
                    help="reference arm: CPU seconds the timed and warm-up steps aim for")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--serial", action="store_true",
                    help="run each window's statistics after its scoring on one stream (no overlap)")
    ap.add_argument("--no-extra", action="store_true", help="skip the top-64 and shared-head lines")
    ap.add_argument("--profile-topk", type=int, metavar="WINDOWS",
                    help="only time the top-64 + tail path on WINDOWS windows (for profiling)")
    ap.add_argument("--profile-sparse", type=int, metavar="ROWS",
                    help="only time the sparse-reference score on ROWS positions (for profiling)")
    ap.add_argument("--profile-capture", type=int, metavar="ROWS",
                    help="only time the sparse capture on ROWS positions (for profiling)")
    ap.add_argument("--profile-batched", action="store_true",
                    help="only time the batched f32 workload (16 windows, 65 GB of logits)")
    ap.add_argument("--profile-paired", action="store_true",
                    help="only time the paired comparison of two candidates over one suite (for profiling)")
    ap.add_argument("--profile-reduce", type=int, metavar="POSITIONS",
                    help="only time the statistics of POSITIONS per-position results (for profiling)")
    ap.add_argument("--profile-head", nargs=2, type=int, metavar=("ROWS", "VOCAB"),
                    help="only time the shared-head path at a reduced size (for profiling)")
    ap.add_argument("--rows", type=int, default=N_ROWS,
                    help="positions per window (default 2047; smaller only for profiling runs)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_topk:
        import torch
        import quantization_fidelity_scoring_b200 as kq
        kq.load_library()
        print(json.dumps(measure_topk(args, kq, torch.device("cuda:0"), windows=args.profile_topk,
                                      steps=args.steps)), flush=True)
        return 0
    if args.profile_sparse:
        import torch
        import quantization_fidelity_scoring_b200 as kq
        kq.load_library()
        print(json.dumps(measure_sparse_ref(args, kq, torch.device("cuda:0"), n_rows=args.profile_sparse,
                                            steps=args.steps)), flush=True)
        return 0
    if args.profile_capture:
        import torch
        import quantization_fidelity_scoring_b200 as kq
        kq.load_library()
        print(json.dumps(measure_sparse_capture(args, kq, torch.device("cuda:0"), n_rows=args.profile_capture,
                                                steps=args.steps)), flush=True)
        return 0
    if args.profile_batched:
        import torch
        import quantization_fidelity_scoring_b200 as kq
        kq.load_library()
        print(json.dumps(measure_batched(args, kq, torch.device("cuda:0"), steps=args.steps)), flush=True)
        return 0
    if args.profile_paired:
        import torch
        import quantization_fidelity_scoring_b200 as kq
        kq.load_library()
        print(json.dumps(measure_paired(args, kq, torch.device("cuda:0"), steps=args.steps)), flush=True)
        return 0
    if args.profile_reduce:
        import torch
        import quantization_fidelity_scoring_b200 as kq
        kq.load_library()
        print(json.dumps(measure_reduce(args, kq, torch.device("cuda:0"), n=args.profile_reduce)), flush=True)
        return 0
    if args.profile_head:
        import torch
        import quantization_fidelity_scoring_b200 as kq
        kq.load_library()
        r = measure_shared_head(args, kq, torch.device("cuda:0"), n_rows=args.profile_head[0],
                                vocab=args.profile_head[1], steps=args.steps)
        print(json.dumps(r), flush=True)
        return 0
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
