#!/usr/bin/env python
"""Benchmark of the AWQ per-layer scale search on B200.

One step = one pass of the whole path over one synthetic layer:
activation statistics -> 20-alpha grid search (tensor cores) -> argmin + pack.

    python bench.py [--gpus N --steps K --warmup W] [--config attn4096] [--impl reference]

Prints ONE JSON line on rank 0.  ``value`` is useful search work
(2 N K T |grid| flops per layer) divided by the device time of the whole step,
summed over ranks (each rank quantizes its own layer: weak scaling, no
collective on the data path).  Inputs live in HBM before the timed region and
L2 is flushed between steps (the layer's W and X fit in the 126 MB L2).

Beside ``value`` the line carries ``layers_per_s`` (whole-job layers per
second), the search kernel's ``roofline`` and, in ``hbm_kernels``, the warm
per-launch HBM rates of the statistics and packing kernels.

``--impl reference`` times the CPU oracle as it stands on this host's cores over
a bounded row sample of the same layer (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "AWQ search TFLOP/s (20-α grid, 4096² layer, T=4096) & % of FP16 TC peak"
UNIT = "TFLOP/s"
LAUNCHES_PER_STEP = 7      # act_stats, alpha_scales, group_params, search, loss_reduce, best_scale, pack
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = ROOT / "profiles" / "search_pair_kernel_traffic.json"
CSRC = ROOT / "awq_activation_aware_b200" / "csrc"


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["awq", "reference"], default="awq")
    p.add_argument("--config", default="attn4096")
    p.add_argument("--e2e-steps", type=int, default=12)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-hbm", action="store_true", help="skip the warm HBM-kernel rates")
    p.add_argument("--shard", choices=["layers", "rows"], default="layers",
                   help="layers: each rank quantizes its own layer (weak scaling, no collective); rows: the "
                        "ranks split one layer's rows and all-reduce the per-alpha losses (strong scaling)")
    p.add_argument("--cpu-rows", type=int, default=0, help="rows of W in the oracle sample (0 = auto)")
    p.add_argument("--cpu-budget-s", type=float, default=15.0)
    p.add_argument("--op", choices=["search", "qlinear", "baselines", "gptq"], default="search",
                   help="search: the AWQ scale-search path (the benchmark); qlinear: the quantized "
                        "linear layer on the packed output vs the fp16 GEMM; baselines: the pages' "
                        "comparisons (RTN, fixed 2x, fp16 1%%, symmetric) on one layer; gptq: AWQ "
                        "followed by GPTQ error compensation, each stage timed")
    p.add_argument("--tokens", default="1,4,16", help="token counts for --op qlinear")
    p.add_argument("--bits", type=int, default=0, help="w_bit for --op gptq (default: the config's)")
    p.add_argument("--group", type=int, default=0, help="group size for --op gptq (default: the config's)")
    return p.parse_args()


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------
def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist


def reduce_max(values, world, device):
    """Element-wise max over ranks of a list of floats."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# host facts
# ---------------------------------------------------------------------------
def load_peaks():
    f = ROOT / "MEASURED_PEAKS.json"
    if f.exists():
        d = json.loads(f.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="awq_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in Path(self.path).read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == len(self.FIELDS):
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        loaded = [r for r in rows if (num(r[3]) or 0) > 0.5 * max(power or [0])] or rows
        sm_loaded = [num(r[1]) for r in loaded if num(r[1]) is not None] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm_loaded) if sm_loaded else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(power) if power else None}


def kernel_source_hash():
    """Hash of the search kernel's source: its namespace block plus the device
    helpers it is built from.  A traffic figure taken from an older build of
    the kernel no longer applies once this changes."""
    kern = (CSRC / "awq_kernels.cuh").read_text()
    a = kern.index("namespace srch2 {")
    b = kern.index("}  // namespace srch2")
    h = hashlib.sha256()
    h.update(kern[a:b].encode())
    h.update((CSRC / "awq_device.cuh").read_bytes())
    return h.hexdigest()[:16]


def search_traffic(cfg_name):
    """DRAM bytes per search launch from a committed ncu capture, or None if the
    kernel sources changed since it was taken (or there is none)."""
    if not TRAFFIC_FILE.exists():
        return None
    d = json.loads(TRAFFIC_FILE.read_text())
    if d.get("source_hash") != kernel_source_hash():
        return None
    e = d.get("per_launch_bytes", {}).get(cfg_name)
    return None if e is None else float(e)


# ---------------------------------------------------------------------------
# oracle sample (CPU baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(cfg, W, X, alphas, rows):
    import oracle
    oracle.build()
    t0 = time.perf_counter()
    a = oracle.act_stats(X)
    r = oracle.search(W, X, a, cfg.bits, cfg.group, alphas, rows=rows)
    oracle.pack(W, a, cfg.bits, cfg.group, alphas, r["losses"], rows=rows)
    return time.perf_counter() - t0


def pick_rows(cfg, W, X, alphas, budget_s):
    """Rows of W for an oracle sample of about budget_s seconds: time two row
    counts over the full grid and fit time = fixed + rows * per_row."""
    import oracle
    oracle.build()
    a = oracle.act_stats(X)
    times = {}
    for r in (16, 64):
        t0 = time.perf_counter()
        oracle.search(W, X, a, cfg.bits, cfg.group, alphas, rows=np.arange(min(r, cfg.N)))
        times[r] = time.perf_counter() - t0
    per_row = max((times[64] - times[16]) / 48.0, 1e-6)
    fixed = max(times[16] - 16 * per_row, 0.0)
    rows = int((budget_s - fixed) / per_row)
    return max(16, min(cfg.N, rows))


def cpu_measure(cfg, W, X, alphas, args):
    rows_n = args.cpu_rows or pick_rows(cfg, W, X, alphas, args.cpu_budget_s)
    rows = np.linspace(0, cfg.N - 1, rows_n).astype(np.int64)
    dt = oracle_sample(cfg, W, X, alphas, rows)
    flops = 2.0 * rows_n * cfg.K * cfg.T * len(alphas)
    return flops / dt / 1e12, dt, rows_n


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def config_dict(cfg, n_alpha, extra=None):
    d = {"workload": f"{cfg.name}, {n_alpha}-alpha grid", "N": cfg.N, "K": cfg.K, "T": cfg.T,
         "bits": cfg.bits, "group_size": cfg.group, "n_alpha": n_alpha,
         "inputs": "seeded synthetic: W ~ N(0, %g^2) fp16; X ~ N(0,1) fp16 with %d outlier channels x10-100"
                   % (cfg.w_std, cfg.n_outliers),
         "l2": "flushed between steps (256 MiB write)"}
    if extra:
        d.update(extra)
    return d


def run_reference(args):
    from awq_activation_aware_b200 import synth
    rank, world, _ = dist_info()
    if rank != 0:
        return 0
    cfg = synth.CONFIGS[args.config]
    W, X, _ = synth.generate(cfg)
    alphas = synth.default_alphas()
    per_step = max(2.0, args.cpu_budget_s * 6 / max(args.steps + args.warmup, 1))
    rows_n = args.cpu_rows or pick_rows(cfg, W, X, alphas, per_step)
    rows = np.linspace(0, cfg.N - 1, rows_n).astype(np.int64)
    for _ in range(args.warmup):
        oracle_sample(cfg, W, X, alphas, rows)
    times = [oracle_sample(cfg, W, X, alphas, rows) for _ in range(args.steps)]
    t = sum(times) / len(times)
    flops = 2.0 * rows_n * cfg.K * cfg.T * len(alphas)
    value = flops / t / 1e12
    sample = f"{rows_n} of {cfg.N} rows of W, all {cfg.K} columns, all {cfg.T} tokens, all {len(alphas)} alphas"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(cfg, len(alphas)),
            "layers_per_s": (rows_n / cfg.N) / t,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def hbm_kernel_rates(awq, torch, cfg, Xd, Wd, s_best, peaks, reps=5):
    """Warm per-launch rates of the two HBM-bound kernels of the path.

    act_stats (reads X) and pack_kernel (awq_pack_scales: reads W and s_best,
    writes codes, scales and zeros) each run over a sequence of distinct copies
    of their input, together more than 4x the 126 MB L2, so every launch reads
    HBM as a model's layers do; CUDA events bracket the whole sequence on the
    stream and a launch's time is the sequence time over its launches.  Bytes
    are the algorithmic ones (each input byte read once, each output
    byte written once)."""
    budget = 512 << 20
    per = 16 if cfg.bits == 2 else 8
    x_bytes = cfg.T * cfg.K * 2
    w_bytes = cfg.N * cfg.K * 2
    Xs = [Xd.clone() for _ in range(max(2, -(-budget // x_bytes)))]
    Ws = [Wd.clone() for _ in range(max(2, -(-budget // w_bytes)))]
    stream = torch.cuda.current_stream()

    def per_launch_s(calls):
        # average launch duration over the back-to-back sequence (events around the
        # whole sequence, so no event sits between two launches); median over reps
        for fn in calls:
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(20_000_000)           # the host queues every launch before the first runs
            b.record(stream)
            for fn in calls:
                fn()
            e.record(stream)
            torch.cuda.synchronize()
            ts.append(b.elapsed_time(e) * 1e-3 / len(calls))
        return statistics.median(ts)

    t_stats = per_launch_s([(lambda x=x: awq.act_stats(x)) for x in Xs])
    t_pack = per_launch_s([(lambda w=w: awq.pack_scales(w, s_best, cfg.bits, cfg.group)) for w in Ws])
    awq.get_status()
    del Xs, Ws
    hbm = peaks.get("hbm_gbs")
    stats_bytes = x_bytes + cfg.K * 4
    pack_bytes = w_bytes + cfg.K * 4 + cfg.N * cfg.K // per * 4 + 2 * cfg.N * (cfg.K // cfg.group) * 2

    def entry(kernel, nbytes, t):
        gbs = nbytes / t / 1e9
        return {"kernel": kernel, "us": t * 1e6, "bytes": nbytes, "GBps": gbs,
                "frac": gbs / hbm if hbm else None}
    return {"act_stats": entry("act_stats_kernel", stats_bytes, t_stats),
            "pack": entry("pack_kernel", pack_bytes, t_pack),
            "peak_GBps": hbm,
            "how": "average launch duration over a back-to-back sequence of distinct input copies "
                   "(> 4x L2), CUDA events around the sequence, median of 5"}


def rank_layer_config(base, rank):
    """Each rank quantizes its own layer of the base shape (independent problems):
    the same recipe with seed + 1000 * rank."""
    from awq_activation_aware_b200 import synth
    return synth.LayerConfig(**{**base.as_dict(), "seed": base.seed + 1000 * rank})


def run_awq(args):
    import torch

    import awq_activation_aware_b200 as awq
    from awq_activation_aware_b200 import synth

    rank, world, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    rows_mode = args.shard == "rows"
    if rows_mode:
        # one layer, its rows split across the ranks; the all-reduce of the
        # per-alpha losses is inside every step (awq_activation_aware_b200.sharded)
        from awq_activation_aware_b200 import sharded
        base = synth.CONFIGS[args.config]
        W_full, X, _ = synth.generate(base)
        r0, r1 = sharded.shard_rows(base.N, world, rank)
        W = np.ascontiguousarray(W_full[r0:r1])
        del W_full
        cfg = synth.LayerConfig(**{**base.as_dict(), "N": r1 - r0})
        if cfg.N < 1:
            raise SystemExit(f"--shard rows: rank {rank} holds no rows of the {base.N}-row layer")
        layer_flops = 2.0 * base.N * base.K * base.T * len(synth.default_alphas())
    else:
        cfg = rank_layer_config(synth.CONFIGS[args.config], rank)
        W, X, _ = synth.generate(cfg)
    alphas_np = synth.default_alphas()
    n_alpha = len(alphas_np)
    flops = 2.0 * cfg.N * cfg.K * cfg.T * n_alpha

    W_h = torch.from_numpy(W).pin_memory()
    X_h = torch.from_numpy(X).pin_memory()
    Wd = W_h.to(dev)
    Xd = X_h.to(dev)
    alphas = torch.from_numpy(alphas_np).to(dev)
    ws = torch.empty(awq.search_workspace_bytes(cfg.N, cfg.K, cfg.T, cfg.bits, cfg.group, n_alpha),
                     dtype=torch.uint8, device=dev)
    losses = torch.empty(n_alpha, dtype=torch.float32, device=dev)
    per = 16 if cfg.bits == 2 else 8
    out = dict(best_idx=torch.empty(1, dtype=torch.int32, device=dev),
               s_best=torch.empty(cfg.K, dtype=torch.float32, device=dev),
               codes=torch.empty((cfg.N, cfg.K // per), dtype=torch.int32, device=dev),
               scales=torch.empty((cfg.N, cfg.K // cfg.group), dtype=torch.float16, device=dev),
               zeros=torch.empty((cfg.N, cfg.K // cfg.group), dtype=torch.float16, device=dev))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(prof=None):
        a = awq.act_stats(Xd)
        if prof is not None:
            awq.profile_next_search(*prof)
        awq.search_layer(Wd, Xd, a, alphas, cfg.bits, cfg.group, workspace=ws, losses_out=losses,
                         rows_total=base.N if rows_mode else None)
        if rows_mode and world > 1:
            import torch.distributed as dist
            dist.all_reduce(losses, op=dist.ReduceOp.SUM)
        awq.pack(Wd, a, alphas, losses, cfg.bits, cfg.group, out=out)

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    awq.get_status()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for b, e in sev:          # materialise the events before handing their handles to the library
        b.record(stream)
        e.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    barrier(world)
    if sampler:
        sampler.start()
    torch.cuda.synchronize()
    barrier(world)
    # a GPU-side pause lets the host queue the steps ahead of the device, so no
    # step waits on the host's launch calls (the pause is outside every event pair)
    torch.cuda._sleep(40_000_000)
    for i in range(K):
        flush.zero_()
        ev[i][0].record(stream)
        step(prof=sev[i])
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    awq.get_status()
    step_ms = [b.elapsed_time(e) for b, e in ev]
    search_ms = [b.elapsed_time(e) for b, e in sev]
    total_ms, search_avg = reduce_max([sum(step_ms), sum(search_ms) / K], world, dev)
    ms_per_step = total_ms / K
    job_flops = layer_flops if rows_mode else world * flops
    value = job_flops / (ms_per_step * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    long_region = total_ms > 1000.0
    peak = peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops")
    achieved = flops / (search_avg * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": search_traffic(args.config),
                "kernel": "search_pair_kernel (tcgen05 cta_group::2 f16 MMA, fused quantize producer, "
                          "on-chip squared-error epilogue)",
                "peak_source": f"{peak_src} {'sustained' if long_region else 'burst'} bf16 dense "
                               f"(fp16 has the same nominal dense rate)",
                "search_ms": search_avg}

    # End to end through the public API with host buffers, as a model's layers are
    # quantized one after another: every step copies its W and X from pinned host
    # memory (H2D), runs the path, and reads the losses, best index, s_best, codes,
    # scales and zeros back (D2H).  The copies run on their own streams with two
    # sets of device buffers, so step i+1's H2D and step i-1's D2H overlap step i's
    # compute; the timed region spans the first H2D to the last D2H.  L2 is flushed
    # before every step's compute.
    e2e = None
    if not args.no_e2e and not rows_mode:
        d2h = (n_alpha * 4 + 4 + cfg.K * 4 + cfg.N * cfg.K // per * 4 + 2 * cfg.N * cfg.K // cfg.group * 2)
        h2d = W_h.numel() * 2 + X_h.numel() * 2
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        bufs = [(torch.empty_like(Wd), torch.empty_like(Xd)) for _ in range(2)]
        outs = [out, {k: torch.empty_like(v) for k, v in out.items()}]
        lss = [losses, torch.empty_like(losses)]
        res_h = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in out.items()} for _ in range(2)]
        loss_h = [torch.empty(n_alpha, dtype=torch.float32).pin_memory() for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n):
            for i in range(n):
                j = i % 2
                Wb, Xb = bufs[j]
                if i >= 2:
                    s_in.wait_event(ev_done[j])           # step i-2 no longer reads these inputs
                with torch.cuda.stream(s_in):
                    Wb.copy_(W_h, non_blocking=True)
                    Xb.copy_(X_h, non_blocking=True)
                    ev_in[j].record(s_in)
                stream.wait_event(ev_in[j])
                if i >= 2:
                    stream.wait_event(ev_out[j])          # step i-2's results have been read back
                flush.zero_()
                a = awq.act_stats(Xb)
                awq.search_layer(Wb, Xb, a, alphas, cfg.bits, cfg.group, workspace=ws, losses_out=lss[j])
                awq.pack(Wb, a, alphas, lss[j], cfg.bits, cfg.group, out=outs[j])
                ev_done[j].record(stream)
                s_out.wait_event(ev_done[j])
                with torch.cuda.stream(s_out):
                    loss_h[j].copy_(lss[j], non_blocking=True)
                    for k in outs[j]:
                        res_h[j][k].copy_(outs[j][k], non_blocking=True)
                    ev_out[j].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        awq.get_status()
        b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        b.record(stream)
        s_in.wait_stream(stream)                          # the first H2D starts inside the timed region
        e2e_run(args.e2e_steps)
        e.record(stream)
        torch.cuda.synchronize()
        awq.get_status()
        e2e_ms = reduce_max([b.elapsed_time(e) / args.e2e_steps], world, dev)[0]
        e2e = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "overlap": "double-buffered: H2D and D2H on their own streams, overlapping compute"}

    hbm_rates = None
    if not args.no_hbm:
        hbm_rates = hbm_kernel_rates(awq, torch, cfg, Xd, Wd, out["s_best"], peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cv, dt, rows_n = cpu_measure(cfg, W, X, alphas_np, args)
        cpu = {"value": cv, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
               "sample": f"{rows_n} of {cfg.N} rows of W x all {cfg.K} columns x all {cfg.T} tokens x "
                         f"{n_alpha} alphas (+ statistics over all of X and packing of the sampled rows): "
                         f"{dt:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "strong" if rows_mode else "weak", "vs_baseline": None, "dtype": "f16",
                "data": "synthetic",
                "config": config_dict(base if rows_mode else cfg, n_alpha),
                "parallelism": (f"one layer's rows split over {world} GPUs, all-reduce of {n_alpha} losses"
                                if rows_mode else
                                f"{world} independent layers, one per GPU" if world > 1 else "1 GPU"),
                "layers_per_s": (1 if rows_mode else world) / (ms_per_step * 1e-3),
                "roofline": roofline, "hbm_kernels": hbm_rates, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": LAUNCHES_PER_STEP * K, "clocks": clocks,
                "pct_of_peak": 100.0 * value / peak}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_qlinear(args):
    """The packed layer as a linear layer at decode token counts: awq_qlinear
    (codes streamed from HBM) against the fp16 GEMM (cuBLAS) on the dequantized
    weights.  Each arm runs a sequence of distinct copies of the layer, as
    the layers of a model run one after another, together more than 4x the L2,
    so every call reads its weights from HBM; the sequence is captured in one
    CUDA graph, so host launch cost is not counted.  One JSON line per token
    count, with the time per call."""
    import torch

    import awq_activation_aware_b200 as awq
    from awq_activation_aware_b200 import synth

    dev = torch.device("cuda", 0)
    cfg = synth.CONFIGS[args.config]
    W, X, _ = synth.generate(cfg)
    Wd = torch.from_numpy(W).to(dev)
    Xd = torch.from_numpy(X).to(dev)
    al = awq.default_alphas(device=dev)
    a = awq.act_stats(Xd)
    losses = awq.search_layer(Wd, Xd, a, al, cfg.bits, cfg.group)
    pk = awq.pack(Wd, a, al, losses, cfg.bits, cfg.group)
    W_hat = awq.quant_dequant(Wd, pk["s_best"], cfg.bits, cfg.group)      # fp16 weights for the cuBLAS arm
    awq.get_status()
    del Wd
    peaks, src = load_peaks()
    hbm = peaks.get("hbm_gbs")
    reps = max(args.steps, 3)
    per = 16 if cfg.bits == 2 else 8
    layer_bytes = (pk["codes"].numel() * pk["codes"].element_size() + pk["scales"].numel() * 2
                   + pk["zeros"].numel() * 2)
    total = 512 << 20                                    # > 4x the 126 MB L2
    n_awq = max(2, -(-total // layer_bytes))
    n_ref = max(2, -(-total // (W_hat.numel() * 2)))
    copies = [{k: pk[k].clone() for k in ("codes", "scales", "zeros", "s_best")} for _ in range(n_awq)]
    refs = [W_hat.clone() for _ in range(n_ref)]
    del W_hat

    def per_call_us(calls):
        for fn in calls:                                 # warm-up, outside capture
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for fn in calls:
                fn()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(1_000_000)
            b.record()
            g.replay()
            e.record()
            torch.cuda.synchronize()
            ts.append(b.elapsed_time(e) * 1e3 / len(calls))
        del g
        return statistics.median(ts)

    def path_and_launches(T):
        # the library's dispatch.  One token: the x' kernel, then one pass of the
        # CUDA-core kernel.  From 2 tokens: the prep kernel (B operand, group sums),
        # then one tensor-core pass per 5, 10 or 16 tokens.
        if T < 2:
            return "cuda-core", 2
        tt = 5 if T <= 5 else 10 if T <= 10 else 16
        return "tensor-core", 1 + -(-T // tt)

    for T in [int(t) for t in args.tokens.split(",")]:
        Xt = Xd[:T].contiguous()
        ws = torch.empty(int(awq.lib().awq_qlinear_workspace_bytes(T, cfg.K, cfg.N)), dtype=torch.uint8, device=dev)
        Y = torch.empty((T, cfg.N), dtype=torch.float32, device=dev)
        Yh = torch.empty((T, cfg.N), dtype=torch.float16, device=dev)
        def timed(tc):
            t = per_call_us([
                (lambda c=c: awq.qlinear(c["codes"], c["scales"], c["zeros"], c["s_best"], Xt, cfg.bits, cfg.group,
                                         workspace=ws, out=Y, tensor_cores=tc)) for c in copies])
            awq.get_status()
            return t
        t_awq, t_cc, t_tc = timed(None), timed(False), timed(True)
        t_ref = per_call_us([(lambda w=w: torch.matmul(Xt, w.t(), out=Yh)) for w in refs])
        nbytes = (cfg.N * cfg.K // per * 4 + 2 * 2 * cfg.N * cfg.K // cfg.group + cfg.K * 4 + T * cfg.K * 2
                  + T * cfg.N * 4)
        gbs = nbytes / (t_awq * 1e-6) / 1e9
        print(json.dumps({"op": "qlinear", "config": cfg.name, "tokens": T, "awq_us": t_awq,
                          "cuda_core_us": t_cc, "tensor_core_us": t_tc,
                          "fp16_gemm_us": t_ref, "speedup_vs_fp16": t_ref / t_awq,
                          "awq_bytes": nbytes, "awq_GBps": gbs, "hbm_frac": gbs / hbm if hbm else None,
                          "hbm_peak_source": src, "layer_copies": [n_awq, n_ref],
                          "path": path_and_launches(T)[0], "launches": path_and_launches(T)[1]}), flush=True)
    awq.get_status()
    return 0


def run_baselines(args):
    """The comparisons of the AWQ pages on one layer (RTN, the fixed 2x scale on
    the salient 1%, fp16 protection of 1% chosen by activation and by weight
    magnitude, the asymmetric and the symmetric grid search), each timed on
    the device with CUDA events after warm-up.  One JSON line with the losses
    and the time of each; value = the searched layer-scale evaluations per
    second of the whole set."""
    import torch

    import awq_activation_aware_b200 as awq
    from awq_activation_aware_b200 import synth

    dev = torch.device("cuda", 0)
    cfg = synth.CONFIGS[args.config]
    W, X, _ = synth.generate(cfg)
    Wd = torch.from_numpy(W).to(dev)
    Xd = torch.from_numpy(X).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 3)

    def timed(fn):
        for _ in range(3):
            flush.zero_()
            out = fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b.record()
            out = fn()
            e.record()
            torch.cuda.synchronize()
            ts.append(b.elapsed_time(e))
        return out, statistics.median(ts)

    r, t_all = timed(lambda: awq.baselines(Wd, Xd, cfg.bits, cfg.group))
    a = awq.act_stats(Xd)
    al = awq.default_alphas(device=dev)
    sym, t_sym = timed(lambda: awq.search_layer(Wd, Xd, a, al, cfg.bits, cfg.group, zero_point=False))
    table = torch.stack([awq.salient_scales(r["mask_act"], 1.0), awq.salient_scales(r["mask_act"], 2.0)])
    _, t_two = timed(lambda: awq.search_scales(Wd, Xd, table, cfg.bits, cfg.group))
    _, t_masked = timed(lambda: awq.search_scales(Wd, Xd, table[:1].contiguous(), cfg.bits, cfg.group,
                                                  mask=r["mask_act"]))
    awq.get_status()
    evals = 2 + 1 + 1 + 20                              # scale vectors searched by baselines()
    flops = 2.0 * cfg.N * cfg.K * cfg.T
    print(json.dumps({
        "op": "baselines", "config": cfg.name, "k_channels": int(r["k"]),
        "losses": {"rtn": float(r["rtn"]), "fixed_2x": float(r["fixed_2x"]), "fp16_act": float(r["fp16_act"]),
                   "fp16_weight": float(r["fp16_weight"]), "awq_grid_best": float(r["awq_grid"].min()),
                   "awq_grid_best_symmetric": float(sym.min())},
        "ms": {"baselines_all": t_all, "grid_symmetric_20": t_sym, "given_scales_2": t_two,
               "given_scales_1_masked": t_masked},
        "tflops": {"baselines_all": evals * flops / (t_all * 1e-3) / 1e12,
                   "grid_symmetric_20": 20 * flops / (t_sym * 1e-3) / 1e12,
                   "given_scales_2": 2 * flops / (t_two * 1e-3) / 1e12,
                   "given_scales_1_masked": flops / (t_masked * 1e-3) / 1e12},
        "l2": "flushed (256 MiB write) before every timed call"}), flush=True)
    return 0


def run_gptq(args):
    """AWQ followed by GPTQ on one layer: each GPU stage timed on the device
    (CUDA events, after warm-up, L2 flushed before each), and the output error
    of RTN, AWQ, GPTQ alone and AWQ+GPTQ.  One JSON line."""
    import torch

    import awq_activation_aware_b200 as awq
    from awq_activation_aware_b200 import synth

    dev = torch.device("cuda", 0)
    cfg = synth.CONFIGS[args.config]
    bits = args.bits or cfg.bits
    group = args.group or cfg.group
    W, X, _ = synth.generate(cfg)
    Wd = torch.from_numpy(W).to(dev)
    Xd = torch.from_numpy(X).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = max(args.steps, 3)

    def timed(fn):
        for _ in range(2):
            flush.zero_()
            out = fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b.record()
            out = fn()
            e.record()
            torch.cuda.synchronize()
            ts.append(b.elapsed_time(e))
        return out, statistics.median(ts)

    res, t_awq = timed(lambda: awq.quantize_layer(Wd, Xd, bits=bits, group=group))
    s = res["s_best"]
    H, t_h = timed(lambda: awq.gptq_hessian(Xd, s))
    U, t_f = timed(lambda: awq.gptq_factor(H))
    q, t_q = timed(lambda: awq.gptq_quantize(Wd, s, U, bits, group))
    loss_both, t_l = timed(lambda: awq.output_error(Wd, q["W_hat"], Xd))
    ones = torch.ones(cfg.K, dtype=torch.float32, device=dev)
    plain = awq.gptq_layer(Wd, Xd, ones, bits, group)
    awq.get_status()
    N, K, T = cfg.N, cfg.K, cfg.T
    print(json.dumps({
        "op": "gptq", "config": cfg.name, "bits": bits, "group": group,
        "losses": {"rtn": float(res["losses"][0]), "awq": float(res["losses"].min()), "gptq": float(plain["loss"]),
                   "awq_gptq": float(loss_both)},
        "ms": {"awq_search_and_pack": t_awq, "hessian": t_h, "factor": t_f, "sweep": t_q, "output_error": t_l},
        "rates": {"hessian_tflops": 2.0 * K * K * T / 2 / (t_h * 1e-3) / 1e12,
                  "factor_gflops": (2.0 / 3.0) * K ** 3 / (t_f * 1e-3) / 1e9,
                  "sweep_tflops": 1.0 * N * K * K / (t_q * 1e-3) / 1e12},
        "l2": "flushed (256 MiB write) before every timed call"}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "qlinear":
        return run_qlinear(args)
    if args.op == "baselines":
        return run_baselines(args)
    if args.op == "gptq":
        return run_gptq(args)
    return run_awq(args)


if __name__ == "__main__":
    sys.exit(main())
