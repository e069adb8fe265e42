#!/usr/bin/env python
"""Throughput of the lookahead importance-scoring path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--cmax C]
    python bench.py --suite ...               # one JSON line per workload
    python bench.py --impl reference ...      # the fp64 CPU oracle on the host cores

One step = the two scoring passes (speckv_row_offsets + speckv_colsum, which
together are speckv_score) + topk_select (pool 7, top-C_max + window) +
kv_compact over every unit of the workload, through the C ABI of
libspeckv.so.  Default workload: the Qwen2.5-32B-shaped SpecKV pass at 64K
context (64 layers, 40/8 heads, head_dim 128, window 64, lookahead 128,
C_max 256), seeded synthetic bf16 inputs resident in HBM (K and V are 8.6 GB
each, far larger than the 126 MB L2, so no L2 flush is needed between steps).
CUDA events are recorded on the launching stream between the kernels of
every timed step, so each kernel's time is measured inside the timed region
and the kernels' times add up to the step.
Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
seed (units are independent, no data-path collective): weak scaling.
Prints one JSON line on rank 0 (one per workload with --suite).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "KV-head-tokens scored+selected+compacted/s at 64K ctx"
SUITE = ("llama3.1-8b_speckv_16k", "qwen2.5-32b_speckv_64k", "qwen2.5-32b_speckv_64k@1024",
         "qwen2.5-32b_speckv_64k@2048", "qwen2.5-32b_speckv_64k+prefill", "qwen2.5-0.5b_specpc_32k",
         "cascade_specpc_speckv_128k", "qwen2.5-32b_decode_compressed", "llama3.1-8b_vs_prefill_16k")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--config", default=W.QWEN32B_64K.name,
                    help="workload name (see workloads.CONFIGS), optionally with @C_max or +prefill")
    ap.add_argument("--layers", type=int, default=None, help="override the workload's layer count (small captures)")
    ap.add_argument("--cmax", type=int, default=None)
    ap.add_argument("--suite", action="store_true", help="one line per workload (headline included)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-full-cache", action="store_true",
                    help="decode workload: skip the full-cache contrast (keeps device memory small)")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="e2e: groups of (batch, layer) whose host-to-device copy overlaps the previous group's work")
    return ap.parse_args(argv)


def config_of(name, cmax=None, layers=None):
    """A workload by name; "<name>@C" sets C_max, "<name>+prefill" runs the
    scoring after the prefill attention of the window and lookahead rows;
    layers overrides the layer count (small profiling captures)."""
    name = name.replace("+prefill", "")
    if "@" in name:
        name, c = name.split("@")
        cmax = int(c)
    if name not in W.CONFIGS:
        raise SystemExit(f"unknown workload {name!r}; one of {sorted(W.CONFIGS)}")
    cfg = W.CONFIGS[name]
    if cmax is not None and isinstance(cfg, W.SpecKVConfig):
        cfg = dataclasses.replace(cfg, c_max=cmax)
    if layers is not None and hasattr(cfg, "layers"):
        cfg = dataclasses.replace(cfg, layers=layers)
    return cfg


# ----------------------------------------------------------------- work and bytes
def specpc_flops(cfg: W.SpecPCConfig) -> float:
    """One Q.K^T product over the causally visible keys of every SpecPC row
    (query position n_in + n_lookahead - 1 - W + i), all query heads and
    layers >= l_skip: 2 * d * sum_i c_i per (batch, layer, query head)."""
    c0 = cfg.n_in + cfg.n_lookahead - cfg.n_rows
    vis = sum(min(cfg.n_in, c0 + i) for i in range(cfg.n_rows))
    return 2.0 * cfg.head_dim * vis * cfg.batch * cfg.layers_used * cfg.hq


def algorithmic_flops(cfg: W.SpecKVConfig) -> float:
    """One Q.K^T product over the causally visible keys of every row:
    2 * d * g * sum_i c_i per unit (each of the two passes does this once)."""
    vis = sum(cfg.n_pre + i + 1 for i in range(cfg.n_window)) + cfg.n_lookahead * cfg.n_in
    return 2.0 * cfg.head_dim * cfg.g * vis * cfg.units


def prefill_flops(cfg: W.SpecKVConfig) -> float:
    """The prefill attention of the window and lookahead rows: Q.K^T and P.V
    over every row's visible keys (input keys, and for lookahead row i the
    lookahead keys up to its own): 2 products x 2 * d * g * sum_i c_i per unit."""
    look = sum(i + 1 for i in range(cfg.n_lookahead))
    return 2.0 * (algorithmic_flops(cfg) + 2.0 * cfg.head_dim * cfg.g * look * cfg.units)


def algorithmic_bytes(cfg: W.SpecKVConfig) -> float:
    """K read once, Q read once, scores written and read once, K and V rows of
    the reduced cache read and written once."""
    d = cfg.head_dim
    per_unit = cfg.n_in * d * 2 + cfg.g * cfg.rows * d * 2 + 8 * cfg.n_pre + 4 * cfg.keep * d * 2
    return per_unit * cfg.units


def topk_bytes(units: int, n_cand: int, out_len: int) -> float:
    """The selection's algorithmic traffic: every score read once, the indices written."""
    return units * (4.0 * n_cand + 4.0 * out_len)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def tensor_peak(peaks):
    """Every kernel is timed per launch (milliseconds each): the roofline
    denominator is the burst bf16 GEMM figure.  The sustained (power-capped,
    seconds-long) figure is reported beside it for context only."""
    return peaks["bf16_tflops"], f"{peaks['source']} bf16 burst (per-launch kernel timing)"


def exp2_peak_per_s():
    """Exponentials per second the SMs can produce: the MUFU gives 16 ex2 per
    clock per SM; the FMA pipe (128 lanes) spends 2 lane-ops per logit on the
    scale and the sum and 7 per polynomial exponential, so the best split
    (40 % polynomial) reaches 16 / 0.6 = 26.7 exponentials per clock per SM."""
    return 148 * (16.0 / 0.6) * 1965e6


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- timed steps
def timed_steps(launches, steps, warmup, stream, barrier=lambda: None):
    """Run `warmup` untimed steps, then `steps` timed ones.  A step runs the
    (name, fn) launches in order; a CUDA event is recorded on `stream` before
    the first launch and after every launch.  Returns the total device time
    of the timed steps (first event to last), each launch's mean time, the
    median step time and the clock summary sampled during the timed steps."""
    import torch
    for _ in range(warmup):
        for _, fn in launches:
            fn()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(launches) + 1)] for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        time.sleep(0.3)
        for s in range(steps):
            ev[s][0].record(stream)
            for i, (_, fn) in enumerate(launches):
                fn()
                ev[s][i + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    total = ev[0][0].elapsed_time(ev[-1][-1])
    per = {name: sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)) / steps
           for i, (name, _) in enumerate(launches)}
    step_ms = sorted(ev[s][0].elapsed_time(ev[s][-1]) for s in range(steps))
    return total, per, step_ms[len(step_ms) // 2], clk.summary()


def check_device(P, when):
    st, site = P.spk_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at site {site} {when}")


# ----------------------------------------------------------------- oracle timing (CPU baseline)
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _oracle_job(job):
    """One oracle sample (fp64, single thread).  The process draws its own
    seeded inputs first (not timed), then runs the oracle:
      ("speckv", cfg, seed, unit, heads): scores -> pool -> top-C + window ->
          gather of K and V for one unit (the rows of its first `heads` query
          heads, or all of them);
      ("specpc", cfg, seed, b, layer, heads): SpecPC scores of one scored
          layer of batch element b (its first `heads` query heads and their
          KV heads, or all of them), then pool + top-K.
    Returns the oracle's wall seconds in this single-threaded process."""
    sys.path.insert(0, ROOT)
    import oracle
    kind, cfg, seed = job[0], job[1], job[2]
    if kind == "speckv":
        u, heads = job[3], job[4]
        qb, kb, vb = W.speckv_unit_numpy(cfg, seed, u)
        if heads is not None:
            qb = np.ascontiguousarray(qb[:heads])
        t0 = time.perf_counter()
        s, p, idx = oracle.speckv_select_unit(qb, kb, cfg.n_window, cfg.n_lookahead, cfg.c_max, cfg.pool)
        oracle.gather_rows(kb, idx)
        oracle.gather_rows(vb, idx)
        return time.perf_counter() - t0
    b, layer, heads = job[3], job[4], job[5]
    qb, kb = W.specpc_layer_numpy(cfg, seed, b, layer)
    if heads is not None:
        qb = np.ascontiguousarray(qb[:heads])
        kb = np.ascontiguousarray(kb[:max(1, heads // cfg.g)])
    w = W.specpc_row_weights(cfg.n_rows).astype(np.float32).astype(np.float64)
    t0 = time.perf_counter()
    s = oracle.specpc_batch(qb[None], kb[None], w, 0, cfg.n_lookahead)
    oracle.topk_with_tail(oracle.maxpool(s, cfg.pool), cfg.keep, 0)
    return time.perf_counter() - t0


def run_oracle_pool(jobs, cores):
    """Run the jobs over `cores` spawned single-threaded processes (spawned,
    so that none inherits a CUDA context); returns each job's oracle seconds."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    with ctx.Pool(processes=cores) as pool:
        pool.map(_oracle_job, jobs[:1])                     # warm: import + build
        return pool.map(_oracle_job, jobs, chunksize=1)


def cpu_baseline_speckv(cfg, seed, cores, full=False):
    """The oracle on all host cores, one single-threaded process per core.
    full: every unit of the workload; else one sample per core, each a unit
    restricted to one query head's rows (1/g of the unit's work).  value =
    the work timed / (the summed oracle seconds / cores)."""
    if full:
        secs = run_oracle_pool([("speckv", cfg, seed, u, None) for u in range(cfg.units)], cores)
        value = cfg.kv_head_tokens / (sum(secs) / cores)
        sample = (f"all {cfg.units} units of {cfg.name}, one process per core on {cores} cores, "
                  f"{sum(secs):.0f} oracle CPU-s")
    else:
        secs = run_oracle_pool([("speckv", cfg, seed, u % 8, 1) for u in range(cores)], cores)
        value = cores * cfg.n_in / cfg.g / (sum(secs) / cores)
        sample = (f"{cores} samples, one per core, each one unit of {cfg.name} restricted to the rows of 1 "
                  f"of its {cfg.g} query heads (1/{cfg.g} unit), {sum(secs):.0f} oracle CPU-s; the full step "
                  f"has {cfg.units} units")
    return {"value": value, "unit": "KV-head-tokens/s", "cores": cores, "kind": "oracle", "sample": sample}


def cpu_baseline_specpc(cfg, seed, cores):
    """The whole SpecPC workload on the host cores: every (batch element,
    scored layer) as its own oracle call; the final mean over layers and max
    over heads (n_in additions per layer) is not timed."""
    jobs = [("specpc", cfg, seed, b, l, None) for b in range(cfg.batch) for l in range(cfg.layers_used)]
    secs = run_oracle_pool(jobs, cores)
    return {"value": cfg.kv_head_tokens / (sum(secs) / cores), "unit": "KV-head-tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"the whole workload: {len(jobs)} (batch, layer) oracle calls of {cfg.name} over {cores} "
                      f"cores, {sum(secs):.0f} oracle CPU-s"}


def cpu_baseline_cascade(cc, seed, cores):
    """Sampled and extrapolated: step 1 timed on one query head (with its KV
    head) of every scored layer of one batch element, step 2 on up to `cores`
    units of the gathered target cache; the CPU-seconds are scaled to the full
    job and spread over the host cores."""
    d, t = cc.draft, cc.target
    s1 = run_oracle_pool([("specpc", d, seed, 0, l, 1) for l in range(d.layers_used)], cores)
    tg = W.SpecKVConfig("cascade_target_2k", batch=t.batch, layers=t.layers, hq=t.hq, hkv=t.hkv,
                        head_dim=t.head_dim, n_in=d.keep, n_window=t.n_window, n_lookahead=t.n_lookahead,
                        c_max=t.c_max, heavy_frac=t.heavy_frac)
    n2 = min(cores, tg.units)
    s2 = run_oracle_pool([("speckv", tg, seed, u, None) for u in range(n2)], cores)
    full_cpu = sum(s1) * d.batch * d.hq + sum(s2) * tg.units / n2
    tokens = t.batch * t.layers * t.hkv * cc.n_in_full
    return {"value": tokens / (full_cpu / cores), "unit": "target KV-head-tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"extrapolated: step 1 timed on 1 of {d.hq} query heads of one batch element "
                      f"({sum(s1):.0f} CPU-s, x {d.batch * d.hq}), step 2 on {n2} of {tg.units} units "
                      f"({sum(s2):.0f} CPU-s); {full_cpu:.0f} CPU-s over {cores} cores"}


def run_reference(args, cfg):
    """--impl reference: the fp64 oracle on the host cores, same metric and
    workload; each step is one sample per core (a unit restricted to one
    query head's rows), all in parallel, and takes as long as its slowest
    sample; the whole run stays within a few minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = host_cores()
    jobs = [("speckv", cfg, args.seed, u % 8, 1) for u in range(cores)]
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    times = []
    with ctx.Pool(processes=cores) as pool:
        pool.map(_oracle_job, jobs[:1])
        for s in range(args.warmup + args.steps):
            secs = pool.map(_oracle_job, jobs, chunksize=1)
            if s >= args.warmup:
                times.append(max(secs))
    step = sum(times) / len(times)
    value = cores * cfg.n_in / cfg.g / step
    sample = (f"{cores} samples per step, one per core, each = one unit of {cfg.name} with the rows of 1 of "
              f"its {cfg.g} query heads (1/{cfg.g} unit of work); a step lasts as long as its slowest sample; "
              f"the full step has {cfg.units} units")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "KV-head-tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "units_per_step": cores, "n_in": cfg.n_in,
                   "c_max": cfg.c_max, "pool": cfg.pool},
        "cpu_baseline": {"value": value, "unit": "KV-head-tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "KV-head-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- multi-rank plumbing
def rank_seed(seed: int, rank: int) -> int:
    """Every rank scores its own batch of units (weak scaling): own seed."""
    return seed + 1000 * rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar (device time) over all ranks."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, units_tokens: int, steps: int, ms_total_max: float) -> float:
    """KV-head-tokens per second over all ranks: every rank processed
    units_tokens per step; the job took the slowest rank's time."""
    return world * units_tokens * steps / (ms_total_max * 1e-3)


def kernel_roofline(name, ms, flops, peaks, traffic=None):
    """Roofline object of a tensor-bound scoring kernel from its in-step time."""
    peak, src = tensor_peak(peaks)
    achieved = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": name, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic, "peak_source": src,
            "sustained_peak": peaks.get("bf16_tflops_sustained"),
            "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                  if peaks.get("bf16_tflops_sustained") else None)}


# ----------------------------------------------------------------- SpecKV workloads
def run_speckv(args, cfg, P, dev, world, rank, headline, prefill=False):
    """SpecKV: scoring passes + selection + compaction.  prefill: the first
    scoring pass is replaced by the prefill attention of the window and
    lookahead rows (which writes the same row offsets), so the step is that
    attention, the column pass, selection and compaction."""
    import torch
    import torch.distributed as dist
    from prompt_compression_b200.pipeline import SpeckvBuffers

    seed = rank_seed(args.seed, rank)
    inp = W.speckv_inputs(cfg, seed=seed, device=dev)
    q, k, v = inp["q"], inp["k"], inp["v"]
    buf = SpeckvBuffers(q, k, v, cfg.n_window, cfg.c_max)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    first = ("score_lse_pass", lambda: P.speckv_row_offsets(q, k, cfg.n_window, buf.ws_score, stream=stream))
    if prefill:
        gen = torch.Generator(device=dev).manual_seed(seed + 17)
        lshape = (cfg.batch, cfg.layers, cfg.hkv, cfg.n_lookahead, cfg.head_dim)
        k_look = torch.randn(lshape, generator=gen, device=dev).to(torch.bfloat16)
        v_look = torch.randn(lshape, generator=gen, device=dev).to(torch.bfloat16)
        attn_out = torch.empty_like(q)
        first = ("prefill_attention", lambda: P.speckv_prefill_attention(
            q, k, v, k_look, v_look, cfg.n_window, out=attn_out, workspace=buf.ws_score, stream=stream))
    launches = [
        first,
        ("score_colsum_pass", lambda: P.speckv_colsum(q, k, cfg.n_window, buf.scores, buf.ws_score,
                                                      stream=stream)),
        ("topk_select", lambda: P.topk_select(buf.scores, cfg.c_max, cfg.n_window, buf.idx, cfg.pool, None,
                                              buf.ws_topk, stream=stream)),
        ("kv_compact", lambda: P.kv_compact(k, v, buf.idx, buf.k_out, buf.v_out, 1, stream=stream)),
    ]
    total, per, med, clocks = timed_steps(launches, args.steps, args.warmup, stream, barrier)
    check_device(P, "in the timed steps")
    ms_total = max_over_ranks(total, world, dev)
    ms_step = ms_total / args.steps
    value = whole_job_value(world, cfg.kv_head_tokens, args.steps, ms_total)

    peaks = load_peaks()
    flops_pass = algorithmic_flops(cfg)
    peak, _ = tensor_peak(peaks)
    kernels = {
        launches[0][0]: {"ms": per[launches[0][0]],
                         "tflops": flops_pass / (per[launches[0][0]] * 1e-3) / 1e12},
        "score_colsum_pass": {"ms": per["score_colsum_pass"],
                              "tflops": flops_pass / (per["score_colsum_pass"] * 1e-3) / 1e12},
        "topk_select": {"ms": per["topk_select"],
                        "gbs": topk_bytes(cfg.units, cfg.n_pre, cfg.keep) / (per["topk_select"] * 1e-3) / 1e9},
        "kv_compact": {"ms": per["kv_compact"],
                       "gbs": cfg.units * 4 * cfg.keep * cfg.head_dim * 2 / (per["kv_compact"] * 1e-3) / 1e9},
    }
    if prefill:
        kernels["prefill_attention"]["tflops"] = prefill_flops(cfg) / (per["prefill_attention"] * 1e-3) / 1e12
    for name in ("score_lse_pass", "score_colsum_pass", "prefill_attention"):
        if name in kernels:
            kernels[name]["frac"] = kernels[name]["tflops"] / peak
    for name in ("topk_select", "kv_compact"):
        kernels[name]["frac_hbm"] = kernels[name]["gbs"] / peaks["hbm_gbs"]
    first_name = launches[0][0]
    first_flops = prefill_flops(cfg) if prefill else flops_pass
    dom = max((first_name, "score_colsum_pass"), key=lambda n: per[n])
    roofline = kernel_roofline(dom, per[dom], first_flops if dom == first_name else flops_pass, peaks,
                               captured_traffic(dom, cfg.name))
    roofline["step_roofline_ms"] = max((first_flops + flops_pass) / (peak * 1e12),
                                       algorithmic_bytes(cfg) / (peaks["hbm_gbs"] * 1e9)) * 1e3
    roofline["step_frac"] = roofline["step_roofline_ms"] / ms_step
    roofline["kernel_ms_sum"] = sum(per.values())

    e2e = None
    if headline and not args.no_e2e:
        e2e = run_e2e(args, cfg, P, q, k, v, dev, stream, world, lambda x: max_over_ranks(x, world, dev), barrier)
    del inp, q, k, v, buf
    torch.cuda.empty_cache()

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline_speckv(cfg, args.seed, host_cores(), full=cfg.n_in <= 16384)

    if prefill:
        metric = (f"KV-head-tokens attended+scored+selected+compacted/s ({cfg.name}: prefill attention of the "
                  f"window and lookahead rows, then the column pass)")
    elif headline:
        metric = METRIC
    else:
        metric = f"KV-head-tokens scored+selected+compacted/s ({cfg.name}, C_max {cfg.c_max})"
    return {
        "metric": metric,
        "value": value, "unit": "KV-head-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "ms_per_step_median": med,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "units": cfg.units, "layers": cfg.layers, "hq": cfg.hq,
                   "hkv": cfg.hkv, "head_dim": cfg.head_dim, "n_in": cfg.n_in, "n_window": cfg.n_window,
                   "n_lookahead": cfg.n_lookahead, "c_max": cfg.c_max, "pool": cfg.pool,
                   "l2": f"inputs larger than L2 (K, V {cfg.units * cfg.n_in * cfg.head_dim * 2 / 1e9:.2f} GB "
                         f"each); no flush",
                   "parallelism": f"units sharded, {world} rank(s), no collective"},
        "roofline": roofline, "kernels": kernels, "gpu_launches": len(launches) * args.steps,
        "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu,
    }


# ----------------------------------------------------------------- SpecPC and the cascade
def run_specpc_like(args, cfg, P, dev):
    """SpecPC (scores + pool + top-K prompt tokens over a draft) or the
    SpecKV-PC cascade (SpecPC on the draft, gather of the target cache,
    SpecKV on the gathered cache), one GPU."""
    import torch
    from prompt_compression_b200.pipeline import SpeckvBuffers
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    cascade = isinstance(cfg, W.CascadeConfig)
    d = cfg.draft if cascade else cfg
    dr = W.specpc_inputs(d, seed=args.seed, device=dev)
    w = torch.from_numpy(W.specpc_row_weights(d.n_rows).astype(np.float32)).to(dev)
    pc_scores = torch.empty((d.batch, d.n_in), dtype=torch.float32, device=dev)
    pc_idx = torch.empty((d.batch, min(d.keep, d.n_in)), dtype=torch.int32, device=dev)
    shape = P.binding.specpc_shape(dr["q"], dr["k"], d.l_skip, d.n_lookahead)
    ws_pc = torch.empty(max(P.specpc_workspace_size(shape), 256), dtype=torch.uint8, device=dev)
    ws_tk = torch.empty(max(P.topk_workspace_size(d.batch, d.n_in), 256), dtype=torch.uint8, device=dev)
    pc_flops = specpc_flops(d)
    # the column pass adds a merge launch when it splits the segments into groups
    offsets = -(-(d.units * (-(-d.g * d.n_rows // 128)) * 4096) // 256) * 256
    merge = ws_pc.numel() > max(offsets, 256)
    launches = [
        ("specpc_lse_pass", lambda: P.specpc_row_offsets(dr["q"], dr["k"], w, ws_pc, d.l_skip, d.n_lookahead,
                                                         stream=stream)),
        ("specpc_colsum_pass", lambda: P.specpc_colsum(dr["q"], dr["k"], pc_scores, ws_pc, d.l_skip,
                                                       d.n_lookahead, stream=stream)),
        ("specpc_topk", lambda: P.topk_select(pc_scores, d.keep, 0, pc_idx, d.pool, None, ws_tk, stream=stream)),
    ]
    if cascade:
        t = cfg.target
        tfull = W.SpecKVConfig("cascade_target_full", batch=t.batch, layers=t.layers, hq=t.hq, hkv=t.hkv,
                               head_dim=t.head_dim, n_in=cfg.n_in_full, n_window=t.n_window,
                               n_lookahead=t.n_lookahead, c_max=t.c_max, heavy_frac=t.heavy_frac)
        tg = W.speckv_inputs(tfull, seed=args.seed + 1, device=dev, heavy_pos=dr["heavy"])
        kg = torch.empty((t.batch, t.layers, t.hkv, d.keep, t.head_dim), dtype=torch.bfloat16, device=dev)
        vg = torch.empty_like(kg)
        buf = SpeckvBuffers(tg["q"], kg, vg, t.n_window, t.c_max)
        tcfg = W.SpecKVConfig("g", batch=t.batch, layers=t.layers, hq=t.hq, hkv=t.hkv, head_dim=t.head_dim,
                              n_in=d.keep, n_window=t.n_window, n_lookahead=t.n_lookahead, c_max=t.c_max)
        launches += [
            ("cascade_gather", lambda: P.kv_compact(tg["k"], tg["v"], pc_idx, kg, vg, t.layers * t.hkv,
                                                    stream=stream)),
            ("target_lse_pass", lambda: P.speckv_row_offsets(tg["q"], kg, t.n_window, buf.ws_score, stream=stream)),
            ("target_colsum_pass", lambda: P.speckv_colsum(tg["q"], kg, t.n_window, buf.scores, buf.ws_score,
                                                           stream=stream)),
            ("target_topk", lambda: P.topk_select(buf.scores, t.c_max, t.n_window, buf.idx, t.pool, None,
                                                  buf.ws_topk, stream=stream)),
            ("target_compact", lambda: P.kv_compact(kg, vg, buf.idx, buf.k_out, buf.v_out, 1, stream=stream)),
        ]
        tokens = t.batch * t.layers * t.hkv * cfg.n_in_full
        metric = "target KV-head-tokens compressed/s (SpecPC 128K -> 2048 -> SpecKV 256 + 64)"
        unit = "target KV-head-tokens/s"
    else:
        tokens = d.kv_head_tokens
        metric = "KV-head-tokens scored+selected/s (SpecPC draft)"
        unit = "KV-head-tokens/s"
    total, per, med, clocks = timed_steps(launches, args.steps, args.warmup, stream)
    check_device(P, "in the timed steps")
    ms_step = total / args.steps
    # each SpecPC pass evaluates one exp2 per visible logit: the exponential
    # stream binds at head_dim 64 (the tensor work per logit is halved)
    exps = pc_flops / (2 * d.head_dim)
    kernels = {}
    for name in ("specpc_lse_pass", "specpc_colsum_pass"):
        kernels[name] = {"ms": per[name], "tflops": pc_flops / (per[name] * 1e-3) / 1e12,
                         "gexp2_per_s": exps / (per[name] * 1e-3) / 1e9}
    for name in per:
        kernels.setdefault(name, {"ms": per[name]})
    dom = max(("specpc_lse_pass", "specpc_colsum_pass"), key=lambda n: per[n])
    peak_exp = exp2_peak_per_s() / 1e9
    ach_exp = exps / (per[dom] * 1e-3) / 1e9
    roofline = {"bound": "alu", "kernel": dom, "achieved": ach_exp, "peak": peak_exp, "unit": "Gexp2/s",
                "frac": ach_exp / peak_exp, "traffic": None,
                "peak_source": "derived: 148 SMs x 26.7 exp2/clk (MUFU 16/clk + FMA-pipe polynomial) x 1965 MHz",
                "tensor_frac": kernels[dom]["tflops"] / tensor_peak(peaks)[0],
                "kernel_ms_sum": sum(per.values())}
    if cascade:
        tf = algorithmic_flops(tcfg)
        for name in ("target_lse_pass", "target_colsum_pass"):
            kernels[name]["tflops"] = tf / (per[name] * 1e-3) / 1e12
        kernels["cascade_gather"]["gbs"] = (2 * 2 * t.batch * t.layers * t.hkv * d.keep * t.head_dim * 2
                                            / (per["cascade_gather"] * 1e-3) / 1e9)
        roofline["step_roofline_ms"] = (2 * pc_flops / (exp2_peak_per_s() * 2 * d.head_dim) * 1e3
                                        + 2 * tf / (tensor_peak(peaks)[0] * 1e12) * 1e3)
        roofline["step_frac"] = roofline["step_roofline_ms"] / ms_step
    else:
        roofline["step_roofline_ms"] = 2 * exps / exp2_peak_per_s() * 1e3
        roofline["step_frac"] = roofline["step_roofline_ms"] / ms_step
    del dr
    if cascade:
        del tg, kg, vg, buf
    torch.cuda.empty_cache()
    cpu = None
    if not args.no_cpu_baseline:
        cpu = cpu_baseline_cascade(cfg, args.seed, host_cores()) if cascade else \
            cpu_baseline_specpc(cfg, args.seed, host_cores())
    return {
        "metric": metric, "value": tokens / (ms_step * 1e-3), "unit": unit, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "ms_per_step_median": med,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "l2": "inputs larger than L2; no flush"},
        "roofline": roofline, "kernels": kernels,
        "gpu_launches": (len(launches) + (1 if merge else 0)) * args.steps,
        "clocks": clocks, "e2e": None, "cpu_baseline": cpu,
    }


# ----------------------------------------------------------------- decode over the compressed cache
def run_decode(args, cfg, P, dev):
    """One decode step over the compressed cache (C_max + window rows per KV
    head) on every (layer, query head); the same step over the full cache is
    timed for contrast.  Four copies of the compressed cache are used in
    rotation so that consecutive launches read 4 x 84 MB, more than the L2;
    the full cache (17 GB) is far larger than the L2."""
    import torch
    stream = torch.cuda.current_stream(dev)
    gen = torch.Generator(device=dev).manual_seed(args.seed)
    B_, L, hq, hkv, d = cfg.batch, cfg.layers, cfg.hq, cfg.hkv, cfg.head_dim

    def rnd(*shape):
        return torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16)

    copies = 4
    qs = [rnd(B_, L, hq, d) for _ in range(copies)]
    kcs = [rnd(B_, L, hkv, cfg.n_kv, d) for _ in range(copies)]
    vcs = [rnd(B_, L, hkv, cfg.n_kv, d) for _ in range(copies)]
    out = torch.empty((B_, L, hq, d), dtype=torch.float32, device=dev)
    scale = d ** -0.5
    # One step is shorter than a Python-level launch, so the steps are
    # captured once in a CUDA graph (the C entry points allocate and
    # synchronise nothing) and the graph is replayed: the device time is the
    # kernels' own, not the host's launch rate.
    reps = 20
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for i in range(copies):             # warm-up outside the capture (first-call set-up)
            P.decode_attention(qs[i], kcs[i], vcs[i], out, scale, side)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=side):
        for i in range(reps):
            P.decode_attention(qs[i % copies], kcs[i % copies], vcs[i % copies], out, scale, side)
    torch.cuda.synchronize()
    launches = [("decode_graph", lambda: graph.replay())]
    total, per, med, clocks = timed_steps(launches, max(args.steps, 20), max(3, args.warmup), stream)
    check_device(P, "in the timed steps")
    steps = max(args.steps, 20) * reps
    ms = total / steps
    del graph
    del kcs, vcs
    ms_full = None
    if not args.no_full_cache:
        kf, vf = rnd(B_, L, hkv, cfg.n_kv_full, d), rnd(B_, L, hkv, cfg.n_kv_full, d)
        tf, _, _, _ = timed_steps([("full", lambda: P.decode_attention(qs[0], kf, vf, out, scale, stream))],
                                  max(args.steps, 5), 3, stream)
        ms_full = tf / max(args.steps, 5)
        del kf, vf
    torch.cuda.empty_cache()
    peaks = load_peaks()
    nbytes = cfg.units * cfg.n_kv * d * 2 * 2 + B_ * L * hq * d * (2 + 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {
        "metric": "decode over the compressed cache: query-head tokens/s", "value": B_ * L * hq / (ms * 1e-3),
        "unit": "query-head tokens/s", "n_gpus": 1, "steps": steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name, "n_kv": cfg.n_kv, "units": cfg.units, "hq": hq, "head_dim": d,
                   "l2": "4 cache copies in rotation (4 x 84 MB > L2); no flush",
                   "timing": f"CUDA graph of {reps} launches replayed; events around each replay"},
        "roofline": {"bound": "hbm", "kernel": "decode_stream_kernel", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peaks['source']} HBM copy"},
        "full_cache": None if ms_full is None else {
            "n_kv": cfg.n_kv_full, "ms_per_step": ms_full,
            "gbs": cfg.units * cfg.n_kv_full * d * 4 / (ms_full * 1e-3) / 1e9},
        "gpu_launches": steps, "clocks": clocks, "e2e": None, "cpu_baseline": None,
    }


# ----------------------------------------------------------------- Vertical-Slash sparse prefill
def vs_tile_work(cfg, vert, sl):
    """Key tiles the kernel processes (slash tiles + vertical tiles, summed over
    items) and the (row, key) pairs the pattern makes visible, from the same
    definitions the kernel and the oracle use."""
    import torch
    n, nq = cfg.n, cfg.n_q
    vert_c, sl_c = vert.cpu().numpy(), sl.cpu().numpy()
    tiles = 0
    visible = 0
    pos = np.arange(n - nq, n)
    for u in range(cfg.units):
        S = np.union1d(sl_c[u], [0])
        V = vert_c[u]
        for rb in range((nq + 127) // 128):
            p0 = n - nq + rb * 128
            p_last = n - nq + min(rb * 128 + 127, nq - 1)
            t = np.arange(p_last // 128 + 1)
            lo, hi = p0 - 128 * t - 127, p_last - 128 * t
            idx = np.searchsorted(S, lo)
            hit = (idx < S.size) & (S[np.minimum(idx, S.size - 1)] <= hi)
            cv = np.searchsorted(V, p_last, side="right")
            tiles += int(hit.sum()) + (cv + 127) // 128
        # visible pairs: diagonals of S u {0} within each row's prefix, plus
        # vertical keys not on those diagonals
        diag = sum(int(np.clip(pos - o + 1, 0, None).astype(bool).sum()) for o in S)
        vv = sum(int(((V <= p) & ~np.isin(p - V, S)).sum()) for p in pos[:: max(1, nq // 64)]) * max(1, nq // 64)
        visible += diag + vv
    return tiles * cfg.g, visible * cfg.g


def run_vs(args, cfg, P, dev):
    """Vertical-Slash sparse prefill over every query row of the sequence,
    one GPU: the vertical rows' gather (kv_compact) and the sparse attention."""
    import torch
    stream = torch.cuda.current_stream(dev)
    gen = torch.Generator(device=dev).manual_seed(args.seed)
    shape_q = (cfg.batch, cfg.layers, cfg.hq, cfg.n_q, cfg.head_dim)
    shape_k = (cfg.batch, cfg.layers, cfg.hkv, cfg.n, cfg.head_dim)
    q = (torch.randn(shape_q, generator=gen, device=dev) / cfg.head_dim ** 0.5).to(torch.bfloat16)
    k = torch.randn(shape_k, generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn(shape_k, generator=gen, device=dev).to(torch.bfloat16)
    vert, sl = W.vs_pattern(cfg, seed=args.seed, device=dev)
    out = torch.empty_like(q)
    ws = torch.empty(P.vs_workspace_size(P.binding.vs_shape(q, k, cfg.n_vertical, cfg.n_slash)), dtype=torch.uint8,
                     device=dev)
    launches = [("vs_sparse_attention", lambda: P.vs_sparse_attention(q, k, v, vert, sl, out=out, workspace=ws,
                                                                      stream=stream))]
    total, per, med, clocks = timed_steps(launches, args.steps, args.warmup, stream)
    check_device(P, "in the timed steps")
    ms = total / args.steps
    tiles, visible = vs_tile_work(cfg, vert, sl)
    peaks = load_peaks()
    peak, src = tensor_peak(peaks)
    tile_flops = tiles * 2 * 2 * 128 * 128 * cfg.head_dim
    useful_flops = visible * 2 * 2 * cfg.head_dim
    dense = cfg.batch * cfg.layers * cfg.hq * sum(range(cfg.n - cfg.n_q + 1, cfg.n + 1)) * 2 * 2 * cfg.head_dim
    del q, k, v, out, ws
    torch.cuda.empty_cache()
    achieved = tile_flops / (ms * 1e-3) / 1e12
    return {
        "metric": "query rows attended/s (Vertical-Slash sparse prefill)",
        "value": cfg.batch * cfg.layers * cfg.hq * cfg.n_q / (ms * 1e-3), "unit": "query-head rows/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_median": med,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "n": cfg.n, "n_q": cfg.n_q, "n_vertical": cfg.n_vertical,
                   "n_slash": cfg.n_slash, "l2": "inputs larger than L2; no flush"},
        "roofline": {"bound": "tensor", "kernel": "vs_attn_kernel (+ vertical gather)", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": captured_traffic("vs_attn_kernel", cfg.name), "peak_source": src,
                     "flops": "executed 128-key tiles x 2 products; useful (visible pairs) and dense-causal "
                              "figures beside it",
                     "useful_tflops": useful_flops / (ms * 1e-3) / 1e12,
                     "density_vs_dense_causal": useful_flops / dense},
        "gpu_launches": 2 * args.steps, "clocks": clocks, "e2e": None, "cpu_baseline": None,
    }


# ----------------------------------------------------------------- traffic bookkeeping
# The files that define each captured kernel (device code and its parameter
# block); profiles/traffic.json records, per kernel, the sha256 of these files
# at the capture, and the traffic is reported only while they are unchanged.
KERNEL_SOURCES = {
    "score_lse_pass": ("common.cuh", "exp2_poly.cuh", "score.cu", "score.cuh"),
    "score_colsum_pass": ("common.cuh", "exp2_poly.cuh", "score.cu", "score.cuh"),
    "prefill_attention": ("attn.cu", "common.cuh", "exp2_poly.cuh", "score.cuh"),
    "vs_attn_kernel": ("common.cuh", "exp2_poly.cuh", "score.cuh", "vs.cu"),
}
SCORING_SOURCES = KERNEL_SOURCES["score_colsum_pass"]


def kernel_source_digest(kernel="score_colsum_pass"):
    """sha256 over the sources of a captured kernel (KERNEL_SOURCES); the
    DRAM traffic captured with ncu is only reported while they are unchanged."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "prompt_compression_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        h.update(name.encode())
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()


def captured_traffic(kernel, workload):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch from
    profiles/traffic.json, or None when absent or captured from other sources."""
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(prof)).get("kernels", {}).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or kernel not in KERNEL_SOURCES or rec.get("source_sha256") != kernel_source_digest(kernel):
        return None
    return rec.get("workloads", {}).get(workload)


# ----------------------------------------------------------------- e2e
def run_e2e(args, cfg, P, q, k, v, dev, stream, world, max_over_ranks, barrier):
    """Same metric end to end from pinned host memory, through the public API.

    Per step, the (batch, layer) pairs are taken in `--e2e-chunks` groups.  Q
    and K of a group are copied to the device on a copy stream; the group is
    scored, selected and compacted (speckv_compress) on the compute stream as
    soon as its copy has landed (the next group's copy overlaps that work);
    the compacted K is gathered from the device copy of K, the compacted V
    straight from the pinned host V (only the selected rows cross the host
    link); the indices and the compacted K/V go back to pinned host memory on
    a third stream.  Each timed step runs from before its first copy to the
    end of its last copy back (events on the compute stream); the line
    reports the mean and the median step.  If the host V cannot be read in
    place, it is copied like K."""
    import torch
    from prompt_compression_b200.pipeline import SpeckvBuffers
    need = (q.numel() + k.numel() + v.numel()) * 2
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = None
    if avail is not None and avail < 2 * need:
        return {"value": None, "unit": "KV-head-tokens/s", "skipped":
                f"host RAM available {avail / 2**30:.0f} GiB < 2 x {need / 2**30:.0f} GiB of pinned inputs"}
    hq_ = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
    hq_.copy_(q)
    hk.copy_(k)
    hv.copy_(v)
    n_bl = q.shape[0] * q.shape[1]
    n_chunks = max(1, min(args.e2e_chunks, n_bl))
    cuts = [round(i * n_bl / n_chunks) for i in range(n_chunks + 1)]

    def group(t, lo, hi):   # (batch, layer) pairs lo..hi-1 as a [1][hi-lo][...] view
        return t.view(n_bl, *t.shape[2:])[lo:hi].view(1, hi - lo, *t.shape[2:])

    dq, dk = torch.empty_like(q), torch.empty_like(k)
    v_in_place = True
    try:
        P.mapped_host_pointer(group(hv, cuts[0], cuts[1]))
    except Exception:
        v_in_place = False
    dv = None if v_in_place else torch.empty_like(v)
    groups = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        gq, gk = group(dq, lo, hi), group(dk, lo, hi)
        gv = group(hv, lo, hi) if v_in_place else group(dv, lo, hi)
        buf = SpeckvBuffers(gq, gk, gv, cfg.n_window, cfg.c_max)
        out = (torch.empty(buf.idx.shape, dtype=buf.idx.dtype, pin_memory=True),
               torch.empty(buf.k_out.shape, dtype=buf.k_out.dtype, pin_memory=True),
               torch.empty(buf.v_out.shape, dtype=buf.v_out.dtype, pin_memory=True))
        groups.append((lo, hi, gq, gk, gv, buf, out))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step():
        s_in.wait_stream(stream)            # the previous step is done with the device inputs
        for lo, hi, gq, gk, gv, buf, out in groups:
            with torch.cuda.stream(s_in):
                gq.copy_(group(hq_, lo, hi), non_blocking=True)
                gk.copy_(group(hk, lo, hi), non_blocking=True)
                if not v_in_place:
                    gv.copy_(group(hv, lo, hi), non_blocking=True)
            stream.wait_stream(s_in)
            P.speckv_compress(gq, gk, gv, cfg.n_window, cfg.c_max, cfg.pool, buffers=buf, stream=stream)
            s_out.wait_stream(stream)
            with torch.cuda.stream(s_out):
                out[0].copy_(buf.idx, non_blocking=True)
                out[1].copy_(buf.k_out, non_blocking=True)
                out[2].copy_(buf.v_out, non_blocking=True)
        stream.wait_stream(s_out)           # the step ends with its last copy back

    step()
    torch.cuda.synchronize()
    barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.e2e_steps + 1)]
    ev[0].record(stream)
    for i in range(args.e2e_steps):
        step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev[0].elapsed_time(ev[-1])) / args.e2e_steps
    per_step = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(args.e2e_steps))
    keep_rows = sum(g[5].idx.numel() for g in groups)
    h2d = (q.numel() + k.numel()) * 2 + (keep_rows * cfg.head_dim * 2 if v_in_place else v.numel() * 2)
    d2h = sum(g[6][0].numel() * 4 + (g[6][1].numel() + g[6][2].numel()) * 2 for g in groups)
    return {"value": world * cfg.kv_head_tokens / (ms * 1e-3), "unit": "KV-head-tokens/s",
            "ms_per_step": ms, "ms_per_step_median": per_step[len(per_step) // 2],
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": args.e2e_steps, "groups": n_chunks,
            "v": "selected rows read in place from pinned host memory" if v_in_place else "copied"}


# ----------------------------------------------------------------- main
def main(argv=None):
    args = parse(argv)
    cfg = config_of(args.config, args.cmax, args.layers)
    if args.impl == "reference":
        if not isinstance(cfg, W.SpecKVConfig):
            print(json.dumps({"impl": "reference", "unavailable":
                              "the CPU reference arm times the SpecKV workloads only"}))
            return
        run_reference(args, cfg)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P

    names = SUITE if args.suite else (args.config + (f"@{args.cmax}" if args.cmax else ""),)
    lines = []
    for name in names:
        c = config_of(name, layers=None if args.suite else args.layers)
        prefill = name.endswith("+prefill")
        headline = (c == W.QWEN32B_64K) and not prefill
        if isinstance(c, W.SpecKVConfig):
            line = run_speckv(args, c, P, dev, world, rank, headline, prefill)
        elif world > 1:
            continue                         # the other workloads are single-GPU lines
        elif isinstance(c, W.DecodeConfig):
            line = run_decode(args, c, P, dev)
        elif isinstance(c, W.VSConfig):
            line = run_vs(args, c, P, dev)
        else:
            line = run_specpc_like(args, c, P, dev)
        lines.append((headline, line))
        if rank == 0 and args.suite:
            print(json.dumps(line), flush=True)
        torch.cuda.empty_cache()
    if rank == 0 and not args.suite:
        print(json.dumps(lines[-1][1]), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
