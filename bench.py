#!/usr/bin/env python
"""Throughput of the lookahead importance-scoring path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--cmax C]
    python bench.py --impl reference ...      # the fp64 CPU oracle on the host cores

One step = speckv_score (row-LSE pass + column-sum pass) + topk_select (pool 7,
top-C_max + window) + kv_compact over every unit of the workload, through the
C ABI of libspeckv.so.  Default workload: the Qwen2.5-32B-shaped SpecKV pass at
64K context (64 layers, 40/8 heads, head_dim 128, window 64, lookahead 128,
C_max 256), seeded synthetic bf16 inputs resident in HBM (K and V are 8.6 GB
each, far larger than the 126 MB L2, so no L2 flush is needed between steps).
Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
seed (units are independent, no data-path collective): weak scaling.
Prints one JSON line on rank 0.
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

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "KV-head-tokens scored+selected+compacted/s at 64K ctx"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--config", default=W.QWEN32B_64K.name, choices=list(W.CONFIGS))
    ap.add_argument("--cmax", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="e2e: groups of (batch, layer) whose host-to-device copy overlaps the previous group's work")
    return ap.parse_args()


def config_of(args):
    import dataclasses
    cfg = W.CONFIGS[args.config]
    if args.cmax is not None and isinstance(cfg, W.SpecKVConfig):
        cfg = dataclasses.replace(cfg, c_max=args.cmax)
    return cfg


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


def algorithmic_bytes(cfg: W.SpecKVConfig) -> float:
    """K read once, Q read once, scores written and read once, K and V rows of
    the reduced cache read and written once."""
    d = cfg.head_dim
    per_unit = cfg.n_in * d * 2 + cfg.g * cfg.rows * d * 2 + 8 * cfg.n_pre + 4 * cfg.keep * d * 2
    return per_unit * cfg.units


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


# ----------------------------------------------------------------- oracle timing
def _oracle_unit_job(payload):
    """Scores -> pool -> top-C_max + window -> gather, for one unit (fp64 oracle)."""
    sys.path.insert(0, ROOT)
    import oracle
    qb, kb, vb, n_window, n_lookahead, c_max, pool = payload
    s, p, idx = oracle.speckv_select_unit(qb, kb, n_window, n_lookahead, c_max, pool)
    oracle.gather_rows(kb, idx)
    oracle.gather_rows(vb, idx)
    return int(idx.size)


def tensor_peak(peaks):
    """The scoring kernels run back to back for the whole timed region (tens of
    milliseconds per step, many steps), under the board power cap: the roofline
    denominator is the sustained bf16 GEMM figure, the burst one only when no
    sustained figure exists."""
    if peaks.get("bf16_tflops_sustained"):
        return peaks["bf16_tflops_sustained"], f"{peaks['source']} bf16 sustained (power-capped, back-to-back GEMM)"
    return peaks["bf16_tflops"], f"{peaks['source']} bf16 burst"


def exp2_peak_per_s():
    """Exponentials per second the SMs can produce: the MUFU gives 16 ex2 per
    clock per SM; the FMA pipe (128 lanes) spends 2 lane-ops per logit on the
    scale and the sum and 7 per polynomial exponential, so the best split
    (40 % polynomial) reaches 16 / 0.6 = 26.7 exponentials per clock per SM."""
    return 148 * (16.0 / 0.6) * 1965e6


# The files that define the scoring kernels and how they are launched.
SCORING_SOURCES = ("api.cu", "common.cuh", "exp2_poly.cuh", "score.cu", "score.cuh")


def kernel_source_digest():
    """sha256 over the scoring kernels' sources (SCORING_SOURCES); the DRAM
    traffic captured with ncu is only reported while they are unchanged."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "prompt_compression_b200", "csrc")
    for name in SCORING_SOURCES:
        h.update(name.encode())
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()


def captured_traffic(kernel, workload):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch from
    profiles/traffic.json, or None when absent or captured from other sources."""
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(prof))
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != kernel_source_digest():
        return None
    return rec.get(kernel, {}).get(workload)


def time_oracle(units_payload, cores):
    """Run the oracle on the given units over `cores` spawned processes; returns seconds."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    with ctx.Pool(processes=cores) as pool:
        pool.map(_oracle_unit_job, units_payload[:1])          # warm: import + build
        t0 = time.perf_counter()
        pool.map(_oracle_unit_job, units_payload, chunksize=1)
        return time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_sample_payload(cfg, seed, n_units):
    payload = []
    for u in range(n_units):
        qb, kb, vb = W.speckv_unit_numpy(cfg, seed, u)
        payload.append((qb, kb, vb, cfg.n_window, cfg.n_lookahead, cfg.c_max, cfg.pool))
    return payload


def run_reference(args, cfg):
    """--impl reference: the fp64 oracle on the host cores, same metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = min(host_cores(), 16)
    per_step = cores                     # one sample per process per step
    # Each sample is one unit restricted to the rows of one query head of its
    # GQA group (1/g of the unit's work; the oracle's cost is linear in rows),
    # so that the whole --steps/--warmup run stays within a few minutes.
    payload = [(qb[:1], kb, vb, nw, nl, c, pl)
               for (qb, kb, vb, nw, nl, c, pl) in cpu_sample_payload(cfg, args.seed, min(per_step, 4))]
    payload = (payload * per_step)[:per_step]
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    times = []
    with ctx.Pool(processes=cores) as pool:
        pool.map(_oracle_unit_job, payload[:1])
        for s in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            pool.map(_oracle_unit_job, payload, chunksize=1)
            if s >= args.warmup:
                times.append(time.perf_counter() - t0)
    step = sum(times) / len(times)
    value = per_step * cfg.n_in / cfg.g / step
    sample = (f"{per_step} samples per step, one per process, each = one unit of {cfg.name} with the "
              f"rows of 1 of its {cfg.g} query heads (1/{cfg.g} unit of work); the full step has "
              f"{cfg.units} units")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "KV-head-tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "units_per_step": per_step, "n_in": cfg.n_in,
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


# ----------------------------------------------------------------- GPU arm
def main():
    args = parse()
    cfg = config_of(args)
    if args.impl == "reference":
        if not isinstance(cfg, W.SpecKVConfig):
            print(json.dumps({"impl": "reference", "unavailable":
                              "the CPU reference arm times the SpecKV workloads only"}))
            return
        run_reference(args, cfg)
        return
    if isinstance(cfg, W.DecodeConfig):
        run_decode(args, cfg)
        return
    if not isinstance(cfg, W.SpecKVConfig):
        run_other(args, cfg)
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
    from prompt_compression_b200.pipeline import SpeckvBuffers

    seed = rank_seed(args.seed, rank)
    inp = W.speckv_inputs(cfg, seed=seed, device=dev)
    q, k, v = inp["q"], inp["k"], inp["v"]
    buf = SpeckvBuffers(q, k, v, cfg.n_window, cfg.c_max)
    stream = torch.cuda.current_stream(dev)

    def step():
        P.speckv_compress(q, k, v, cfg.n_window, cfg.c_max, cfg.pool, buffers=buf, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_ranks(x: float) -> float:
        return max_over_ranks(x, world, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, site = P.spk_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at site {site} during warm-up")

    # ---- timed region: K steps, events on the launching stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = max_ranks(e0.elapsed_time(e1))
    ms_step = ms_total / args.steps
    value = whole_job_value(world, cfg.kv_head_tokens, args.steps, ms_total)

    # ---- per-kernel timing: pass 1 alone (row LSE), then the whole score call
    lse2 = torch.empty((cfg.units, cfg.g * cfg.rows), dtype=torch.float32, device=dev)

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    n_k = max(3, min(args.steps, 10))
    ms_lse = timed(lambda: P.speckv_row_lse(q, k, cfg.n_window, lse2, stream=stream), n_k)
    ms_score = timed(lambda: P.speckv_score(q, k, cfg.n_window, buf.scores, None, buf.ws_score,
                                            stream=stream), n_k)
    ms_topk = timed(lambda: P.topk_select(buf.scores, cfg.c_max, cfg.n_window, buf.idx, cfg.pool, None,
                                          buf.ws_topk, stream=stream), n_k)
    ms_compact = timed(lambda: P.kv_compact(k, v, buf.idx, buf.k_out, buf.v_out, 1, stream=stream), n_k)
    ms_colsum = ms_score - ms_lse
    st, site = P.spk_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at site {site}")

    peaks = load_peaks()
    flops_pass = algorithmic_flops(cfg)
    kernels = {
        "score_lse_pass": {"ms": ms_lse, "tflops": flops_pass / (ms_lse * 1e-3) / 1e12},
        "score_colsum_pass": {"ms": ms_colsum, "tflops": flops_pass / (ms_colsum * 1e-3) / 1e12},
        "topk_select": {"ms": ms_topk},
        "kv_compact": {"ms": ms_compact,
                       "gbs": cfg.units * 4 * cfg.keep * cfg.head_dim * 2 / (ms_compact * 1e-3) / 1e9},
    }
    dom = "score_lse_pass" if ms_lse >= ms_colsum else "score_colsum_pass"
    achieved = kernels[dom]["tflops"]
    peak, peak_src = tensor_peak(peaks)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": captured_traffic(dom, cfg.name),
                "peak_source": peak_src,
                "step_roofline_ms": max(2 * flops_pass / (peak * 1e12),
                                        algorithmic_bytes(cfg) / (peaks["hbm_gbs"] * 1e9)) * 1e3}
    roofline["step_frac"] = roofline["step_roofline_ms"] / ms_step

    # ---- e2e through the C ABI with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, cfg, P, q, k, v, dev, stream, world, max_ranks, barrier)

    # ---- CPU baseline (oracle), rank 0 at N = 1 only
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cores = host_cores()
        n_units = max(1, min(cores, 8))
        payload = cpu_sample_payload(cfg, args.seed, n_units)
        secs = time_oracle(payload, n_units)
        cpu = {"value": n_units * cfg.n_in / secs, "unit": "KV-head-tokens/s", "cores": n_units,
               "kind": "oracle",
               "sample": f"{n_units} units of {cfg.name} (one per process, seeded host inputs), "
                         f"{secs:.1f} s wall; the full step has {cfg.units} units"}

    launches = 4 * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "KV-head-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "units": cfg.units, "layers": cfg.layers, "hq": cfg.hq,
                   "hkv": cfg.hkv, "head_dim": cfg.head_dim, "n_in": cfg.n_in, "n_window": cfg.n_window,
                   "n_lookahead": cfg.n_lookahead, "c_max": cfg.c_max, "pool": cfg.pool,
                   "l2": f"inputs larger than L2 (K, V {k.numel() * 2 / 1e9:.1f} GB each); no flush",
                   "parallelism": f"units sharded, {world} rank(s), no collective"},
        "roofline": roofline, "kernels": kernels, "gpu_launches": launches,
        "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_other(args, cfg):
    """SpecPC (scores + pool + top-K prompt tokens over a draft) and the
    SpecKV-PC cascade (SpecPC on the draft, gather of the target cache, SpecKV
    on the gathered cache), one GPU, one JSON line."""
    import torch
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    from prompt_compression_b200.pipeline import SpeckvBuffers
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
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
    flops = 2 * specpc_flops(d)
    launches_per_step = 3
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
        flops += 2 * algorithmic_flops(tcfg)
        launches_per_step += 1 + 4
        tokens = t.batch * t.layers * t.hkv * cfg.n_in_full
        metric = "target KV-head-tokens compressed/s (SpecPC 128K -> 2048 -> SpecKV 256 + 64)"
    else:
        tokens = d.kv_head_tokens
        metric = "KV-head-tokens scored+selected/s (SpecPC draft)"

    def step():
        P.specpc_score(dr["q"], dr["k"], w, pc_scores, d.l_skip, d.n_lookahead, ws_pc, stream=stream)
        P.topk_select(pc_scores, d.keep, 0, pc_idx, d.pool, None, ws_tk, stream=stream)
        if cascade:
            P.kv_compact(tg["k"], tg["v"], pc_idx, kg, vg, t.layers * t.hkv, stream=stream)
            P.speckv_compress(tg["q"], kg, vg, t.n_window, t.c_max, t.pool, buffers=buf, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, site = P.spk_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at site {site} during warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        time.sleep(0.3)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms_step = e0.elapsed_time(e1) / args.steps
    achieved = flops / (ms_step * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "whole step (scoring passes dominate)", "achieved": achieved,
                "peak": tensor_peak(peaks)[0], "unit": "TFLOP/s", "frac": achieved / tensor_peak(peaks)[0],
                "traffic": None, "peak_source": tensor_peak(peaks)[1]}
    if not cascade:
        # head_dim 64 halves the tensor work per logit, so the exponential
        # stream (one exp2 per visible logit per pass) is the binding ceiling
        exps = 2 * specpc_flops(d) / (2 * d.head_dim)
        peak_exp = exp2_peak_per_s() / 1e9
        ach_exp = exps / (ms_step * 1e-3) / 1e9
        roofline = {"bound": "alu", "kernel": "whole step (scoring passes dominate)", "achieved": ach_exp,
                    "peak": peak_exp, "unit": "Gexp2/s", "frac": ach_exp / peak_exp, "traffic": None,
                    "peak_source": "derived: 148 SMs x 26.7 exp2/clk (MUFU 16/clk + FMA-pipe polynomial) x 1965 MHz",
                    "tensor_frac": achieved / tensor_peak(peaks)[0]}
    line = {
        "metric": metric, "value": tokens / (ms_step * 1e-3), "unit": "KV-head-tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "l2": "inputs larger than L2; no flush"},
        "roofline": roofline,
        "gpu_launches": launches_per_step * args.steps, "clocks": clk.summary(), "e2e": None,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def run_decode(args, cfg):
    """One decode step over the compressed cache (C_max + window rows per KV
    head) on every (layer, query head), one JSON line; the same step over the
    full cache is timed for contrast.  Four copies of the compressed cache are
    used in rotation so that consecutive launches read 4 x 84 MB, more than
    the L2; the full cache (17 GB) is far larger than the L2."""
    import torch
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
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

    def timed(fn, n):
        for i in range(max(3, args.warmup)):
            fn(i)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    steps = max(args.steps, 20) * 10
    with ClockSampler(dev.index) as clk:
        time.sleep(0.3)
        ms = timed(lambda i: P.decode_attention(qs[i % copies], kcs[i % copies], vcs[i % copies], out, scale,
                                                stream), steps)
    st, site = P.spk_device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} at site {site}")
    del kcs, vcs
    kf, vf = rnd(B_, L, hkv, cfg.n_kv_full, d), rnd(B_, L, hkv, cfg.n_kv_full, d)
    ms_full = timed(lambda i: P.decode_attention(qs[0], kf, vf, out, scale, stream), max(args.steps, 5))
    del kf, vf
    peaks = load_peaks()
    nbytes = cfg.units * cfg.n_kv * d * 2 * 2 + B_ * L * hq * d * (2 + 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "decode over the compressed cache: query-head tokens/s", "value": B_ * L * hq / (ms * 1e-3),
        "unit": "query-head tokens/s", "n_gpus": 1, "steps": steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name, "n_kv": cfg.n_kv, "units": cfg.units, "hq": hq, "head_dim": d,
                   "l2": "4 cache copies in rotation (4 x 84 MB > L2); no flush"},
        "roofline": {"bound": "hbm", "kernel": "decode_kernel", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peaks['source']} HBM copy"},
        "full_cache": {"n_kv": cfg.n_kv_full, "ms_per_step": ms_full,
                       "gbs": cfg.units * cfg.n_kv_full * d * 4 / (ms_full * 1e-3) / 1e9},
        "gpu_launches": steps, "clocks": clk.summary(), "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def run_e2e(args, cfg, P, q, k, v, dev, stream, world, max_over_ranks, barrier):
    """Same metric end to end from pinned host memory, through the public API.

    Per step, the (batch, layer) pairs are taken in `--e2e-chunks` groups.  Q
    and K of a group are copied to the device on a copy stream; the group is
    scored, selected and compacted on the compute stream as soon as its copy
    has landed (the next group's copy overlaps that work); the compacted K is
    gathered from the device copy of K, the compacted V straight from the
    pinned host V (only the selected rows cross the host link); the indices
    and the compacted K/V go back to pinned host memory on a third stream.
    The timed region runs from before the first copy to the end of the last
    copy back.  If the host V cannot be read in place, it is copied like K."""
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
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b)) / args.e2e_steps
    keep_rows = sum(g[5].idx.numel() for g in groups)
    h2d = (q.numel() + k.numel()) * 2 + (keep_rows * cfg.head_dim * 2 if v_in_place else v.numel() * 2)
    d2h = sum(g[6][0].numel() * 4 + (g[6][1].numel() + g[6][2].numel()) * 2 for g in groups)
    return {"value": world * cfg.kv_head_tokens / (ms * 1e-3), "unit": "KV-head-tokens/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": args.e2e_steps, "groups": n_chunks,
            "v": "selected rows read in place from pinned host memory" if v_in_place else "copied"}


if __name__ == "__main__":
    main()
