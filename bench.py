"""Benchmark of the lazy-update looped decode step (one JSON line on rank 0).

Workload: the decode step of an 8-sequence batch over a 4096-token context
with a shared block of 4 layers (d_model 2048, 16 query / 4 KV heads,
head_dim 128, SwiGLU 5632) applied K = 4 times; rho = 0.10, c = 256 key
columns, int4 KV residuals (group 64); random-init weights ~N(0, 0.02) and a
synthetic base + residual context (seeded, see cross_loop_sparsity_b200.synth).
A step is one decode step: 8 new tokens through all K loops and the LM head.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl flashloop|reference]

N > 1 (launched with torchrun) runs one independent replica per GPU (the
decode step has no cross-GPU exchange): weak scaling, max-over-ranks time.
The `reference` arm times the CPU oracle on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from cross_loop_sparsity_b200 import synth  # noqa: E402

WORKLOAD = "c2"
METRIC = "looped decode tokens/s at K loops; KV-cache bytes/token; % of HBM/TC roofline"
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "gemm_decode_c2.md")
GEMM_SOURCE = os.path.join(ROOT, "cross_loop_sparsity_b200", "csrc", "fl_gemm.cu")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["flashloop", "reference"], default="flashloop")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-looped GPU baseline")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    return ap.parse_args()


def workload_desc(cfg):
    return (f"decode step, B={cfg.batch} sequences x {cfg.ctx_len}-token context, d_model={cfg.d_model}, "
            f"{cfg.n_heads}q/{cfg.n_kv_heads}kv heads x {cfg.head_dim}, ffn={cfg.ffn_dim}, "
            f"{cfg.n_layers} shared layers x K={cfg.n_loops} loops, rho={cfg.rho}, c={cfg.c_cols}, "
            f"int{cfg.resid_bits} residual g{cfg.group_size}, vocab={cfg.vocab}")


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def gemm_traffic():
    """Per-launch DRAM bytes of the decode GEMM from the committed ncu summary,
    or None when the summary is missing or the GEMM source changed since."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    txt = open(PROFILE_SUMMARY).read()
    m = re.search(r"gemm_source_sha256:\s*([0-9a-f]{64})", txt)
    t = re.search(r"traffic_bytes_per_step:\s*([0-9.eE+]+)", txt)
    if not m or not t:
        return None
    cur = hashlib.sha256(open(GEMM_SOURCE, "rb").read()).hexdigest()
    return float(t.group(1)) if m.group(1) == cur else None


def gemm_algorithmic_bytes(cfg, n_first, n_sel):
    """Bytes a decode step's GEMMs must move: every weight once per loop, plus
    the bf16 inputs and fp32 / bf16 outputs of the token rows."""
    d, f, hq, qkv = cfg.d_model, cfg.ffn_dim, cfg.n_heads * cfg.head_dim, cfg.qkv_rows
    w_layer = 2 * (qkv * d + d * hq + 2 * f * d + d * f)

    def acts(n):
        return n * (2 * d + 4 * qkv + 2 * hq + 8 * d + 2 * d + 2 * f + 2 * f + 8 * d)

    total = 0
    for l in range(1, cfg.n_loops + 1):
        n = n_first if l == 1 else n_sel
        total += cfg.n_layers * (w_layer + acts(n))
    total += 2 * cfg.vocab * d + n_first * (2 * d + 4 * cfg.vocab)
    return total


class ClockSampler:
    """nvidia-smi clocks / throttle reasons every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ replicas (one per GPU)
from cross_loop_sparsity_b200 import replicas  # noqa: E402

barrier = replicas.barrier
max_over_ranks = replicas.max_over_ranks


# ------------------------------------------------------------------ the library arm
def setup_engine(cfg, dense, stream):
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    w = synth.make_weights(cfg)
    rng = w["rng"]
    lens = [cfg.ctx_len] * cfg.batch
    ccfg = cfg.with_(resid_bits=16) if dense else cfg
    ctx = synth.make_dense_context(ccfg, rng, lens) if dense else synth.make_context(cfg, rng, lens)
    h0 = synth.make_h0(cfg, rng, cfg.batch)
    eng = fl.FlashLoop(ccfg, fl.upload_weights(w), max_batch=cfg.batch, max_ctx=cfg.ctx_len + 1, stream=stream)
    eng.load_context(ctx, dense)
    del ctx
    return eng, lens, h0, w


def time_steps(eng, lens, h0_dev, logits, stream, steps, warmup, world, sampler=None):
    import torch
    B = len(lens)
    for _ in range(warmup):
        eng.reset(lens, stream=stream)
        eng.decode_step(h0_dev, B, None, logits, stream=stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        eng.reset(lens, stream=stream)
        eng.decode_step(h0_dev, B, None, logits, stream=stream)
    end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    clocks = sampler.stop() if sampler else None
    return max_over_ranks(world, ms), clocks


def run_library(args, world, rank, local):
    import torch
    from cross_loop_sparsity_b200 import build
    from cross_loop_sparsity_b200 import flashloop as fl
    build.build()
    cfg = synth.config(WORKLOAD)
    B = cfg.batch
    stream = torch.cuda.Stream()
    eng, lens, h0, w = setup_engine(cfg, False, stream)
    h0_dev = torch.from_numpy(h0).cuda()
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    sampler = ClockSampler(local)
    ms, clocks = time_steps(eng, lens, h0_dev, logits, stream, args.steps, args.warmup, world, sampler)
    ms_step = ms / args.steps
    assert eng.sync_status(stream) == 0, "a kernel reported an error"
    launches_per_step = eng.kernels_per_call() + 1          # + the length-reset kernel

    # profiled pass: per-kind device time from CUDA events around each kernel
    prof, prof_mode = None, None
    for use_graph in (1, 0):
        try:
            prof = profile_pass(eng, fl, lens, h0_dev, logits, stream, max(3, min(10, args.steps)), use_graph)
            prof_mode = "graph replay with event-record nodes" if use_graph else "direct launches"
            break
        except Exception as e:  # graph event nodes refused: profile direct launches instead
            print(f"profile pass ({'graph' if use_graph else 'direct'}) failed: {e}", file=sys.stderr)
            torch.cuda.synchronize()
    eng.set_option(fl.FL_OPT_PROFILE, 0)
    eng.set_option(fl.FL_OPT_USE_GRAPH, 1)
    prof = prof or {}

    # end to end through the C ABI with pinned host buffers (copies inside the timed region)
    h0_host = torch.from_numpy(h0).pin_memory()
    logits_host = torch.empty((B, cfg.vocab), dtype=torch.float32).pin_memory()
    e2e_ms, _ = time_steps(eng, lens, h0_host, logits_host, stream, args.steps, 2, world)
    e2e_tps = world * B / (e2e_ms / args.steps / 1e3)

    tot, per, dense_per = eng.kv_bytes()
    n_sel = max(1, min(B, math.ceil(cfg.rho * B - 1e-9)))
    eng.close()
    del eng
    torch.cuda.empty_cache()

    dense = None
    if not args.no_dense:
        deng, dlens, dh0, _ = setup_engine(cfg, True, stream)
        dms, _ = time_steps(deng, dlens, torch.from_numpy(dh0).cuda(), logits, stream, max(5, args.steps // 2),
                            max(3, args.warmup // 2), world)
        dsteps = max(5, args.steps // 2)
        dense = {"tokens_per_s": world * B / (dms / dsteps / 1e3), "ms_per_step": dms / dsteps,
                 "kv_bytes_per_token_per_layer": dense_per, "what": "rho=1, per-loop bf16 KV, full attention "
                 "every loop, same kernels"}
        deng.close()
        del deng
        torch.cuda.empty_cache()

    hbm, tc, peak_kind = measured_peaks()
    gemm = prof.get("gemm", {"ms_per_step": float("nan"), "launches_per_step": 0})
    gbytes = gemm_algorithmic_bytes(cfg, B, n_sel)
    achieved = gbytes / (gemm["ms_per_step"] / 1e3) / 1e9
    n_launch = max(1, gemm["launches_per_step"])
    traffic = gemm_traffic()
    roofline = {"kernel": "k_gemm_tc (all tcgen05 GEMMs of the step: QKV, O, gate/up, down, LM head)",
                "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_source": f"{peak_kind} hbm_gbs", "traffic": None if traffic is None else traffic / n_launch,
                "algorithmic_bytes_per_launch": gbytes / n_launch, "launches_per_step": n_launch,
                "avg_launch_us": gemm["ms_per_step"] * 1e3 / n_launch}
    step_bytes = gbytes + kv_bytes_read(cfg, n_sel)
    whole = {"bytes_per_step": step_bytes, "roofline_ms": step_bytes / hbm / 1e6,
             "frac_of_hbm_roofline": (step_bytes / hbm / 1e6) / ms_step}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(cfg, w, 1)
    out = {
        "metric": METRIC, "value": replicas.job_throughput(world, B, ms_step), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "global_batch": world * B, "ctx": cfg.ctx_len,
                   "loops": cfg.n_loops, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: each step streams 1.57 GB of weights and 0.27 GB of KV",
                   "graph": "decode step captured as one CUDA graph, replayed"},
        "kv_bytes": {"per_token_per_layer": per, "dense_per_token_per_layer": dense_per,
                     "reduction": dense_per / per, "cache_total": tot},
        "roofline": roofline, "whole_step": whole, "profile": prof, "profile_mode": prof_mode,
        "e2e": {"value": e2e_tps, "unit": "tokens/s", "h2d_bytes_per_step": B * cfg.d_model * 4,
                "d2h_bytes_per_step": B * cfg.vocab * 4},
        "gpu_launches": launches_per_step * args.steps, "gpu_launches_per_step": launches_per_step,
        "dense_baseline": dense,
        "speedup_vs_dense": None if dense is None else (world * B / (ms_step / 1e3)) / dense["tokens_per_s"],
        "cpu_baseline": cpu, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)


def profile_pass(eng, fl, lens, h0_dev, logits, stream, steps, use_graph):
    eng.set_option(fl.FL_OPT_USE_GRAPH, use_graph)
    eng.set_option(fl.FL_OPT_PROFILE, 1)
    acc = {}
    for i in range(steps + 2):
        eng.reset(lens, stream=stream)
        eng.decode_step(h0_dev, len(lens), None, logits, stream=stream)
        p = eng.profile(stream)
        if i >= 2:
            for k, (t, n) in p.items():
                a = acc.setdefault(k, [0.0, 0])
                a[0] += t
                a[1] = n
    return {k: {"ms_per_step": v[0] / steps, "launches_per_step": v[1]} for k, v in acc.items()}


def kv_bytes_read(cfg, n_sel):
    """KV bytes a lazy decode step reads: loop-1 base K/V for every sequence,
    the delta-score pass over the K chain and the correction's column rows."""
    M, Hkv, hd, T, B = cfg.n_layers, cfg.n_kv_heads, cfg.head_dim, cfg.ctx_len + 1, cfg.batch
    res = hd * cfg.resid_bits // 8 + 2 * hd // cfg.group_size
    base = M * B * Hkv * T * hd * 2 * 2
    # first recompute at loop 2: K chain (base + 1 residual) for the selected tokens' sequences
    dscore = M * n_sel * Hkv * T * (hd * 2 + res)
    corr = 0
    for l in range(2, cfg.n_loops + 1):
        corr += M * n_sel * Hkv * cfg.c_cols * 2 * (hd * 2 + (l - 1) * res) * 2
    return base + dscore + corr


# ------------------------------------------------------------------ the oracle on the host
def cpu_baseline(cfg, w, n_steps):
    """The CPU oracle, as it stands, on the host cores: one decode step of the
    same workload (all 8 tokens), after its one-off weight and cache set-up."""
    from oracle import flashloop_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    rng = np.random.default_rng(cfg.seed + 1000)
    W = orc.prepare_weights(w)
    lens = [cfg.ctx_len] * cfg.batch
    ctx = synth.make_context(cfg, rng, lens)
    cache = orc.KVCache.from_context(cfg, ctx, cfg.ctx_len + 1)
    del ctx
    h0 = synth.make_h0(cfg, rng, cfg.batch)
    times = []
    for _ in range(n_steps):
        cache.lens[:] = cfg.ctx_len
        t0 = time.perf_counter()
        orc.decode_step(cfg, W, cache, h0)
        times.append(time.perf_counter() - t0)
    t = float(np.mean(times))
    return {"value": cfg.batch / t, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n_steps} full decode step(s) of the workload ({cfg.batch} tokens, fp64 numpy oracle); "
                      f"{t:.2f} s per step"}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    from oracle import flashloop_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    cfg = synth.config(WORKLOAD)
    w = synth.make_weights(cfg)
    rng = w["rng"]
    W = orc.prepare_weights(w)
    # each step is a bounded sample: one sequence of the batch (its token through all K loops)
    sample_b = 1
    lens = [cfg.ctx_len] * sample_b
    ctx = synth.make_context(cfg, rng, lens)
    cache = orc.KVCache.from_context(cfg, ctx, cfg.ctx_len + 1)
    del ctx
    h0 = synth.make_h0(cfg, rng, sample_b)
    for _ in range(args.warmup):
        cache.lens[:] = cfg.ctx_len
        orc.decode_step(cfg, W, cache, h0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cache.lens[:] = cfg.ctx_len
        orc.decode_step(cfg, W, cache, h0)
    dt = time.perf_counter() - t0
    tps = sample_b * args.steps / dt
    sample = (f"each step: one sequence of the {cfg.batch}-sequence batch ({sample_b} token through all "
              f"{cfg.n_loops} loops over the {cfg.ctx_len}-token context), fp64 numpy oracle")
    out = {"impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": workload_desc(cfg), "global_batch": cfg.batch, "ctx": cfg.ctx_len,
                      "loops": cfg.n_loops},
           "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    world, rank, local = replicas.init()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_library(args, world, rank, local)
    finally:
        replicas.finish(world)


if __name__ == "__main__":
    main()
