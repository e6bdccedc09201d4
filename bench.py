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
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from cross_loop_sparsity_b200 import synth  # noqa: E402
from cross_loop_sparsity_b200.clocks import ClockSampler  # noqa: E402

WORKLOAD = "c2"
METRIC = "looped decode tokens/s at K loops; KV-cache bytes/token; % of HBM/TC roofline"
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "gemm_decode_c2_traffic.json")
GEMM_SOURCE = os.path.join(ROOT, "cross_loop_sparsity_b200", "csrc", "fl_gemm.cu")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["flashloop", "reference"], default="flashloop")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-looped GPU baseline")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--workload", default=None, choices=["c1", "c2", "c3", "c4", "c5", "c5_int2"],
                    help="time this one workload as the line's headline (default: c2, with every other "
                         "workload summarised under per_config)")
    ap.add_argument("--no-per-config", action="store_true", help="time the headline workload only")
    ap.add_argument("--resid-layout", choices=["sparse", "dense"], default="sparse",
                    help="lazy-path KV residual storage: rows for recomputed tokens only (sparse) or every position")
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


def gemm_traffic_ratio():
    """DRAM bytes per algorithmic byte of the decode GEMM, from the committed
    ncu capture (profiles/gemm_decode_c2_traffic.json), or None when the file
    is missing or the GEMM source changed since it was taken."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    d = json.load(open(TRAFFIC_JSON))
    cur = hashlib.sha256(open(GEMM_SOURCE, "rb").read()).hexdigest()
    return float(d["dram_bytes_per_algorithmic_byte"]) if d.get("gemm_source_sha256") == cur else None


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


# ------------------------------------------------------------------ replicas (one per GPU)
from cross_loop_sparsity_b200 import replicas  # noqa: E402

barrier = replicas.barrier
max_over_ranks = replicas.max_over_ranks


# ------------------------------------------------------------------ the library arm
def lazy_cfg(cfg, layout):
    """The lazy arm's config: sparse residual storage sized to the synthetic
    context's recompute rate plus the batch's new tokens, or every position."""
    return cfg.with_(resid_rows=synth.sparse_rows(cfg, cfg.batch)) if layout == "sparse" else cfg


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
    stream = torch.cuda.Stream()
    if args.workload and args.workload != WORKLOAD:
        return run_single(args.workload, args, world, rank, local, stream)
    cfg = lazy_cfg(synth.config(WORKLOAD), args.resid_layout)
    B = cfg.batch
    eng, lens, h0, w = setup_engine(cfg, False, stream)
    h0_dev = torch.from_numpy(h0).cuda()
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    sampler = ClockSampler(local)
    ms, clocks = time_steps(eng, lens, h0_dev, logits, stream, args.steps, args.warmup, world, sampler)
    ms_step = ms / args.steps
    assert eng.sync_status(stream) == 0, "a kernel reported an error"
    launches_per_step = eng.kernels_per_call() + (2 if cfg.resid_rows else 1)   # + the reset (lengths, pool counts)
    # then, in replays of the same step after the timed region, the GEMMs stamp
    # their own start (dependency released) and end on the GPU's global timer:
    # two atomics per CTA, kept out of the timed steps
    eng.set_option(fl.FL_OPT_GEMM_TIMES, 1)
    gemm_ms, gemm_n = gemm_time_per_step(eng, lens, h0_dev, logits, stream, args.steps)
    assert gemm_ms <= ms_step * 1.001, (gemm_ms, ms_step)   # launches never overlap in the sum
    eng.set_option(fl.FL_OPT_GEMM_TIMES, 0)

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
        deng, dlens, dh0, _ = setup_engine(cfg.with_(resid_rows=0), True, stream)
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
    gbytes = gemm_algorithmic_bytes(cfg, B, n_sel)
    achieved = gbytes / (gemm_ms / 1e3) / 1e9
    n_launch = max(1, gemm_n)
    ratio = gemm_traffic_ratio()
    roofline = {"kernel": "k_gemm_tc (all tcgen05 GEMMs of the step: QKV, O, gate/up, down, LM head)",
                "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_source": f"{peak_kind} hbm_gbs",
                "traffic": None if ratio is None else ratio * gbytes / n_launch,
                "algorithmic_bytes_per_launch": gbytes / n_launch, "launches_per_step": n_launch,
                "avg_launch_us": gemm_ms * 1e3 / n_launch, "gemm_ms_per_step": gemm_ms,
                "gemm_share_of_step": gemm_ms / ms_step,
                "timing": "per launch: last CTA's end - first CTA's return from the dependency wait, stamped by "
                          "the kernel on the global timer in graph replays of the timed step run right after the "
                          "timed region; summed per step"}
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
        "roofline": roofline, "whole_step": whole,
        "e2e": {"value": e2e_tps, "unit": "tokens/s", "h2d_bytes_per_step": B * cfg.d_model * 4,
                "d2h_bytes_per_step": B * cfg.vocab * 4},
        "gpu_launches": launches_per_step * args.steps, "gpu_launches_per_step": launches_per_step,
        "dense_baseline": dense,
        "speedup_vs_dense": None if dense is None else (world * B / (ms_step / 1e3)) / dense["tokens_per_s"],
        "cpu_baseline": cpu, "clocks": clocks,
    }
    # every other workload: lazy and dense-looped throughput, speedup, KV bytes, roofline, clocks
    per = {WORKLOAD: {"workload": workload_desc(cfg), "unit": "tokens/s",
                      "lazy": {"tokens_per_s": out["value"], "ms_per_step": ms_step,
                               "kv_bytes_per_token_per_layer": out["kv_bytes"]["per_token_per_layer"],
                               "roofline": decode_roofline(cfg, ms_step, n_sel), "clocks": clocks},
                      "dense_looped": None if dense is None else {
                          "tokens_per_s": dense["tokens_per_s"], "ms_per_step": dense["ms_per_step"],
                          "kv_bytes_per_token_per_layer": dense_per,
                          "roofline": decode_roofline(cfg, dense["ms_per_step"], B, True)},
                      "speedup_vs_dense": out["speedup_vs_dense"],
                      "kv_bytes_reduction": out["kv_bytes"]["reduction"]}}
    if not args.no_per_config and args.workload is None:
        for nm in PER_CONFIG:
            try:
                per[nm] = measure_workload(nm, args, world, local, stream)
            except Exception as e:     # one workload failing must not hide the others
                per[nm] = {"error": f"{type(e).__name__}: {e}"}
                torch.cuda.synchronize()
                torch.cuda.empty_cache()
    out["per_config"] = per
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_single(name, args, world, rank, local, stream):
    """One workload as the line's headline (its lazy throughput), with its dense-looped baseline."""
    r = measure_workload(name, args, world, local, stream)
    lazy = r["lazy"]
    ms = lazy.get("ms_per_step", lazy.get("ms_per_call"))
    cfg = synth.config(name)
    units = cfg.batch if cfg.mode == "decode" else cfg.batch * cfg.seq_len
    rl = lazy["roofline"]
    out = {"metric": METRIC, "value": lazy["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
           "steps": r.get("timed_steps", r.get("timed_calls")), "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (device-drawn weights and context)",
           "config": {"workload": r["workload"], "global_batch": world * cfg.batch, "units_per_step": units,
                      "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
           "roofline": {"kernel": "whole step", "bound": rl["bound"], "frac": rl["frac"], "peak": rl["peak"],
                        "peak_source": rl["peak_source"]},
           "gpu_launches": None, "speedup_vs_dense": r["speedup_vs_dense"], "dense_baseline": r["dense_looped"],
           "kv_bytes_reduction": r["kv_bytes_reduction"], "clocks": lazy["clocks"], "detail": r}
    if rank == 0:
        print(json.dumps(out), flush=True)


def gemm_time_per_step(eng, lens, h0_dev, logits, stream, steps):
    """Mean over `steps` replays of the step's summed GEMM device time (the
    kernels' own global-timer stamps), and the GEMM launches per step."""
    tot, n = 0.0, 0
    reps = max(3, min(steps, 20))
    for _ in range(reps):
        eng.reset(lens, stream=stream)
        eng.decode_step(h0_dev, len(lens), None, logits, stream=stream)
        ms, n = eng.gemm_times(stream)
        tot += ms
    return tot / reps, n


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


# ------------------------------------------------------------------ every workload (per_config)
PER_CONFIG = ["c1", "c3", "c4", "c5", "c5_int2"]


def dense_kv_bytes_read(cfg):
    """KV bytes a dense-looped decode step reads: every loop's own K/V of every column."""
    return cfg.n_layers * cfg.n_loops * cfg.batch * cfg.n_kv_heads * (cfg.ctx_len + 1) * cfg.head_dim * 2 * 2


def decode_roofline(cfg, ms, n_sel, dense=False):
    """Whole-step algorithmic bytes against the HBM peak (decode is bandwidth-bound)."""
    hbm, _, kind = measured_peaks()
    B = cfg.batch
    if dense:
        nbytes = gemm_algorithmic_bytes(cfg, B, B) + dense_kv_bytes_read(cfg)
    else:
        nbytes = gemm_algorithmic_bytes(cfg, B, n_sel) + kv_bytes_read(cfg, n_sel)
    t_roof = nbytes / hbm / 1e6
    return {"bound": "hbm", "bytes_per_step": nbytes, "roofline_ms": t_roof, "frac": t_roof / ms,
            "peak": hbm, "peak_source": f"{kind} hbm_gbs"}


def prefill_flops(cfg, sel=None):
    """Algorithmic FLOPs of one prefill call.  Dense (sel None): K loops of every
    token's GEMMs and causal attention.  Lazy: loop 1 dense; each later loop the
    recomputed tokens' GEMMs, the delta-score products of tiles choosing their
    column set (q_l.K_l and q_last.K_last over the query's causal columns) and
    the correction over c columns; every call ends with the last rows' LM head."""
    d, f, hq, qkv, H, hd = cfg.d_model, cfg.ffn_dim, cfg.n_heads * cfg.head_dim, cfg.qkv_rows, cfg.n_heads, cfg.head_dim
    B, T, M, K = cfg.batch, cfg.seq_len, cfg.n_layers, cfg.n_loops
    gemm_tok = 2 * (d * qkv + hq * d + 2 * d * f + f * d)
    attn = 4 * H * hd * B * T * (T + 1) / 2
    head = 2 * d * cfg.vocab * B
    if sel is None:
        return K * M * (B * T * gemm_tok + attn) + head
    total = M * (B * T * gemm_tok + attn) + head
    tps = (T + cfg.q_tile - 1) // cfg.q_tile
    chosen = set()
    for l in range(2, K + 1):
        S = np.asarray(sel[l - 2])
        tiles = (S // T) * tps + (S % T) // cfg.q_tile
        new = [t for t in np.unique(tiles) if t not in chosen]
        pos = S % T
        for t in new:
            total += M * 4 * hd * H * float(np.sum(pos[tiles == t] + 1))
        chosen.update(new)
        total += M * len(S) * (gemm_tok + 8 * H * hd * cfg.c_cols)
    return total


def measure_decode(name, args, world, local, stream):
    """Lazy and dense-looped decode steps of one workload on device-drawn inputs."""
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    cfg = lazy_cfg(synth.config(name), args.resid_layout)
    B, d = cfg.batch, cfg.d_model
    lens = [cfg.ctx_len] * B
    steps, warm = (10, 3) if cfg.n_layers * cfg.d_model > 65536 else (20, 5)
    w = synth.make_weights_device(cfg)
    g = torch.Generator(device="cuda")
    g.manual_seed(cfg.seed + 11)
    h0 = torch.randn((B, d), generator=g, device="cuda", dtype=torch.float32)
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    res = {"workload": workload_desc(cfg), "unit": "tokens/s", "timed_steps": steps}
    for dense in (False, True):
        ecfg = cfg.with_(resid_rows=0) if dense else cfg
        eng = fl.FlashLoop(ecfg, w, max_batch=B, max_ctx=cfg.ctx_len + 1, resid_bits=16 if dense else None,
                           stream=stream)
        eng.load_context_device(lens, dense=dense)
        ms, clocks = time_steps(eng, lens, h0, logits, stream, steps, warm, world, ClockSampler(local))
        assert eng.sync_status(stream) == 0, f"{name}: a kernel reported an error"
        ms_step = ms / steps
        tot, per, dense_per = eng.kv_bytes()
        n_sel = B if dense else max(1, min(B, math.ceil(cfg.rho * B - 1e-9)))
        part = {"tokens_per_s": replicas.job_throughput(world, B, ms_step), "ms_per_step": ms_step,
                "kv_bytes_per_token_per_layer": per, "roofline": decode_roofline(cfg, ms_step, n_sel, dense),
                "gpu_launches_per_step": eng.kernels_per_call() + (2 if ecfg.resid_rows else 1), "clocks": clocks}
        eng.close()
        del eng
        torch.cuda.empty_cache()
        res["dense_looped" if dense else "lazy"] = part
    res["speedup_vs_dense"] = res["lazy"]["tokens_per_s"] / res["dense_looped"]["tokens_per_s"]
    res["kv_bytes_reduction"] = (res["dense_looped"]["kv_bytes_per_token_per_layer"] /
                                 res["lazy"]["kv_bytes_per_token_per_layer"])
    del w
    torch.cuda.empty_cache()
    return res


def measure_prefill(name, args, world, local, stream):
    """Lazy and dense-looped prefill calls of one workload (B sequences of T tokens)."""
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    cfg = synth.config(name)
    if args.resid_layout == "sparse":   # room for every recomputed token of the call in one sequence's pool
        cfg = cfg.with_(resid_rows=min(cfg.seq_len, int(math.ceil(cfg.rho * cfg.batch * cfg.seq_len - 1e-9))))
    B, T, d = cfg.batch, cfg.seq_len, cfg.d_model
    big = B * T * cfg.n_layers > 100000
    steps, warm = (3, 1) if big else (20, 5)
    w = synth.make_weights_device(cfg)
    g = torch.Generator(device="cuda")
    g.manual_seed(cfg.seed + 13)
    h0 = torch.randn((B * T, d), generator=g, device="cuda", dtype=torch.float32)
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    _, tc, kind = measured_peaks()
    res = {"workload": (f"prefill, B={B} x {T} tokens, d_model={d}, {cfg.n_heads}q/{cfg.n_kv_heads}kv heads x "
                        f"{cfg.head_dim}, ffn={cfg.ffn_dim}, {cfg.n_layers} shared layers x K={cfg.n_loops} loops, "
                        f"rho={cfg.rho}, c={cfg.c_cols} per {cfg.q_tile}-query tile, int{cfg.resid_bits} g"
                        f"{cfg.group_size}"), "unit": "tokens/s", "timed_calls": steps}
    for dense in (False, True):
        eng = fl.FlashLoop(cfg.with_(resid_rows=0) if dense else cfg, w, max_batch=B, max_ctx=T, max_tokens=B * T,
                           resid_bits=16 if dense else None, stream=stream)
        for _ in range(warm):
            eng.reset(None, stream=stream)
            eng.prefill(h0, B, T, None, logits, stream=stream)
        torch.cuda.synchronize()
        barrier(world)
        sampler = ClockSampler(local)
        sampler.start()
        time.sleep(0.3)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            eng.reset(None, stream=stream)
            eng.prefill(h0, B, T, None, logits, stream=stream)
        e1.record(stream)
        e1.synchronize()
        clocks = sampler.stop()
        ms = max_over_ranks(world, e0.elapsed_time(e1)) / steps
        assert eng.sync_status(stream) == 0, f"{name}: a kernel reported an error"
        sel = None
        if not dense and cfg.n_loops > 1:
            n_sel = max(1, min(B * T, math.ceil(cfg.rho * B * T - 1e-9)))
            sel, _, _, _ = eng.read_trace(B * T, n_sel, B * ((T + cfg.q_tile - 1) // cfg.q_tile), stream=stream)
        flops = prefill_flops(cfg, None if dense else sel)
        _, per, _ = eng.kv_bytes()
        t_roof = flops / (tc * 1e12) * 1e3
        res["dense_looped" if dense else "lazy"] = {
            "tokens_per_s": replicas.job_throughput(world, B * T, ms), "ms_per_call": ms,
            "kv_bytes_per_token_per_layer": per, "gpu_launches_per_call": eng.kernels_per_call() + 1,
            "roofline": {"bound": "tensor", "flops_per_call": flops, "roofline_ms": t_roof, "frac": t_roof / ms,
                         "peak": tc, "peak_source": f"{kind} bf16_tflops"},
            "clocks": clocks}
        eng.close()
        del eng
        torch.cuda.empty_cache()
    res["speedup_vs_dense"] = res["lazy"]["tokens_per_s"] / res["dense_looped"]["tokens_per_s"]
    res["kv_bytes_reduction"] = (res["dense_looped"]["kv_bytes_per_token_per_layer"] /
                                 res["lazy"]["kv_bytes_per_token_per_layer"])
    del w
    torch.cuda.empty_cache()
    return res


def measure_workload(name, args, world, local, stream):
    return (measure_prefill if synth.config(name).mode == "prefill" else measure_decode)(name, args, world, local,
                                                                                       stream)


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
    # each step is one full decode step of the workload: all B tokens through all K loops
    # (about a second on the host cores, so the driver's warm-up + timed steps stay within a minute)
    sample_b = cfg.batch
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
    sample = (f"each step: the full decode step of the workload ({sample_b} tokens through all {cfg.n_loops} "
              f"loops over the {cfg.ctx_len}-token context), fp64 numpy oracle")
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
