"""Kernel-level measurements against the B200 roofline (one JSON line per kernel).

  python -m cross_loop_sparsity_b200.kernel_bench [--reps N]

* ``gemm_wide``: the persistent tcgen05 GEMM (128 x 256 output tiles, two TMEM
  accumulators) at the long-prefill shapes (16384 tokens x d_model 2048: QKV
  3072, O 2048, gate or up 5632, down from 5632), TFLOP/s against the measured
  dense bf16 peak.
* ``gemm_skinny``: the split-K swap-AB GEMM at the decode shapes (8 tokens),
  weight GB/s against the measured HBM bandwidth.
* ``topk``: the top-c column selection (bit pattern descending, index
  ascending) of one decode layer's column keys (4 KV heads x 4097 keys,
  c = 256) and of a 65537-key row (c = 1024); microseconds per launch.
* ``attn_decode``: the loop-1 decode attention measured in situ inside the
  decode step (CUDA events around each kernel of the replayed graph) at the
  long-context decode shape (1 token, 65536-token context, 4 KV heads x 128,
  134 MB of K and V per launch) and at the 8 x 4096 shape (67 MB per launch);
  the cache is the zero-initialised workspace at full length (the values do
  not change the work).
* ``quantize_residual``: the residual quantiser on a c5-shaped KV update
  (65536 tokens x 4 layers x 4 KV heads x (K, V) rows of 128): reads the new
  fp32 rows and the previous bf16 rows (1.61 GB), writes packed int4 codes and
  fp16 scales (0.14 GB); bytes moved against HBM.
* ``quantize``: the KV-residual quantiser over a residual shaped like the
  65536-token context (65536 tokens x 4 layers x 2 (K, V) x 4 KV heads rows of
  128 fp32, int4 / int2, group 64), bytes moved against HBM.
* ``decode_step_capture`` and ``lazy_call_capture`` (only on request, for ncu;
  no measurement): one decode step at the decode GEMM shapes with one shared
  layer and a 512-token context, and one lazy call of ``--workload`` with
  ``--layers`` shared layers; kernels launched directly, a few GB on the device.

Every operand set is rotated over copies whose total exceeds L2 (126 MB), so
each timed launch reads from HBM; times are CUDA events around ``reps``
launches after warm-up, on one stream.  Every line carries the SM clocks and
throttle reasons sampled while its kernel group ran (``clocks``).
"""
from __future__ import annotations

import argparse
import json
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def _time(fn, reps, warmup=3):
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(reps):
        fn(i)
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / reps


def gemm_wide(reps):
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    hbm, tc, src = _peaks()
    out = []
    M = 16384
    for name, n, k in (("qkv", 3072, 2048), ("o", 2048, 2048), ("gate_or_up", 5632, 2048), ("down", 2048, 5632)):
        A = torch.randn((M, k), device="cuda").to(torch.bfloat16)
        Bs = [torch.randn((n, k), device="cuda").mul_(0.02).to(torch.bfloat16) for _ in range(2)]
        D = torch.empty((M, n), dtype=torch.float32, device="cuda")
        import ctypes
        L = fl.lib()

        def run(i, B=Bs):
            st = L.fl_test_gemm(ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(B[i % 2].data_ptr()),
                                ctypes.c_void_p(D.data_ptr()), M, n, k, 0, None, 0, None)
            assert st == 0
        ms = _time(run, reps)
        tflops = 2.0 * M * n * k / (ms * 1e-3) / 1e12
        out.append({"kernel": "gemm_wide", "shape": f"{name}: {M}x{n}x{k}", "ms": ms, "achieved": tflops,
                    "unit": "TFLOP/s", "peak": tc, "frac": tflops / tc, "peak_source": f"{src} bf16_tflops"})
    return out


def gemm_skinny(reps):
    import ctypes
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    hbm, tc, src = _peaks()
    L = fl.lib()
    out = []
    m = 8
    for name, n, k in (("qkv", 3072, 2048), ("o", 2048, 2048), ("gate_or_up", 5632, 2048), ("down", 2048, 5632),
                       ("lm_head", 32000, 2048)):
        copies = max(2, int(np.ceil(300e6 / (n * k * 2))))
        Bs = [torch.randn((n, k), device="cuda").mul_(0.02).to(torch.bfloat16) for _ in range(copies)]
        A = torch.randn((m, k), device="cuda").to(torch.bfloat16)
        D = torch.empty((m, n), dtype=torch.float32, device="cuda")
        nb = int(L.fl_test_gemm_scratch_bytes(m, n, k, 1))
        scratch = torch.empty(max(nb, 256) + 256, dtype=torch.uint8, device="cuda")
        sp = scratch.data_ptr() + ((-scratch.data_ptr()) % 256)

        def run(i):
            st = L.fl_test_gemm(ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(Bs[i % copies].data_ptr()),
                                ctypes.c_void_p(D.data_ptr()), m, n, k, 1, ctypes.c_void_p(sp), nb, None)
            assert st == 0
        ms = _time(run, reps)
        gbs = (n * k * 2 + m * k * 2 + m * n * 4) / (ms * 1e-3) / 1e9
        out.append({"kernel": "gemm_skinny", "shape": f"{name}: {m}x{n}x{k}", "ms": ms, "achieved": gbs,
                    "unit": "GB/s", "peak": hbm, "frac": gbs / hbm, "peak_source": f"{src} hbm_gbs",
                    "note": "standalone launch (ticket split-K path, no programmatic overlap)"})
        del Bs
        torch.cuda.empty_cache()
    return out


def topk(reps):
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl, synth
    out = []
    for n_seg, n, k in ((4, 4097, 256), (4, 65537, 1024)):
        keys = torch.from_numpy(np.stack([synth.make_keys(3 + s, n, "distinct") for s in range(n_seg)])).cuda()

        def run(i):
            fl.topk(keys, k)
        ms = _time(run, reps)
        out.append({"kernel": "topk", "shape": f"{n_seg} rows x {n} keys, k={k}", "ms": ms, "us": ms * 1e3,
                    "note": "includes the output allocation of the binding"})
    return out


def quantize(reps):
    import ctypes
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    hbm, tc, src = _peaks()
    L = fl.lib()
    out = []
    rows, width, g = 65536 * 4 * 2 * 4, 128, 64
    r = torch.randn((rows, width), device="cuda")
    for bits in (4, 2):
        codes = torch.empty((rows, width * bits // 8), dtype=torch.uint8, device="cuda")
        scales = torch.empty((rows, width // g), dtype=torch.int16, device="cuda")

        def run(i):
            st = L.fl_test_quantize(ctypes.c_void_p(r.data_ptr()), rows, width, g, bits,
                                    ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()), None)
            assert st == 0
        ms = _time(run, reps)
        moved = rows * width * 4 + rows * width * bits // 8 + rows * (width // g) * 2
        gbs = moved / (ms * 1e-3) / 1e9
        out.append({"kernel": "quantize", "shape": f"int{bits}: {rows} rows x {width}, g{g}", "ms": ms,
                    "achieved": gbs, "unit": "GB/s", "peak": hbm, "frac": gbs / hbm,
                    "peak_source": f"{src} hbm_gbs"})
    return out


def attn_decode(reps):
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl, synth
    hbm, tc, src = _peaks()
    out = []
    for name in ("c5", "c2"):
        cfg = synth.config(name)
        w = synth.make_weights(cfg)
        stream = torch.cuda.Stream()
        eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=cfg.batch, max_ctx=cfg.ctx_len + 1, stream=stream)
        lens = [cfg.ctx_len] * cfg.batch
        h0 = torch.from_numpy(synth.make_h0(cfg, w["rng"], cfg.batch)).cuda()
        logits = torch.empty((cfg.batch, cfg.vocab), dtype=torch.float32, device="cuda")
        eng.set_option(fl.FL_OPT_PROFILE, 1)
        acc, n = 0.0, 0
        for i in range(reps + 2):
            eng.reset(lens, stream=stream)
            eng.decode_step(h0, cfg.batch, None, logits, stream=stream)
            p = eng.profile(stream)
            if i >= 2 and "attn" in p:
                acc += p["attn"][0]
                n = p["attn"][1]
        ms = acc / reps / max(1, n)
        moved = cfg.batch * cfg.n_kv_heads * (cfg.ctx_len + 1) * cfg.head_dim * 2 * 2
        gbs = moved / (ms * 1e-3) / 1e9
        out.append({"kernel": "attn_decode", "shape": f"{name}: {cfg.batch} token(s) x {cfg.ctx_len + 1} keys, "
                    f"{cfg.n_kv_heads} KV heads x {cfg.head_dim}", "ms": ms, "bytes": moved, "achieved": gbs,
                    "unit": "GB/s", "peak": hbm, "frac": gbs / hbm, "peak_source": f"{src} hbm_gbs",
                    "note": "in situ, event-bracketed launch inside the replayed decode graph"})
        eng.close()
        del eng, w
        torch.cuda.empty_cache()
    return out


def quantize_residual(reps):
    import ctypes
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    hbm, tc, src = _peaks()
    L = fl.lib()
    rows, width, g, bits = 65536 * 4 * 4 * 2, 128, 64, 4
    x = torch.randn((rows, width), device="cuda")
    prev = (x + 0.05 * torch.randn_like(x)).to(torch.bfloat16)
    codes = torch.empty((rows, width * bits // 8), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, width // g), dtype=torch.int16, device="cuda")

    def run(i):
        st = L.fl_test_quantize_residual(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(prev.data_ptr()), rows, width,
                                         g, bits, ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                         None)
        assert st == 0
    ms = _time(run, reps)
    moved = rows * width * (4 + 2) + rows * width * bits // 8 + rows * (width // g) * 2
    gbs = moved / (ms * 1e-3) / 1e9
    return [{"kernel": "quantize_residual", "shape": f"int{bits}: {rows} rows x {width}, g{g}", "ms": ms,
             "achieved": gbs, "unit": "GB/s", "peak": hbm, "frac": gbs / hbm, "peak_source": f"{src} hbm_gbs"}]


def decode_step_capture(reps):
    """One decode step at the decode workload's GEMM shapes (8 tokens, d_model
    2048, ffn 5632, vocab 32000) with one shared layer and a 512-token context,
    kernels launched directly (no graph), for an ncu capture of the first GEMM
    launches: a few GB on the device.  Prints no measurement."""
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl, synth
    cfg = synth.config("c2").with_(n_layers=1, ctx_len=512)
    w = synth.make_weights(cfg)
    eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=cfg.batch, max_ctx=cfg.ctx_len + 1)
    eng.load_context(synth.make_context(cfg, w["rng"], [cfg.ctx_len] * cfg.batch))
    eng.set_option(fl.FL_OPT_USE_GRAPH, 0)
    h0 = torch.from_numpy(synth.make_h0(cfg, w["rng"], cfg.batch)).cuda()
    eng.decode_step(h0, cfg.batch)
    torch.cuda.synchronize()
    assert eng.sync_status() == 0
    eng.close()
    return []


CAPTURE = {"workload": "c3", "layers": 2}


def lazy_call_capture(reps):
    """One lazy call of a workload (prefill or decode, sparse residual storage,
    kernels launched directly) after one warm-up call, for ncu captures of its
    lazy-loop kernels: the workload's shapes with `--layers` shared layers, so
    the device holds a few GB at most.  Prints the call's duration (under ncu:
    not a measurement)."""
    import math
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl, synth
    cfg = synth.config(CAPTURE["workload"])
    if CAPTURE["layers"]:
        cfg = cfg.with_(n_layers=CAPTURE["layers"])
    w = synth.make_weights_device(cfg)
    if cfg.mode == "prefill":
        B, T = cfg.batch, cfg.seq_len
        cfg = cfg.with_(resid_rows=min(T, int(math.ceil(cfg.rho * B * T - 1e-9))))
        eng = fl.FlashLoop(cfg, w, max_batch=B, max_ctx=T, max_tokens=B * T)
        h0 = torch.randn((B * T, cfg.d_model), device="cuda")
        run = lambda: (eng.reset(None), eng.prefill(h0, B, T))
    else:
        B = cfg.batch
        cfg = cfg.with_(resid_rows=synth.sparse_rows(cfg, B))
        lens = [cfg.ctx_len] * B
        eng = fl.FlashLoop(cfg, w, max_batch=B, max_ctx=cfg.ctx_len + 1)
        eng.load_context_device(lens)
        eng.set_option(fl.FL_OPT_USE_GRAPH, 0)
        h0 = torch.randn((B, cfg.d_model), device="cuda")
        run = lambda: (eng.reset(lens), eng.decode_step(h0, B))
    run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    run()
    b.record()
    b.synchronize()
    assert eng.sync_status() == 0
    eng.close()
    return [{"kernel": "lazy call", "workload": CAPTURE["workload"], "layers": cfg.n_layers,
             "ms": a.elapsed_time(b), "note": "kernels launched directly, for ncu captures"}]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--only", default="", help="comma-separated subset, e.g. gemm_wide,topk")
    ap.add_argument("--workload", default="c3", help="lazy_call_capture: the workload")
    ap.add_argument("--layers", type=int, default=2, help="lazy_call_capture: shared layers (0: the workload's)")
    args = ap.parse_args()
    CAPTURE.update(workload=args.workload, layers=args.layers)
    from cross_loop_sparsity_b200 import build
    build.build()
    import time
    import torch
    from cross_loop_sparsity_b200.clocks import ClockSampler
    fns = (gemm_wide, gemm_skinny, topk, attn_decode, quantize_residual, quantize, decode_step_capture,
           lazy_call_capture)
    captures = (decode_step_capture, lazy_call_capture)
    only = {x for x in args.only.split(",") if x}
    for fn in fns:
        if (only and fn.__name__ not in only) or (not only and fn in captures):
            continue
        sampler = ClockSampler(torch.cuda.current_device())
        sampler.start()
        time.sleep(0.3)
        lines = fn(args.reps)
        clocks = sampler.stop()
        for line in lines:
            line["clocks"] = clocks
            print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
