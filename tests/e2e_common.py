"""Shared drivers for the end-to-end GPU parity tests.

Each driver draws one seeded workload from ``synth``, runs the CPU oracle on
it, runs the CUDA library on the same arrays through the C ABI, and returns
both.  In "forced" mode the library is handed the oracle's own integer
decisions -- token selections, column sets and residual codes with their
scales (the oracle's outputs become the library's inputs, never the reverse)
-- so the comparison is of arithmetic rather than of decisions that small
floating-point differences flip (a perturbation of 1e-6 of the inputs moves
the oracle's own early-position states by 2% of RMS through code flips).  The
library still computes every key and every residual itself; its selection and
quantiser are checked bit-exactly on identical inputs elsewhere.
"""
import numpy as np

from cross_loop_sparsity_b200 import synth

TOL = 2e-2   # max |gpu - oracle| <= TOL * RMS(oracle), for hidden states and logits

def rel_err(got, want):
    want = np.asarray(want, np.float64)
    rms = float(np.sqrt(np.mean(want ** 2)))
    return float(np.max(np.abs(np.asarray(got, np.float64) - want))) / rms


def top_valid(keys, k, chosen):
    """True when `chosen` (ascending) is a valid top-k of fp32 `keys` under
    (bit pattern desc, index asc) -- checked with a plain sort, not the oracle."""
    keys = np.ascontiguousarray(keys, np.float32)
    bits = keys.view(np.uint32).astype(np.int64)
    order = np.lexsort((np.arange(len(keys)), -bits))
    return np.array_equal(np.sort(order[:k]).astype(np.int32), np.asarray(chosen, np.int32))


def forced_arrays(cfg, trace, n_tiles):
    sel = np.stack([trace["sel"][l] for l in range(2, cfg.n_loops + 1)])
    cols = np.zeros((cfg.n_layers, n_tiles, cfg.n_kv_heads, cfg.c_cols), np.int32)
    ncols = np.zeros((cfg.n_layers, n_tiles, cfg.n_kv_heads), np.int32)
    for key, C in trace["cols"].items():
        j, t, g = key
        cols[j, t, g, :len(C)] = C
        ncols[j, t, g] = len(C)
    return sel, cols, ncols


def forced_codes(cfg, cache, trace, seq, pos):
    """The oracle's residual codes and scales of each loop's recomputed tokens,
    in selection order: [M][K-1][n_sel][2][Hkv][hd] and [..][hd/g]."""
    M, K = cfg.n_layers, cfg.n_loops
    S2 = trace["sel"][2]
    n_sel = len(S2)
    codes = np.zeros((M, K - 1, n_sel, 2, cfg.n_kv_heads, cfg.head_dim), np.int8)
    scales = np.zeros((M, K - 1, n_sel, 2, cfg.n_kv_heads, cfg.head_dim // cfg.group_size), np.float16)
    for l in range(2, K + 1):
        for a, t in enumerate(trace["sel"][l]):
            for kv, nm in enumerate(("k", "v")):
                codes[:, l - 2, a, kv] = getattr(cache, "codes_" + nm)[:, l - 2, seq[t], :, pos[t]]
                scales[:, l - 2, a, kv] = getattr(cache, "scales_" + nm)[:, l - 2, seq[t], :, pos[t]]
    return codes, scales


def run_prefill(cfg, B, T, forced=True, dense=False):
    """forced: True hands over selections, column sets and codes; "sel" hands
    over selections and codes only; False hands over nothing."""
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    from oracle import flashloop_oracle as orc
    if dense:
        cfg = cfg.with_(resid_bits=16)
    w = synth.make_weights(cfg)
    h0 = synth.make_h0(cfg, w["rng"], B * T)
    W = orc.prepare_weights(w)
    ocache = orc.KVCache(cfg, B, T)
    ref = orc.prefill(cfg, W, ocache, h0, B, T)
    eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=B, max_ctx=T, max_tokens=B * T)
    n_tiles = B * ((T + cfg.q_tile - 1) // cfg.q_tile)
    if forced and not dense and cfg.n_loops > 1:
        sel, cols, ncols = forced_arrays(cfg, ref.trace, n_tiles)
        if forced == "sel":   # token selections and codes handed over, column sets left free
            eng.force_selection(sel)
        else:
            eng.force_selection(sel, cols, ncols, n_tiles=n_tiles)
        seq, pos = np.repeat(np.arange(B), T), np.tile(np.arange(T), B)
        eng.force_codes(*forced_codes(cfg, ocache, ref.trace, seq, pos))
    h_out = torch.empty((B * T, cfg.d_model), dtype=torch.float32, device="cuda")
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    eng.prefill(torch.from_numpy(h0).cuda(), B, T, h_out, logits)
    torch.cuda.synchronize()
    out = {"h": h_out.cpu().numpy(), "logits": logits.cpu().numpy(), "status": eng.sync_status(),
           "n_tiles": n_tiles}
    if not dense:
        n_sel = orc.n_select(cfg.rho, B * T)
        out["sel"], out["keys"], out["cols"], out["ncols"] = eng.read_trace(B * T, n_sel, n_tiles)
    return cfg, ref, eng, out


def load_context(eng, cfg, ctx, dense=False):
    """Import a synthetic context into the library's cache (device buffers)."""
    eng.load_context(ctx, dense)


def run_decode(cfg, lens, forced=True, dense=False, steps=1, extra_ctx=0, options=None):
    """forced: True hands over selections, column sets and codes; "sel" hands
    over selections and codes only; False hands over nothing.  options: library
    options (FL_OPT_*) set on the context first."""
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    from oracle import flashloop_oracle as orc
    if dense:
        cfg = cfg.with_(resid_bits=16)
    B = len(lens)
    w = synth.make_weights(cfg)
    rng = w["rng"]
    W = orc.prepare_weights(w)
    tmax = int(max(lens)) + steps + extra_ctx
    ctx = synth.make_dense_context(cfg, rng, lens) if dense else synth.make_context(cfg, rng, lens)
    cache = orc.KVCache.from_dense_context(cfg, ctx, tmax) if dense else orc.KVCache.from_context(cfg, ctx, tmax)
    eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=B, max_ctx=tmax, max_tokens=0)
    for opt, val in (options or {}).items():
        eng.set_option(opt, val)
    load_context(eng, cfg, ctx, dense)
    results = []
    for _ in range(steps):
        h0 = synth.make_h0(cfg, rng, B)
        pos = cache.lens[:B].copy()
        ref = orc.decode_step(cfg, W, cache, h0)
        if forced and not dense and cfg.n_loops > 1:
            sel, cols, ncols = forced_arrays(cfg, ref.trace, B)
            if forced == "sel":   # token selections and codes handed over, column sets left free
                eng.force_selection(sel)
            else:
                eng.force_selection(sel, cols, ncols, n_tiles=B)
            eng.force_codes(*forced_codes(cfg, cache, ref.trace, np.arange(B), pos))
        h_out = torch.empty((B, cfg.d_model), dtype=torch.float32, device="cuda")
        logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
        eng.decode_step(torch.from_numpy(h0).cuda(), B, h_out, logits)
        torch.cuda.synchronize()
        out = {"h": h_out.cpu().numpy(), "logits": logits.cpu().numpy(), "status": eng.sync_status()}
        if not dense:
            n_sel = orc.n_select(cfg.rho, B)
            out["sel"], out["keys"], out["cols"], out["ncols"] = eng.read_trace(B, n_sel, B)
        results.append((ref, out))
    return cfg, cache, eng, results


def run_calls(cfg, B, ctx_lens, chunks, dense=False, decode_after=0, forced=True):
    """Oracle and library through the same calls: an optional synthetic context,
    prefill chunks of the given sizes, then decode steps."""
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    from oracle import flashloop_oracle as orc
    if dense:
        cfg = cfg.with_(resid_bits=16)
    w = synth.make_weights(cfg)
    rng = w["rng"]
    W = orc.prepare_weights(w)
    tmax = max(ctx_lens) + sum(chunks) + decode_after
    if max(ctx_lens) > 0:
        ctx = synth.make_dense_context(cfg, rng, ctx_lens) if dense else synth.make_context(cfg, rng, ctx_lens)
        cache = (orc.KVCache.from_dense_context if dense else orc.KVCache.from_context)(cfg, ctx, tmax)
    else:
        ctx, cache = None, orc.KVCache(cfg, B, tmax)
    eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=B, max_ctx=tmax, max_tokens=B * max(chunks, default=0))
    if ctx is not None:
        eng.load_context(ctx, dense)
    out = []
    for T in chunks:
        h0 = synth.make_h0(cfg, rng, B * T)
        start = cache.lens[:B].copy()
        ref = orc.prefill(cfg, W, cache, h0, B, T)
        n_tiles = B * ((T + cfg.q_tile - 1) // cfg.q_tile)
        if forced and not dense and cfg.n_loops > 1:
            eng.force_selection(*forced_arrays(cfg, ref.trace, n_tiles), n_tiles=n_tiles)
            seq = np.repeat(np.arange(B), T)
            pos = start[seq] + np.tile(np.arange(T), B)
            eng.force_codes(*forced_codes(cfg, cache, ref.trace, seq, pos))
        h_out = torch.empty((B * T, cfg.d_model), dtype=torch.float32, device="cuda")
        logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
        eng.prefill(torch.from_numpy(h0).cuda(), B, T, h_out, logits)
        torch.cuda.synchronize()
        out.append((ref, {"h": h_out.cpu().numpy(), "logits": logits.cpu().numpy(), "status": eng.sync_status()}))
    for _ in range(decode_after):
        h0 = synth.make_h0(cfg, rng, B)
        pos = cache.lens[:B].copy()
        ref = orc.decode_step(cfg, W, cache, h0)
        if forced and not dense and cfg.n_loops > 1:
            sel, cols, ncols = forced_arrays(cfg, ref.trace, B)
            eng.force_selection(sel, cols, ncols, n_tiles=B)
            eng.force_codes(*forced_codes(cfg, cache, ref.trace, np.arange(B), pos))
        h_out = torch.empty((B, cfg.d_model), dtype=torch.float32, device="cuda")
        logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
        eng.decode_step(torch.from_numpy(h0).cuda(), B, h_out, logits)
        torch.cuda.synchronize()
        out.append((ref, {"h": h_out.cpu().numpy(), "logits": logits.cpu().numpy(), "status": eng.sync_status()}))
    eng.close()
    return out


def check_all(results, tol=TOL):
    """Every call's hidden states and logits within tol x RMS of the oracle's."""
    for ref, o in results:
        assert o["status"] == 0
        eh, el = rel_err(o["h"], ref.h), rel_err(o["logits"], ref.logits)
        assert eh <= tol, eh
        assert el <= tol, el
