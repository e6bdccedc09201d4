"""Seeded synthetic inputs for the looped-block workloads.

This module draws random numbers and nothing else: it holds shapes, seeds and
draws, and no step of the lazy-update method (no selection, no quantiser, no
attention, no chain reconstruction).  Both the CPU checker and the CUDA path
take their inputs from here, so the two are fed identical arrays.

Draw recipe (fixed, so that the two sides agree bit for bit):

* ``numpy.random.default_rng(seed)`` (PCG64).
* Per layer, in this order: attention-norm gain (all ones, no draw), W_qkv,
  W_o, MLP-norm gain (ones), W_gate, W_up, W_down; then W_out; then h0; then
  the synthetic decode context.  Each weight is ``sigma * N(0, 1)`` drawn in
  float32 and rounded to bfloat16 (round to nearest even); weights are
  returned as the raw bfloat16 bit patterns (``uint16``).
* h0 is ``N(0, 1)`` in float32.
* Decode context (a cache as a lazy prefill would have left it): base K/V are
  ``N(0, 1)`` rounded to bfloat16; for every loop l = 2..K, a uniformly random
  ``ceil(rho * ctx)`` subset of each sequence's context tokens carries
  residual codes drawn uniformly from [-qmax, qmax] (qmax = 2**(bits-1) - 1)
  with per-group scales ``U[0.01, 0.03]`` rounded to float16; every other
  token has zero codes and zero scales.  The dense per-loop baseline context
  is an independent ``N(0, 1)`` bfloat16 K/V per loop.

Linear weights are row-major ``[out_features, in_features]``.  The QKV rows
are the H query heads, then the Hkv key heads, then the Hkv value heads, each
``head_dim`` rows.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "LoopConfig", "CONFIGS", "config", "bf16_bits", "bf16_bits_to_f32",
    "make_weights", "make_h0", "make_context", "make_dense_context",
    "make_keys", "make_residuals", "make_weights_device", "context_slices_device",
]


@dataclasses.dataclass(frozen=True)
class LoopConfig:
    """Shapes and knobs of one looped-block workload."""
    name: str
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    n_layers: int          # M: layers in the shared block
    n_loops: int           # K: applications of the block
    rho: float             # fraction of tokens recomputed at loops >= 2
    c_cols: int            # key columns kept per (query tile, KV head)
    resid_bits: int = 4    # 4 or 2; 16 = dense per-loop bfloat16 KV
    group_size: int = 64
    q_tile: int = 128
    resid_scale: float = 0.3
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0
    vocab: int = 32000
    sigma: float = 0.02
    seed: int = 0
    mode: str = "decode"   # "prefill" or "decode"
    batch: int = 1
    seq_len: int = 0       # prefill tokens per sequence
    ctx_len: int = 0       # existing context per sequence (decode)
    kv_mode: int = 0       # dense path: 0 per_loop KV, 1 last_loop (one KV per layer, overwritten each loop)
    # variants around the looped core: independent layers before (prelude) and
    # after (coda) the loop, a per-loop input embedding, and input injection
    n_prelude: int = 0
    n_coda: int = 0
    loop_embed: int = 0        # 1: loop k's input is h + e_k
    inject_scale: float = 0.0  # gamma: loop k's input also adds gamma * (the state entering the loop)
    resid_rows: int = 0        # sparse residual storage: rows per pool (0: one row per position)

    @property
    def qkv_rows(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def max_ctx(self) -> int:
        return self.ctx_len + self.seq_len + (1 if self.mode == "decode" else 0)

    def with_(self, **kw) -> "LoopConfig":
        return dataclasses.replace(self, **kw)


_C2_BLOCK = dict(d_model=2048, n_heads=16, n_kv_heads=4, head_dim=128, ffn_dim=5632)

CONFIGS = {
    # tiny looped block, prefill of 128 tokens (the oracle finishes in seconds)
    "c1": LoopConfig("c1", d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, ffn_dim=688,
                     n_layers=2, n_loops=4, rho=0.25, c_cols=32, resid_bits=4, group_size=32,
                     sigma=0.02, seed=0, mode="prefill", batch=1, seq_len=128),
    # decode step: 8 sequences over a 4096-token context
    "c2": LoopConfig("c2", **_C2_BLOCK, n_layers=4, n_loops=4, rho=0.10, c_cols=256,
                     resid_bits=4, group_size=64, sigma=0.02, seed=1, mode="decode",
                     batch=8, ctx_len=4096),
    # long prefill: 22 layers x 2 passes over 16384 tokens
    "c3": LoopConfig("c3", **_C2_BLOCK, n_layers=22, n_loops=2, rho=0.15, c_cols=512,
                     resid_bits=4, group_size=64, sigma=0.02, seed=2, mode="prefill",
                     batch=1, seq_len=16384),
    # deep recurrence: 48 layers x 4 loops, decode over 8192 tokens
    "c4": LoopConfig("c4", d_model=4096, n_heads=32, n_kv_heads=8, head_dim=128, ffn_dim=11008,
                     n_layers=48, n_loops=4, rho=0.05, c_cols=256, resid_bits=4, group_size=128,
                     sigma=0.01, seed=3, mode="decode", batch=4, ctx_len=8192),
    # KV-residual stress: K=8 loops, decode at a 65536-token context (int4 and int2)
    "c5": LoopConfig("c5", **_C2_BLOCK, n_layers=4, n_loops=8, rho=0.05, c_cols=1024,
                     resid_bits=4, group_size=64, sigma=0.02, seed=4, mode="decode",
                     batch=1, ctx_len=65536),
    "c5_int2": LoopConfig("c5_int2", **_C2_BLOCK, n_layers=4, n_loops=8, rho=0.05, c_cols=1024,
                          resid_bits=2, group_size=64, sigma=0.02, seed=4, mode="decode",
                          batch=1, ctx_len=65536),
}


def config(name: str, **overrides) -> LoopConfig:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg


def sparse_rows(cfg: LoopConfig, extra: int) -> int:
    """Rows per sparse residual pool for a cache of cfg.max_ctx positions whose
    tokens were recomputed at rate rho (the synthetic context's rate), plus
    `extra` rows for tokens appended later."""
    return min(cfg.max_ctx, int(math.ceil(cfg.rho * cfg.max_ctx - 1e-9)) + extra)


# ----------------------------------------------------------------------------
# bfloat16 bit patterns (input preparation: weights and KV are bf16 data)
# ----------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (NaN kept quiet)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    nan = (u & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = ((u[nan] >> np.uint32(16)) | np.uint32(0x40)).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, sigma: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return bf16_bits(x)


# ----------------------------------------------------------------------------
# weights, inputs, context
# ----------------------------------------------------------------------------

def make_weights(cfg: LoopConfig, rng: np.random.Generator | None = None) -> dict:
    """All block weights as bfloat16 bit patterns; norm gains are float32 ones."""
    rng = np.random.default_rng(cfg.seed) if rng is None else rng
    d = cfg.d_model
    out = {
        "layers": [_draw_layer(cfg, rng) for _ in range(cfg.n_layers)],
        "final_norm": np.ones(d, np.float32),
        "w_out": _normal_bf16(rng, (cfg.vocab, d), cfg.sigma),
        "rng": rng,
    }
    # variants, drawn after everything above so the plain looped block's draws
    # do not move: prelude layers, coda layers, then the loop embeddings
    # e_1..e_K ~ N(0, 1) float32 (the scale of the residual stream)
    if cfg.n_prelude:
        out["prelude"] = [_draw_layer(cfg, rng) for _ in range(cfg.n_prelude)]
    if cfg.n_coda:
        out["coda"] = [_draw_layer(cfg, rng) for _ in range(cfg.n_coda)]
    if cfg.loop_embed:
        out["loop_embed"] = rng.standard_normal(size=(cfg.n_loops, d), dtype=np.float32)
    return out


def _draw_layer(cfg: LoopConfig, rng: np.random.Generator) -> dict:
    """One layer's weights in the draw order of the recipe."""
    d, f, hq = cfg.d_model, cfg.ffn_dim, cfg.n_heads * cfg.head_dim
    lw = {}
    lw["attn_norm"] = np.ones(d, np.float32)
    lw["w_qkv"] = _normal_bf16(rng, (cfg.qkv_rows, d), cfg.sigma)
    lw["w_o"] = _normal_bf16(rng, (d, hq), cfg.sigma)
    lw["mlp_norm"] = np.ones(d, np.float32)
    lw["w_gate"] = _normal_bf16(rng, (f, d), cfg.sigma)
    lw["w_up"] = _normal_bf16(rng, (f, d), cfg.sigma)
    lw["w_down"] = _normal_bf16(rng, (d, f), cfg.sigma)
    return lw


def make_h0(cfg: LoopConfig, rng: np.random.Generator, n_tokens: int) -> np.ndarray:
    return rng.standard_normal(size=(n_tokens, cfg.d_model), dtype=np.float32)


def make_context(cfg: LoopConfig, rng: np.random.Generator, ctx_lens) -> dict:
    """Synthetic base + residual cache for ``len(ctx_lens)`` sequences.

    Arrays are sized to ``max(ctx_lens)``; rows at or past a sequence's own
    length are zero.  Shapes (M layers, K loops, B sequences):
      base_k, base_v : uint16 bf16 bits [M, B, Hkv, T, hd]
      codes_k, codes_v : int8 [M, K-1, B, Hkv, T, hd]
      scales_k, scales_v : float16 [M, K-1, B, Hkv, T, hd/g]
    """
    lens = np.asarray(ctx_lens, dtype=np.int64)
    B, T = len(lens), int(lens.max()) if len(lens) else 0
    M, K, Hkv, hd, g = cfg.n_layers, cfg.n_loops, cfg.n_kv_heads, cfg.head_dim, cfg.group_size
    qmax = (1 << (cfg.resid_bits - 1)) - 1
    base_k = np.zeros((M, B, Hkv, T, hd), np.uint16)
    base_v = np.zeros_like(base_k)
    codes_k = np.zeros((M, max(K - 1, 0), B, Hkv, T, hd), np.int8)
    codes_v = np.zeros_like(codes_k)
    scales_k = np.zeros((M, max(K - 1, 0), B, Hkv, T, hd // g), np.float16)
    scales_v = np.zeros_like(scales_k)
    for j in range(M):
        for b in range(B):
            n = int(lens[b])
            base_k[j, b, :, :n] = _normal_bf16(rng, (Hkv, n, hd), 1.0)
            base_v[j, b, :, :n] = _normal_bf16(rng, (Hkv, n, hd), 1.0)
        for li in range(K - 1):
            for b in range(B):
                n = int(lens[b])
                m = min(n, int(math.ceil(cfg.rho * n - 1e-9)))
                rows = np.sort(rng.choice(n, size=m, replace=False)) if m > 0 else np.zeros(0, np.int64)
                for codes, scales in ((codes_k, scales_k), (codes_v, scales_v)):
                    c_view = codes[j, li, b]      # [Hkv, T, hd]
                    s_view = scales[j, li, b]     # [Hkv, T, hd/g]
                    c_view[:, rows] = rng.integers(-qmax, qmax + 1, size=(Hkv, len(rows), hd),
                                                   dtype=np.int8)
                    s_view[:, rows] = rng.uniform(0.01, 0.03, size=(Hkv, len(rows), hd // g)
                                                  ).astype(np.float16)
    out = {"lens": lens, "base_k": base_k, "base_v": base_v, "codes_k": codes_k, "codes_v": codes_v,
           "scales_k": scales_k, "scales_v": scales_v}
    out.update(_extra_context(cfg, rng, lens))
    return out


def _extra_context(cfg: LoopConfig, rng: np.random.Generator, lens) -> dict:
    """KV of the prelude and coda layers (one pass each): uint16 bf16 bits
    [P+Q, B, Hkv, T, hd] of N(0, 1), drawn after the looped layers' context."""
    X = cfg.n_prelude + cfg.n_coda
    if X == 0:
        return {}
    B, T = len(lens), int(max(lens)) if len(lens) else 0
    xk = np.zeros((X, B, cfg.n_kv_heads, T, cfg.head_dim), np.uint16)
    xv = np.zeros_like(xk)
    for x in range(X):
        for b in range(B):
            n = int(lens[b])
            xk[x, b, :, :n] = _normal_bf16(rng, (cfg.n_kv_heads, n, cfg.head_dim), 1.0)
            xv[x, b, :, :n] = _normal_bf16(rng, (cfg.n_kv_heads, n, cfg.head_dim), 1.0)
    return {"extra_k": xk, "extra_v": xv}


def make_dense_context(cfg: LoopConfig, rng: np.random.Generator, ctx_lens) -> dict:
    """bf16 K/V context for the dense looped baseline: uint16 [M, KS, B, Hkv, T, hd],
    KS = K loop slots (per_loop) or 1 (last_loop)."""
    lens = np.asarray(ctx_lens, dtype=np.int64)
    B, T = len(lens), int(lens.max()) if len(lens) else 0
    M, Hkv, hd = cfg.n_layers, cfg.n_kv_heads, cfg.head_dim
    K = 1 if cfg.kv_mode == 1 else cfg.n_loops
    kv_k = np.zeros((M, K, B, Hkv, T, hd), np.uint16)
    kv_v = np.zeros_like(kv_k)
    for j in range(M):
        for l in range(K):
            for b in range(B):
                n = int(lens[b])
                kv_k[j, l, b, :, :n] = _normal_bf16(rng, (Hkv, n, hd), 1.0)
                kv_v[j, l, b, :, :n] = _normal_bf16(rng, (Hkv, n, hd), 1.0)
    out = {"lens": lens, "kv_k": kv_k, "kv_v": kv_v}
    out.update(_extra_context(cfg, rng, lens))
    return out


# ----------------------------------------------------------------------------
# unit-test inputs
# ----------------------------------------------------------------------------

def make_keys(seed: int, n: int, kind: str = "ties") -> np.ndarray:
    """float32 selection keys.  ``ties`` mixes many duplicates and zeros."""
    rng = np.random.default_rng(seed)
    if kind == "ties":
        pool = rng.standard_normal(max(1, n // 8), dtype=np.float32) ** 2
        keys = rng.choice(pool, size=n)
        keys[rng.random(n) < 0.25] = 0.0
        return keys.astype(np.float32)
    if kind == "distinct":
        return (rng.standard_normal(n, dtype=np.float32) ** 2).astype(np.float32)
    raise ValueError(kind)


def make_residuals(seed: int, n_rows: int, width: int, scale_mix: bool = True) -> np.ndarray:
    """float32 residual rows with varied magnitudes, exact zeros and ties."""
    rng = np.random.default_rng(seed)
    r = rng.standard_normal((n_rows, width), dtype=np.float32)
    if scale_mix:
        mags = np.float32(10.0) ** rng.uniform(-6, 2, size=(n_rows, 1)).astype(np.float32)
        r *= mags
        r[rng.random((n_rows, width)) < 0.05] = 0.0
        zero_rows = rng.random(n_rows) < 0.05
        r[zero_rows] = 0.0
    return r.astype(np.float32)


# ----------------------------------------------------------------------------
# device-drawn inputs for benchmark workloads too large to draw on the host
# ----------------------------------------------------------------------------
# The same distributions as above, drawn on the GPU with torch's seeded
# generator (Philox) instead of PCG64, so the 17 GB of deep-recurrence weights
# or a 65536-token context take seconds, not minutes.  The parity tests use the
# host draws; the benchmark's timings do not depend on which generator drew the
# values.

def _dev_gen(seed: int, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _dev_normal_bf16(g, shape, sigma: float, device):
    import torch
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(torch.bfloat16).view(torch.int16)     # round to nearest even, bit patterns


def make_weights_device(cfg: LoopConfig, device="cuda", seed: int | None = None) -> dict:
    """Block weights stacked over layers on the device (bf16 bits as int16,
    gains float32 ones), in the layout ``flashloop.upload_weights`` returns."""
    import torch
    g = _dev_gen(cfg.seed if seed is None else seed, device)
    M, d, f, hq = cfg.n_layers, cfg.d_model, cfg.ffn_dim, cfg.n_heads * cfg.head_dim
    out = {"attn_norm": torch.ones((M, d), dtype=torch.float32, device=device),
           "mlp_norm": torch.ones((M, d), dtype=torch.float32, device=device),
           "final_norm": torch.ones((d,), dtype=torch.float32, device=device)}
    shapes = {"w_qkv": (cfg.qkv_rows, d), "w_o": (d, hq), "w_gate": (f, d), "w_up": (f, d), "w_down": (d, f)}
    for name, shp in shapes.items():
        t = torch.empty((M,) + shp, dtype=torch.int16, device=device)
        for j in range(M):              # one layer at a time keeps the fp32 draw small
            t[j] = _dev_normal_bf16(g, shp, cfg.sigma, device)
        out[name] = t
    out["w_out"] = _dev_normal_bf16(g, (cfg.vocab, d), cfg.sigma, device)
    return out


def context_slices_device(cfg: LoopConfig, ctx_lens, device="cuda", seed: int | None = None, dense: bool = False):
    """Yield one (layer, sequence) slice of a synthetic decode context at a time,
    drawn on the device, in the import layout of ``flashloop_import_lazy``
    (``dense``: ``flashloop_import_dense``):
      lazy : (j, b, base_k, base_v, codes_k, codes_v, scales_k, scales_v) with base
             bf16 bits [Hkv][n][hd], codes int8 [K-1][Hkv][n][hd], scales fp16 bits
             [K-1][Hkv][n][hd/g]; for each loop a uniformly random ceil(rho*n)
             subset of the rows carries codes uniform in [-qmax, qmax] and scales
             U[0.01, 0.03], the other rows zero (the recipe of ``make_context``)
      dense: (j, b, kv_k, kv_v) with bf16 bits [KS][Hkv][n][hd], N(0, 1), KS = K loop
             slots (per_loop) or 1 (last_loop)."""
    import torch
    g = _dev_gen((cfg.seed if seed is None else seed) + 7919, device)
    M, K, Hkv, hd = cfg.n_layers, cfg.n_loops, cfg.n_kv_heads, cfg.head_dim
    KS = 1 if (dense and cfg.kv_mode == 1) else K
    for j in range(M):
        for b, n in enumerate(ctx_lens):
            n = int(n)
            if n == 0:
                continue
            if dense:
                yield (j, b, _dev_normal_bf16(g, (KS, Hkv, n, hd), 1.0, device),
                       _dev_normal_bf16(g, (KS, Hkv, n, hd), 1.0, device))
                continue
            ng = hd // cfg.group_size
            qmax = (1 << (cfg.resid_bits - 1)) - 1
            m = min(n, int(math.ceil(cfg.rho * n - 1e-9)))
            base = [_dev_normal_bf16(g, (Hkv, n, hd), 1.0, device) for _ in range(2)]
            codes = [torch.zeros((max(K - 1, 0), Hkv, n, hd), dtype=torch.int8, device=device) for _ in range(2)]
            scales = [torch.zeros((max(K - 1, 0), Hkv, n, ng), dtype=torch.float16, device=device) for _ in range(2)]
            for li in range(K - 1):
                rows = torch.sort(torch.randperm(n, generator=g, device=device)[:m]).values
                for w in range(2):
                    codes[w][li][:, rows] = torch.randint(-qmax, qmax + 1, (Hkv, m, hd), generator=g, device=device,
                                                          dtype=torch.int8)
                    scales[w][li][:, rows] = (torch.rand((Hkv, m, ng), generator=g, device=device) * 0.02 + 0.01
                                              ).to(torch.float16)
            yield (j, b, base[0], base[1], codes[0], codes[1], scales[0].view(torch.int16),
                   scales[1].view(torch.int16))
