"""CPU oracle of FlashLoop's lazy-update looped-Transformer inference step.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
calls it and shares no code with it; its inputs come from the seeded
generators (``cross_loop_sparsity_b200.synth``) and never from the GPU.

Plain, slow and meant to be read against the pages:

* "FlashLoop: Fast and Memory-Efficient Looped Transformers via Lazy Updates"
  (abstract) -- the method: token-sparse updates, sparse attention over a
  fixed small set of key columns, and each loop's KV kept as a low-bit
  residual over the previous loop's.  It gives no equations; the concrete rules below (ranking by
  the squared change norm, top-c columns by |delta score|, per-group absmax
  int4/int2 codes) are the plainest reading of it, and every open point is
  listed with the reading taken in the design notes.
* "Looped Transformer 教程：权重共享、循环次数与推理成本怎么读", 第一步 (the
  looped forward ``for _ in range(num_passes): h = shared_stack(h)``) and
  第四步 (per-loop KV cache, ``per_loop`` mode) -- the dense looped baseline.
* "循环Transformer解析：参数不变，推理深度翻倍", the ``forward_looped`` sketch
  -- the same dense loop over a shared stack of layers.
* "从'堆层数'到'循环复用'：FlashLoop 到底在解决什么问题", §3.2 (rotary position
  encoding inside the loop body; residual connection carries the state) and
  §8 (pre-norm placement) -- the layer: pre-RMSNorm, RoPE attention, SwiGLU
  MLP, scaled residual adds.

Precision: floating point is fp64, except where floating point decides an
integer -- the quantiser (residual, scale and code are taken in IEEE fp32, as
the kernels take them) and the selection keys (rounded to fp32 and ordered by
their bit pattern).  The residual chain is defined as fp32 accumulation in loop
order, base first; bf16 storage of base / per-loop KV is modelled by
round-to-nearest-even.  Activations are never rounded: the oracle is the plain
high-precision statement of the step, whatever precision the GPU computes in.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against a definition other than itself (dense limit, brute force, closed
forms, a torch restatement of a plain block).
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64
F32 = np.float32


# ============================================================================
# scalar rules
# ============================================================================

def n_select(rho: float, n: int) -> int:
    """Number of tokens recomputed at a lazy loop: ceil(rho*N), at least 1, at most N.

    Token-sparse updates ("FlashLoop ...", abstract).  The 1e-9 guard keeps
    an exact product such as 0.25*128 from rounding up to 33.
    """
    if n <= 0:
        return 0
    k = int(math.ceil(rho * n - 1e-9))
    return max(1, min(n, k))


def select_top(keys: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest fp32 keys, returned in ascending index order.

    Order: the key's IEEE-754 bit pattern read as an unsigned integer,
    descending (so NaN sorts above +inf), ties to the lower index.  Used for
    the top-rho tokens and for the top-c key columns ("FlashLoop ...",
    abstract: few tokens carry most of a loop's state change, and few key
    columns carry most of the change in attention output).
    """
    keys = np.ascontiguousarray(keys, dtype=F32)
    n = keys.shape[0]
    k = max(0, min(int(k), n))
    bits = keys.view(np.uint32).astype(np.uint64)
    order = np.lexsort((np.arange(n), np.uint64(0xFFFFFFFF) - bits))
    return np.sort(order[:k]).astype(np.int32)


# ============================================================================
# number formats
# ============================================================================

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 value (ties to even), returned as float64.

    Models bf16 storage of the base / per-loop KV cache.  Works on the fp32
    bit pattern: add 0x7FFF plus the lowest kept bit, drop 16 bits.
    """
    u = np.ascontiguousarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return (r.astype(np.uint32)).view(F32).astype(F64)


def fp16_round_up(x: np.ndarray) -> np.ndarray:
    """Smallest IEEE binary16 value >= x, for finite fp32 x >= 0 (result float16).

    Definition-based: take the nearest binary16 value, and if it lies below x
    step to the next representable binary16 value towards +inf.  Values above
    the largest finite binary16 give +inf.
    """
    x = np.asarray(x, dtype=F32)
    with np.errstate(over="ignore"):
        y = x.astype(np.float16)
        below = y.astype(F32) < x
        if np.any(below):
            y = np.where(below, np.nextafter(y, np.float16(np.inf)), y)
    return y.astype(np.float16)


def qmax_of(bits: int) -> int:
    return (1 << (bits - 1)) - 1


def quantize_groups(r: np.ndarray, bits: int, g: int):
    """Per-group symmetric absmax quantiser of a KV residual.

    r: fp32 [..., hd] with hd % g == 0.  For each contiguous group of g
    elements: s = fp16_RU(fp32(absmax / qmax)) (s = 0 when absmax = 0) and
    code = clamp(rint(fp32(r / s)), -qmax, qmax) with rint ties-to-even.
    Returns (codes int8 [..., hd], scales float16 [..., hd/g]).
    KV-residual quantisation ("FlashLoop ...", abstract).
    """
    r = np.ascontiguousarray(r, dtype=F32)
    hd = r.shape[-1]
    assert hd % g == 0
    qm = qmax_of(bits)
    rg = r.reshape(r.shape[:-1] + (hd // g, g))
    amax = np.max(np.abs(rg), axis=-1).astype(F32)
    s32 = (amax / F32(qm)).astype(F32)
    s16 = fp16_round_up(s32)
    s = s16.astype(F32)
    safe = np.where(s > 0, s, F32(1))
    q = (rg / safe[..., None]).astype(F32)
    codes = np.clip(np.rint(q), -qm, qm)
    codes = np.where(s[..., None] > 0, codes, 0).astype(np.int8)
    return codes.reshape(r.shape), s16


def dequant_groups(codes: np.ndarray, scales: np.ndarray, g: int) -> np.ndarray:
    """code * scale per element, in fp32 (exact: |code| <= 7, 11-bit scale)."""
    s = np.repeat(np.asarray(scales, dtype=F32), g, axis=-1)
    return (np.asarray(codes, dtype=F32) * s).astype(F32)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack two's-complement codes along the last axis into bytes.

    int4: element 2i in the low nibble of byte i, element 2i+1 in the high
    nibble.  int2: element 4i+j in bits 2j..2j+1 of byte i.
    """
    c = np.asarray(codes, dtype=np.int64) & ((1 << bits) - 1)
    per = 8 // bits
    c = c.reshape(c.shape[:-1] + (c.shape[-1] // per, per))
    out = np.zeros(c.shape[:-1], dtype=np.int64)
    for j in range(per):
        out |= c[..., j] << (bits * j)
    return out.astype(np.uint8)


def unpack_codes(packed: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of ``pack_codes`` (sign-extends each field)."""
    p = np.asarray(packed, dtype=np.int64)
    per = 8 // bits
    mask = (1 << bits) - 1
    fields = [(p >> (bits * j)) & mask for j in range(per)]
    c = np.stack(fields, axis=-1)
    c = np.where(c >= (1 << (bits - 1)), c - (1 << bits), c)
    return c.reshape(p.shape[:-1] + (p.shape[-1] * per,)).astype(np.int8)


# ============================================================================
# layer pieces (fp64)
# ============================================================================

def rmsnorm(h: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """x = gain * h / sqrt(mean(h^2) + eps) over the last axis (pre-norm)."""
    h = np.asarray(h, dtype=F64)
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + eps) * np.asarray(gain, dtype=F64)


def rope_angles(pos: np.ndarray, hd: int, theta: float) -> np.ndarray:
    """angle[t, i] = pos_t * theta^(-2i/hd) for i < hd/2 (fp64)."""
    i = np.arange(hd // 2, dtype=F64)
    inv_freq = theta ** (-2.0 * i / hd)
    return np.asarray(pos, dtype=F64)[:, None] * inv_freq[None, :]


def apply_rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE: pair (i, i + hd/2) rotated by angle(pos, i).

    x: [n, heads, hd]; pos: [n] absolute positions (the same every loop).
    """
    hd = x.shape[-1]
    half = hd // 2
    ang = rope_angles(pos, hd, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def prepare_weights(w: dict) -> dict:
    """bf16 bit patterns -> float64 arrays (once per test)."""
    def f(b):
        return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(F32).astype(F64)
    out = {"layers": []}
    for lw in w["layers"]:
        out["layers"].append({
            "attn_norm": np.asarray(lw["attn_norm"], F64), "mlp_norm": np.asarray(lw["mlp_norm"], F64),
            "w_qkv": f(lw["w_qkv"]), "w_o": f(lw["w_o"]), "w_gate": f(lw["w_gate"]),
            "w_up": f(lw["w_up"]), "w_down": f(lw["w_down"]),
        })
    out["final_norm"] = np.asarray(w["final_norm"], F64)
    out["w_out"] = f(w["w_out"])
    for part in ("prelude", "coda"):
        if part in w:
            out[part] = prepare_weights({"layers": w[part], "final_norm": w["final_norm"],
                                         "w_out": w["w_out"][:1]})["layers"]
    if "loop_embed" in w:
        out["loop_embed"] = np.asarray(w["loop_embed"], F64)
    return out


def _qkv(cfg, lw, h, pos):
    """Pre-norm, fused QKV projection, RoPE on q and k.  Returns q [n,H,hd], k, v [n,Hkv,hd]."""
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    x = rmsnorm(h, lw["attn_norm"], cfg.rms_eps)
    y = x @ lw["w_qkv"].T
    q = y[:, :H * hd].reshape(-1, H, hd)
    k = y[:, H * hd:(H + Hkv) * hd].reshape(-1, Hkv, hd)
    v = y[:, (H + Hkv) * hd:].reshape(-1, Hkv, hd)
    return apply_rope(q, pos, cfg.rope_theta), apply_rope(k, pos, cfg.rope_theta), v


def _mlp_update(cfg, lw, h):
    """h + s * W_down(silu(W_gate x) * W_up x), x = RMSNorm(h)."""
    x = rmsnorm(h, lw["mlp_norm"], cfg.rms_eps)
    a = silu(x @ lw["w_gate"].T) * (x @ lw["w_up"].T)
    return h + cfg.resid_scale * (a @ lw["w_down"].T)


def _attn_full(q_i, keys, vals, tau):
    """Plain softmax attention of one query over n columns, all heads.

    q_i [H, hd]; keys, vals [Hkv, n, hd].  Returns O [H, hd], lse [H].
    """
    Hkv, n, hd = keys.shape
    grp = q_i.shape[0] // Hkv
    qg = q_i.reshape(Hkv, grp, hd)
    s = tau * np.einsum("gqd,gtd->gqt", qg, keys)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=-1, keepdims=True)
    o = np.einsum("gqt,gtd->gqd", e, vals) / z
    lse = (m + np.log(z))[..., 0]
    return o.reshape(-1, hd), lse.reshape(-1)


# ============================================================================
# KV cache (per layer: bf16 base + residual per loop; or dense per-loop KV)
# ============================================================================

class KVCache:
    """Cache rows per (layer, sequence, KV head, position).

    Lazy layout (bits 2/4, or 32 = exact fp64 residual, checker-only):
      base_k/v [M, B, Hkv, T, hd]   -- loop-1 KV (bf16 values unless exact)
      codes_k/v [M, K-1, B, Hkv, T, hd] int8 and scales_k/v [.., hd/g] float16
      res_k/v  [M, K-1, B, Hkv, T, hd] -- dequantised residual (fp32, or fp64 when exact)
    Dense layout (bits 16): kv_k/v [M, KS, B, Hkv, T, hd] (bf16 values unless
    exact), KS = K with per-loop KV ("Looped Transformer 教程", 第四步:
    per_loop), or 1 in last_loop mode, where each loop overwrites the one slot
    with its own KV and only the last pass is kept (第四步: last_loop).
    """

    def __init__(self, cfg, B: int, tmax: int, kv_exact: bool = False):
        self.cfg, self.B, self.tmax = cfg, B, tmax
        self.kv_exact = kv_exact
        self.lens = np.zeros(B, dtype=np.int64)
        M, K, Hkv, hd = cfg.n_layers, cfg.n_loops, cfg.n_kv_heads, cfg.head_dim
        # prelude and coda layers: one pass of KV each, [P+Q, B, Hkv, T, hd]
        X = getattr(cfg, "n_prelude", 0) + getattr(cfg, "n_coda", 0)
        self.xk = np.zeros((X, B, Hkv, tmax, hd), F64)
        self.xv = np.zeros_like(self.xk)
        self.dense = cfg.resid_bits == 16
        if self.dense:
            self.last_loop = getattr(cfg, "kv_mode", 0) == 1
            self.kv_k = np.zeros((M, 1 if self.last_loop else K, B, Hkv, tmax, hd), F64)
            self.kv_v = np.zeros_like(self.kv_k)
        else:
            exact = cfg.resid_bits == 32
            rdt = F64 if exact else F32
            self.base_k = np.zeros((M, B, Hkv, tmax, hd), F64 if kv_exact else F32)
            self.base_v = np.zeros_like(self.base_k)
            self.res_k = np.zeros((M, K - 1, B, Hkv, tmax, hd), rdt)
            self.res_v = np.zeros_like(self.res_k)
            if not exact:
                g = cfg.group_size
                self.codes_k = np.zeros((M, K - 1, B, Hkv, tmax, hd), np.int8)
                self.codes_v = np.zeros_like(self.codes_k)
                self.scales_k = np.zeros((M, K - 1, B, Hkv, tmax, hd // g), np.float16)
                self.scales_v = np.zeros_like(self.scales_k)

    # -- synthetic context -------------------------------------------------
    @classmethod
    def from_context(cls, cfg, ctx: dict, tmax: int):
        """Load a synthetic lazy context (base bf16 bits, int8 codes, fp16 scales)."""
        lens = np.asarray(ctx["lens"])
        c = cls(cfg, len(lens), tmax)
        T = ctx["base_k"].shape[3]
        to32 = lambda b: (b.astype(np.uint32) << 16).view(F32)
        c.base_k[:, :, :, :T] = to32(ctx["base_k"])
        c.base_v[:, :, :, :T] = to32(ctx["base_v"])
        g = cfg.group_size
        for name in ("k", "v"):
            codes, scales = ctx["codes_" + name], ctx["scales_" + name]
            getattr(c, "codes_" + name)[..., :T, :] = codes
            getattr(c, "scales_" + name)[..., :T, :] = scales
            getattr(c, "res_" + name)[..., :T, :] = dequant_groups(codes, scales, g)
        c._load_extra(ctx, T)
        c.lens[:] = lens
        return c

    def _load_extra(self, ctx, T):
        if "extra_k" in ctx:
            to64 = lambda b: (b.astype(np.uint32) << 16).view(F32).astype(F64)
            self.xk[..., :T, :] = to64(ctx["extra_k"])
            self.xv[..., :T, :] = to64(ctx["extra_v"])

    @classmethod
    def from_dense_context(cls, cfg, ctx: dict, tmax: int):
        lens = np.asarray(ctx["lens"])
        c = cls(cfg, len(lens), tmax)
        T = ctx["kv_k"].shape[4]
        to64 = lambda b: (b.astype(np.uint32) << 16).view(F32).astype(F64)
        c.kv_k[..., :T, :] = to64(ctx["kv_k"])
        c.kv_v[..., :T, :] = to64(ctx["kv_v"])
        c._load_extra(ctx, T)
        c.lens[:] = lens
        return c

    def slot(self, l: int) -> int:
        """Dense KV slot of loop l (1..K): its own, or the single last_loop slot."""
        return 0 if self.last_loop else l - 1

    # -- storage rules -----------------------------------------------------
    def store_kv(self, x: np.ndarray) -> np.ndarray:
        """Value a base / per-loop KV row takes when stored."""
        return np.asarray(x, F64) if self.kv_exact else bf16_round(x)

    def chain(self, which: str, j: int, m: int, b: int, rows) -> np.ndarray:
        """Reconstructed KV of loop m for rows of sequence b: [Hkv, n, hd].

        base, then + residual of loops 2..m in that order; each add rounded to
        fp32 (fp64 in the exact mode).  KV_l = KV_{l-1} + deq(q(r_l))
        ("FlashLoop ...", abstract: each loop's KV as a residual over the
        previous loop's).
        """
        base = getattr(self, "base_" + which)[j, b][:, rows]
        res = getattr(self, "res_" + which)
        exact = self.cfg.resid_bits == 32
        acc = base.astype(F64 if exact else F32)
        for l in range(2, m + 1):
            r = res[j, l - 2, b][:, rows]
            acc = (acc + r) if exact else (acc + r).astype(F32)
        return acc.astype(F64)


# ============================================================================
# variants around the looped core
# ============================================================================

def _independent_layer(cfg, lw, cache: KVCache, x: int, h, seq, pos):
    """One prelude or coda layer: applied once to every token, its own weights
    and its own one-pass KV (slot x of cache.xk / xv), otherwise the same
    pre-norm layer as the shared block ("从'堆层数'到'循环复用'", §3.1: the
    independent first P and last Q layers around the R looped layers)."""
    tau = 1.0 / math.sqrt(cfg.head_dim)
    N = h.shape[0]
    q, k, v = _qkv(cfg, lw, h, pos)
    for i in range(N):
        cache.xk[x, seq[i], :, pos[i]] = cache.store_kv(k[i])
        cache.xv[x, seq[i], :, pos[i]] = cache.store_kv(v[i])
    O = np.zeros((N, cfg.n_heads, cfg.head_dim))
    for i in range(N):
        O[i], _ = _attn_full(q[i], cache.xk[x, seq[i]][:, :pos[i] + 1], cache.xv[x, seq[i]][:, :pos[i] + 1], tau)
    h = h + cfg.resid_scale * (O.reshape(N, -1) @ lw["w_o"].T)
    return _mlp_update(cfg, lw, h)


def _loop_input(cfg, W, l: int, h_rows, x_rows):
    """The state a token enters loop l with: h + e_l when loop embeddings are on
    (same page, §3.2 and §4.1: each loop's input adds a learned loop
    embedding) + gamma * x with input injection ("Looped Transformer 教程",
    第三步: every loop also receives the input representation), x being the
    token's state when it entered the loop stack."""
    u = np.asarray(h_rows, F64)
    if "loop_embed" in W:
        u = u + W["loop_embed"][l - 1]
    if getattr(cfg, "inject_scale", 0.0):
        u = u + cfg.inject_scale * np.asarray(x_rows, F64)
    return u


def _prelude(cfg, W, cache, h, seq, pos):
    for x, lw in enumerate(W.get("prelude", [])):
        h = _independent_layer(cfg, lw, cache, x, h, seq, pos)
    return h


def _coda(cfg, W, cache, h, seq, pos):
    P = len(W.get("prelude", []))
    for x, lw in enumerate(W.get("coda", [])):
        h = _independent_layer(cfg, lw, cache, P + x, h, seq, pos)
    return h


# ============================================================================
# one call: prefill (T tokens per sequence) or decode (one token per sequence)
# ============================================================================

class Result:
    def __init__(self, h, logits, trace):
        self.h, self.logits, self.trace = h, logits, trace


def _logits(cfg, W, h_rows):
    x = rmsnorm(h_rows, W["final_norm"], cfg.rms_eps)
    return x @ W["w_out"].T


def _run_lazy(cfg, W, cache: KVCache, h0, seq, pos, tile, forced=None):
    """The lazy-update looped forward over the call's N tokens.

    Loop 1 is dense.  At loops l = 2..K: select the top-n_sel tokens by the
    fp32 key ||h_{l-1} - h_{l-2}||^2 (carried tokens have key 0); unselected
    tokens carry h forward and store a zero residual; selected tokens run the
    block, store a quantised KV residual against the reconstructed chain, and
    update their attention by a correction over the fixed column set C of
    their (query tile, KV head), chosen at the tile's first recomputation as
    the top-c columns by max |delta score|.
    """
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    grp = H // Hkv
    tau = 1.0 / math.sqrt(hd)
    M, K, s_res = cfg.n_layers, cfg.n_loops, cfg.resid_scale
    exact = cfg.resid_bits == 32
    N = h0.shape[0]
    h = _prelude(cfg, W, cache, np.asarray(h0, F64).copy(), seq, pos)
    x_in = h.copy()                     # the state entering the loop stack
    h = _loop_input(cfg, W, 1, h, x_in)
    O = np.zeros((M, N, H, hd))
    lse = np.zeros((M, N, H))
    qlast = np.zeros((M, N, H, hd))
    last = np.ones(N, dtype=np.int64)
    cols = {}
    trace = {"sel": {}, "keys": {}, "cols": {}, "col_keys": {}, "applications": 0}

    # ---- loop 1: every token, full causal attention over the base KV ----
    for j, lw in enumerate(W["layers"]):
        q, k, v = _qkv(cfg, lw, h, pos)
        for i in range(N):
            cache.base_k[j, seq[i], :, pos[i]] = cache.store_kv(k[i])
            cache.base_v[j, seq[i], :, pos[i]] = cache.store_kv(v[i])
        for i in range(N):
            rows = np.arange(pos[i] + 1)
            kk = cache.chain("k", j, 1, seq[i], rows)
            vv = cache.chain("v", j, 1, seq[i], rows)
            O[j, i], lse[j, i] = _attn_full(q[i], kk, vv, tau)
        qlast[j] = q
        h = h + s_res * (O[j].reshape(N, H * hd) @ lw["w_o"].T)
        h = _mlp_update(cfg, lw, h)
        trace["applications"] += 1
    key = np.sum((h - x_in) ** 2, axis=1).astype(F32)
    trace["h"] = {1: h.copy()}

    n_sel = n_select(cfg.rho, N)
    for l in range(2, K + 1):
        trace["keys"][l] = key.copy()
        if forced is not None and l in forced.get("sel", {}):
            S = np.asarray(forced["sel"][l], dtype=np.int64)
        else:
            S = select_top(key, n_sel).astype(np.int64)
        trace["sel"][l] = S.astype(np.int32)
        h_prev = h[S].copy()
        h[S] = _loop_input(cfg, W, l, h[S], x_in[S])
        for j, lw in enumerate(W["layers"]):
            q, k, v = _qkv(cfg, lw, h[S], pos[S])
            # residual rows of loop l: zero for every token of the call ...
            for i in range(N):
                for nm in ("k", "v"):
                    getattr(cache, "res_" + nm)[j, l - 2, seq[i], :, pos[i]] = 0
                    if not exact:
                        getattr(cache, "codes_" + nm)[j, l - 2, seq[i], :, pos[i]] = 0
                        getattr(cache, "scales_" + nm)[j, l - 2, seq[i], :, pos[i]] = 0
            # ... and the quantised residual against the chain for selected ones
            for a, i in enumerate(S):
                b, p = seq[i], pos[i]
                for nm, x in (("k", k[a]), ("v", v[a])):
                    prev = cache.chain(nm, j, l - 1, b, [p])[:, 0]
                    if exact:
                        r = x - prev
                        getattr(cache, "res_" + nm)[j, l - 2, b, :, p] = r
                    else:
                        r = (x.astype(F32) - prev.astype(F32)).astype(F32)
                        codes, scales = quantize_groups(r, cfg.resid_bits, cfg.group_size)
                        getattr(cache, "codes_" + nm)[j, l - 2, b, :, p] = codes
                        getattr(cache, "scales_" + nm)[j, l - 2, b, :, p] = scales
                        getattr(cache, "res_" + nm)[j, l - 2, b, :, p] = dequant_groups(
                            codes, scales, cfg.group_size)
            # column sets for tiles recomputed for the first time
            sel_pos = {int(i): a for a, i in enumerate(S)}
            for t_id in sorted(set(int(tile[i]) for i in S)):
                if (j, t_id) in cols:
                    continue
                members = [int(i) for i in S if tile[i] == t_id]
                b = seq[members[0]]
                maxpos = max(pos[i] for i in members)
                rows = np.arange(maxpos + 1)
                knew = cache.chain("k", j, l, b, rows)
                for gk in range(Hkv):
                    colkey = np.full(maxpos + 1, -np.inf)
                    for i in members:
                        kold = cache.chain("k", j, last[i], b, rows)
                        for hh in range(gk * grp, (gk + 1) * grp):
                            ds = np.abs(tau * (knew[gk] @ q[sel_pos[i], hh]
                                               - kold[gk] @ qlast[j, i, hh]))
                            ds[pos[i] + 1:] = -np.inf
                            colkey = np.maximum(colkey, ds)
                    ck = colkey.astype(F32)
                    n_elig = maxpos + 1
                    C = np.arange(n_elig, dtype=np.int32) if n_elig <= cfg.c_cols \
                        else select_top(ck, cfg.c_cols)
                    cols[(j, t_id, gk)] = C
                    trace["cols"][(j, t_id, gk)] = C
                    trace["col_keys"][(j, t_id, gk)] = ck
                cols[(j, t_id)] = True
            if forced is not None:
                for key_, C in forced.get("cols", {}).items():
                    if key_[0] == j and key_ in cols:
                        cols[key_] = np.asarray(C, dtype=np.int32)
                        trace["cols"][key_] = cols[key_]
            # sparse-column correction of O and lse
            for a, i in enumerate(S):
                b = seq[i]
                for hh in range(H):
                    gk = hh // grp
                    C = cols[(j, int(tile[i]), gk)]
                    C = C[C <= pos[i]]
                    kn = cache.chain("k", j, l, b, C)[gk]
                    vn = cache.chain("v", j, l, b, C)[gk]
                    ko = cache.chain("k", j, last[i], b, C)[gk]
                    vo = cache.chain("v", j, last[i], b, C)[gk]
                    s_new = tau * (kn @ q[a, hh])
                    s_old = tau * (ko @ qlast[j, i, hh])
                    L = lse[j, i, hh]
                    mx = max([L] + list(s_new) + list(s_old))
                    e_new, e_old = np.exp(s_new - mx), np.exp(s_old - mx)
                    z = math.exp(L - mx) - e_old.sum() + e_new.sum()
                    assert z > 0, "corrected softmax denominator must stay positive"
                    num = math.exp(L - mx) * O[j, i, hh] - e_old @ vo + e_new @ vn
                    O[j, i, hh] = num / z
                    lse[j, i, hh] = mx + math.log(z)
                qlast[j, i] = q[a]
            hs = h[S] + s_res * (O[j, S].reshape(len(S), H * hd) @ lw["w_o"].T)
            h[S] = _mlp_update(cfg, lw, hs)
            trace["applications"] += 1
        last[S] = l
        key = np.zeros(N, F32)
        key[S] = np.sum((h[S] - h_prev) ** 2, axis=1).astype(F32)
        trace["h"][l] = h.copy()
    trace["O"], trace["lse"] = O, lse
    h = _coda(cfg, W, cache, h, seq, pos)
    trace["independent"] = len(W.get("prelude", [])) + len(W.get("coda", []))
    return h, trace


def _run_dense(cfg, W, cache: KVCache, h0, seq, pos):
    """Dense looped forward with a per-loop KV cache: h_l = block(h_{l-1}), l = 1..K.

    "Looped Transformer 教程", 第一步 and 第四步 (per_loop KV); "循环Transformer
    解析", forward_looped.  Every loop recomputes every token and attends over
    that loop's own KV.
    """
    H, hd = cfg.n_heads, cfg.head_dim
    tau = 1.0 / math.sqrt(hd)
    N = h0.shape[0]
    h = _prelude(cfg, W, cache, np.asarray(h0, F64).copy(), seq, pos)
    x_in = h.copy()
    apps = 0
    for l in range(1, cfg.n_loops + 1):
        h = _loop_input(cfg, W, l, h, x_in)
        for j, lw in enumerate(W["layers"]):
            q, k, v = _qkv(cfg, lw, h, pos)
            sl = cache.slot(l)
            for i in range(N):
                cache.kv_k[j, sl, seq[i], :, pos[i]] = cache.store_kv(k[i])
                cache.kv_v[j, sl, seq[i], :, pos[i]] = cache.store_kv(v[i])
            O = np.zeros((N, H, hd))
            for i in range(N):
                kk = cache.kv_k[j, sl, seq[i]][:, :pos[i] + 1]
                vv = cache.kv_v[j, sl, seq[i]][:, :pos[i] + 1]
                O[i], _ = _attn_full(q[i], kk, vv, tau)
            h = h + cfg.resid_scale * (O.reshape(N, H * hd) @ lw["w_o"].T)
            h = _mlp_update(cfg, lw, h)
            apps += 1
    h = _coda(cfg, W, cache, h, seq, pos)
    return h, {"applications": apps, "independent": len(W.get("prelude", [])) + len(W.get("coda", []))}


def _call(cfg, W, cache, h0, seq, pos, tile, forced):
    if cache.dense:
        return _run_dense(cfg, W, cache, h0, seq, pos)
    return _run_lazy(cfg, W, cache, h0, seq, pos, tile, forced)


def prefill(cfg, W, cache: KVCache, h0: np.ndarray, B: int, T: int, forced=None) -> Result:
    """Prefill a chunk of T tokens onto each of sequences 0..B-1; h0 is [B*T, d]
    (sequence-major).  Token t of sequence b sits at position lens[b] + t, after
    what the sequence already holds (nothing for a fresh prompt; a later chunk
    of the prompt, or decoded tokens, otherwise) and attends to every earlier
    position.  Query tiles are q_tile consecutive tokens of one sequence's
    chunk, counted from the chunk's first token; the token ranking pools all
    B*T tokens by flat index b*T + t.  Logits are for the last position of each
    sequence.
    """
    start = cache.lens[:B].copy()
    assert np.all(start + T <= cache.tmax), "the chunk does not fit the cache"
    seq = np.repeat(np.arange(B), T)
    rel = np.tile(np.arange(T), B)
    pos = start[seq] + rel
    tile = seq * ((T + cfg.q_tile - 1) // cfg.q_tile) + rel // cfg.q_tile
    h, trace = _call(cfg, W, cache, h0, seq, pos, tile, forced)
    cache.lens[:B] = start + T
    last_rows = np.arange(B) * T + (T - 1)
    return Result(h, _logits(cfg, W, h[last_rows]), trace)


def decode_step(cfg, W, cache: KVCache, h0: np.ndarray, forced=None) -> Result:
    """Append one token to each of the B sequences; h0 is [B, d].

    Each new token is its own query tile; the token ranking pools the B new
    tokens of the call.
    """
    B = h0.shape[0]
    seq = np.arange(B)
    pos = cache.lens[:B].copy()
    assert np.all(pos < cache.tmax)
    h, trace = _call(cfg, W, cache, h0, seq, pos, seq.copy(), forced)
    cache.lens[:B] += 1
    return Result(h, _logits(cfg, W, h), trace)
