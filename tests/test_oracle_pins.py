"""Pins of the CPU oracle against definitions other than itself (no GPU).

Each test ties one oracle function to an independent statement of what it
must compute: brute force on small inputs, a library routine for a special
case (torch bfloat16 casts, torch scaled-dot-product attention, complex
rotation), closed-form invariants, or the dense looped forward that the lazy
method must reduce to when nothing is skipped.
"""
import math

import numpy as np
import pytest
import torch

from cross_loop_sparsity_b200 import synth
from oracle import flashloop_oracle as orc

F32 = np.float32


# ----------------------------------------------------------------------------
# selection: top-k by (fp32 bit pattern desc, index asc)
# ----------------------------------------------------------------------------

def _select_by_counting(keys, k):
    """Element i is selected iff fewer than k elements beat it (brute force)."""
    bits = keys.astype(F32).view(np.uint32).astype(np.int64)
    n = len(keys)
    out = []
    for i in range(n):
        beats = sum(1 for j in range(n) if bits[j] > bits[i] or (bits[j] == bits[i] and j < i))
        if beats < k:
            out.append(i)
    return np.array(out, dtype=np.int32)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_matches_counting_every_k(seed):
    for n in (1, 2, 7, 33, 64):
        keys = synth.make_keys(seed * 100 + n, n, "ties")
        for k in range(0, n + 1):
            assert np.array_equal(orc.select_top(keys, k), _select_by_counting(keys, k))


def test_select_large_ties_matches_python_sort():
    keys = synth.make_keys(7, 70000, "ties")
    bits = keys.view(np.uint32)
    order = sorted(range(len(keys)), key=lambda i: (-int(bits[i]), i))
    for k in (1, 10, 4097, 35000, 70000):
        assert np.array_equal(orc.select_top(keys, k), np.sort(np.array(order[:k], dtype=np.int32)))


def test_select_nan_inf_zero_order():
    keys = np.array([0.0, np.inf, np.nan, 1.0, 0.0, np.inf], dtype=F32)
    assert list(orc.select_top(keys, 1)) == [2]          # NaN bit pattern above +inf
    assert list(orc.select_top(keys, 3)) == [1, 2, 5]
    assert list(orc.select_top(keys, 5)) == [0, 1, 2, 3, 5]   # zero tie -> lower index


def test_n_select_rule():
    assert orc.n_select(0.25, 128) == 32
    assert orc.n_select(0.10, 8) == 1
    assert orc.n_select(0.15, 16384) == 2458
    assert orc.n_select(0.05, 4) == 1
    assert orc.n_select(0.05, 1) == 1
    assert orc.n_select(1.0, 5) == 5
    assert orc.n_select(1e-9, 5) == 1
    assert orc.n_select(0.5, 0) == 0


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def test_bf16_round_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100000).astype(F32) * F32(10.0) ** rng.integers(-30, 30, 100000),
                        np.array([0.0, -0.0, 1.0, 3.0e38, 1e-40, -2.5], F32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = orc.bf16_round(x)
    assert np.array_equal(got, ref)


def _fp16_table():
    allv = np.arange(0, 0x7C01, dtype=np.uint16).view(np.float16).astype(np.float64)  # +0 .. +inf
    return np.sort(allv)


def test_fp16_round_up_brute_force():
    table = _fp16_table()
    rng = np.random.default_rng(4)
    xs = [rng.uniform(0, 1, 20000), 10.0 ** rng.uniform(-9, 4.8, 20000),
          table[1:-1][rng.integers(0, len(table) - 2, 5000)],                   # exact fp16 values
          (table[1:-2] + table[2:-1])[rng.integers(0, len(table) - 3, 5000)] / 2.0]  # midpoints
    x = np.concatenate(xs).astype(F32)
    x = np.concatenate([x, np.array([0.0, 65504.0, 65504.5, 70000.0, 5.9604645e-08, 1e-12], F32)])
    got = orc.fp16_round_up(x).astype(np.float64)
    want = table[np.searchsorted(table, x.astype(np.float64), side="left")]
    assert np.array_equal(got, want)


def test_fp16_round_up_overflow_is_inf():
    assert np.isinf(orc.fp16_round_up(np.array([65520.0], F32))[0])


# ----------------------------------------------------------------------------
# quantiser
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("bits,g", [(4, 32), (4, 64), (4, 128), (2, 64)])
def test_quantizer_brute_force_and_bounds(bits, g):
    qm = (1 << (bits - 1)) - 1
    r = synth.make_residuals(11 + bits + g, 300, 128)
    codes, s16 = orc.quantize_groups(r, bits, g)
    table = _fp16_table()
    rg = r.reshape(300, 128 // g, g)
    amax = np.abs(rg).max(axis=-1)
    q32 = (amax / F32(qm)).astype(F32)
    # scale: the smallest fp16 value >= fp32(absmax/qmax), by table search
    want_s = table[np.searchsorted(table, q32.astype(np.float64), side="left")]
    assert np.array_equal(s16.astype(np.float64), want_s)
    s = s16.astype(F32)
    cg = codes.reshape(300, 128 // g, g).astype(np.int64)
    assert np.all(np.abs(cg) <= qm)
    # code: the integer in [-qmax, qmax] nearest the fp32 quotient, ties to even (brute force)
    for row in range(0, 300, 7):
        for gi in range(128 // g):
            if s[row, gi] == 0:
                assert np.all(cg[row, gi] == 0)
                continue
            quot = (rg[row, gi] / s[row, gi]).astype(F32).astype(np.float64)
            for e in range(g):
                best = min(range(-qm, qm + 1), key=lambda c: (abs(quot[e] - c), c % 2, c))
                assert cg[row, gi, e] == best
    # error bound |r - code*s| <= s/2 * (1 + 2^-20), in exact (fp64) arithmetic
    err = np.abs(rg.astype(np.float64) - cg * s[..., None].astype(np.float64))
    assert np.all(err <= s[..., None].astype(np.float64) / 2 * (1 + 2.0 ** -20))


def test_quantizer_zero_group_and_exact_grid():
    r = np.zeros((2, 64), F32)
    r[1, :32] = np.arange(-7, 9, dtype=F32).repeat(2)[:32] * F32(0.5)   # multiples of 0.5 up to 4
    codes, s = orc.quantize_groups(r, 4, 32)
    assert np.all(codes[0] == 0) and np.all(s[0] == 0)
    assert s[1, 0] == np.float16(4.0 / 7.0) or s[1, 0] >= np.float32(4.0 / 7.0)
    deq = orc.dequant_groups(codes, s, 32)
    assert np.all(np.abs(deq - r) <= s.astype(F32).repeat(32, axis=-1) / 2 * (1 + 2 ** -20))


def test_pack_layout_and_roundtrip():
    assert orc.pack_codes(np.array([1, -1, 7, -7], np.int8), 4).tolist() == [0xF1, 0x97]
    assert orc.pack_codes(np.array([1, -1, 0, 1], np.int8), 2).tolist() == [0x4D]
    rng = np.random.default_rng(5)
    for bits in (4, 2):
        qm = (1 << (bits - 1)) - 1
        c = rng.integers(-qm, qm + 1, size=(17, 128)).astype(np.int8)
        p = orc.pack_codes(c, bits)
        assert p.shape == (17, 128 * bits // 8)
        assert np.array_equal(orc.unpack_codes(p, bits), c)


# ----------------------------------------------------------------------------
# layer pieces
# ----------------------------------------------------------------------------

def test_rope_matches_complex_rotation_and_relative_position():
    rng = np.random.default_rng(6)
    hd, theta = 64, 10000.0
    x = rng.standard_normal((5, 3, hd))
    pos = np.array([0, 1, 17, 4095, 65536])
    got = orc.apply_rope(x, pos, theta)
    z = x[..., :hd // 2] + 1j * x[..., hd // 2:]
    freqs = theta ** (-np.arange(0, hd, 2) / hd)
    z = z * np.exp(1j * pos[:, None, None] * freqs[None, None, :])
    want = np.concatenate([z.real, z.imag], axis=-1)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    # <rope(q, p1), rope(k, p2)> depends on p1 - p2 only
    q, k = rng.standard_normal((1, 1, hd)), rng.standard_normal((1, 1, hd))
    a = np.sum(orc.apply_rope(q, np.array([10]), theta) * orc.apply_rope(k, np.array([3]), theta))
    b = np.sum(orc.apply_rope(q, np.array([107]), theta) * orc.apply_rope(k, np.array([100]), theta))
    assert abs(a - b) < 1e-10


def _torch_block_forward(cfg, W, h):
    """A plain pre-norm Llama-style layer stack written with torch library ops (fp64)."""
    op = lambda t: t
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    T = h.shape[0]
    x = torch.from_numpy(np.asarray(h, np.float64))
    freqs = cfg.rope_theta ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    rot = torch.polar(torch.ones(T, hd // 2, dtype=torch.float64),
                      torch.arange(T, dtype=torch.float64)[:, None] * freqs[None, :])

    def rope(t):   # t [T, heads, hd] in rotate-half pairing
        z = torch.complex(t[..., :hd // 2], t[..., hd // 2:]) * rot[:, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    for lw in W["layers"]:
        a = op(torch.nn.functional.rms_norm(x, (cfg.d_model,), torch.from_numpy(lw["attn_norm"]), cfg.rms_eps))
        y = a @ torch.from_numpy(lw["w_qkv"]).T
        q = rope(y[:, :H * hd].reshape(T, H, hd))
        k = rope(y[:, H * hd:(H + Hkv) * hd].reshape(T, Hkv, hd))
        v = y[:, (H + Hkv) * hd:].reshape(T, Hkv, hd)
        o = torch.nn.functional.scaled_dot_product_attention(
            q.transpose(0, 1)[None], k.transpose(0, 1)[None], v.transpose(0, 1)[None],
            is_causal=True, enable_gqa=True)[0].transpose(0, 1).reshape(T, H * hd)
        x = x + cfg.resid_scale * (op(o) @ torch.from_numpy(lw["w_o"]).T)
        m = op(torch.nn.functional.rms_norm(x, (cfg.d_model,), torch.from_numpy(lw["mlp_norm"]), cfg.rms_eps))
        act = op(torch.nn.functional.silu(m @ torch.from_numpy(lw["w_gate"]).T) * (m @ torch.from_numpy(lw["w_up"]).T))
        x = x + cfg.resid_scale * (act @ torch.from_numpy(lw["w_down"]).T)
    return x.numpy()


def _tiny_cfg(**kw):
    base = dict(d_model=32, n_heads=4, n_kv_heads=2, head_dim=8, ffn_dim=48, n_layers=2, n_loops=3,
                rho=0.25, c_cols=4, resid_bits=4, group_size=8, q_tile=8, vocab=40, sigma=0.2,
                seed=9, mode="prefill", batch=1, seq_len=16)
    base.update(kw)
    return synth.LoopConfig("tiny", **base)


def _weights(cfg):
    w = synth.make_weights(cfg)
    return orc.prepare_weights(w), w["rng"]


@pytest.mark.parametrize("K", [1, 3])
def test_dense_looped_forward_is_k_plain_blocks(K):
    cfg = _tiny_cfg(n_loops=K, resid_bits=16)
    W, rng = _weights(cfg)
    h0 = synth.make_h0(cfg, rng, cfg.seq_len)
    cache = orc.KVCache(cfg, 1, cfg.seq_len, kv_exact=True)
    res = orc.prefill(cfg, W, cache, h0, 1, cfg.seq_len)
    want = np.asarray(h0, np.float64)
    for _ in range(K):
        want = _torch_block_forward(cfg, W, want)
    np.testing.assert_allclose(res.h, want, rtol=0, atol=1e-11 * np.abs(want).max())
    assert res.trace["applications"] == cfg.n_layers * K
    x = want[-1] / np.sqrt(np.mean(want[-1] ** 2) + cfg.rms_eps)
    np.testing.assert_allclose(res.logits[0], W["w_out"] @ x, atol=1e-11)


def test_block_applications_golden():
    rows = [tuple(int(v) for v in ln.split()) for ln in open(
        __file__.replace("test_oracle_pins.py", "golden/block_applications.txt"))
        if ln.strip() and not ln.startswith("#")]
    for M, K, apps in rows:
        cfg = _tiny_cfg(d_model=16, n_heads=2, n_kv_heads=1, head_dim=8, ffn_dim=16, n_layers=M,
                        n_loops=K, seq_len=4, q_tile=4, rho=0.5, c_cols=2, group_size=8)
        W, rng = _weights(cfg)
        h0 = synth.make_h0(cfg, rng, 4)
        res = orc.prefill(cfg, W, orc.KVCache(cfg, 1, 4), h0, 1, 4)
        assert res.trace["applications"] == apps


# ----------------------------------------------------------------------------
# dense limit: rho = 1, every column, exact residual  ==  dense looped forward
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("B,T,qt", [(1, 16, 8), (2, 12, 16)])
def test_lazy_prefill_dense_limit(B, T, qt):
    cfg = _tiny_cfg(rho=1.0, c_cols=10 ** 6, resid_bits=32, q_tile=qt, seq_len=T, batch=B, n_loops=4)
    W, rng = _weights(cfg)
    h0 = synth.make_h0(cfg, rng, B * T)
    lazy = orc.prefill(cfg, W, orc.KVCache(cfg, B, T, kv_exact=True), h0, B, T)
    dcfg = cfg.with_(resid_bits=16)
    dense = orc.prefill(dcfg, W, orc.KVCache(dcfg, B, T, kv_exact=True), h0, B, T)
    scale = np.sqrt(np.mean(dense.h ** 2))
    assert np.max(np.abs(lazy.h - dense.h)) <= 1e-9 * scale
    np.testing.assert_allclose(lazy.logits, dense.logits, atol=1e-9 * np.abs(dense.logits).max())


def test_lazy_decode_dense_limit():
    cfg = _tiny_cfg(rho=1.0, c_cols=10 ** 6, resid_bits=32, mode="decode", batch=3, ctx_len=9, seq_len=0,
                    n_loops=4)
    W, rng = _weights(cfg)
    lens = np.array([9, 5, 1])
    tmax = 10
    M, K, Hkv, hd = cfg.n_layers, cfg.n_loops, cfg.n_kv_heads, cfg.head_dim
    lazy_c = orc.KVCache(cfg, 3, tmax, kv_exact=True)
    dcfg = cfg.with_(resid_bits=16)
    dense_c = orc.KVCache(dcfg, 3, tmax, kv_exact=True)
    base_k = rng.standard_normal((M, 3, Hkv, tmax, hd))
    base_v = rng.standard_normal((M, 3, Hkv, tmax, hd))
    res_k = rng.standard_normal((M, K - 1, 3, Hkv, tmax, hd)) * 0.1
    res_v = rng.standard_normal((M, K - 1, 3, Hkv, tmax, hd)) * 0.1
    for b in range(3):
        base_k[:, b, :, lens[b]:] = base_v[:, b, :, lens[b]:] = 0
        res_k[:, :, b, :, lens[b]:] = res_v[:, :, b, :, lens[b]:] = 0
    lazy_c.base_k[:], lazy_c.base_v[:], lazy_c.res_k[:], lazy_c.res_v[:] = base_k, base_v, res_k, res_v
    # dense per-loop context KV = base + sum of residuals up to that loop (independent cumulative sum)
    dense_c.kv_k[:, 0], dense_c.kv_v[:, 0] = base_k, base_v
    dense_c.kv_k[:, 1:] = base_k[:, None] + np.cumsum(res_k, axis=1)
    dense_c.kv_v[:, 1:] = base_v[:, None] + np.cumsum(res_v, axis=1)
    lazy_c.lens[:] = lens
    dense_c.lens[:] = lens
    h0 = synth.make_h0(cfg, rng, 3)
    a = orc.decode_step(cfg, W, lazy_c, h0)
    b = orc.decode_step(dcfg, W, dense_c, h0)
    assert np.max(np.abs(a.h - b.h)) <= 1e-9 * np.sqrt(np.mean(b.h ** 2))
    np.testing.assert_allclose(a.logits, b.logits, atol=1e-9 * np.abs(b.logits).max())


# ----------------------------------------------------------------------------
# materialised brute force of the lazy path (independent restatement)
# ----------------------------------------------------------------------------

def _brute_lazy_prefill(cfg, W, h0, T, quant):
    """Tiny lazy prefill (B = 1) holding each query's score vector and value rows explicitly.

    Every query keeps, per layer and head, the score and the value row of every
    causal column as last written; its attention output is the softmax of that
    vector.  Recomputing a query overwrites the entries of its tile's column set
    with the new loop's scores and values.  The column set is the top-c columns
    by max |new score - stored score|, chosen once per tile.  Written without
    the running (O, lse) form that the oracle uses.
    """
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    grp, tau, M = H // Hkv, 1 / math.sqrt(hd), cfg.n_layers
    pos = np.arange(T)
    tiles = pos // cfg.q_tile
    h = np.asarray(h0, np.float64).copy()
    # chain[j] = list over loops of (K, V) [Hkv, T, hd] reconstructed values
    chain = [[] for _ in range(M)]
    scores = np.zeros((M, T, H, T))
    values = np.zeros((M, T, H, T, hd))
    colset = {}

    def out_of(j, i):
        s = scores[j, i][:, :i + 1]
        w = np.exp(s - s.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
        return np.einsum("ht,htd->hd", w, values[j, i][:, :i + 1])

    def layer_tail(lw, hs, o):
        hs = hs + cfg.resid_scale * (o.reshape(len(hs), H * hd) @ lw["w_o"].T)
        return orc._mlp_update(cfg, lw, hs)

    for j, lw in enumerate(W["layers"]):
        q, k, v = orc._qkv(cfg, lw, h, pos)
        kb, vb = orc.bf16_round(k).transpose(1, 0, 2), orc.bf16_round(v).transpose(1, 0, 2)
        chain[j].append((kb, vb))
        for i in range(T):
            for hh in range(H):
                scores[j, i, hh, :i + 1] = tau * (kb[hh // grp, :i + 1] @ q[i, hh])
                values[j, i, hh, :i + 1] = vb[hh // grp, :i + 1]
        o = np.stack([out_of(j, i) for i in range(T)])
        h = layer_tail(lw, h, o)
    key = np.sum((h - h0) ** 2, axis=1).astype(F32)
    n_sel = max(1, min(T, math.ceil(cfg.rho * T - 1e-9)))
    sels = {}
    for l in range(2, cfg.n_loops + 1):
        bits = key.view(np.uint32)
        S = np.array(sorted(sorted(range(T), key=lambda t: (-int(bits[t]), t))[:n_sel]))
        sels[l] = S
        hprev = h[S].copy()
        for j, lw in enumerate(W["layers"]):
            q, k, v = orc._qkv(cfg, lw, h[S], pos[S])
            kp, vp = chain[j][-1]
            kn, vn = kp.copy(), vp.copy()
            for a, t in enumerate(S):
                for arr, new, prev in ((kn, k[a], kp), (vn, v[a], vp)):
                    r = (new.astype(F32) - prev[:, t].astype(F32)).astype(F32)
                    c, s = quant(r)
                    arr[:, t] = (prev[:, t].astype(F32) + orc.dequant_groups(c, s, cfg.group_size)).astype(F32)
            chain[j].append((kn, vn))
            for tl in sorted(set(tiles[S])):
                if (j, tl) in colset:
                    continue
                mem = [a for a, t in enumerate(S) if tiles[t] == tl]
                mp = max(S[a] for a in mem)
                for gk in range(Hkv):
                    ck = np.full(mp + 1, -np.inf)
                    for a in mem:
                        t = S[a]
                        for hh in range(gk * grp, (gk + 1) * grp):
                            d = np.abs(tau * (kn[gk, :t + 1] @ q[a, hh]) - scores[j, t, hh, :t + 1])
                            ck[:t + 1] = np.maximum(ck[:t + 1], d)
                    ck = ck.astype(F32)
                    if mp + 1 <= cfg.c_cols:
                        colset[(j, tl, gk)] = np.arange(mp + 1)
                    else:
                        b2 = ck.view(np.uint32)
                        colset[(j, tl, gk)] = np.array(sorted(sorted(range(mp + 1),
                                                                     key=lambda c: (-int(b2[c]), c))[:cfg.c_cols]))
                colset[(j, tl)] = True
            for a, t in enumerate(S):
                for hh in range(H):
                    C = colset[(j, tiles[t], hh // grp)]
                    C = C[C <= t]
                    scores[j, t, hh, C] = tau * (kn[hh // grp, C] @ q[a, hh])
                    values[j, t, hh, C] = vn[hh // grp, C]
            o = np.stack([out_of(j, t) for t in S])
            h[S] = layer_tail(lw, h[S], o)
        key = np.zeros(T, F32)
        key[S] = np.sum((h[S] - hprev) ** 2, axis=1).astype(F32)
    return h, sels, colset


@pytest.mark.parametrize("seed,T,qt,c", [(21, 16, 8, 3), (22, 20, 16, 5), (23, 12, 4, 2)])
def test_lazy_prefill_matches_materialised_brute_force(seed, T, qt, c):
    cfg = _tiny_cfg(seed=seed, seq_len=T, q_tile=qt, c_cols=c, rho=0.3, n_loops=4)
    W, rng = _weights(cfg)
    h0 = synth.make_h0(cfg, rng, T)
    res = orc.prefill(cfg, W, orc.KVCache(cfg, 1, T), h0, 1, T)
    quant = lambda r: orc.quantize_groups(r, cfg.resid_bits, cfg.group_size)
    bh, bsel, bcols = _brute_lazy_prefill(cfg, W, h0, T, quant)
    for l, S in bsel.items():
        assert np.array_equal(res.trace["sel"][l], S)
    for key_, C in res.trace["cols"].items():
        assert np.array_equal(C, bcols[key_])
    assert np.max(np.abs(res.h - bh)) <= 1e-9 * np.sqrt(np.mean(bh ** 2))


def _brute_lazy_call(cfg, W, h0, seq, pos, tile, ctx, quant):
    """A lazy call over N tokens of B sequences, each query's attention held as an
    explicit score vector and value rows over its causal columns.

    seq / pos / tile: per call token (flat index = position in the call, the
    pooled ranking's tie-break).  ctx: None (empty sequences, prefill) or a
    synthetic context (bf16 base bits, int8 codes, fp16 scales of loops 2..K)
    whose rows before each sequence's length hold that sequence's history.
    Every KV level of every column is kept materialised: level m of a context
    column is its base plus the dequantised residuals of loops 2..m, added one at
    a time in fp32; a call token's level m is its level m-1 plus the residual it
    stored at loop m (zero when carried).  A recomputed query overwrites the
    entries of its tile's column set with the new loop's scores and values; the
    set is the top-c columns by max |new score - stored score| over the tile's
    selected queries and the group's heads, chosen once per tile.  Written
    without the running (O, lse) form and without the oracle's cache class.
    Returns h, selections, column sets and the residual codes stored per
    (layer, loop, token, K/V).
    """
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    grp, tau, M, K = H // Hkv, 1 / math.sqrt(hd), cfg.n_layers, cfg.n_loops
    N = len(seq)
    B = int(max(seq)) + 1
    tlen = [int(max(pos[i] for i in range(N) if seq[i] == b)) + 1 for b in range(B)]
    # lev[j][b][m]: (K, V) of level m = 1..K, [Hkv, tlen_b, hd] float32
    lev = [[[None] + [(np.zeros((Hkv, tlen[b], hd), F32), np.zeros((Hkv, tlen[b], hd), F32)) for _ in range(K)]
            for b in range(B)] for _ in range(M)]
    if ctx is not None:
        f32 = lambda bits: (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(F32)
        g = cfg.group_size
        for j in range(M):
            for b in range(B):
                n = int(ctx["lens"][b])
                kb, vb = f32(ctx["base_k"][j, b][:, :n]), f32(ctx["base_v"][j, b][:, :n])
                lev[j][b][1][0][:, :n], lev[j][b][1][1][:, :n] = kb, vb
                for m in range(2, K + 1):
                    for w, nm in enumerate(("k", "v")):
                        codes = ctx["codes_" + nm][j, m - 2, b][:, :n].astype(F32)
                        sc = np.repeat(ctx["scales_" + nm][j, m - 2, b][:, :n].astype(F32), g, axis=-1)
                        lev[j][b][m][w][:, :n] = (lev[j][b][m - 1][w][:, :n] + codes * sc).astype(F32)
    h = np.asarray(h0, np.float64).copy()
    scores = [[np.zeros((H, pos[i] + 1)) for i in range(N)] for _ in range(M)]
    values = [[np.zeros((H, pos[i] + 1, hd)) for i in range(N)] for _ in range(M)]
    stored = {}

    def out_of(j, i):
        s = scores[j][i]
        w = np.exp(s - s.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
        return np.einsum("ht,htd->hd", w, values[j][i])

    def layer_tail(lw, hs, o):
        hs = hs + cfg.resid_scale * (o.reshape(len(hs), H * hd) @ lw["w_o"].T)
        return orc._mlp_update(cfg, lw, hs)

    for j, lw in enumerate(W["layers"]):
        q, k, v = orc._qkv(cfg, lw, h, pos)
        for i in range(N):
            b, p = seq[i], pos[i]
            for m in range(1, K + 1):      # a new token's later levels start equal to its base
                lev[j][b][m][0][:, p] = orc.bf16_round(k[i])
                lev[j][b][m][1][:, p] = orc.bf16_round(v[i])
        for i in range(N):
            b, p = seq[i], pos[i]
            for hh in range(H):
                scores[j][i][hh] = tau * (lev[j][b][1][0][hh // grp, :p + 1].astype(np.float64) @ q[i, hh])
                values[j][i][hh] = lev[j][b][1][1][hh // grp, :p + 1]
        o = np.stack([out_of(j, i) for i in range(N)])
        h = layer_tail(lw, h, o)
    key = np.sum((h - h0) ** 2, axis=1).astype(F32)
    n_sel = max(1, min(N, math.ceil(cfg.rho * N - 1e-9)))
    sels, colset = {}, {}
    for l in range(2, K + 1):
        kbits = key.view(np.uint32)
        S = np.array(sorted(sorted(range(N), key=lambda t: (-int(kbits[t]), t))[:n_sel]))
        sels[l] = S
        hprev = h[S].copy()
        for j, lw in enumerate(W["layers"]):
            q, k, v = orc._qkv(cfg, lw, h[S], pos[S])
            for i in range(N):          # carried: level l = level l-1 (a zero residual)
                b, p = seq[i], pos[i]
                for w in (0, 1):
                    lev[j][b][l][w][:, p] = lev[j][b][l - 1][w][:, p]
            for a, i in enumerate(S):
                b, p = seq[i], pos[i]
                for w, new in ((0, k[a]), (1, v[a])):
                    prev = lev[j][b][l - 1][w][:, p]
                    r = (new.astype(F32) - prev).astype(F32)
                    c, s = quant(r)
                    stored[(j, l, int(i), w)] = (c, s)
                    lev[j][b][l][w][:, p] = (prev + orc.dequant_groups(c, s, cfg.group_size)).astype(F32)
            for tl in sorted(set(int(tile[i]) for i in S)):
                if (j, tl) in colset:
                    continue
                mem = [a for a, i in enumerate(S) if tile[i] == tl]
                b = seq[S[mem[0]]]
                mp = max(pos[S[a]] for a in mem)
                kn = lev[j][b][l][0].astype(np.float64)
                for gk in range(Hkv):
                    ck = np.full(mp + 1, -np.inf)
                    for a in mem:
                        i, p = S[a], pos[S[a]]
                        for hh in range(gk * grp, (gk + 1) * grp):
                            d = np.abs(tau * (kn[gk, :p + 1] @ q[a, hh]) - scores[j][i][hh])
                            ck[:p + 1] = np.maximum(ck[:p + 1], d)
                    ck = ck.astype(F32)
                    if mp + 1 <= cfg.c_cols:
                        colset[(j, tl, gk)] = np.arange(mp + 1)
                    else:
                        b2 = ck.view(np.uint32)
                        colset[(j, tl, gk)] = np.array(sorted(sorted(range(mp + 1),
                                                                     key=lambda c: (-int(b2[c]), c))[:cfg.c_cols]))
                colset[(j, tl)] = True
            for a, i in enumerate(S):
                b, p = seq[i], pos[i]
                for hh in range(H):
                    C = colset[(j, int(tile[i]), hh // grp)]
                    C = C[C <= p]
                    scores[j][i][hh, C] = tau * (lev[j][b][l][0][hh // grp, C].astype(np.float64) @ q[a, hh])
                    values[j][i][hh, C] = lev[j][b][l][1][hh // grp, C]
            o = np.stack([out_of(j, i) for i in S])
            h[S] = layer_tail(lw, h[S], o)
        key = np.zeros(N, F32)
        key[S] = np.sum((h[S] - hprev) ** 2, axis=1).astype(F32)
    return h, sels, {k_: v_ for k_, v_ in colset.items() if len(k_) == 3}, stored


def _compare_with_brute(cfg, res, cache, seq, pos, bh, bsel, bcols, bstored):
    assert set(res.trace["sel"]) == set(bsel)
    for l, S in bsel.items():
        assert np.array_equal(res.trace["sel"][l], S), l
    assert set(res.trace["cols"]) == set(bcols)
    for key_, C in res.trace["cols"].items():
        assert np.array_equal(C, bcols[key_]), key_
    for (j, l, i, w), (c, s) in bstored.items():
        nm = "k" if w == 0 else "v"
        assert np.array_equal(getattr(cache, "codes_" + nm)[j, l - 2, seq[i], :, pos[i]], c)
        assert np.array_equal(getattr(cache, "scales_" + nm)[j, l - 2, seq[i], :, pos[i]].view(np.uint16),
                              np.asarray(s, np.float16).view(np.uint16))
    assert np.max(np.abs(res.h - bh)) <= 1e-9 * np.sqrt(np.mean(bh ** 2))


@pytest.mark.parametrize("seed,bits,lens,rho,c", [(61, 4, [9, 4, 13], 0.5, 3), (62, 2, [6, 11, 1, 8], 0.5, 4),
                                                  (63, 4, [12, 12], 1.0, 5), (64, 2, [3, 15, 7], 0.3, 2)])
def test_lazy_decode_over_residual_context_matches_materialised_brute_force(seed, bits, lens, rho, c):
    """Decode over a context whose tokens already hold residual levels 2..K,
    pooled over ragged sequences, rho < 1 and c below the context length."""
    cfg = _tiny_cfg(seed=seed, rho=rho, c_cols=c, resid_bits=bits, mode="decode", batch=len(lens), seq_len=0,
                    ctx_len=max(lens), n_loops=4)
    W, rng = _weights(cfg)
    ctx = synth.make_context(cfg, rng, lens)
    tmax = max(lens) + 1
    cache = orc.KVCache.from_context(cfg, ctx, tmax)
    h0 = synth.make_h0(cfg, rng, len(lens))
    res = orc.decode_step(cfg, W, cache, h0)
    B = len(lens)
    seq, pos = np.arange(B), np.asarray(lens)
    quant = lambda r: orc.quantize_groups(r, cfg.resid_bits, cfg.group_size)
    bh, bsel, bcols, bstored = _brute_lazy_call(cfg, W, h0, seq, pos, seq.copy(), ctx, quant)
    assert len(bstored) == cfg.n_layers * (cfg.n_loops - 1) * 2 * orc.n_select(rho, B)
    _compare_with_brute(cfg, res, cache, seq, pos, bh, bsel, bcols, bstored)


def test_lazy_decode_pooled_ties_go_to_the_lower_sequence():
    """Identical sequences (same context, same input row) give bit-identical
    change keys, so the pooled ranking is decided by the tie-break alone: the
    lower flat index (sequence) wins, in the oracle and in the brute force."""
    B, n = 4, 9
    cfg = _tiny_cfg(seed=65, rho=0.5, c_cols=3, resid_bits=4, mode="decode", batch=B, seq_len=0, ctx_len=n,
                    n_loops=3)
    W, rng = _weights(cfg)
    ctx = synth.make_context(cfg, rng, [n] * B)
    for name in ("base_k", "base_v"):
        ctx[name][:, 1:] = ctx[name][:, :1]
    for name in ("codes_k", "codes_v", "scales_k", "scales_v"):
        ctx[name][:, :, 1:] = ctx[name][:, :, :1]
    h0 = np.repeat(synth.make_h0(cfg, rng, 1), B, axis=0)
    cache = orc.KVCache.from_context(cfg, ctx, n + 1)
    res = orc.decode_step(cfg, W, cache, h0)
    seq, pos = np.arange(B), np.full(B, n)
    quant = lambda r: orc.quantize_groups(r, cfg.resid_bits, cfg.group_size)
    bh, bsel, bcols, bstored = _brute_lazy_call(cfg, W, h0, seq, pos, seq.copy(), ctx, quant)
    assert len(set(res.trace["keys"][2].tolist())) == 1           # every key ties
    assert np.array_equal(bsel[2], [0, 1])
    _compare_with_brute(cfg, res, cache, seq, pos, bh, bsel, bcols, bstored)


@pytest.mark.parametrize("seed,B,T,qt,c,bits", [(71, 2, 10, 4, 2, 4), (72, 3, 7, 8, 3, 2)])
def test_lazy_prefill_pooled_sequences_match_materialised_brute_force(seed, B, T, qt, c, bits):
    """Prefill of several sequences: the ranking pools all B*T tokens by flat
    index b*T + t and query tiles never span two sequences."""
    cfg = _tiny_cfg(seed=seed, seq_len=T, batch=B, q_tile=qt, c_cols=c, rho=0.3, n_loops=4, resid_bits=bits)
    W, rng = _weights(cfg)
    h0 = synth.make_h0(cfg, rng, B * T)
    cache = orc.KVCache(cfg, B, T)
    res = orc.prefill(cfg, W, cache, h0, B, T)
    seq, pos = np.repeat(np.arange(B), T), np.tile(np.arange(T), B)
    tile = seq * ((T + qt - 1) // qt) + pos // qt
    quant = lambda r: orc.quantize_groups(r, cfg.resid_bits, cfg.group_size)
    bh, bsel, bcols, bstored = _brute_lazy_call(cfg, W, h0, seq, pos, tile, None, quant)
    _compare_with_brute(cfg, res, cache, seq, pos, bh, bsel, bcols, bstored)
    # the pooled selection really crosses sequences (some loop takes tokens of two sequences)
    assert any(len(set(seq[S])) > 1 for S in bsel.values())


# ----------------------------------------------------------------------------
# chunked prefill onto an existing cache, and the last_loop KV mode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("seed,lens,T,qt,c,bits", [(81, [7, 3], 6, 4, 3, 4), (82, [5, 9, 2], 5, 8, 4, 2)])
def test_lazy_chunked_prefill_over_residual_context_matches_materialised_brute_force(seed, lens, T, qt, c, bits):
    """A prefill chunk continues sequences that already hold tokens with
    residual levels: positions lens[b] + t, tiles counted from the chunk start,
    columns over the whole causal prefix (context and chunk)."""
    B = len(lens)
    cfg = _tiny_cfg(seed=seed, seq_len=T, batch=B, q_tile=qt, c_cols=c, rho=0.3, n_loops=4, resid_bits=bits,
                    ctx_len=max(lens))
    W, rng = _weights(cfg)
    ctx = synth.make_context(cfg, rng, lens)
    cache = orc.KVCache.from_context(cfg, ctx, max(lens) + T)
    h0 = synth.make_h0(cfg, rng, B * T)
    res = orc.prefill(cfg, W, cache, h0, B, T)
    assert np.array_equal(cache.lens, np.asarray(lens) + T)
    seq = np.repeat(np.arange(B), T)
    rel = np.tile(np.arange(T), B)
    pos = np.asarray(lens)[seq] + rel
    tile = seq * ((T + qt - 1) // qt) + rel // qt
    quant = lambda r: orc.quantize_groups(r, cfg.resid_bits, cfg.group_size)
    bh, bsel, bcols, bstored = _brute_lazy_call(cfg, W, h0, seq, pos, tile, ctx, quant)
    _compare_with_brute(cfg, res, cache, seq, pos, bh, bsel, bcols, bstored)
    # the column sets really reach into the context
    assert any(C.min() < min(lens) for C in bcols.values())


def test_lazy_chunked_prefill_dense_limit():
    """rho = 1, every column and an exact residual: a chunk over a residual
    context equals the dense per-loop chunk over the same context."""
    lens, T = np.array([6, 2]), 5
    cfg = _tiny_cfg(rho=1.0, c_cols=10 ** 6, resid_bits=32, seq_len=T, batch=2, n_loops=3, q_tile=4)
    W, rng = _weights(cfg)
    M, K, Hkv, hd = cfg.n_layers, cfg.n_loops, cfg.n_kv_heads, cfg.head_dim
    tmax = int(lens.max()) + T
    lazy_c = orc.KVCache(cfg, 2, tmax, kv_exact=True)
    dcfg = cfg.with_(resid_bits=16)
    dense_c = orc.KVCache(dcfg, 2, tmax, kv_exact=True)
    base_k, base_v = (rng.standard_normal((M, 2, Hkv, tmax, hd)) for _ in range(2))
    res_k, res_v = (rng.standard_normal((M, K - 1, 2, Hkv, tmax, hd)) * 0.1 for _ in range(2))
    for b in range(2):
        base_k[:, b, :, lens[b]:] = base_v[:, b, :, lens[b]:] = 0
        res_k[:, :, b, :, lens[b]:] = res_v[:, :, b, :, lens[b]:] = 0
    lazy_c.base_k[:], lazy_c.base_v[:], lazy_c.res_k[:], lazy_c.res_v[:] = base_k, base_v, res_k, res_v
    dense_c.kv_k[:, 0], dense_c.kv_v[:, 0] = base_k, base_v
    dense_c.kv_k[:, 1:] = base_k[:, None] + np.cumsum(res_k, axis=1)
    dense_c.kv_v[:, 1:] = base_v[:, None] + np.cumsum(res_v, axis=1)
    lazy_c.lens[:] = dense_c.lens[:] = lens
    h0 = synth.make_h0(cfg, rng, 2 * T)
    a = orc.prefill(cfg, W, lazy_c, h0, 2, T)
    b = orc.prefill(dcfg, W, dense_c, h0, 2, T)
    assert np.max(np.abs(a.h - b.h)) <= 1e-9 * np.sqrt(np.mean(b.h ** 2))
    np.testing.assert_allclose(a.logits, b.logits, atol=1e-9 * np.abs(b.logits).max())


def test_dense_chunked_prefill_equals_the_whole_prompt():
    """The dense looped forward is causal through every loop, so a prompt
    prefilled in chunks gives the same states, caches and logits as in one call."""
    cfg = _tiny_cfg(resid_bits=16, n_loops=3, seq_len=12, batch=2, seed=83)
    W, rng = _weights(cfg)
    T = cfg.seq_len
    h0 = synth.make_h0(cfg, rng, 2 * T)
    whole_c = orc.KVCache(cfg, 2, T)
    whole = orc.prefill(cfg, W, whole_c, h0, 2, T)
    parts_c = orc.KVCache(cfg, 2, T)
    hp = h0.reshape(2, T, -1)
    outs = []
    for a, b in ((0, 5), (5, 9), (9, 12)):
        r = orc.prefill(cfg, W, parts_c, hp[:, a:b].reshape(-1, cfg.d_model), 2, b - a)
        outs.append(r.h.reshape(2, b - a, -1))
    scale = np.abs(whole.h).max()
    np.testing.assert_allclose(np.concatenate(outs, axis=1).reshape(2 * T, -1), whole.h, atol=1e-12 * scale)
    np.testing.assert_allclose(r.logits, whole.logits, atol=1e-12 * np.abs(whole.logits).max())
    np.testing.assert_allclose(parts_c.kv_k, whole_c.kv_k, atol=1e-12 * np.abs(whole_c.kv_k).max())


def test_last_loop_prefill_of_a_fresh_prompt_equals_per_loop():
    """Within one call every token is at the same loop, so overwriting one KV
    slot per loop (last_loop) gives exactly the per-loop result."""
    cfg = _tiny_cfg(resid_bits=16, n_loops=3, seq_len=10, batch=2, seed=84)
    W, rng = _weights(cfg)
    h0 = synth.make_h0(cfg, rng, 20)
    per = orc.prefill(cfg, W, orc.KVCache(cfg, 2, 10), h0, 2, 10)
    lcfg = cfg.with_(kv_mode=1)
    lc = orc.KVCache(lcfg, 2, 10)
    last = orc.prefill(lcfg, W, lc, h0, 2, 10)
    assert np.array_equal(per.h, last.h) and np.array_equal(per.logits, last.logits)
    assert lc.kv_k.shape[1] == 1


def test_last_loop_decode_sees_the_context_last_pass_at_every_loop():
    """Over a context, last_loop attends to the context's one stored pass at
    every loop: the same as per_loop with every loop slot holding that pass."""
    cfg = _tiny_cfg(resid_bits=16, n_loops=3, mode="decode", batch=3, seq_len=0, ctx_len=8, seed=85, kv_mode=1)
    W, rng = _weights(cfg)
    lens = [8, 3, 6]
    ctx = synth.make_dense_context(cfg, rng, lens)
    assert ctx["kv_k"].shape[1] == 1
    last_c = orc.KVCache.from_dense_context(cfg, ctx, 9)
    pcfg = cfg.with_(kv_mode=0)
    rep = {"lens": ctx["lens"], "kv_k": np.repeat(ctx["kv_k"], cfg.n_loops, axis=1),
           "kv_v": np.repeat(ctx["kv_v"], cfg.n_loops, axis=1)}
    per_c = orc.KVCache.from_dense_context(pcfg, rep, 9)
    h0 = synth.make_h0(cfg, rng, 3)
    a = orc.decode_step(cfg, W, last_c, h0)
    b = orc.decode_step(pcfg, W, per_c, h0)
    assert np.array_equal(a.h, b.h)
    # and the new token's stored pass is its last loop's KV
    np.testing.assert_array_equal(last_c.kv_k[:, 0, :, :, 8], per_c.kv_k[:, -1, :, :, 8])


# ----------------------------------------------------------------------------
# variants around the looped core: prelude / coda layers, loop embedding,
# input injection
# ----------------------------------------------------------------------------

def test_sandwich_depth_golden():
    """The page's worked example: applications of independent and shared layers
    add up to the effective depth; the weights are P + R + Q layers."""
    rows = [tuple(int(v) for v in ln.split()) for ln in open(
        __file__.replace("test_oracle_pins.py", "golden/sandwich_depth.txt"))
        if ln.strip() and not ln.startswith("#")]
    for P, R, K, Q, depth, weight_layers in rows:
        cfg = _tiny_cfg(d_model=16, n_heads=2, n_kv_heads=1, head_dim=8, ffn_dim=16, n_layers=R, n_loops=K,
                        n_prelude=P, n_coda=Q, seq_len=4, q_tile=4, rho=0.5, c_cols=2, group_size=8)
        w = synth.make_weights(cfg)
        W = orc.prepare_weights(w)
        h0 = synth.make_h0(cfg, w["rng"], 4)
        res = orc.prefill(cfg, W, orc.KVCache(cfg, 1, 4), h0, 1, 4)
        assert res.trace["applications"] + res.trace["independent"] == depth
        assert len(W["prelude"]) + len(W["layers"]) + len(W["coda"]) == weight_layers
        dense = orc.prefill(cfg.with_(resid_bits=16), W, orc.KVCache(cfg.with_(resid_bits=16), 1, 4), h0, 1, 4)
        assert dense.trace["applications"] + dense.trace["independent"] == depth


@pytest.mark.parametrize("embed,gamma", [(0, 0.0), (1, 0.0), (1, 0.5), (0, 0.7)])
def test_sandwich_with_loop_embedding_and_injection_matches_torch(embed, gamma):
    """Dense variants against a torch restatement: the prelude, then per loop
    the shared stack applied to h + e_k + gamma * x (x: the prelude output),
    then the coda, each stack a plain pre-norm block sequence."""
    cfg = _tiny_cfg(resid_bits=16, n_loops=3, n_prelude=2, n_coda=1, loop_embed=embed, inject_scale=gamma, seed=87,
                    seq_len=10)
    w = synth.make_weights(cfg)
    W = orc.prepare_weights(w)
    h0 = synth.make_h0(cfg, w["rng"], 10)
    res = orc.prefill(cfg, W, orc.KVCache(cfg, 1, 10, kv_exact=True), h0, 1, 10)
    sub = lambda layers: {"layers": layers}
    x = _torch_block_forward(cfg, sub(W["prelude"]), np.asarray(h0, np.float64))
    h = x.copy()
    for k in range(cfg.n_loops):
        u = h + (W["loop_embed"][k] if embed else 0.0) + gamma * x
        h = _torch_block_forward(cfg, W, u)
    want = _torch_block_forward(cfg, sub(W["coda"]), h)
    np.testing.assert_allclose(res.h, want, rtol=0, atol=1e-11 * np.abs(want).max())
    if embed or gamma:      # the variant really changes the result
        plain = orc.prefill(cfg.with_(loop_embed=0, inject_scale=0.0), {k_: v_ for k_, v_ in W.items()
                            if k_ != "loop_embed"}, orc.KVCache(cfg, 1, 10, kv_exact=True), h0, 1, 10)
        assert np.max(np.abs(plain.h - res.h)) > 1e-3 * np.abs(want).max()


@pytest.mark.parametrize("mode", ["prefill", "decode"])
def test_lazy_variants_dense_limit(mode):
    """rho = 1, every column, exact residuals: the lazy path with prelude, coda,
    loop embedding and input injection equals the dense one."""
    cfg = _tiny_cfg(rho=1.0, c_cols=10 ** 6, resid_bits=32, n_loops=3, n_prelude=1, n_coda=2, loop_embed=1,
                    inject_scale=0.4, seed=88, seq_len=9, batch=2)
    dcfg = cfg.with_(resid_bits=16)
    w = synth.make_weights(cfg)
    rng = w["rng"]
    W = orc.prepare_weights(w)
    if mode == "prefill":
        h0 = synth.make_h0(cfg, rng, 18)
        a = orc.prefill(cfg, W, orc.KVCache(cfg, 2, 9, kv_exact=True), h0, 2, 9)
        b = orc.prefill(dcfg, W, orc.KVCache(dcfg, 2, 9, kv_exact=True), h0, 2, 9)
    else:
        lazy_c = orc.KVCache(cfg, 2, 12, kv_exact=True)
        dense_c = orc.KVCache(dcfg, 2, 12, kv_exact=True)
        pre = synth.make_h0(cfg, rng, 18)       # a dense prompt fills both caches identically
        orc.prefill(cfg, W, lazy_c, pre, 2, 9)
        orc.prefill(dcfg, W, dense_c, pre, 2, 9)
        h0 = synth.make_h0(cfg, rng, 2)
        a = orc.decode_step(cfg, W, lazy_c, h0)
        b = orc.decode_step(dcfg, W, dense_c, h0)
    assert np.max(np.abs(a.h - b.h)) <= 1e-9 * np.sqrt(np.mean(b.h ** 2))
    np.testing.assert_allclose(a.logits, b.logits, atol=1e-9 * np.abs(b.logits).max())


# ----------------------------------------------------------------------------
# invariants of the lazy path
# ----------------------------------------------------------------------------

def test_lazy_invariants_carry_and_keys():
    cfg = _tiny_cfg(seed=31, seq_len=24, q_tile=8, c_cols=6, rho=0.25, n_loops=4)
    W, rng = _weights(cfg)
    h0 = synth.make_h0(cfg, rng, 24)
    cache = orc.KVCache(cfg, 1, 24)
    res = orc.prefill(cfg, W, cache, h0, 1, 24)
    n_sel = orc.n_select(cfg.rho, 24)
    hs = res.trace["h"]
    for l in range(2, cfg.n_loops + 1):
        S = res.trace["sel"][l]
        assert len(S) == n_sel
        carried = np.setdiff1d(np.arange(24), S)
        assert np.array_equal(hs[l][carried], hs[l - 1][carried])        # bit-identical carry
        if l + 1 in res.trace["keys"]:
            assert np.all(res.trace["keys"][l + 1][carried] == 0)
        for j in range(cfg.n_layers):
            nz = np.any(cache.codes_k[j, l - 2, 0] != 0, axis=(0, 2)) | np.any(
                cache.scales_k[j, l - 2, 0] != 0, axis=(0, 2))
            assert np.all(np.isin(np.nonzero(nz)[0], S))
            assert nz.sum() <= n_sel
    np.testing.assert_array_equal(res.h, hs[cfg.n_loops])


def test_correction_identity_full_columns_equals_softmax():
    """With C = every column, the corrected output equals softmax attention on the new scores."""
    cfg = _tiny_cfg(seed=41, seq_len=10, q_tile=16, c_cols=10 ** 6, rho=1.0, n_loops=2)
    W, rng = _weights(cfg)
    h0 = synth.make_h0(cfg, rng, 10)
    cache = orc.KVCache(cfg, 1, 10)
    res = orc.prefill(cfg, W, cache, h0, 1, 10)
    # recompute loop 2's attention of layer 0 directly from the cache and loop-1 state
    lw = W["layers"][0]
    q, _, _ = orc._qkv(cfg, lw, res.trace["h"][1], np.arange(10))
    tau = 1 / math.sqrt(cfg.head_dim)
    for i in range(10):
        kk = cache.chain("k", 0, 2, 0, np.arange(i + 1))
        vv = cache.chain("v", 0, 2, 0, np.arange(i + 1))
        o, lse = orc._attn_full(q[i], kk, vv, tau)
        np.testing.assert_allclose(res.trace["O"][0, i], o, atol=1e-12)
        np.testing.assert_allclose(res.trace["lse"][0, i], lse, atol=1e-12)
