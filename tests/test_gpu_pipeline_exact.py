"""Free-running, bit-exact checks of the integer decisions the pipeline takes.

Nothing is handed to the library here: it selects tokens, chooses column sets
and quantises KV residuals itself.  Through the check buffers of
``flashloop_set_trace`` it reports the inputs of those decisions -- the rotated
fp32 K/V rows each lazy loop quantised and the delta-score key of every
eligible column -- and the tests recompute every decision on the CPU from those
inputs and the library's exported cache:

* KV-residual quantisation ("FlashLoop: Fast and Memory-Efficient Looped
  Transformers via Lazy Updates", abstract: each loop's KV kept as a low-bit
  residual over the previous loop's): the previous level is rebuilt from the exported base and
  residual codes / scales of loops 2..l-1 (fp32 adds in loop order), r =
  fp32(x - prev), and the oracle's quantiser and packer must give the exported
  codes and scales bit for bit.  Tokens not recomputed at loop l must hold a
  zero residual row.
* Column sets (the abstract's sparse, stable subset of key columns): every set
  must be the top-c of the library's own keys under (bit pattern desc, index
  asc), checked with a plain sort.
* Token selections: a valid top-n_sel of the library's own change keys.

Prefill (wide GEMM) and decode (split-K GEMM) both feed the RoPE / KV kernel,
whose quantiser is covered at int4 and int2, head_dim 64 and 128 (two and four
values per lane), groups 32 and 64, loops 2..8.
"""
import numpy as np
import pytest

import e2e_common as E
from cross_loop_sparsity_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from cross_loop_sparsity_b200 import build
    build.build()


def _f32_of_bf16(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


class _Exports:
    """Exported cache slices, fetched once per (layer, loop, sequence, K/V)."""

    def __init__(self, eng, n_of_seq):
        self.eng, self.n_of_seq, self.memo = eng, n_of_seq, {}

    def get(self, j, l, b, kv):
        key = (j, l, b, kv)
        if key not in self.memo:
            self.memo[key] = self.eng.export_slice(j, l, b, kv, self.n_of_seq[b])
        return self.memo[key]


def _check_codes(cfg, eng, sel, kv_trace, seq_of, pos_of, call_tokens, n_of_seq):
    """Every recomputed token's exported codes and scales at every lazy loop
    equal the oracle quantiser applied to (library row - rebuilt previous level);
    every other token of the call holds a zero residual row."""
    from oracle import flashloop_oracle as orc
    bits, g, K = cfg.resid_bits, cfg.group_size, cfg.n_loops
    ex = _Exports(eng, n_of_seq)
    checked = 0
    for j in range(cfg.n_layers):
        for l in range(2, K + 1):
            S = np.asarray(sel[l - 2])
            for kv in (0, 1):
                for b in sorted(set(int(seq_of[t]) for t in call_tokens)):
                    slots = [a for a, t in enumerate(S) if seq_of[t] == b]
                    mine = [t for t in call_tokens if seq_of[t] == b]
                    codes_l, scales_l = ex.get(j, l, b, kv)
                    # carried tokens of this call: zero residual row at loop l
                    carried = [pos_of[t] for t in mine if t not in set(S.tolist())]
                    if carried:
                        assert not np.any(codes_l[:, carried]), (j, l, b, kv)
                        assert not np.any(scales_l[:, carried].view(np.uint16)), (j, l, b, kv)
                    if not slots:
                        continue
                    p = np.array([pos_of[S[a]] for a in slots])
                    base, _ = ex.get(j, 1, b, kv)
                    prev = _f32_of_bf16(base[:, p])                            # [Hkv][n][hd]
                    for l2 in range(2, l):
                        c2, s2 = ex.get(j, l2, b, kv)
                        deq = orc.dequant_groups(orc.unpack_codes(c2[:, p], bits), s2[:, p], g)
                        prev = (prev + deq).astype(np.float32)
                    x = kv_trace[j, l - 2, slots, kv].transpose(1, 0, 2)       # [Hkv][n][hd]
                    r = (x - prev).astype(np.float32)
                    want_c, want_s = orc.quantize_groups(r, bits, g)
                    assert np.array_equal(scales_l[:, p].view(np.uint16), want_s.view(np.uint16)), (j, l, b, kv)
                    assert np.array_equal(codes_l[:, p], orc.pack_codes(want_c, bits)), (j, l, b, kv)
                    checked += len(slots)
    return checked


def _check_column_sets(cfg, sel, cols, ncols, ck_trace, tile_of, pos_of):
    """Each tile's set is chosen at its first recomputation in the call from the
    keys of columns 0..(largest position among that loop's selected members)."""
    chosen_at = {}
    for l in range(2, cfg.n_loops + 1):
        members = {}
        for t in sel[l - 2]:
            members.setdefault(int(tile_of[t]), []).append(int(t))
        for tl, ts in members.items():
            if tl not in chosen_at:
                chosen_at[tl] = max(pos_of[t] for t in ts) + 1
    for tl, n in chosen_at.items():
        for j in range(cfg.n_layers):
            for gk in range(cfg.n_kv_heads):
                k = min(cfg.c_cols, n)
                assert ncols[j, tl, gk] == k, (j, tl, gk)
                got = cols[j, tl, gk, :k]
                assert E.top_valid(ck_trace[j, tl, gk, :n], k, got), (j, tl, gk)
    return len(chosen_at)


def _traces(torch, cfg, n_slots, n_tiles, max_ctx):
    kv = torch.zeros((cfg.n_layers, cfg.n_loops - 1, n_slots, 2, cfg.n_kv_heads, cfg.head_dim),
                     dtype=torch.float32, device="cuda")
    ck = torch.zeros((cfg.n_layers, n_tiles, cfg.n_kv_heads, max_ctx), dtype=torch.float32, device="cuda")
    return kv, ck


@pytest.mark.parametrize("case", ["c1_two_sequences", "c3_block_1024", "c1_chunk_onto_context"])
def test_prefill_free_running_codes_and_column_sets_bit_exact(case):
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    from oracle import flashloop_oracle as orc
    lens = None
    if case == "c1_two_sequences":
        cfg, B, T = synth.config("c1").with_(seq_len=200, seed=41), 2, 200
    elif case == "c3_block_1024":
        cfg, B, T = synth.config("c3").with_(n_layers=2, n_loops=3, seq_len=1024, seed=43), 1, 1024
    else:   # a chunk continuing sequences whose context already holds residual levels
        cfg, B, T, lens = synth.config("c1").with_(seq_len=150, seed=45, c_cols=24), 2, 150, [220, 60]
    w = synth.make_weights(cfg)
    rng = w["rng"]
    ctx = synth.make_context(cfg, rng, lens) if lens else None
    h0 = synth.make_h0(cfg, rng, B * T)
    lens = lens or [0] * B
    eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=B, max_ctx=max(lens) + T, max_tokens=B * T)
    if ctx is not None:
        eng.load_context(ctx)
    N = B * T
    n_sel = orc.n_select(cfg.rho, N)
    tps = (T + cfg.q_tile - 1) // cfg.q_tile
    n_tiles = B * tps
    kv, ck = _traces(torch, cfg, n_sel, n_tiles, max(lens) + T)
    eng.set_trace(kv, n_sel, ck, n_tiles)
    eng.prefill(torch.from_numpy(h0).cuda(), B, T)
    torch.cuda.synchronize()
    assert eng.sync_status() == 0
    sel, keys, cols, ncols = eng.read_trace(N, n_sel, n_tiles)
    for l in range(2, cfg.n_loops + 1):
        assert E.top_valid(keys[l - 2], n_sel, sel[l - 2]), l
    seq_of, rel = np.repeat(np.arange(B), T), np.tile(np.arange(T), B)
    pos_of = np.asarray(lens)[seq_of] + rel
    tile_of = seq_of * tps + rel // cfg.q_tile
    n = _check_codes(cfg, eng, sel, kv.cpu().numpy(), seq_of, pos_of, list(range(N)), [l + T for l in lens])
    assert n == cfg.n_layers * (cfg.n_loops - 1) * 2 * n_sel
    assert _check_column_sets(cfg, sel, cols, ncols, ck.cpu().numpy(), tile_of, pos_of) > 0
    eng.close()


DECODE_CASES = {
    # tiny block, int4 g32, head_dim 64, ragged contexts, several recomputed tokens
    "c1_ragged": (synth.config("c1").with_(mode="decode", batch=3, rho=0.5, c_cols=24, seed=47, seq_len=0),
                  [300, 77, 1], 2),
    # the full decode workload: 8 x 4096, int4 g64, head_dim 128
    "c2_full": (synth.config("c2"), [4096] * 8, 1),
    # ragged contexts of the decode block, two recomputed tokens per loop
    "c2_ragged": (synth.config("c2").with_(ctx_len=1500, seed=53, rho=0.5), [1500, 700, 3, 1200], 1),
    # K = 8 loops, int2, ragged contexts, two recomputed tokens per loop
    "c5_int2_ragged": (synth.config("c5_int2").with_(batch=3, rho=0.5, ctx_len=3000, seed=59), [3000, 1700, 64], 2),
    # contexts longer than one shared-memory slice of column keys: the top-c is
    # taken per slice and then over the slices' candidates
    "c5_long_slices": (synth.config("c5").with_(batch=2, rho=0.5, ctx_len=40000, seed=61), [40000, 20001], 1),
    # the full decode workload with sparse residual storage (rows for recomputed tokens only)
    "c2_full_sparse": (synth.config("c2").with_(resid_rows=synth.sparse_rows(synth.config("c2"), 8)), [4096] * 8, 1),
}


@pytest.mark.parametrize("case", list(DECODE_CASES))
def test_decode_free_running_codes_and_column_sets_bit_exact(case):
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    from oracle import flashloop_oracle as orc
    cfg, lens, steps = DECODE_CASES[case]
    B = len(lens)
    w = synth.make_weights(cfg)
    rng = w["rng"]
    ctx = synth.make_context(cfg, rng, lens)
    max_ctx = max(lens) + steps
    eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=B, max_ctx=max_ctx)
    eng.load_context(ctx)
    del ctx
    n_sel = orc.n_select(cfg.rho, B)
    kv, ck = _traces(torch, cfg, n_sel, B, max_ctx)
    eng.set_trace(kv, n_sel, ck, B)
    total = 0
    for step in range(steps):
        kv.zero_()
        ck.zero_()
        h0 = torch.from_numpy(synth.make_h0(cfg, rng, B)).cuda()
        eng.decode_step(h0, B)
        torch.cuda.synchronize()
        assert eng.sync_status() == 0
        sel, keys, cols, ncols = eng.read_trace(B, n_sel, B)
        for l in range(2, cfg.n_loops + 1):
            assert E.top_valid(keys[l - 2], n_sel, sel[l - 2]), (step, l)
        pos_of = np.array([lens[b] + step for b in range(B)])
        seq_of = np.arange(B)
        total += _check_codes(cfg, eng, sel, kv.cpu().numpy(), seq_of, pos_of, list(range(B)),
                              [int(p) + 1 for p in pos_of])
        assert _check_column_sets(cfg, sel, cols, ncols, ck.cpu().numpy(), seq_of, pos_of) > 0
    assert total == steps * cfg.n_layers * (cfg.n_loops - 1) * 2 * n_sel
    eng.close()
