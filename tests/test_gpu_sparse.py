"""Sparse residual storage on the GPU.

With resid_rows > 0 the cache keeps KV residual rows only for the tokens a loop
recomputed (a pool of rows per layer, loop, K/V, sequence and KV head, and a
row index per position), which is where the KV-cache memory reduction of
"FlashLoop: Fast and Memory-Efficient Looped Transformers via Lazy Updates"
(abstract) comes from.  Storage changes nothing else: the same calls, free
running, must give bit-identical hidden states, logits, selections and cache
contents (exported by position) with the dense layout and with the sparse one,
and a pool that is too small must be reported, not overrun.
"""
import numpy as np
import pytest

from cross_loop_sparsity_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from cross_loop_sparsity_b200 import build
    build.build()


def _run(cfg, B, ctx_lens, chunks, decode_steps, rows):
    """Free-running calls; returns every output and the exported cache."""
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    w = synth.make_weights(cfg)
    rng = w["rng"]
    ctx = synth.make_context(cfg, rng, ctx_lens) if max(ctx_lens) else None
    tmax = max(ctx_lens) + sum(chunks) + decode_steps
    eng = fl.FlashLoop(cfg.with_(resid_rows=rows), fl.upload_weights(w), max_batch=B, max_ctx=tmax,
                       max_tokens=B * max(chunks, default=0))
    if ctx is not None:
        eng.load_context(ctx)
    outs, lens = [], list(ctx_lens)
    for T in chunks:
        h0 = torch.from_numpy(synth.make_h0(cfg, rng, B * T)).cuda()
        h_out = torch.empty((B * T, cfg.d_model), dtype=torch.float32, device="cuda")
        lg = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
        eng.prefill(h0, B, T, h_out, lg)
        torch.cuda.synchronize()
        n_sel = max(1, min(B * T, int(np.ceil(cfg.rho * B * T - 1e-9))))
        n_tiles = B * ((T + cfg.q_tile - 1) // cfg.q_tile)
        outs += [h_out.cpu().numpy(), lg.cpu().numpy()] + list(eng.read_trace(B * T, n_sel, n_tiles))
        lens = [x + T for x in lens]
    for _ in range(decode_steps):
        h0 = torch.from_numpy(synth.make_h0(cfg, rng, B)).cuda()
        h_out = torch.empty((B, cfg.d_model), dtype=torch.float32, device="cuda")
        lg = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
        eng.decode_step(h0, B, h_out, lg)
        torch.cuda.synchronize()
        n_sel = max(1, min(B, int(np.ceil(cfg.rho * B - 1e-9))))
        outs += [h_out.cpu().numpy(), lg.cpu().numpy()] + list(eng.read_trace(B, n_sel, B))
        lens = [x + 1 for x in lens]
    status = eng.sync_status()
    cache = []
    for j in range(cfg.n_layers):
        for loop in range(1, cfg.n_loops + 1):
            for b in range(B):
                for which in (0, 1):
                    c, s = eng.export_slice(j, loop, b, which, lens[b])
                    cache.append(c)
                    if s is not None:
                        cache.append(s.view(np.uint16))
    eng.close()
    return status, outs, cache


CASES = {
    # ragged decode over a context holding residual levels, several recomputed tokens
    "c2_ragged_decode": (synth.config("c2").with_(ctx_len=1500, rho=0.5, seed=121), 4, [1500, 700, 3, 1200], [], 3),
    # K = 8 loops, int2, decode over ragged contexts
    "c5_int2_decode": (synth.config("c5_int2").with_(batch=3, rho=0.5, ctx_len=2000, seed=123), 3, [2000, 900, 64],
                       [], 2),
    # prefill of two fresh sequences, then decode
    "c1_prefill_decode": (synth.config("c1").with_(seq_len=200, seed=125), 2, [0, 0], [200], 2),
    # a chunk onto a residual context (the large-call path assigns the rows)
    "c1_chunk_onto_context": (synth.config("c1").with_(seq_len=150, seed=127, c_cols=24), 2, [220, 60], [150], 1),
}


@pytest.mark.parametrize("case", list(CASES))
def test_sparse_storage_is_bit_identical_to_the_dense_layout(case):
    cfg, B, ctx_lens, chunks, steps = CASES[case]
    tmax = max(ctx_lens) + sum(chunks) + steps
    # room for the context's recomputed rows and every token the calls add
    rows = min(tmax, int(np.ceil(cfg.rho * tmax)) + sum(chunks) + steps)
    st_d, outs_d, cache_d = _run(cfg, B, ctx_lens, chunks, steps, 0)
    st_s, outs_s, cache_s = _run(cfg, B, ctx_lens, chunks, steps, rows)
    assert st_d == 0 and st_s == 0
    assert len(outs_d) == len(outs_s) and len(cache_d) == len(cache_s)
    for a, b in zip(outs_d, outs_s):
        assert np.array_equal(a, b)
    for a, b in zip(cache_d, cache_s):
        assert np.array_equal(a, b)


def test_sparse_pool_overflow_is_reported():
    """A pool smaller than the context's recomputed rows: the import and the
    calls keep what fits, record the overflow, and sync_status reports
    FL_ERR_CAPACITY; nothing is written outside the pool."""
    cfg = synth.config("c2").with_(ctx_len=600, rho=0.5, seed=129)
    status, outs, _ = _run(cfg, 4, [600, 300, 80, 600], [], 1, 16)
    assert status == 2
    for o in outs:
        assert np.all(np.isfinite(o))
