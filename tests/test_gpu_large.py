"""The large workloads on the GPU.

* The long prefill (16384 tokens, 22 layers x 2 loops) at full size, checked
  through properties that hold at any size plus sampled outputs the oracle can
  compute one by one (layer-0 keys from h0).
* The long-prefill and deep-recurrence block shapes at reduced depth and
  length, compared element by element with the oracle (forced selections).
"""
import math

import numpy as np
import pytest

import e2e_common as E
from cross_loop_sparsity_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from cross_loop_sparsity_b200 import build
    build.build()


def test_prefill_long_block_reduced_depth_forced():
    cfg = synth.config("c3").with_(n_layers=2, seq_len=1024, seed=21)
    cfg, ref, eng, out = E.run_prefill(cfg, 1, 1024)
    assert out["status"] == 0
    assert E.rel_err(out["h"], ref.h) <= E.TOL
    assert E.rel_err(out["logits"], ref.logits) <= E.TOL


def test_decode_deep_block_reduced_depth_forced():
    cfg = synth.config("c4").with_(n_layers=2, ctx_len=512, seed=31)
    cfg, cache, eng, results = E.run_decode(cfg, [512, 300, 77, 511])
    for ref, out in results:
        assert out["status"] == 0
        assert E.rel_err(out["h"], ref.h) <= E.TOL
        assert E.rel_err(out["logits"], ref.logits) <= E.TOL


def test_prefill_long_full_size_properties():
    import torch
    from cross_loop_sparsity_b200 import flashloop as fl
    from oracle import flashloop_oracle as orc
    cfg = synth.config("c3")
    T, d = cfg.seq_len, cfg.d_model
    w = synth.make_weights(cfg)
    h0 = synth.make_h0(cfg, w["rng"], T)
    eng = fl.FlashLoop(cfg, fl.upload_weights(w), max_batch=1, max_ctx=T, max_tokens=T)
    h_out = torch.empty((T, d), dtype=torch.float32, device="cuda")
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    eng.prefill(torch.from_numpy(h0).cuda(), 1, T, h_out, logits)
    torch.cuda.synchronize()
    assert eng.sync_status() == 0
    h = h_out.cpu().numpy()
    assert np.all(np.isfinite(h)) and np.all(np.isfinite(logits.cpu().numpy()))
    n_sel = math.ceil(cfg.rho * T - 1e-9)
    assert n_sel == 2458
    tiles = T // cfg.q_tile
    sel, keys, cols, ncols = eng.read_trace(T, n_sel, tiles)
    # (1) the recomputed tokens are a valid top-rho of the library's own change keys
    assert E.top_valid(keys[0], n_sel, sel[0])
    # (2) a carried token's final state is its loop-1 state: its change key is
    #     ||h_final - h0||^2 (fp32 on the GPU, fp64 here)
    carried = np.setdiff1d(np.arange(T), sel[0])
    dk = np.sum((h[carried].astype(np.float64) - h0[carried]) ** 2, axis=1)
    assert np.allclose(keys[0][carried], dk, rtol=1e-4, atol=1e-6)
    # (3) every recomputed query tile has min(c, eligible) ascending causal columns
    sel_tiles = np.unique(sel[0] // cfg.q_tile)
    for j in range(cfg.n_layers):
        for t in sel_tiles:
            members = sel[0][sel[0] // cfg.q_tile == t]
            elig = int(members.max()) + 1
            for g in range(cfg.n_kv_heads):
                n = ncols[j, t, g]
                assert n == min(cfg.c_cols, elig)
                C = cols[j, t, g, :n]
                assert np.all(np.diff(C) > 0) and C[0] >= 0 and C[-1] < elig
    # (4) loop-2 residuals: zero for carried tokens, int4 codes in [-7, 7] for recomputed ones
    for j in (0, cfg.n_layers - 1):
        for which in (0, 1):
            codes, scales = eng.export_slice(j, 2, 0, which, T)
            assert np.all(codes[:, carried] == 0) and np.all(scales[:, carried] == 0)
            nib = np.stack([codes[:, sel[0]] & 0xF, codes[:, sel[0]] >> 4])
            assert not np.any(nib == 0x8)
    # (5) sampled outputs the oracle computes one by one: layer-0 keys from h0
    rows = np.array([0, 1, 127, 128, 4095, 9999, T - 1])
    Wq = orc.prepare_weights({"layers": [w["layers"][0]], "final_norm": w["final_norm"], "w_out": w["w_out"][:1]})
    lw = Wq["layers"][0]
    _, k_ref, v_ref = orc._qkv(cfg, lw, h0[rows], rows)
    base_k, _ = eng.export_slice(0, 1, 0, 0, T)
    base_v, _ = eng.export_slice(0, 1, 0, 1, T)
    to_f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    k_gpu = to_f(base_k[:, rows]).transpose(1, 0, 2)
    v_gpu = to_f(base_v[:, rows]).transpose(1, 0, 2)
    assert E.rel_err(k_gpu, k_ref) <= E.TOL
    assert E.rel_err(v_gpu, v_ref) <= E.TOL
