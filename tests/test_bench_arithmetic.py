"""Host arithmetic of bench.py's roofline entries, against figures derived by hand.

The bytes and FLOPs below were worked out from the workloads' shapes alone:
weights are 2 bytes per parameter, streamed once per loop; the dense-looped
decode reads every loop's own bf16 K and V of every column; a prefill performs
the GEMMs and causal attention of every token at every loop.  They are the
denominators of the reported roofline fractions, so a slip in bench.py's
formulas would misstate every fraction without failing any GPU test.
"""
import importlib.util
import math
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def _cfg(name):
    from cross_loop_sparsity_b200 import synth
    return synth.config(name)


# (workload, weight GB over all loops, LM head GB, dense-looped KV GB read per step)
DECODE = [
    ("c2", 1.4428, 0.1311, 1.0740),   # 4 loops x 360.7 MB; 8 x 4097 columns x 4 layers x 4 loops
    ("c4", 68.048, 0.2621, 25.773),   # 4 loops x 17.01 GB (d 4096, ffn 11008, 48 layers)
    ("c5", 2.8857, 0.1311, 4.2950),   # 8 loops x 360.7 MB; 65 537 columns x 4 layers x 8 loops
]


@pytest.mark.parametrize("name,weights_gb,head_gb,dense_kv_gb", DECODE)
def test_decode_bytes_match_hand_derived(bench, name, weights_gb, head_gb, dense_kv_gb):
    cfg = _cfg(name)
    B = cfg.batch
    n_sel = max(1, min(B, math.ceil(cfg.rho * B - 1e-9)))
    assert bench.dense_kv_bytes_read(cfg) / 1e9 == pytest.approx(dense_kv_gb, rel=2e-4)
    # the GEMM bytes are the weights and the LM head plus the token rows' activations (well under 1 %)
    g = bench.gemm_algorithmic_bytes(cfg, B, n_sel) / 1e9
    assert weights_gb + head_gb <= g <= (weights_gb + head_gb) * 1.01
    # the lazy step reads at least the loop-1 base K/V of every column, and less than the dense step
    base = cfg.n_layers * B * cfg.n_kv_heads * (cfg.ctx_len + 1) * cfg.head_dim * 2 * 2
    kv = bench.kv_bytes_read(cfg, n_sel)
    assert base < kv < bench.dense_kv_bytes_read(cfg)


def test_dense_prefill_flops_match_hand_derived(bench):
    # c3: 22 layers x 2 loops over 16 384 tokens: 2 x (QKV + O + 3 FFN GEMMs) per token plus causal attention
    assert bench.prefill_flops(_cfg("c3")) / 1e12 == pytest.approx(113.39, rel=2e-4)


def test_lazy_prefill_flops_count_each_tile_once(bench):
    """The Δscore products are counted once per tile, at the loop that first recomputes it."""
    cfg = _cfg("c1")
    T, K = cfg.seq_len, cfg.n_loops
    dense = bench.prefill_flops(cfg)
    one_tile = np.arange(0, min(T, cfg.q_tile), dtype=np.int64)   # the first query tile only
    again = [one_tile] * (K - 1)
    first_only = [one_tile] + [np.zeros(0, dtype=np.int64)] * (K - 2)
    lazy_again = bench.prefill_flops(cfg, again)
    lazy_first = bench.prefill_flops(cfg, first_only)
    # recomputing the same tile at later loops adds its GEMMs and corrections, never a second Δscore
    d, f, hq, qkv, H, hd = (cfg.d_model, cfg.ffn_dim, cfg.n_heads * cfg.head_dim, cfg.qkv_rows, cfg.n_heads,
                            cfg.head_dim)
    per_tok = 2 * (d * qkv + hq * d + 2 * d * f + f * d) + 8 * H * hd * cfg.c_cols
    assert lazy_again - lazy_first == pytest.approx(cfg.n_layers * (K - 2) * len(one_tile) * per_tok, rel=1e-12)
    assert lazy_first < dense
